// spec_verify_chain_noalloc: chain verification over a scratch that lives inside the library.
//
// Some callers cannot hand the library a workspace:
//   - code recording a stream capture it does not own, where an allocation would either
//     be refused or become part of the captured graph;
//   - plain C hosts that hold only the tensors they pass and have no device allocator;
//   - decode loops whose memory pool is fixed at start-up, where cudaMalloc may
//     synchronise the device or fail outright.
// For them this entry point runs spec_verify_chain unchanged, with its workspace carved from
// one statically sized __device__ array (one instance per device the module is loaded on).
// It allocates nothing: no cudaMalloc/cudaFree, no allocating library routine. The array's
// address is looked up once per device with cudaGetSymbolAddress, with that device
// current, and cached; the logits must be device memory of the current device (checked
// before any launch). What must start at zero (the status word and the fallback count)
// spec_verify_chain clears on every call; everything else it writes before reading.
#include <cuda_runtime.h>

#include <mutex>

#include "specverify.h"

namespace {

__device__ __align__(256) unsigned char g_static_scratch[SPEC_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};  // per device; nullptr until looked up

// The scratch of the current device, or nullptr if its address cannot be obtained.
void* device_scratch() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

// True when p is device (or managed) memory of the current device. The scratch is chosen
// by the current device, so logits on another device would have this call's kernels write
// the wrong device's array.
bool on_current_device(const void* p) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaPointerAttributes at = {};
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();  // a failed query leaves a (non-sticky) error behind: clear it
    return false;
  }
  return (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) && at.device == dev;
}

}  // namespace

extern "C" spec_status spec_verify_chain_noalloc(
    const void* target_logits, const void* draft_logits, spec_dtype dtype, int B, int K, int V,
    const int32_t* draft_tokens, const float* uniforms, float temp, int top_k, float top_p,
    int32_t* accepted_len, int32_t* out_tokens, void* stream) {
  if (B <= 0 || K <= 0 || V <= 0 || !target_logits) return SPEC_ERR_INVALID_ARG;
  const size_t need = spec_workspace_size(B, K, V);
  if (need == 0) return SPEC_ERR_INVALID_ARG;
  if (need > SPEC_STATIC_SCRATCH_BYTES) return SPEC_ERR_WORKSPACE;  // before any CUDA call
  if (!on_current_device(target_logits)) return SPEC_ERR_INVALID_ARG;
  void* scratch = device_scratch();
  if (!scratch) return SPEC_ERR_CUDA;
  return spec_verify_chain(target_logits, draft_logits, dtype, B, K, V, draft_tokens, uniforms,
                           temp, top_k, top_p, accepted_len, out_tokens, scratch,
                           SPEC_STATIC_SCRATCH_BYTES, stream);
}
