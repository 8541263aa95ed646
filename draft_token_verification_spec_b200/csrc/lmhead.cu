// spec_verify_chain_lmhead: chain verification straight from hidden states, with the LM head
// product on the tensor cores and the verification statistics in its epilogue (lmhead.cuh).
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <map>
#include <mutex>

#include "lmhead.cuh"
#include "specverify.h"

namespace {

using sv::kThreads;

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// Work split of one product: row tiles x vocabulary chunks, the chunk size chosen so the
// busiest of G CTAs carries the fewest 256-column tiles (chunks x k <= the merge's capacity).
struct Split {
  int m_tiles, n_tiles, nchunk, tpc;
};

Split plan_split(int M, int V, int k, int G) {
  Split s;
  s.m_tiles = (M + sv::kLmBM - 1) / sv::kLmBM;
  s.n_tiles = (V + sv::kLmBN - 1) / sv::kLmBN;
  const int max_chunks = std::max(1, std::min(s.n_tiles, sv::kLmMergeCap / k));
  long long best = -1;
  s.nchunk = 1;
  s.tpc = s.n_tiles;
  for (int nc = 1; nc <= max_chunks; ++nc) {
    const int tpc = (s.n_tiles + nc - 1) / nc;
    const int chunks = (s.n_tiles + tpc - 1) / tpc;
    const long long items = (long long)s.m_tiles * chunks;
    const long long load = ((items + G - 1) / G) * tpc;  // tiles of the busiest CTA
    if (best < 0 || load < best) {
      best = load;
      s.nchunk = chunks;
      s.tpc = tpc;
    }
  }
  return s;
}

struct LmLayout {
  size_t part_val, part_id, rows, kept_val, kept_id, total;
};

LmLayout lm_layout(long long rows, int k, int nchunk_max) {
  LmLayout w;
  w.part_val = 256;  // the status word lives at offset 0
  w.part_id = w.part_val + up256(size_t(rows) * nchunk_max * k * 4);
  w.rows = w.part_id + up256(size_t(rows) * nchunk_max * k * 4);
  w.kept_val = w.rows + up256(size_t(rows) * sizeof(sv::LmRow));
  w.kept_id = w.kept_val + up256(size_t(rows) * k * 4);
  w.total = w.kept_id + up256(size_t(rows) * k * 4);
  return w;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// A K-major bf16 matrix [rows][d] as a TMA tensor map with (64 x box_rows) boxes and the
// 128-byte swizzle the MMA descriptors expect.
bool make_map(CUtensorMap* map, const void* base, long long rows, int d, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cuuint64_t(d), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(d) * 2};
  cuuint32_t box[2] = {cuuint32_t(sv::kLmBK), cuuint32_t(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

int sm_count(cudaError_t* err) {
  static std::mutex mu;
  static std::map<int, int> cache;
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(dev);
  if (it != cache.end()) return it->second;
  int n = 0;
  *err = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (*err != cudaSuccess) return 0;
  cache[dev] = n;
  return n;
}

// One product (hidden [M][d] x weight [V][d]^T) into per-chunk top-k lists of rows
// [row0, row0 + M) of the workspace.
cudaError_t run_product(const void* hidden, const void* weight, int M, int V, int d, int k,
                        int G, float* part_val, int32_t* part_id, int nchunk_stride,
                        float* logits_out, int32_t* dev_status, cudaStream_t s, Split* used) {
  CUtensorMap mh, mw;
  if (!make_map(&mh, hidden, M, d, sv::kLmBM) || !make_map(&mw, weight, V, d, sv::kLmBN))
    return cudaErrorInvalidValue;
  const Split sp = plan_split(M, V, k, G);
  *used = sp;
  sv::LmJob j = {};
  j.M = M;
  j.V = V;
  j.d = d;
  j.k = k;
  j.nchunk = sp.nchunk;
  j.tiles_per_chunk = sp.tpc;
  j.n_tiles = sp.n_tiles;
  j.m_tiles = sp.m_tiles;
  j.part_val = part_val;
  j.part_id = part_id;
  j.logits_out = logits_out;
  j.dev_status = dev_status;
  (void)nchunk_stride;
  cudaError_t e = cudaFuncSetAttribute(sv::lmhead_topk_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(sv::kLmSmem));
  if (e != cudaSuccess) return e;
  const int items = sp.m_tiles * sp.nchunk;
  sv::lmhead_topk_kernel<<<std::min(G, items), sv::kLmThreads, sv::kLmSmem, s>>>(mh, mw, j);
  return cudaGetLastError();
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

size_t spec_lmhead_workspace_size(int B, int K, int V, int d, int top_k) {
  if (B <= 0 || K <= 0 || V <= 0 || d <= 0) return 0;
  const int k = top_k >= 1 ? top_k : 1;
  const long long rows = (long long)B * (2LL * K + 1);
  return lm_layout(rows, k, sv::kLmMergeCap / k).total;
}

spec_status spec_verify_chain_lmhead(const void* target_hidden, const void* draft_hidden,
                                     const void* target_weight, const void* draft_weight, int B,
                                     int K, int V, int d, const int32_t* draft_tokens,
                                     const float* uniforms, float temp, int top_k,
                                     int32_t* accepted_len, int32_t* out_tokens,
                                     float* logits_out, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  const bool greedy = temp == 0.0f;
  if (!target_hidden || !target_weight || (!greedy && (!draft_hidden || !draft_weight)) ||
      B <= 0 || K <= 0 || V <= 0 || d <= 0 || !draft_tokens || !uniforms || !accepted_len ||
      !out_tokens || !std::isfinite(temp) || temp < 0.0f)
    return SPEC_ERR_INVALID_ARG;
  // the fused path keeps a top-k list per row: the argmax (temperature 0), or top-k sampling
  if (!greedy && (top_k < 1 || top_k > sv::kLmKMax || top_k >= V)) return SPEC_ERR_UNSUPPORTED;
  if (d % sv::kLmBK != 0 || V > SPEC_MAX_VOCAB || !aligned16(target_hidden) ||
      !aligned16(target_weight) || (!greedy && (!aligned16(draft_hidden) || !aligned16(draft_weight))))
    return SPEC_ERR_UNSUPPORTED;
  const int k = greedy ? 1 : top_k;
  const long long rows_t = (long long)B * (K + 1), rows_d = greedy ? 0 : (long long)B * K;
  if (rows_t + rows_d > 0x7fffffffLL) return SPEC_ERR_UNSUPPORTED;
  const int cap = sv::kLmMergeCap / k;
  const LmLayout wl = lm_layout(rows_t + rows_d, k, cap);
  if (!workspace || !aligned16(workspace) ||
      workspace_bytes < spec_lmhead_workspace_size(B, K, V, d, top_k))
    return SPEC_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  int32_t* dev_status = reinterpret_cast<int32_t*>(ws);
  float* part_val = reinterpret_cast<float*>(ws + wl.part_val);
  int32_t* part_id = reinterpret_cast<int32_t*>(ws + wl.part_id);
  sv::LmRow* lrows = reinterpret_cast<sv::LmRow*>(ws + wl.rows);
  float* kept_val = reinterpret_cast<float*>(ws + wl.kept_val);
  int32_t* kept_id = reinterpret_cast<int32_t*>(ws + wl.kept_id);
  if (cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s) != cudaSuccess) return SPEC_ERR_CUDA;
  cudaError_t e = cudaSuccess;
  const int G = sm_count(&e);
  if (e != cudaSuccess || G < 1) return SPEC_ERR_CUDA;

  // target rows, then draft rows: per-chunk lists, then the exact top-k of each row
  Split st, sd;
  e = run_product(target_hidden, target_weight, int(rows_t), V, d, k, G, part_val, part_id, cap,
                  logits_out, dev_status, s, &st);
  if (e != cudaSuccess) return e == cudaErrorInvalidValue ? SPEC_ERR_INVALID_ARG : SPEC_ERR_CUDA;
  sv::LmMergeJob mj = {part_val, part_id, int(rows_t), st.nchunk, k, temp, lrows, kept_val,
                       kept_id};
  sv::lmhead_merge_kernel<<<unsigned(rows_t), kThreads, 0, s>>>(mj);
  if (cudaGetLastError() != cudaSuccess) return SPEC_ERR_CUDA;
  if (!greedy) {
    const size_t po = size_t(rows_t) * st.nchunk * k;
    e = run_product(draft_hidden, draft_weight, int(rows_d), V, d, k, G, part_val + po,
                    part_id + po, cap,
                    logits_out ? logits_out + size_t(rows_t) * V : nullptr, dev_status, s, &sd);
    if (e != cudaSuccess) return e == cudaErrorInvalidValue ? SPEC_ERR_INVALID_ARG : SPEC_ERR_CUDA;
    sv::LmMergeJob md = {part_val + po, part_id + po, int(rows_d), sd.nchunk, k, temp,
                         lrows + rows_t, kept_val + size_t(rows_t) * k,
                         kept_id + size_t(rows_t) * k};
    sv::lmhead_merge_kernel<<<unsigned(rows_d), kThreads, 0, s>>>(md);
    if (cudaGetLastError() != cudaSuccess) return SPEC_ERR_CUDA;
  }
  sv::LmChainJob cj = {B, K, k, lrows, kept_val, kept_id, draft_tokens, uniforms, temp, V,
                       accepted_len, out_tokens};
  sv::lmhead_chain_kernel<<<B, kThreads, 0, s>>>(cj);
  return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ERR_CUDA;
}

}  // extern "C"
