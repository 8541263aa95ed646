// libspecverify C ABI: argument checks, workspace layout and kernel launches.
// The operations and their sources are documented in include/specverify.h.
#include <atomic>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include "chain.cuh"
#include "lstate.cuh"
#include "probs.cuh"
#include "refine.cuh"
#include "row_stats.cuh"
#include "specverify.h"
#include "stream.cuh"
#include "tree.cuh"
#include "tree_sample.cuh"

namespace {

using sv::kThreads;

// Cluster kernel (spec_logits_to_probs, the exact finisher of listed rows, top-k above
// the streaming limit): a slice of a logit row per CTA; each CTA keeps sv::kNBuf slices in
// flight, and two CTAs share an SM, so one CTA's computation overlaps the other's copies
// and its own next rows' copies.
#ifndef SV_SLICE_KB
#define SV_SLICE_KB 40
#endif
constexpr size_t kSliceTargetBytes = SV_SLICE_KB * 1024;
constexpr size_t kMaxDynSmem = 227 * 1024 - sizeof(sv::RowAux) - 1024;
constexpr size_t kStatsOffset = 256;  // the device status word lives at offset 0

std::atomic<void*> g_ev_before{nullptr};
std::atomic<void*> g_ev_after{nullptr};

struct RowPlan {
  int C;             // CTAs per cluster (one cluster per row at a time)
  int slice;         // elements per CTA
  int slice_bytes;   // bytes per slice buffer
  size_t dyn;        // dynamic shared memory per CTA (the ring of slice buffers)
};

bool plan_rows(int V, int elem_bytes, RowPlan* pl) {
  int C = 1;
  while (C < sv::kMaxCluster && size_t((V + C - 1) / C) * elem_bytes > kSliceTargetBytes) C *= 2;
  const int slice = ((V + C - 1) / C + 15) / 16 * 16;
  const int slice_bytes = int((size_t(slice) * elem_bytes + 16 + 127) / 128 * 128);
  const size_t dyn = size_t(slice_bytes) * sv::kNBuf;
  if (dyn > kMaxDynSmem) return false;
  *pl = RowPlan{C, slice, slice_bytes, dyn};
  return true;
}

// Lets the row kernel take any ring size this build plans (per function and device; the
// largest value, so a later, smaller launch can never lower it below a cached shape).
template <typename T>
cudaError_t allow_row_kernel_smem() {
  auto k = sv::row_stats_kernel<T>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(kMaxDynSmem));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

// Clusters of the row kernel that fit on the device at once (cached per device and shape).
template <typename T>
int resident_clusters(const RowPlan& pl, cudaError_t* err) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, size_t>, int> cache;
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return 0;
  const auto key = std::make_tuple(dev, pl.C, pl.dyn);
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  auto k = sv::row_stats_kernel<T>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(pl.C), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = pl.dyn;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = unsigned(pl.C);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  *err = cudaOccupancyMaxActiveClusters(&n, k, &cfg);
  if (*err != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  cache[key] = n;
  return n;
}

template <typename T>
cudaError_t launch_row_stats(const sv::RowJob& job, const RowPlan& pl, cudaStream_t s) {
  auto k = sv::row_stats_kernel<T>;
  cudaError_t e = allow_row_kernel_smem<T>();
  if (e != cudaSuccess) return e;
  const int clusters = resident_clusters<T>(pl, &e);
  if (e != cudaSuccess) return e;
  if (clusters < 1) return cudaErrorInvalidConfiguration;
  const long long G = job.rows < clusters ? job.rows : clusters;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(G * pl.C), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = pl.dyn;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = unsigned(pl.C);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, job);
}

cudaError_t launch_row_stats_dt(spec_dtype dt, const sv::RowJob& job, const RowPlan& pl,
                                cudaStream_t s) {
  return dt == SPEC_BF16 ? launch_row_stats<__nv_bfloat16>(job, pl, s)
                         : launch_row_stats<float>(job, pl, s);
}

// ------------------------------------------------------------------ streaming kernel
int stream_mode(const sv::RowJob& rj) {
  if (rj.flags & sv::RS_GREEDY) return sv::SM_GREEDY;
  if (rj.top_k >= 1 && rj.top_k < rj.V) return sv::SM_TOPK;
  if (rj.top_p < 1.0f) return sv::SM_TOPP;
  return sv::SM_SUMS;
}

template <typename T, int M>
struct StreamKernel {
  // Resident CTAs (cached per device): the kernel is persistent.
  static int grid(cudaError_t* err) {
    static std::mutex mu;
    static std::map<int, int> cache;
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return 0;
    {
      std::lock_guard<std::mutex> lock(mu);
      auto it = cache.find(dev);
      if (it != cache.end()) return it->second;
    }
    auto k = sv::stream_rows_kernel<T, M>;
    const size_t dyn = sv::stream_dyn_bytes(M);
    *err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(dyn));
    if (*err != cudaSuccess) return 0;
    int per_sm = 0, sms = 0;
    *err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, sv::kStreamThreads, dyn);
    if (*err == cudaSuccess)
      *err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (*err != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    cache[dev] = per_sm * sms;
    return per_sm * sms;
  }

  static cudaError_t launch(const sv::StreamJob& job, cudaStream_t s) {
    cudaError_t e = cudaSuccess;
    const int g = grid(&e);
    if (e != cudaSuccess) return e;
    if (g < 1) return cudaErrorInvalidConfiguration;
    auto k = sv::stream_rows_kernel<T, M>;
    const size_t dyn = sv::stream_dyn_bytes(M);
    // set on every launch: the attribute is per device, the cache is not
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(dyn));
    if (e != cudaSuccess) return e;
    const long long n = job.r.rows < g ? job.r.rows : g;
    k<<<unsigned(n), sv::kStreamThreads, dyn, s>>>(job);
    return cudaGetLastError();
  }
};

template <typename T>
cudaError_t launch_stream(const sv::StreamJob& job, int mode, cudaStream_t s) {
  switch (mode) {
    case sv::SM_GREEDY: return StreamKernel<T, sv::SM_GREEDY>::launch(job, s);
    case sv::SM_SUMS: return StreamKernel<T, sv::SM_SUMS>::launch(job, s);
    case sv::SM_TOPK: return StreamKernel<T, sv::SM_TOPK>::launch(job, s);
    default: return StreamKernel<T, sv::SM_TOPP>::launch(job, s);
  }
}

// The top-p refinement. bfloat16 rows: the exact normalisers (eight blocks per SM over the
// (row, slice) items), then one block per listed row (one per SM, each walking the list).
// float32 rows: one block per SM, each walking the listed rows.
template <typename T>
cudaError_t launch_refine(const sv::RefineJob& j, cudaStream_t s) {
  static std::mutex mu;
  static std::map<int, int> sms_of;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int sms = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = sms_of.find(dev);
    if (it != sms_of.end()) sms = it->second;
  }
  if (sms == 0) {
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    sms_of[dev] = sms;
  }
  const long long g = j.r.rows < sms ? j.r.rows : sms;
  if constexpr (sizeof(T) == 2) {
    const long long items = j.r.rows * sv::kZSlices;
    const long long gz = items < 8LL * sms ? items : 8LL * sms;
    sv::topp_zexact_kernel<T><<<unsigned(gz), kThreads, 0, s>>>(j);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    sv::topp_finalize_kernel<T><<<unsigned(g), sv::kFinThreads, 0, s>>>(j);
    return cudaGetLastError();
  } else {
    const size_t dyn = sv::refine_smem<T>();
    e = cudaFuncSetAttribute(sv::topp_refine_kernel<T>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(dyn));
    if (e != cudaSuccess) return e;
    sv::topp_refine_kernel<T><<<unsigned(g), kThreads, dyn, s>>>(j);
    return cudaGetLastError();
  }
}

// Row statistics for a verify call. The streaming kernel settles the rows it can; in the
// candidate modes it lists the rest, which the cluster kernel then finishes exactly. A
// top-k above the candidate path's limit goes to the cluster kernel for every row. Pure
// top-p rows whose boundary was placed with fp32 masses too close to call (and every top-p
// row the cluster kernel settled) then get it placed again in double precision
// (refine_rows, when given).
cudaError_t row_stage(spec_dtype dt, sv::RowJob rj, const RowPlan& pl, int32_t* fb_rows,
                      int32_t* fb_count, int32_t* refine_rows, int32_t* refine_count,
                      unsigned long long* refine_z, int32_t* unresolved, cudaStream_t s) {
  const bool refine = refine_rows && rj.top_p < 1.0f && rj.top_k == 0 &&
                      !(rj.flags & sv::RS_GREEDY);
  rj.refine_rows = refine ? refine_rows : nullptr;
  rj.refine_count = refine ? refine_count : nullptr;
  rj.refine_z = refine ? refine_z : nullptr;
  const int mode = stream_mode(rj);
  sv::RefineJob rf = {};
  rf.r = rj;
  rf.rows = refine_rows;
  rf.count = refine_count;
  rf.unresolved = unresolved;
  // top-k above the candidate path's limit, and float32 top-p rows: the cluster kernel
  // settles every row (then the refinement, for top-p)
  if ((mode == sv::SM_TOPK && rj.top_k > sv::kStreamMaxTopK) ||
      (mode == sv::SM_TOPP && dt != SPEC_BF16)) {
    cudaError_t e = launch_row_stats_dt(dt, rj, pl, s);
    if (e != cudaSuccess || !refine) return e;
    return dt == SPEC_BF16 ? launch_refine<__nv_bfloat16>(rf, s) : launch_refine<float>(rf, s);
  }
  const int E = dt == SPEC_BF16 ? 2 : 4;
  sv::StreamJob sj = {};
  sj.r = rj;
  sj.chunk = sv::stream_chunk_bytes(mode) / E;
  sj.nchunk = (rj.V + sj.chunk - 1) / sj.chunk;
  sj.topp_span = rj.top_p < 1.0f
                     ? float(std::log(double(rj.V) / (1.0 - double(rj.top_p))) / rj.inv_t)
                     : 0.0f;
  sj.fb_rows = fb_rows;
  sj.fb_count = fb_count;
  cudaError_t e = dt == SPEC_BF16 ? launch_stream<__nv_bfloat16>(sj, mode, s)
                                  : launch_stream<float>(sj, mode, s);
  if (e != cudaSuccess || (mode != sv::SM_TOPK && mode != sv::SM_TOPP)) return e;
  sv::RowJob fj = rj;
  fj.row_list = fb_rows;
  fj.row_count = fb_count;
  e = launch_row_stats_dt(dt, fj, pl, s);
  if (e != cudaSuccess || !refine) return e;
  return dt == SPEC_BF16 ? launch_refine<__nv_bfloat16>(rf, s) : launch_refine<float>(rf, s);
}

int elem_bytes(spec_dtype dt) { return dt == SPEC_BF16 ? 2 : 4; }

bool dtype_ok(int dt) { return dt == SPEC_F32 || dt == SPEC_BF16; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Workspace: [header | RowStats per row | kept-id count per row | kept ids per row |
// fallback row list | refinement row list | exact normalisers of refined rows (Fx128)].
// Header words (int32): 0 the device status,
// 1 the fallback count, 2 the tree row-list count, 3 the refinement count, 4 rows left
// unrefined; the rest of the 256 bytes is unused.
struct WsLayout {
  size_t stats, kept_n, kept_ids, fb_rows, refine_rows, refine_z, total;
};
constexpr int kHeaderWords = 5;

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

WsLayout ws_layout(long long rows) {
  WsLayout w;
  w.stats = kStatsOffset;
  w.kept_n = w.stats + up256(size_t(rows) * sizeof(sv::RowStats));
  w.kept_ids = w.kept_n + up256(size_t(rows) * sizeof(int32_t));
  w.fb_rows = w.kept_ids + up256(size_t(rows) * sv::kKeptCap * sizeof(int32_t));
  w.refine_rows = w.fb_rows + up256(size_t(rows) * sizeof(int32_t));
  w.refine_z = w.refine_rows + up256(size_t(rows) * sizeof(int32_t));
  w.total = w.refine_z + up256(size_t(rows) * 2 * sizeof(unsigned long long));
  return w;
}

size_t stats_bytes(long long rows) { return ws_layout(rows).total; }

bool rows_fit(long long rows, int) { return rows <= 0x7fffffffLL; }

spec_status check_launch(cudaError_t e) { return e == cudaSuccess ? SPEC_OK : SPEC_ERR_CUDA; }

// Tree verification, typical or greedy acceptance (the two public calls below).
spec_status verify_tree(const void* target_logits, spec_dtype dtype, int B, int N, int V,
                        const int32_t* node_tokens, const int32_t* parent_idx, float eps,
                        float delta, bool greedy, int32_t* best_path, int path_cap,
                        int32_t* accepted_len, int32_t* next_token, void* workspace,
                        size_t workspace_bytes, void* stream) {
  if (!target_logits || !dtype_ok(dtype) || B <= 0 || N <= 0 || V <= 0 || !node_tokens ||
      !parent_idx || !best_path || path_cap <= 0 || !accepted_len ||
      (!greedy && (!std::isfinite(eps) || !std::isfinite(delta))))
    return SPEC_ERR_INVALID_ARG;
  if (V > SPEC_MAX_VOCAB || N > SPEC_MAX_TREE_NODES) return SPEC_ERR_UNSUPPORTED;
  const long long rows = (long long)B * N;
  if (!workspace || !aligned16(workspace) || workspace_bytes < stats_bytes(rows))
    return SPEC_ERR_WORKSPACE;
  RowPlan pl;
  if (!plan_rows(V, elem_bytes(dtype), &pl) || !rows_fit(rows, pl.C)) return SPEC_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* dev_status = static_cast<int32_t*>(workspace);
  const WsLayout wl = ws_layout(rows);  // the kept-id area (unused by trees) holds the row map
  char* ws = static_cast<char*>(workspace);
  sv::RowStats* stats = reinterpret_cast<sv::RowStats*>(ws + wl.stats);
  if (cudaMemsetAsync(dev_status, 0, kHeaderWords * sizeof(int32_t), s) != cudaSuccess)
    return SPEC_ERR_CUDA;

  sv::RowJob rj = {};
  rj.base0 = target_logits;
  rj.base1 = target_logits;
  rj.rows0 = rows;
  rj.rows = rows;
  rj.V = V;
  rj.slice = pl.slice;
  rj.slice_bytes = pl.slice_bytes;
  rj.c = greedy ? 0.0f : sv::kLog2e;
  rj.inv_t = greedy ? 0.0f : 1.0f;
  rj.temp = 1.0f;
  rj.top_k = 0;
  rj.top_p = 1.0f;
  rj.flags = greedy ? sv::RS_GREEDY : sv::RS_ENTROPY;
  rj.stats = stats;
  rj.dev_status = dev_status;
  if (!greedy) {
    // typical acceptance reads only the rows of nodes with a child (greedy also reads the
    // deepest accepted node's own row, which may be a leaf): list them on the device
    int32_t* map = reinterpret_cast<int32_t*>(ws + wl.kept_ids);
    int32_t* count = dev_status + 2;
    sv::tree_parent_rows_kernel<<<1, kThreads, 0, s>>>(parent_idx, N, B, map, count);
    if (cudaGetLastError() != cudaSuccess) return SPEC_ERR_CUDA;
    rj.row_list = map;
    rj.row_count = count;
  }
  void* evb = g_ev_before.load();
  void* eva = g_ev_after.load();
  if (evb) cudaEventRecord(static_cast<cudaEvent_t>(evb), s);
  if (row_stage(dtype, rj, pl, reinterpret_cast<int32_t*>(ws + wl.fb_rows), dev_status + 1,
                nullptr, nullptr, nullptr, nullptr, s) != cudaSuccess)
    return SPEC_ERR_CUDA;
  if (eva) cudaEventRecord(static_cast<cudaEvent_t>(eva), s);

  sv::TreeJob tj = {};
  tj.target = target_logits;
  tj.B = B;
  tj.N = N;
  tj.V = V;
  tj.tokens = node_tokens;
  tj.parent = parent_idx;
  tj.eps = eps;
  tj.delta = delta;
  tj.stats = stats;
  tj.best_path = best_path;
  tj.path_cap = path_cap;
  tj.accepted_len = accepted_len;
  tj.greedy = greedy ? 1 : 0;
  tj.next_token = next_token;
  const size_t dyn = size_t(N) * (4 + 4 + 1 + 1) + 16;
  if (dtype == SPEC_BF16)
    sv::tree_finish_kernel<__nv_bfloat16><<<B, kThreads, dyn, s>>>(tj);
  else
    sv::tree_finish_kernel<float><<<B, kThreads, dyn, s>>>(tj);
  return check_launch(cudaGetLastError());
}

template <int R>
cudaError_t launch_commit(const sv::LsCommitJob& j, cudaStream_t s) {
  const size_t dyn = sv::lstate_commit_smem(j.S, 16 * R);
  cudaError_t e = cudaFuncSetAttribute(sv::lstate_commit_kernel<R>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(dyn));
  if (e != cudaSuccess) return e;
  const long long blocks = (long long)j.B * j.H * j.tiles;
  sv::lstate_commit_kernel<R><<<unsigned(blocks), kThreads, dyn, s>>>(j);
  return cudaGetLastError();
}
}  // namespace

extern "C" {

const char* spec_status_string(int status) {
  switch (status) {
    case SPEC_OK: return "SPEC_OK";
    case SPEC_ERR_INVALID_ARG: return "SPEC_ERR_INVALID_ARG";
    case SPEC_ERR_UNSUPPORTED: return "SPEC_ERR_UNSUPPORTED";
    case SPEC_ERR_CUDA: return "SPEC_ERR_CUDA";
    case SPEC_ERR_WORKSPACE: return "SPEC_ERR_WORKSPACE";
    case SPEC_ERR_DEVICE_TIMEOUT: return "SPEC_ERR_DEVICE_TIMEOUT";
    default: return "unknown spec_status";
  }
}

size_t spec_workspace_size(int B, int K_or_N, int V) {
  if (B <= 0 || K_or_N <= 0 || V <= 0) return 0;
  return stats_bytes((long long)B * (2LL * K_or_N + 1));
}

spec_status spec_verify_chain(const void* target_logits, const void* draft_logits,
                              spec_dtype dtype, int B, int K, int V,
                              const int32_t* draft_tokens, const float* uniforms, float temp,
                              int top_k, float top_p, int32_t* accepted_len,
                              int32_t* out_tokens, void* workspace, size_t workspace_bytes,
                              void* stream) {
  const bool greedy = temp == 0.0f;
  if (!target_logits || (!greedy && !draft_logits) || !dtype_ok(dtype) || B <= 0 || K <= 0 ||
      V <= 0 || !draft_tokens || !uniforms || !accepted_len || !out_tokens ||
      !std::isfinite(temp) || temp < 0.0f || !(top_p > 0.0f))
    return SPEC_ERR_INVALID_ARG;
  if (V > SPEC_MAX_VOCAB) return SPEC_ERR_UNSUPPORTED;
  const long long rows = (long long)B * (greedy ? K + 1 : 2LL * K + 1);
  if (!workspace || !aligned16(workspace) || workspace_bytes < stats_bytes(rows))
    return SPEC_ERR_WORKSPACE;
  RowPlan pl;
  if (!plan_rows(V, elem_bytes(dtype), &pl) || !rows_fit(rows, pl.C) || B > 0x7fffffff)
    return SPEC_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* dev_status = static_cast<int32_t*>(workspace);
  const WsLayout wl = ws_layout(rows);
  char* ws = static_cast<char*>(workspace);
  sv::RowStats* stats = reinterpret_cast<sv::RowStats*>(ws + wl.stats);
  if (cudaMemsetAsync(dev_status, 0, kHeaderWords * sizeof(int32_t), s) != cudaSuccess)
    return SPEC_ERR_CUDA;

  sv::RowJob rj = {};
  rj.kept_n = reinterpret_cast<int32_t*>(ws + wl.kept_n);
  rj.kept_ids = reinterpret_cast<int32_t*>(ws + wl.kept_ids);
  rj.base0 = target_logits;
  rj.base1 = draft_logits;
  rj.rows0 = (long long)B * (K + 1);
  rj.rows = rows;
  rj.V = V;
  rj.slice = pl.slice;
  rj.slice_bytes = pl.slice_bytes;
  rj.c = greedy ? 0.0f : sv::kLog2e / temp;
  rj.inv_t = greedy ? 0.0f : 1.0f / temp;
  rj.temp = temp;
  rj.top_k = (top_k >= 1 && top_k < V) ? top_k : 0;
  rj.top_p = top_p < 1.0f ? top_p : 1.0f;
  rj.flags = greedy ? sv::RS_GREEDY : 0;
  rj.stats = stats;
  rj.dev_status = dev_status;
  void* evb = g_ev_before.load();
  void* eva = g_ev_after.load();
  if (evb) cudaEventRecord(static_cast<cudaEvent_t>(evb), s);
  if (row_stage(dtype, rj, pl, reinterpret_cast<int32_t*>(ws + wl.fb_rows), dev_status + 1,
                reinterpret_cast<int32_t*>(ws + wl.refine_rows), dev_status + 3,
                reinterpret_cast<unsigned long long*>(ws + wl.refine_z), dev_status + 4,
                s) != cudaSuccess)
    return SPEC_ERR_CUDA;
  if (eva) cudaEventRecord(static_cast<cudaEvent_t>(eva), s);

  sv::ChainJob cj = {};
  cj.target = target_logits;
  cj.draft = draft_logits;
  cj.B = B;
  cj.K = K;
  cj.V = V;
  cj.tokens = draft_tokens;
  cj.uniforms = uniforms;
  cj.stats = stats;
  cj.kept_n = rj.kept_n;
  cj.kept_ids = rj.kept_ids;
  cj.greedy = greedy ? 1 : 0;
  cj.temp = temp;
  if (!greedy && rj.top_k == 0 && rj.top_p >= 1.0f) {
    // untruncated rows: the streaming kernel's fp32 normaliser sums, per consumer thread,
    // n = ceil(V / kThreads) weights in order (at most n roundings of 2^-24), each from ex2
    // (relative error < 2^-22.7) of an exponent whose roundings shift it by at most
    // 2^-24 (|l| + |m|) c (the |m| part is added per row by the finisher; the mean of
    // |l - m| c under the row's own distribution is at most log2 V), and rescales the sum
    // by ex2 at most once per 16-byte vector, n / 4 times (2^-22 each)
    const double n = double((V + kThreads - 1) / kThreads);
    cj.zguard = float(std::ldexp(n + std::log2(double(V)) + 16.0, -24) +
                      std::ldexp(n / 4.0 + 8.0, -22));
  }
  cj.accepted_len = accepted_len;
  cj.out_tokens = out_tokens;
  if (dtype == SPEC_BF16)
    sv::chain_finish_kernel<__nv_bfloat16><<<B, kThreads, 0, s>>>(cj);
  else
    sv::chain_finish_kernel<float><<<B, kThreads, 0, s>>>(cj);
  return check_launch(cudaGetLastError());
}

spec_status spec_verify_tree_typical(const void* target_logits, spec_dtype dtype, int B, int N,
                                     int V, const int32_t* node_tokens,
                                     const int32_t* parent_idx, float eps, float delta,
                                     int32_t* best_path, int path_cap, int32_t* accepted_len,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  return verify_tree(target_logits, dtype, B, N, V, node_tokens, parent_idx, eps, delta, false,
                     best_path, path_cap, accepted_len, nullptr, workspace, workspace_bytes,
                     stream);
}

spec_status spec_verify_tree_greedy(const void* target_logits, spec_dtype dtype, int B, int N,
                                    int V, const int32_t* node_tokens, const int32_t* parent_idx,
                                    int32_t* best_path, int path_cap, int32_t* accepted_len,
                                    int32_t* next_token, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  return verify_tree(target_logits, dtype, B, N, V, node_tokens, parent_idx, 0.0f, 0.0f, true,
                     best_path, path_cap, accepted_len, next_token, workspace, workspace_bytes,
                     stream);
}

spec_status spec_verify_tree_sampling(const void* target_logits, const void* draft_logits,
                                      spec_dtype dtype, int B, int N, int V,
                                      const int32_t* node_tokens, const int32_t* parent_idx,
                                      const float* uniforms, float temp, int top_k, float top_p,
                                      int32_t* best_path, int path_cap, int32_t* accepted_len,
                                      int32_t* next_token, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  const bool greedy = temp == 0.0f;
  if (!target_logits || (!greedy && !draft_logits) || !dtype_ok(dtype) || B <= 0 || N <= 0 ||
      V <= 0 || !node_tokens || !parent_idx || !uniforms || !best_path || path_cap <= 0 ||
      !accepted_len || !std::isfinite(temp) || temp < 0.0f || !(top_p > 0.0f))
    return SPEC_ERR_INVALID_ARG;
  if (V > SPEC_MAX_VOCAB || N > SPEC_MAX_TREE_NODES) return SPEC_ERR_UNSUPPORTED;
  const long long rows = (long long)B * N * (greedy ? 1 : 2);
  if (!workspace || !aligned16(workspace) || workspace_bytes < stats_bytes(rows))
    return SPEC_ERR_WORKSPACE;
  RowPlan pl;
  if (!plan_rows(V, elem_bytes(dtype), &pl) || !rows_fit(rows, pl.C) || B > 0x7fffffff)
    return SPEC_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* dev_status = static_cast<int32_t*>(workspace);
  const WsLayout wl = ws_layout(rows);
  char* ws = static_cast<char*>(workspace);
  sv::RowStats* stats = reinterpret_cast<sv::RowStats*>(ws + wl.stats);
  if (cudaMemsetAsync(dev_status, 0, kHeaderWords * sizeof(int32_t), s) != cudaSuccess)
    return SPEC_ERR_CUDA;

  sv::RowJob rj = {};
  rj.kept_n = reinterpret_cast<int32_t*>(ws + wl.kept_n);
  rj.kept_ids = reinterpret_cast<int32_t*>(ws + wl.kept_ids);
  rj.base0 = target_logits;
  rj.base1 = draft_logits;
  rj.rows0 = (long long)B * N;
  rj.rows = rows;
  rj.V = V;
  rj.slice = pl.slice;
  rj.slice_bytes = pl.slice_bytes;
  rj.c = greedy ? 0.0f : sv::kLog2e / temp;
  rj.inv_t = greedy ? 0.0f : 1.0f / temp;
  rj.temp = temp;
  rj.top_k = (top_k >= 1 && top_k < V) ? top_k : 0;
  rj.top_p = top_p < 1.0f ? top_p : 1.0f;
  rj.flags = greedy ? sv::RS_GREEDY : 0;
  rj.stats = stats;
  rj.dev_status = dev_status;
  void* evb = g_ev_before.load();
  void* eva = g_ev_after.load();
  if (evb) cudaEventRecord(static_cast<cudaEvent_t>(evb), s);
  if (row_stage(dtype, rj, pl, reinterpret_cast<int32_t*>(ws + wl.fb_rows), dev_status + 1,
                reinterpret_cast<int32_t*>(ws + wl.refine_rows), dev_status + 3,
                reinterpret_cast<unsigned long long*>(ws + wl.refine_z), dev_status + 4,
                s) != cudaSuccess)
    return SPEC_ERR_CUDA;
  if (eva) cudaEventRecord(static_cast<cudaEvent_t>(eva), s);

  sv::TreeSampleJob tj = {};
  tj.target = target_logits;
  tj.draft = draft_logits;
  tj.B = B;
  tj.N = N;
  tj.V = V;
  tj.tokens = node_tokens;
  tj.parent = parent_idx;
  tj.uniforms = uniforms;
  tj.stats = stats;
  tj.kept_n = rj.kept_n;
  tj.kept_ids = rj.kept_ids;
  tj.greedy = greedy ? 1 : 0;
  tj.temp = temp;
  tj.best_path = best_path;
  tj.path_cap = path_cap;
  tj.accepted_len = accepted_len;
  tj.next_token = next_token;
  const size_t dyn = size_t(N) * 20 + 16;  // normalisers (double), child lists, path
  cudaError_t e;
  if (dtype == SPEC_BF16) {
    e = cudaFuncSetAttribute(sv::tree_sample_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(dyn));
    if (e == cudaSuccess) sv::tree_sample_kernel<__nv_bfloat16><<<B, kThreads, dyn, s>>>(tj);
  } else {
    e = cudaFuncSetAttribute(sv::tree_sample_kernel<float>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(dyn));
    if (e == cudaSuccess) sv::tree_sample_kernel<float><<<B, kThreads, dyn, s>>>(tj);
  }
  if (e != cudaSuccess) return SPEC_ERR_CUDA;
  return check_launch(cudaGetLastError());
}

spec_status spec_logits_to_probs(const void* logits, spec_dtype dtype, int rows, int V,
                                 float temp, int top_k, float top_p, float* probs,
                                 float* entropy, void* stream) {
  if (!logits || !dtype_ok(dtype) || rows <= 0 || V <= 0 || !probs || !std::isfinite(temp) ||
      temp < 0.0f || !(top_p > 0.0f))
    return SPEC_ERR_INVALID_ARG;
  if (V > SPEC_MAX_VOCAB) return SPEC_ERR_UNSUPPORTED;
  RowPlan pl;
  if (!plan_rows(V, elem_bytes(dtype), &pl) || !rows_fit(rows, pl.C)) return SPEC_ERR_UNSUPPORTED;
  const bool greedy = temp == 0.0f;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  sv::RowJob rj = {};
  rj.base0 = logits;
  rj.base1 = logits;
  rj.rows0 = rows;
  rj.rows = rows;
  rj.V = V;
  rj.slice = pl.slice;
  rj.slice_bytes = pl.slice_bytes;
  rj.c = greedy ? 0.0f : sv::kLog2e / temp;
  rj.inv_t = greedy ? 0.0f : 1.0f / temp;
  rj.temp = temp;
  rj.top_k = (top_k >= 1 && top_k < V) ? top_k : 0;
  rj.top_p = top_p < 1.0f ? top_p : 1.0f;
  rj.dev_status = nullptr;
  // bfloat16 rows: the row statistics by the streaming kernel (with its exact finisher and
  // the exact top-p placement), kept in the probability buffer itself (its first `head` rows),
  // then the probabilities in three launches: the rows past the head (their statistics are not
  // overwritten meanwhile), the head rows but for row 0's first segment (which holds the head
  // rows' statistics: kStatsOffset + head * sizeof(RowStats) bytes at most), and that segment
  const long long R = rows;
  const size_t o_stats = kStatsOffset;
  const size_t o_fb = o_stats + up256(size_t(R) * sizeof(sv::RowStats));
  const size_t o_ref = o_fb + up256(size_t(R) * sizeof(int32_t));
  const size_t o_refz = o_ref + up256(size_t(R) * sizeof(int32_t));
  const size_t scratch = o_refz + up256(size_t(R) * 2 * sizeof(unsigned long long));
  const long long head = (long long)((scratch + size_t(V) * 4 - 1) / (size_t(V) * 4));
  const size_t seg0_bytes = size_t(V < sv::kProbsSeg ? V : sv::kProbsSeg) * 4;
  const bool streamed = dtype == SPEC_BF16 && !greedy && V % 8 == 0 && V >= 2048 &&
                        aligned16(logits) && aligned16(probs) &&
                        scratch <= size_t(R) * V * 4 &&
                        o_stats + size_t(head) * sizeof(sv::RowStats) <= seg0_bytes;
  if (!streamed) {
    rj.flags = sv::RS_WRITE_PROBS | (greedy ? sv::RS_GREEDY : 0) |
               ((entropy && !greedy) ? sv::RS_ENTROPY : 0);
    rj.stats = nullptr;
    rj.probs = probs;
    rj.entropy = entropy;
    return check_launch(launch_row_stats_dt(dtype, rj, pl, s));
  }
  char* ws = reinterpret_cast<char*>(probs);
  int32_t* hdr = reinterpret_cast<int32_t*>(ws);
  if (cudaMemsetAsync(hdr, 0, kHeaderWords * sizeof(int32_t), s) != cudaSuccess)
    return SPEC_ERR_CUDA;
  rj.flags = entropy ? sv::RS_ENTROPY : 0;
  rj.stats = reinterpret_cast<sv::RowStats*>(ws + o_stats);
  rj.dev_status = hdr;
  if (row_stage(dtype, rj, pl, reinterpret_cast<int32_t*>(ws + o_fb), hdr + 1,
                reinterpret_cast<int32_t*>(ws + o_ref), hdr + 3,
                reinterpret_cast<unsigned long long*>(ws + o_refz), hdr + 4, s) != cudaSuccess)
    return SPEC_ERR_CUDA;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return SPEC_ERR_CUDA;
  const int seg = (V + sv::kProbsSeg - 1) / sv::kProbsSeg;
  sv::ProbsJob pj = {logits, rj.stats, probs, entropy, head, R, -1, V};
  for (int part = 0; part < 2; ++part) {
    const long long n = pj.r_end - pj.r_begin;
    if (n > 0) {
      // about 16 blocks per SM in all, 65,535 row groups at most
      long long gy = (16LL * sms + seg - 1) / seg;
      gy = gy < n ? gy : n;
      gy = gy < 65535 ? gy : 65535;
      sv::probs_write_kernel<<<dim3(unsigned(seg), unsigned(gy)), kThreads, 0, s>>>(pj);
      if (cudaGetLastError() != cudaSuccess) return SPEC_ERR_CUDA;
    }
    pj.r_begin = 0;
    pj.r_end = head < R ? head : R;
    pj.skip_row = 0;
  }
  sv::probs_write_first_kernel<<<1, kThreads, 0, s>>>(pj);
  return check_launch(cudaGetLastError());
}

spec_status spec_residual_sample(const float* p, const float* q, int rows, int V,
                                 const float* uniforms, int32_t* tokens, void* stream) {
  if (!p || rows <= 0 || V <= 0 || !uniforms || !tokens) return SPEC_ERR_INVALID_ARG;
  if (V > SPEC_MAX_VOCAB) return SPEC_ERR_UNSUPPORTED;
  sv::ResidualJob j = {p, q, rows, V, uniforms, tokens};
  sv::residual_sample_kernel<<<rows, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(j);
  return check_launch(cudaGetLastError());
}

spec_status spec_linear_state_factors(const float* alpha, const float* beta, const float* keys,
                                      const float* values, int B, int H, int S, int dk, int dv,
                                      float* w, float* u, float* gamma, void* stream) {
  if (!alpha || !beta || !keys || !values || !w || !u || !gamma || B <= 0 || H <= 0 || S <= 0 ||
      dk <= 0 || dv <= 0)
    return SPEC_ERR_INVALID_ARG;
  if (S > sv::kLsMaxSteps || dk > sv::kLsMaxDk || (long long)B * H > 0x7fffffffLL)
    return SPEC_ERR_UNSUPPORTED;
  sv::LsFactorJob j = {alpha, beta, keys, values, B, H, S, dk, dv, w, u, gamma};
  const size_t dyn = sv::lstate_factors_smem(S, dk);
  if (cudaFuncSetAttribute(sv::lstate_factors_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(dyn)) != cudaSuccess)
    return SPEC_ERR_CUDA;
  sv::lstate_factors_kernel<<<unsigned(B * H), kThreads, dyn,
                              static_cast<cudaStream_t>(stream)>>>(j);
  return check_launch(cudaGetLastError());
}

spec_status spec_commit_linear_state(float* state, int B, int H, int dk, int dv, int S,
                                     const float* keys, const float* w, const float* u,
                                     const float* gamma, const int32_t* steps, void* stream) {
  if (!state || !keys || !w || !u || !gamma || !steps || B <= 0 || H <= 0 || S <= 0 || dk <= 0 ||
      dv <= 0)
    return SPEC_ERR_INVALID_ARG;
  if (S > sv::kLsMaxSteps || dv % 4 != 0 || !aligned16(state) || !aligned16(keys) ||
      !aligned16(w) || !aligned16(u) ||
      (dk != 32 && dk != 64 && dk != 128 && dk != 256))
    return SPEC_ERR_UNSUPPORTED;
  const long long blocks = (long long)B * H * ((dv + sv::kLsCols - 1) / sv::kLsCols);
  if (blocks > 0x7fffffffLL) return SPEC_ERR_UNSUPPORTED;
  sv::LsCommitJob j = {state, B, H, S, dk, dv, keys, w, u, gamma, steps,
                       (dv + sv::kLsCols - 1) / sv::kLsCols};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  switch (dk) {
    case 32: e = launch_commit<2>(j, s); break;
    case 64: e = launch_commit<4>(j, s); break;
    case 128: e = launch_commit<8>(j, s); break;
    default: e = launch_commit<16>(j, s); break;
  }
  return check_launch(e);
}

spec_status spec_get_device_status(const void* workspace, int32_t* status_out, void* stream) {
  if (!workspace || !status_out) return SPEC_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t h = 0;
  if (cudaMemcpyAsync(&h, workspace, sizeof h, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return SPEC_ERR_CUDA;
  *status_out = h ? SPEC_ERR_DEVICE_TIMEOUT : SPEC_OK;
  return SPEC_OK;
}

void spec_set_row_kernel_events(void* before, void* after) {
  g_ev_before.store(before);
  g_ev_after.store(after);
}

int spec_kernels_per_call(const char* entry_point) {
  if (!entry_point) return -1;
  if (!std::strcmp(entry_point, "spec_verify_chain")) return 4;
  if (!std::strcmp(entry_point, "spec_verify_tree_typical")) return 3;
  if (!std::strcmp(entry_point, "spec_verify_tree_greedy")) return 2;
  if (!std::strcmp(entry_point, "spec_verify_tree_sampling")) return 4;
  if (!std::strcmp(entry_point, "spec_logits_to_probs")) return 1;
  if (!std::strcmp(entry_point, "spec_residual_sample")) return 1;
  if (!std::strcmp(entry_point, "spec_linear_state_factors")) return 1;
  if (!std::strcmp(entry_point, "spec_commit_linear_state")) return 1;
  return -1;
}

}  // extern "C"
