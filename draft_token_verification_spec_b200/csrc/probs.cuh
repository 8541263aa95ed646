// Inverse-CDF draw from explicit probability rows: norm(max(0, p - q)), or p when q
// is absent or the residual is empty ("Speculative Sampling", spec-decoding-i notes).
// One thread block per row; the same deterministic draw as chain verification, on the
// exact double differences of the float inputs.
#pragma once

#include "draw.cuh"

namespace sv {

struct ResidualJob {
  const float* p;          // [rows][V]
  const float* q;          // [rows][V] or NULL
  int rows, V;
  const float* uniforms;   // [rows]
  int32_t* tokens;         // [rows]
};

__global__ void __launch_bounds__(kThreads) residual_sample_kernel(const ResidualJob j) {
  __shared__ DrawSmem sm;
  const int row = blockIdx.x, V = j.V;
  const float* pr = j.p + size_t(row) * V;
  const float* qr = j.q ? j.q + size_t(row) * V : nullptr;
  int bad = 0, pos = 0;
  for (int v = threadIdx.x; v < V; v += kThreads) {
    const float a = pr[v];
    if (!(a >= 0.0f && a <= 1.0f)) bad = 1;
    if (a > 0.0f) pos = 1;
    if (qr) {
      const float c = qr[v];
      if (!(c >= 0.0f && c <= 1.0f)) bad = 1;
    }
  }
  bad = __syncthreads_or(bad);
  pos = __syncthreads_or(pos);
  if (bad || !pos) {
    if (threadIdx.x == 0) j.tokens[row] = -1;
    return;
  }
  const float w = j.uniforms[row];
  int tok = -1;
  if (qr) {
    tok = inverse_cdf_draw(
        [&](int v0, Fx128* r) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int v = v0 + k;
            r[k] = (v < V) ? fx_from(fmax(double(pr[v]) - double(qr[v]), 0.0)) : fx_zero();
          }
        },
        V, w, sm);
  }
  if (tok < 0) {
    tok = inverse_cdf_draw(
        [&](int v0, Fx128* r) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int v = v0 + k;
            r[k] = (v < V) ? fx_from(double(pr[v])) : fx_zero();
          }
        },
        V, w, sm);
  }
  if (threadIdx.x == 0) j.tokens[row] = tok;
}

// Probability rows from row statistics (spec_logits_to_probs after the streaming kernel):
// p(v) = kept(v) ? exp2(l_v c - mc) / z : 0, NaN for rows whose statistics are not valid;
// entropy[row] from the statistics. Work items are (row, segment of kProbsSeg entries),
// numbered row * seg + segment; each thread takes 8 consecutive entries (one 16-byte load of
// bfloat16 logits, two 16-byte stores). V % 8 == 0, rows 16-byte aligned.
constexpr int kProbsSeg = 8 * kThreads;
struct ProbsJob {
  const void* logits;       // [rows][V] bfloat16
  const RowStats* stats;    // [rows]
  float* probs;             // [rows][V]
  float* entropy;           // [rows] or NULL
  long long item_begin, item_end;
  int V, seg;               // seg = ceil(V / kProbsSeg)
};

__device__ __forceinline__ void probs_write8(const ProbsJob& j, const RowStats& s, long long row,
                                             int v0) {
  const uint4 w = __ldg(reinterpret_cast<const uint4*>(
      static_cast<const __nv_bfloat16*>(j.logits) + size_t(row) * j.V + v0));
  float x[8], o[8];
  Elem<__nv_bfloat16>::unpack(w, x);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    if (s.status != ROW_OK)
      o[k] = NAN;
    else
      o[k] = kept(Elem<__nv_bfloat16>::key(x[k]), v0 + k, s.thr_key, s.cutoff)
                 ? weight(x[k], s.c, s.mc) / s.z
                 : 0.0f;
  }
  float4* out = reinterpret_cast<float4*>(j.probs + size_t(row) * j.V + v0);
  out[0] = make_float4(o[0], o[1], o[2], o[3]);
  out[1] = make_float4(o[4], o[5], o[6], o[7]);
}

// Items [item_begin, item_end); none of them may overwrite the statistics of its own rows.
__global__ void __launch_bounds__(kThreads) probs_write_kernel(const ProbsJob j) {
  for (long long it = j.item_begin + blockIdx.x; it < j.item_end; it += gridDim.x) {
    const long long row = it / j.seg;
    const int v0 = int(it - row * j.seg) * kProbsSeg + 8 * int(threadIdx.x);
    const RowStats s = j.stats[row];
    if (v0 < j.V) probs_write8(j, s, row, v0);
    if (j.entropy && v0 == 0) j.entropy[row] = s.status != ROW_OK ? NAN : s.entropy;
  }
}

// Item 0 (the first segment of row 0, which holds the statistics of the first rows): one
// block reads row 0's statistics before it overwrites them.
__global__ void __launch_bounds__(kThreads) probs_write_first_kernel(const ProbsJob j) {
  const RowStats s = j.stats[0];
  __syncthreads();
  const int v0 = 8 * int(threadIdx.x);
  if (v0 < j.V) probs_write8(j, s, 0, v0);
  if (j.entropy && threadIdx.x == 0) j.entropy[0] = s.status != ROW_OK ? NAN : s.entropy;
}

}  // namespace sv
