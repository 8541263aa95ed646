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
// entropy[row] from the statistics. A row is cut into segments of kProbsSeg entries; block
// (x, y) of the grid writes segment x of rows r_begin + y, r_begin + y + gridDim.y, ... Each
// thread loads its kProbsVecs 16-byte vectors of bfloat16 logits (8 entries each, kThreads
// vectors apart) before it computes and stores any, so that several loads are in flight.
// V % 8 == 0, rows 16-byte aligned.
constexpr int kProbsVecs = 4;
constexpr int kProbsSeg = 8 * kProbsVecs * kThreads;  // 8,192 entries
struct ProbsJob {
  const void* logits;       // [rows][V] bfloat16
  const RowStats* stats;    // [rows]
  float* probs;             // [rows][V]
  float* entropy;           // [rows] or NULL
  long long r_begin, r_end;
  long long skip_row;       // the row whose first segment the launch leaves out, or -1
  int V;
};

__device__ __forceinline__ void probs_write_seg(const ProbsJob& j, const RowStats& s,
                                                long long row, int v_base) {
  const __nv_bfloat16* lg = static_cast<const __nv_bfloat16*>(j.logits) + size_t(row) * j.V;
  float* out = j.probs + size_t(row) * j.V;
  uint4 w[kProbsVecs];
#pragma unroll
  for (int u = 0; u < kProbsVecs; ++u) {
    const int v0 = v_base + u * 8 * kThreads;
    w[u] = v0 < j.V ? __ldg(reinterpret_cast<const uint4*>(lg + v0)) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int u = 0; u < kProbsVecs; ++u) {
    const int v0 = v_base + u * 8 * kThreads;
    if (v0 >= j.V) continue;
    float x[8], o[8];
    Elem<__nv_bfloat16>::unpack(w[u], x);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (s.status != ROW_OK)
        o[k] = NAN;
      else
        o[k] = kept(Elem<__nv_bfloat16>::key(x[k]), v0 + k, s.thr_key, s.cutoff)
                   ? weight(x[k], s.c, s.mc) / s.z
                   : 0.0f;
    }
    float4* o4 = reinterpret_cast<float4*>(out + v0);
    o4[0] = make_float4(o[0], o[1], o[2], o[3]);
    o4[1] = make_float4(o[4], o[5], o[6], o[7]);
  }
}

// Rows [r_begin, r_end) but the first segment of skip_row; no block may overwrite the
// statistics of a row it writes.
__global__ void __launch_bounds__(kThreads) probs_write_kernel(const ProbsJob j) {
  const int v_base = int(blockIdx.x) * kProbsSeg + 8 * int(threadIdx.x);
  for (long long row = j.r_begin + blockIdx.y; row < j.r_end; row += gridDim.y) {
    if (row == j.skip_row && blockIdx.x == 0) continue;
    const RowStats s = j.stats[row];
    probs_write_seg(j, s, row, v_base);
    if (j.entropy && blockIdx.x == 0 && threadIdx.x == 0)
      j.entropy[row] = s.status != ROW_OK ? NAN : s.entropy;
  }
}

// The first segment of row 0, which holds the statistics of the first rows: one block reads
// row 0's statistics before it overwrites them.
__global__ void __launch_bounds__(kThreads) probs_write_first_kernel(const ProbsJob j) {
  const RowStats s = j.stats[0];
  __syncthreads();
  probs_write_seg(j, s, 0, 8 * int(threadIdx.x));
  if (j.entropy && threadIdx.x == 0) j.entropy[0] = s.status != ROW_OK ? NAN : s.entropy;
}

}  // namespace sv
