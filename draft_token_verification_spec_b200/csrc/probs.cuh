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

}  // namespace sv
