// Linear-attention state commit after verification (the SpecLA summary, gist.science: a
// linear-attention model keeps one dense state per head that every token updates; after the
// verdict the state is brought to the accepted prefix from small per-step "factors" saved
// during verification, instead of replaying the accepted tokens).
//
// The state of one sequence and head, S in R^{dk x dv}, follows the gated delta rule
//   S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T.
// With G_t = alpha_1 ... alpha_t and the WY vectors
//   w_t = beta_t (k_t - sum_{s<t} (k_t . k_s) w_s)                 (length dk)
//   u_t = beta_t (v_t / G_t - sum_{s<t} (k_t . k_s) u_s)           (length dv)
// every prefix of a steps has the closed form
//   S_a = G_a (S_0 + sum_{t<=a} k_t (u_t - S_0^T w_t)^T),
// because prod_{t=a..1} (I - beta_t k_t k_t^T) = I - sum_{t<=a} k_t w_t^T and the rescaled
// state S_t / G_t follows the same rule with values v_t / G_t. The vectors of step t depend
// only on steps <= t, so one set of factors serves every acceptance length.
//
//   lstate_factors_kernel: one block per (sequence, head); the Gram products k_t . k_s, the
//     gates G_t, then w_t and u_t by forward substitution over the steps, one column per
//     thread (the earlier steps of a column stay in shared memory).
//   lstate_commit_kernel: one block per (sequence, head, 64-column tile of S); the tile stays
//     in registers: M = U_a - W_a S_0 (a x 64; partial sums per thread over its rows, then
//     over the warp's two row groups and the eight warps), then S_a = G_a (S_0 + K_a^T M),
//     written back in place. A
//     sequence committing 0 steps (or an invalid length) is not touched. Bandwidth-bound:
//     one read and one write of the state per committed sequence.
#pragma once

#include "common.cuh"

namespace sv {

constexpr int kLsMaxSteps = 32;   // steps per round (drafts + the deferred token)
constexpr int kLsMaxDk = 256;
constexpr int kLsCols = 64;       // columns of S per commit block

struct LsFactorJob {
  const float* alpha;   // [B][H][S]
  const float* beta;    // [B][H][S]
  const float* keys;    // [B][H][S][dk]
  const float* values;  // [B][H][S][dv]
  int B, H, S, dk, dv;
  float* w;             // [B][H][S][dk]
  float* u;             // [B][H][S][dv]
  float* gamma;         // [B][H][S]: G_t for t = 1..S
};

// Dynamic shared memory of a factor block: the keys [S][dk] (overwritten in place by w, each
// thread's own entries), the Gram products [S][S], and the u values of the thread's current
// column [S][kThreads].
__host__ __device__ constexpr size_t lstate_factors_smem(int S, int dk) {
  return (size_t(S) * dk + size_t(S) * S + size_t(S) * kThreads) * 4;
}

__global__ void __launch_bounds__(kThreads) lstate_factors_kernel(const LsFactorJob j) {
  extern __shared__ __align__(16) float fsm[];
  __shared__ float g[kLsMaxSteps], gi[kLsMaxSteps], bs[kLsMaxSteps];
  const int bh = blockIdx.x, S = j.S, dk = j.dk, dv = j.dv;
  float* kk = fsm;                          // [S][dk]: k_t, overwritten in place by w_t
  float* gram = kk + size_t(S) * dk;        // [S][S]: k_t . k_s for s < t
  float* us = gram + size_t(S) * S;         // [S][kThreads]: v_t, overwritten by u_t
  // the keys, gates and step weights are loaded before anything is stored, and the values of
  // a column all at once before its substitution (the outputs may not be assumed apart from
  // the inputs, so a load placed after a store could not be moved ahead of it)
  const float* kin = j.keys + size_t(bh) * S * dk;
  for (int i = threadIdx.x; i < S * dk; i += kThreads) kk[i] = kin[i];
  if (threadIdx.x < S) {
    g[threadIdx.x] = j.alpha[size_t(bh) * S + threadIdx.x];
    bs[threadIdx.x] = j.beta[size_t(bh) * S + threadIdx.x];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float acc = 1.0f;
    for (int t = 0; t < S; ++t) {
      acc *= g[t];
      g[t] = acc;
      gi[t] = 1.0f / acc;
      j.gamma[size_t(bh) * S + t] = acc;
    }
  }
  // Gram products k_t . k_s (s < t), one warp per pair
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int p = warp; p < S * S; p += kWarps) {
    const int t = p / S, s = p % S;
    if (s >= t) continue;
    float acc = 0.0f;
    for (int i = lane; i < dk; i += 32) acc += kk[t * dk + i] * kk[s * dk + i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) gram[t * S + s] = acc;
  }
  __syncthreads();
  float* wout = j.w + size_t(bh) * S * dk;
  float* uout = j.u + size_t(bh) * S * dv;
  const float* vin = j.values + size_t(bh) * S * dv;
  // w_t and u_t by forward substitution over the steps, one column per thread: the earlier
  // steps of a column are the thread's own shared-memory entries
  for (int i = threadIdx.x; i < dk; i += kThreads) {
    for (int t = 0; t < S; ++t) {
      float x = kk[t * dk + i];
#pragma unroll 8
      for (int s = 0; s < t; ++s) x -= gram[t * S + s] * kk[s * dk + i];
      x = bs[t] * x;
      kk[t * dk + i] = x;
      wout[t * dk + i] = x;
    }
  }
  for (int i0 = 0; i0 < dv; i0 += kThreads) {
    const int i = i0 + int(threadIdx.x);
    if (i < dv) {
      for (int t = 0; t < S; ++t) us[t * kThreads + threadIdx.x] = vin[t * dv + i];
      for (int t = 0; t < S; ++t) {
        float x = us[t * kThreads + threadIdx.x] * gi[t];
#pragma unroll 8
        for (int s = 0; s < t; ++s) x -= gram[t * S + s] * us[s * kThreads + threadIdx.x];
        x = bs[t] * x;
        us[t * kThreads + threadIdx.x] = x;
        uout[t * dv + i] = x;
      }
    }
  }
}

struct LsCommitJob {
  float* state;         // [B][H][dk][dv], updated in place
  int B, H, S, dk, dv;
  const float* keys;    // [B][H][S][dk]
  const float* w;       // [B][H][S][dk]
  const float* u;       // [B][H][S][dv]
  const float* gamma;   // [B][H][S]
  const int32_t* steps; // [B]: steps to commit (0..S; anything else leaves the state)
  int tiles;            // column tiles per head: ceil(dv / kLsCols)
};

// Thread layout of a commit block: 16 column quads (64 columns) x 16 row groups; the thread
// with quad q = tid % 16 and row group g = tid / 16 holds rows g, g + 16, ..., g + 16 (R - 1)
// (dk = 16 R) of columns 4q .. 4q + 3 of the tile. A warp's load or store of one of its rows
// then covers two whole 256-byte row segments of the tile.
// Dynamic shared memory: keys and w of S steps (S x dk each), M (S x kLsCols), and the warps'
// partial sums of M (S x kWarps x kLsCols).
__host__ __device__ constexpr size_t lstate_commit_smem(int S, int dk) {
  return size_t(S) * dk * 8 + size_t(S) * kLsCols * 4 + size_t(S) * kWarps * kLsCols * 4;
}

// 16-byte global -> shared copy that bypasses the registers (and L1).
__device__ __forceinline__ void ls_copy16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}

template <int R>
__global__ void __launch_bounds__(kThreads) lstate_commit_kernel(const LsCommitJob j) {
  extern __shared__ __align__(16) float lsm[];
  constexpr int dk = 16 * R;
  float* ks = lsm;                                            // [S][dk]
  float* ws = ks + size_t(j.S) * dk;                          // [S][dk]
  float (*mt)[kLsCols] = reinterpret_cast<float (*)[kLsCols]>(ws + size_t(j.S) * dk);
  float4* red = reinterpret_cast<float4*>(ws + size_t(j.S) * dk + size_t(j.S) * kLsCols);
  // red[(t * kWarps + warp) * 16 + q]: warp's partial sum of M[t][4q .. 4q + 3]
  const long long blk = blockIdx.x;
  const int tile = int(blk % j.tiles);
  const long long bh = blk / j.tiles;
  const int b = int(bh / j.H);
  const int a = j.steps[b];
  if (a <= 0 || a > j.S) return;  // nothing to commit (uniform)
  const int S = j.S, dv = j.dv;
  const int c0 = tile * kLsCols;
  // every load is issued before any is waited for: the factors go to shared memory by
  // asynchronous copies (keys and w of the first a steps, and this tile's columns of u; a
  // tile past dv reads zeros), and the state tile goes to registers meanwhile
  {
    const float4* kin = reinterpret_cast<const float4*>(j.keys + size_t(bh) * S * dk);
    const float4* win = reinterpret_cast<const float4*>(j.w + size_t(bh) * S * dk);
    for (int i = threadIdx.x; i < a * dk / 4; i += kThreads) {
      ls_copy16(ks + 4 * i, kin + i);
      ls_copy16(ws + 4 * i, win + i);
    }
    const float* urow = j.u + size_t(bh) * S * dv;
    for (int i = threadIdx.x; i < a * (kLsCols / 4); i += kThreads) {
      const int t = i / (kLsCols / 4), c = 4 * (i % (kLsCols / 4));
      if (c0 + c < dv)
        ls_copy16(&mt[t][c], urow + size_t(t) * dv + c0 + c);
      else
        *reinterpret_cast<float4*>(&mt[t][c]) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  const float ga = j.gamma[size_t(bh) * S + a - 1];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int q = threadIdx.x & 15;                    // column quad: columns 4q .. 4q + 3
  const int rg = threadIdx.x >> 4;                   // row group: rows rg, rg + 16, ...
  const int col = c0 + 4 * q;
  const bool live = col < dv;                        // dv % 4 == 0: a quad is all in or out
  float* base = j.state + size_t(bh) * dk * dv;
  float4 x[R];
#pragma unroll
  for (int r = 0; r < R; ++r)
    x[r] = live ? *reinterpret_cast<const float4*>(base + size_t(rg + 16 * r) * dv + col)
                : make_float4(0.f, 0.f, 0.f, 0.f);
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  // M[t][c] = U[t][c] - sum_i W[t][i] S[i][c]: partial sums over this thread's rows, the two
  // row groups of the warp (lanes l and l ^ 16), then the warps' sums in warp order
  for (int t = 0; t < a; ++t) {
    float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float wv = ws[t * dk + rg + 16 * r];
      p.x = fmaf(wv, x[r].x, p.x);
      p.y = fmaf(wv, x[r].y, p.y);
      p.z = fmaf(wv, x[r].z, p.z);
      p.w = fmaf(wv, x[r].w, p.w);
    }
    p.x += __shfl_xor_sync(0xffffffffu, p.x, 16);
    p.y += __shfl_xor_sync(0xffffffffu, p.y, 16);
    p.z += __shfl_xor_sync(0xffffffffu, p.z, 16);
    p.w += __shfl_xor_sync(0xffffffffu, p.w, 16);
    if (lane < 16) red[(t * kWarps + warp) * 16 + q] = p;
  }
  __syncthreads();
  for (int o = threadIdx.x; o < a * 16; o += kThreads) {
    const int t = o >> 4, qq = o & 15;
    float4 sum = red[(t * kWarps) * 16 + qq];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) {
      const float4 v = red[(t * kWarps + w) * 16 + qq];
      sum.x += v.x;
      sum.y += v.y;
      sum.z += v.z;
      sum.w += v.w;
    }
    float4* m = reinterpret_cast<float4*>(&mt[t][4 * qq]);
    const float4 u4 = *m;
    *m = make_float4(u4.x - sum.x, u4.y - sum.y, u4.z - sum.z, u4.w - sum.w);
  }
  __syncthreads();
  // S_a = G_a (S_0 + K^T M)
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float4 y = x[r];
    for (int t = 0; t < a; ++t) {
      const float kv = ks[t * dk + rg + 16 * r];
      const float4 m = *reinterpret_cast<const float4*>(&mt[t][4 * q]);
      y.x = fmaf(kv, m.x, y.x);
      y.y = fmaf(kv, m.y, y.y);
      y.z = fmaf(kv, m.z, y.z);
      y.w = fmaf(kv, m.w, y.w);
    }
    y.x *= ga;
    y.y *= ga;
    y.z *= ga;
    y.w *= ga;
    if (live) *reinterpret_cast<float4*>(base + size_t(rg + 16 * r) * dv + col) = y;
  }
}

}  // namespace sv
