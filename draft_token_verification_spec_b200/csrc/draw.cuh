// Deterministic inverse-CDF draw over one vocabulary row (one thread block), and the
// double-precision view of a transformed row that the sampling decisions use.
//
// The draw returns the smallest token id v (ascending) with res[v] > 0 whose
// cumulative mass C_v exceeds w * S, S the total; if rounding leaves none, the largest
// v with res[v] > 0. Masses are doubles held as 128-bit fixed point (Fx128), so every
// partial sum is exact and the result does not depend on how the sum is split across
// threads. The row is read in chunks of kThreads * m groups of 8 entries (m groups per
// thread, m = 1 unless the row has more than kMaxDrawChunks such chunks). The first pass
// records each warp's share of each chunk's mass with no block barrier; one barrier later
// the chunk totals locate the chunk that holds the crossing, and only that chunk is read
// again. This is the resampling step of "Speculative Decoding" / "Speculative Sampling"
// (spec-decoding-i notes) with the reading that the draw walks token ids in ascending
// order.
#pragma once

#include <climits>

#include "common.cuh"

namespace sv {

constexpr int kMaxDrawChunks = 128;
constexpr int kSparseCap = kThreads;                    // support of a sparse draw

struct DrawSmem {
  Fx128 wchunk[kMaxDrawChunks][kWarps];   // per-warp mass of each chunk
  int ids[kSparseCap];
  Fx128 scr[kWarps];
  Fx128 total;
  Fx128 sel_before;
  int sel_chunk;
  int fallback;
  int best;
};

// f(v0, r) fills r[0..7] with the masses of entries v0..v0+7 (0 past V).
// Returns -1 when the whole row has zero mass.
template <typename F>
__device__ int inverse_cdf_draw(F&& f, int V, float w, DrawSmem& sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = (V + 7) / 8;
  const int m = max(1, (G + kThreads * kMaxDrawChunks - 1) / (kThreads * kMaxDrawChunks));
  const int CG = kThreads * m;  // groups per chunk
  const int nch = (G + CG - 1) / CG;
  for (int ch = 0; ch < nch; ++ch) {
    Fx128 t = fx_zero();
    for (int i = 0; i < m; ++i) {
      const int g = ch * CG + i * kThreads + int(threadIdx.x);  // coalesced within a warp
      if (g < G) {
        Fx128 r[8];
        f(g * 8, r);
#pragma unroll
        for (int k = 0; k < 8; ++k) t = fx_add(t, r[k]);
      }
    }
    t = warp_sum_fx(t);
    if (lane == 0) sm.wchunk[ch][warp] = t;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    Fx128 S = fx_zero();
    for (int ch = 0; ch < nch; ++ch)
      for (int ww = 0; ww < kWarps; ++ww) S = fx_add(S, sm.wchunk[ch][ww]);
    const double target = double(w) * fx_to_double(S);
    Fx128 cum = fx_zero(), sel_before = fx_zero(), last_before = fx_zero();
    int sel = -1, last = -1;
    for (int ch = 0; ch < nch; ++ch) {
      Fx128 c = fx_zero();
      for (int ww = 0; ww < kWarps; ++ww) c = fx_add(c, sm.wchunk[ch][ww]);
      if (!fx_is_zero(c)) {
        last = ch;
        last_before = cum;
        if (sel < 0 && fx_to_double(fx_add(cum, c)) > target) {
          sel = ch;
          sel_before = cum;
        }
      }
      cum = fx_add(cum, c);
    }
    sm.fallback = sel < 0;
    if (sel < 0) {
      sel = last;
      sel_before = last_before;
    }
    sm.sel_chunk = sel;
    sm.sel_before = sel_before;
    sm.total = S;
    sm.best = sm.fallback ? -1 : INT_MAX;
  }
  __syncthreads();
  const int sel = sm.sel_chunk;
  if (sel < 0) {
    __syncthreads();
    return -1;
  }
  const double target = double(w) * fx_to_double(sm.total);
  // the chunk again, in token order: thread t takes groups t, t + kThreads, ... of it;
  // group j of the chunk is entry range [8 (sel * CG + j), +8)
  Fx128 rr[8];
  Fx128 before = sm.sel_before;
  const bool fallback = sm.fallback;
  for (int i = 0; i < m; ++i) {
    const int g = sel * CG + i * kThreads + int(threadIdx.x);
    if (g < G) {
      f(g * 8, rr);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) rr[k] = fx_zero();
    }
    Fx128 own = fx_zero();
#pragma unroll
    for (int k = 0; k < 8; ++k) own = fx_add(own, rr[k]);
    Fx128 total;
    Fx128 cum = fx_add(before, block_exclusive_scan_fx(own, sm.scr, &total));
    if (fallback) {
      int lst = -1;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (!fx_is_zero(rr[k])) lst = g * 8 + k;
      if (lst >= 0) atomicMax(&sm.best, lst);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        cum = fx_add(cum, rr[k]);
        if (!fx_is_zero(rr[k]) && fx_to_double(cum) > target) {
          atomicMin(&sm.best, g * 8 + k);
          break;
        }
      }
    }
    before = fx_add(before, total);
  }
  __syncthreads();
  const int tok = sm.best;
  __syncthreads();
  return tok;
}

// The same draw when every entry outside ids[0..n) (distinct ids, any order, n <= kThreads)
// has mass 0: the support is sorted by id and one block-wide prefix sum replaces the pass
// over the row. mass(v) gives the Fx128 mass of entry v; the result is identical to
// inverse_cdf_draw over the whole row with the same masses.
template <typename F>
__device__ int sparse_draw(const int32_t* ids, int n, F&& mass, float w, DrawSmem& sm) {
  const int t = threadIdx.x;
  const int my = t < n ? ids[t] : INT_MAX;
  if (t < n) sm.ids[t] = my;
  if (t == 0) sm.best = INT_MAX;
  __syncthreads();
  int rank = 0;
  if (t < n)
    for (int j = 0; j < n; ++j) rank += sm.ids[j] < my ? 1 : 0;
  __syncthreads();
  if (t < n) sm.ids[rank] = my;
  __syncthreads();
  const int v = t < n ? sm.ids[t] : -1;
  const Fx128 r = t < n ? mass(v) : fx_zero();
  Fx128 S;
  const Fx128 ex = block_exclusive_scan_fx(r, sm.scr, &S);
  const double target = double(w) * fx_to_double(S);
  if (!fx_is_zero(r) && fx_to_double(fx_add(ex, r)) > target) atomicMin(&sm.best, v);
  __syncthreads();
  int tok = sm.best;
  if (fx_is_zero(S)) {
    tok = -1;
  } else if (tok == INT_MAX) {  // rounding left none: the largest id with mass
    __syncthreads();
    if (t == 0) sm.best = -1;
    __syncthreads();
    if (!fx_is_zero(r)) atomicMax(&sm.best, v);
    __syncthreads();
    tok = sm.best;
  }
  __syncthreads();
  return tok;
}

// Loads entries v0..v0+7 of a logit row as floats (-inf past V): 16-byte vector loads
// when the row is 16-byte aligned and the 8 entries are inside it.
template <typename T>
__device__ __forceinline__ void load8(const T* row, int v0, int V, bool aligned, float* x) {
  if (aligned && v0 + 8 <= V) {
    constexpr int P = Elem<T>::kPerVec;
    const uint4* p = reinterpret_cast<const uint4*>(row + v0);
#pragma unroll
    for (int q = 0; q < 8 / P; ++q) Elem<T>::unpack(__ldg(p + q), x + q * P);
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) x[k] = (v0 + k < V) ? Elem<T>::load(row, size_t(v0 + k)) : -INFINITY;
  }
}

// Probability of entry v under the transformed distribution described by s (fp32).
template <typename T>
__device__ __forceinline__ float prob(const RowStats& s, float l, int v) {
  return kept(Elem<T>::key(l), v, s.thr_key, s.cutoff) ? weight(l, s.c, s.mc) / s.z : 0.0f;
}

// ------------------------------------------------------------------ double-precision view
// Unnormalised weight exp((l - m) / T) of a kept entry, in double (l - m is exact).
__device__ __forceinline__ double weight_d(float l, float m, double T) {
  return exp((double(l) - double(m)) / T);
}

// Weight of entry v of the row described by s (0 outside the kept set).
template <typename T>
__device__ __forceinline__ double kept_weight_d(const RowStats& s, double Tt, float l, int v) {
  return kept(Elem<T>::key(l), v, s.thr_key, s.cutoff) ? weight_d(l, s.m, Tt) : 0.0;
}

// Probability of entry v in double: kept weight / zd.
template <typename T>
__device__ __forceinline__ double prob_d(const RowStats& s, double zd, double Tt, float l, int v) {
  return kept_weight_d<T>(s, Tt, l, v) / zd;
}

// The double normaliser of one row (every thread of the block calls it, gets the sum):
// s.zd when the row statistics hold it, else the sum over the kept set, by a pass over the
// row with exact Fx128 accumulation.
template <typename T>
__device__ double row_zd(const RowStats& s, const T* row, int V, double Tt, Fx128* scr) {
  if (s.zd >= 0.0) return s.zd;
  const bool al = (reinterpret_cast<uintptr_t>(row) & 15u) == 0;
  Fx128 acc = fx_zero();
  for (int v0 = int(threadIdx.x) * 8; v0 < V; v0 += kThreads * 8) {
    float x[8];
    load8<T>(row, v0, V, al, x);
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (v0 + k < V) acc = fx_add(acc, fx_from(kept_weight_d<T>(s, Tt, x[k], v0 + k)));
  }
  return fx_to_double(block_sum_fx(acc, scr));
}

}  // namespace sv
