// Deterministic inverse-CDF draw over one vocabulary row (one thread block).
//
// The draw returns the smallest token id v (ascending) with res[v] > 0 whose
// cumulative mass C_v exceeds w * S, S the total; if rounding leaves none, the largest
// v with res[v] > 0. Masses are fixed point (42 fraction bits), so every partial sum
// is exact and the result does not depend on how the sum is split across threads.
// The row is read in chunks of kThreads * m groups of 8 entries (m groups per thread,
// m = 1 unless the row has more than kMaxDrawChunks such chunks). The first pass records
// each warp's share of each chunk's mass with no block barrier; one barrier later the
// chunk totals locate the chunk that holds the crossing, and only that chunk is read
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
  unsigned long long wchunk[kMaxDrawChunks][kWarps];   // per-warp mass of each chunk
  int ids[kSparseCap];
  unsigned long long scr[kWarps];
  unsigned long long total;
  unsigned long long sel_before;
  int sel_chunk;
  int fallback;
  int best;
};

// f(v0, r) fills r[0..7] with the fixed-point masses of entries v0..v0+7 (0 past V).
// Returns -1 when the whole row has zero mass.
template <typename F>
__device__ int inverse_cdf_draw(F&& f, int V, float w, DrawSmem& sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = (V + 7) / 8;
  const int m = max(1, (G + kThreads * kMaxDrawChunks - 1) / (kThreads * kMaxDrawChunks));
  const int CG = kThreads * m;  // groups per chunk
  const int nch = (G + CG - 1) / CG;
  for (int ch = 0; ch < nch; ++ch) {
    unsigned long long t = 0;
    for (int i = 0; i < m; ++i) {
      const int g = ch * CG + i * kThreads + int(threadIdx.x);  // coalesced within a warp
      if (g < G) {
        unsigned long long r[8];
        f(g * 8, r);
#pragma unroll
        for (int k = 0; k < 8; ++k) t += r[k];
      }
    }
    t = warp_sum_u64(t);
    if (lane == 0) sm.wchunk[ch][warp] = t;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long S = 0;
    for (int ch = 0; ch < nch; ++ch)
      for (int ww = 0; ww < kWarps; ++ww) S += sm.wchunk[ch][ww];
    const double target = double(w) * double(S);
    unsigned long long cum = 0, sel_before = 0, last_before = 0;
    int sel = -1, last = -1;
    for (int ch = 0; ch < nch; ++ch) {
      unsigned long long c = 0;
      for (int ww = 0; ww < kWarps; ++ww) c += sm.wchunk[ch][ww];
      if (c > 0) {
        last = ch;
        last_before = cum;
        if (sel < 0 && double(cum + c) > target) {
          sel = ch;
          sel_before = cum;
        }
      }
      cum += c;
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
  const double target = double(w) * double(sm.total);
  // the chunk again, in token order: thread t takes groups t, t + kThreads, ... of it;
  // group j of the chunk is entry range [8 (sel * CG + j), +8)
  unsigned long long rr[8];
  unsigned long long own = 0;  // this thread's mass, in the order that scans below expect
  // order within the chunk: i-major (i * kThreads + t), so a scan per i keeps token order
  unsigned long long before = sm.sel_before;
  for (int i = 0; i < m; ++i) {
    const int g = sel * CG + i * kThreads + int(threadIdx.x);
    if (g < G) {
      f(g * 8, rr);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) rr[k] = 0ull;
    }
    own = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) own += rr[k];
    unsigned long long total;
    unsigned long long cum = before + block_exclusive_scan<unsigned long long>(own, sm.scr, &total);
    if (sm.fallback) {
      int lst = -1;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (rr[k] > 0) lst = g * 8 + k;
      if (lst >= 0) atomicMax(&sm.best, lst);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        cum += rr[k];
        if (rr[k] > 0 && double(cum) > target) {
          atomicMin(&sm.best, g * 8 + k);
          break;
        }
      }
    }
    before += total;
  }
  __syncthreads();
  const int tok = sm.best;
  __syncthreads();
  return tok;
}

// The same draw when every entry outside ids[0..n) (distinct ids, any order, n <= kThreads)
// has mass 0: the support is sorted by id and one block-wide prefix sum replaces the pass
// over the row. mass(v) gives the fixed-point mass of entry v; the result is identical
// to inverse_cdf_draw over the whole row with the same masses.
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
  const unsigned long long r = t < n ? mass(v) : 0ull;
  unsigned long long S;
  const unsigned long long ex = block_exclusive_scan<unsigned long long>(r, sm.scr, &S);
  const double target = double(w) * double(S);
  if (r > 0 && double(ex + r) > target) atomicMin(&sm.best, v);
  __syncthreads();
  int tok = sm.best;
  if (S == 0) {
    tok = -1;
  } else if (tok == INT_MAX) {  // rounding left none: the largest id with mass
    __syncthreads();
    if (t == 0) sm.best = -1;
    __syncthreads();
    if (r > 0) atomicMax(&sm.best, v);
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

// Probability of entry v under the transformed distribution described by s.
template <typename T>
__device__ __forceinline__ float prob(const RowStats& s, float l, int v) {
  return kept(Elem<T>::key(l), v, s.thr_key, s.cutoff) ? weight(l, s.c, s.mc) / s.z : 0.0f;
}

}  // namespace sv
