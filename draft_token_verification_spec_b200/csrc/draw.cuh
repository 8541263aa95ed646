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
constexpr int kSparsePer = 8;                           // support entries per thread
constexpr int kSparseCap = kSparsePer * kThreads;       // support of a sparse draw

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

// Ids below this many are sorted through a bitmap in the draw's chunk table (16 KB).
constexpr int kBitmapIds = kMaxDrawChunks * kWarps * 16 * 8;

// The same draw when every entry outside ids[0..n) (distinct ids, any order,
// n <= kPer * kThreads) has mass 0: the support is sorted by id and one block-wide prefix
// sum replaces the pass over the row, thread t holding sorted positions [kPer t, kPer (t + 1)).
// The sort: long lists of ids below V <= kBitmapIds set bits in a bitmap that the block then
// reads in order; other lists count for each id the smaller ones. mass(v) gives the Fx128
// mass of entry v; the result is identical to inverse_cdf_draw over the whole row with the
// same masses.
template <int kPer, typename F>
__device__ int sparse_draw_n(const int32_t* ids, int n, F&& mass, float w, DrawSmem& sm,
                             int V) {
  const int t = threadIdx.x;
  int my[kPer];
  const bool bitmap = n > 128 && V > 0 && V <= kBitmapIds;  // (uniform)
  uint32_t* bm = reinterpret_cast<uint32_t*>(&sm.wchunk[0][0]);
  const int nw = (V + 31) >> 5;
  if (bitmap)
    for (int i = t; i < nw; i += kThreads) bm[i] = 0u;
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    const int i = q * kThreads + t;
    my[q] = i < n ? ids[i] : INT_MAX;
    if (i < n && !bitmap) sm.ids[i] = my[q];
  }
  if (t == 0) sm.best = INT_MAX;
  __syncthreads();
  if (bitmap) {
#pragma unroll
    for (int q = 0; q < kPer; ++q)
      if (q * kThreads + t < n) atomicOr(&bm[my[q] >> 5], 1u << (my[q] & 31));
    __syncthreads();
    // thread t reads words [t per, (t + 1) per) and writes their ids from its exclusive
    // prefix count on
    const int per = (nw + kThreads - 1) / kThreads;
    int cnt = 0;
    for (int i = t * per; i < min(nw, (t + 1) * per); ++i) cnt += __popc(bm[i]);
    const int lane = t & 31, warp = t >> 5;
    int inc = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int up = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += up;
    }
    int* wsum = reinterpret_cast<int*>(sm.scr);
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    int pos = inc - cnt;
    for (int ww = 0; ww < warp; ++ww) pos += wsum[ww];
    for (int i = t * per; i < min(nw, (t + 1) * per); ++i)
      for (uint32_t bits = bm[i]; bits != 0u; bits &= bits - 1u) sm.ids[pos++] = 32 * i + __ffs(bits) - 1;
  } else {
    int rank[kPer];
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      rank[q] = 0;
      if (q * kThreads + t < n)
        for (int j = 0; j < n; ++j) rank[q] += sm.ids[j] < my[q] ? 1 : 0;
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < kPer; ++q)
      if (q * kThreads + t < n) sm.ids[rank[q]] = my[q];
  }
  __syncthreads();
  Fx128 r[kPer];
  Fx128 own = fx_zero();
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    const int p = kPer * t + q;
    r[q] = p < n ? mass(sm.ids[p]) : fx_zero();
    own = fx_add(own, r[q]);
  }
  Fx128 S;
  Fx128 cum = block_exclusive_scan_fx(own, sm.scr, &S);
  const double target = double(w) * fx_to_double(S);
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    cum = fx_add(cum, r[q]);
    if (!fx_is_zero(r[q]) && fx_to_double(cum) > target) {
      atomicMin(&sm.best, sm.ids[kPer * t + q]);
      break;
    }
  }
  __syncthreads();
  int tok = sm.best;
  if (fx_is_zero(S)) {
    tok = -1;
  } else if (tok == INT_MAX) {  // rounding left none: the largest id with mass
    __syncthreads();
    if (t == 0) sm.best = -1;
    __syncthreads();
#pragma unroll
    for (int q = 0; q < kPer; ++q)
      if (!fx_is_zero(r[q])) atomicMax(&sm.best, sm.ids[kPer * t + q]);
    __syncthreads();
    tok = sm.best;
  }
  __syncthreads();
  return tok;
}

// Dispatch on the support size: four entries per thread up to 4 * kThreads, else eight
// (fewer registers for the common short lists).
template <typename F>
__device__ int sparse_draw(const int32_t* ids, int n, F&& mass, float w, DrawSmem& sm,
                           int V = 0) {
  if (n <= 4 * kThreads) return sparse_draw_n<4>(ids, n, mass, w, sm, V);
  return sparse_draw_n<kSparsePer>(ids, n, mass, w, sm, V);
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

// G groups of 8 entries at v0, v0 + stride, ..., v0 + (G - 1) stride (-inf past V). When
// every group lies inside an aligned row the G vector loads are issued together, ahead of
// any use, so that their latencies overlap; otherwise group by group.
template <typename T, int G>
__device__ __forceinline__ void load8xG(const T* row, int v0, int stride, int V, bool aligned,
                                        float (&x)[G][8]) {
  constexpr int P = Elem<T>::kPerVec;
  if (aligned && v0 + (G - 1) * stride + 8 <= V) {
    uint4 w[G][8 / P];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int q = 0; q < 8 / P; ++q)
        w[g][q] = __ldg(reinterpret_cast<const uint4*>(row + v0 + g * stride) + q);
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int q = 0; q < 8 / P; ++q) Elem<T>::unpack(w[g][q], x[g] + q * P);
  } else {
#pragma unroll
    for (int g = 0; g < G; ++g) load8<T>(row, v0 + g * stride, V, aligned, x[g]);
  }
}

// Probability of entry v under the transformed distribution described by s (fp32).
template <typename T>
__device__ __forceinline__ float prob(const RowStats& s, float l, int v) {
  return kept(Elem<T>::key(l), v, s.thr_key, s.cutoff) ? weight(l, s.c, s.mc) / s.z : 0.0f;
}

// ------------------------------------------------------------------ double-precision view
// 2^(j/64), j = 0..63, each the double nearest the exact value (computed to 60 digits).
static __device__ const double kExp2J[64] = {
    0x1.0000000000000p+0, 0x1.02c9a3e778061p+0, 0x1.059b0d3158574p+0, 0x1.0874518759bc8p+0,
    0x1.0b5586cf9890fp+0, 0x1.0e3ec32d3d1a2p+0, 0x1.11301d0125b51p+0, 0x1.1429aaea92de0p+0,
    0x1.172b83c7d517bp+0, 0x1.1a35beb6fcb75p+0, 0x1.1d4873168b9aap+0, 0x1.2063b88628cd6p+0,
    0x1.2387a6e756238p+0, 0x1.26b4565e27cddp+0, 0x1.29e9df51fdee1p+0, 0x1.2d285a6e4030bp+0,
    0x1.306fe0a31b715p+0, 0x1.33c08b26416ffp+0, 0x1.371a7373aa9cbp+0, 0x1.3a7db34e59ff7p+0,
    0x1.3dea64c123422p+0, 0x1.4160a21f72e2ap+0, 0x1.44e086061892dp+0, 0x1.486a2b5c13cd0p+0,
    0x1.4bfdad5362a27p+0, 0x1.4f9b2769d2ca7p+0, 0x1.5342b569d4f82p+0, 0x1.56f4736b527dap+0,
    0x1.5ab07dd485429p+0, 0x1.5e76f15ad2148p+0, 0x1.6247eb03a5585p+0, 0x1.6623882552225p+0,
    0x1.6a09e667f3bcdp+0, 0x1.6dfb23c651a2fp+0, 0x1.71f75e8ec5f74p+0, 0x1.75feb564267c9p+0,
    0x1.7a11473eb0187p+0, 0x1.7e2f336cf4e62p+0, 0x1.82589994cce13p+0, 0x1.868d99b4492edp+0,
    0x1.8ace5422aa0dbp+0, 0x1.8f1ae99157736p+0, 0x1.93737b0cdc5e5p+0, 0x1.97d829fde4e50p+0,
    0x1.9c49182a3f090p+0, 0x1.a0c667b5de565p+0, 0x1.a5503b23e255dp+0, 0x1.a9e6b5579fdbfp+0,
    0x1.ae89f995ad3adp+0, 0x1.b33a2b84f15fbp+0, 0x1.b7f76f2fb5e47p+0, 0x1.bcc1e904bc1d2p+0,
    0x1.c199bdd85529cp+0, 0x1.c67f12e57d14bp+0, 0x1.cb720dcef9069p+0, 0x1.d072d4a07897cp+0,
    0x1.d5818dcfba487p+0, 0x1.da9e603db3285p+0, 0x1.dfc97337b9b5fp+0, 0x1.e502ee78b3ff6p+0,
    0x1.ea4afa2a490dap+0, 0x1.efa1bee615a27p+0, 0x1.f50765b6e4540p+0, 0x1.fa7c1819e90d8p+0,
};

// e^x for x <= 0 in double, by Tang's table-driven method (P. T. P. Tang, "Table-driven
// implementation of the exponential function in IEEE floating-point arithmetic", ACM TOMS
// 15(2), 1989): x = (64 k + j) ln2 / 64 + r with |r| <= ln2 / 128 (ln2 / 64 split into a
// 32-bit head and a tail, so n * head is exact), e^x = 2^k 2^(j/64) e^r, and e^r by its
// Taylor series to r^5 (the remainder is below 4e-17 of it). Relative error within a few
// units in the last place; x below -745 (and -inf) gives 0.
__device__ __forceinline__ double exp_neg(double x) {
  if (!(x > -745.0)) return 0.0;
  const double n = rint(x * 92.33248261689366);  // 64 / ln2
  double r = fma(-n, 0x1.62e42fee00000p-7, x);
  r = fma(-n, 0x1.a39ef35793c76p-39, r);
  const int ni = int(n);
  double p = fma(r, 1.0 / 120.0, 1.0 / 24.0);
  p = fma(p, r, 1.0 / 6.0);
  p = fma(p, r, 0.5);
  p = fma(p, r, 1.0);
  p = fma(p, r, 1.0);
  const double t = __ldg(&kExp2J[ni & 63]) * p;
  const int k = ni >> 6;  // floor(n / 64)
  if (k >= -1022) return t * __longlong_as_double((long long)(k + 1023) << 52);
  return ldexp(t, k);
}

// Unnormalised weight exp((l - m) / T) of a kept entry, in double (l - m is exact); iT = 1 / T.
__device__ __forceinline__ double weight_d(float l, float m, double iT) {
  return exp_neg((double(l) - double(m)) * iT);
}

// Weight of entry v of the row described by s (0 outside the kept set).
template <typename T>
__device__ __forceinline__ double kept_weight_d(const RowStats& s, double iT, float l, int v) {
  return kept(Elem<T>::key(l), v, s.thr_key, s.cutoff) ? weight_d(l, s.m, iT) : 0.0;
}

// Probability of entry v in double: kept weight times izd = 1 / zd.
template <typename T>
__device__ __forceinline__ double prob_d(const RowStats& s, double izd, double iT, float l, int v) {
  return kept_weight_d<T>(s, iT, l, v) * izd;
}

// The double normaliser of one row (every thread of the block calls it, gets the sum):
// s.zd when the row statistics hold it; else the sum over the kept set with exact Fx128
// accumulation, over the row's listed kept ids (nk > 0 of them at ids) or by a pass over the
// row.
template <typename T>
__device__ double row_zd(const RowStats& s, const T* row, int V, double iT, Fx128* scr,
                         const int32_t* ids = nullptr, int nk = 0) {
  if (s.zd >= 0.0) return s.zd;
  if (ids && nk > 0) {
    Fx128 acc = fx_zero();
    for (int i = threadIdx.x; i < nk; i += kThreads) {
      const int v = ids[i];
      acc = fx_add(acc, fx_from(kept_weight_d<T>(s, iT, Elem<T>::load(row, size_t(v)), v)));
    }
    return fx_to_double(block_sum_fx(acc, scr));
  }
  const bool al = (reinterpret_cast<uintptr_t>(row) & 15u) == 0;
  Fx128 acc = fx_zero();
  // four groups of 8 per iteration, all loaded before any is used
  for (int v00 = int(threadIdx.x) * 8; v00 < V; v00 += 4 * kThreads * 8) {
    float x[4][8];
    load8xG<T, 4>(row, v00, kThreads * 8, V, al, x);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const int v0 = v00 + g * kThreads * 8;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (v0 + k < V) acc = fx_add(acc, fx_from(kept_weight_d<T>(s, iT, x[g][k], v0 + k)));
    }
  }
  return fx_to_double(block_sum_fx(acc, scr));
}

}  // namespace sv
