// Double-precision placement of top-p boundaries ("Speculative Sampling", spec-decoding-i
// notes: the probabilities are transformed, here truncated to the nucleus, before the
// rejection scheme; the nucleus is the shortest prefix in (probability desc, id asc) order
// whose mass reaches top_p, the crossing token kept).
//
// The streaming kernel places the boundary with fp32 masses. Rows where that placement lies
// within its error guard of the target, and rows the exact finisher settled, are listed;
// here one thread block per listed row places the boundary again with double weights
// exp((l - m) / T) summed exactly (Fx128):
//   - one pass over the row collects, as (key << 32 | ~id) composites, the entries of a
//     window of three log-weight bins around the listed boundary's bin (the same fp32 bin
//     function the streaming kernel used, so the classification is identical), notes the
//     lightest entry above the window and the heaviest below it, and lists the ids above
//     the window. It also gathers the total mass Z and the mass above the window: for
//     bfloat16 rows through a histogram of the row's codes (each distinct code weighed once,
//     hist.cuh), for float32 rows entry by entry;
//   - the window is sorted (bitonic, descending composite = descending probability, then
//     ascending id) and scanned: the first entry whose cumulative mass reaches top_p * Z is
//     the boundary. A crossing just outside the window is taken from the noted neighbours.
// The row statistics get the new boundary and the double normaliser of the kept set, and
// the row's kept-id list is rewritten for the new boundary (emptied when it does not fit).
// A row whose window overflows, or whose crossing lies further out, keeps its fp32 boundary
// and is counted in *unresolved.
#pragma once

#include "draw.cuh"
#include "hist.cuh"
#include "stream.cuh"

namespace sv {

constexpr int kRefineCap = 4096;  // window entries one block sorts

struct RefineJob {
  RowJob r;                 // rows, element type, temperature, top_p, statistics, kept lists
  const int32_t* rows;      // listed rows
  const int32_t* count;     // number of listed rows
  int32_t* unresolved;      // rows left at their fp32 boundary (may be NULL)
};

// Dynamic shared memory: the window, then (bfloat16 rows) the code histogram: one block per
// SM.
template <typename T>
__host__ __device__ constexpr size_t refine_smem() {
  return size_t(kRefineCap) * 8 + (sizeof(T) == 2 ? kHistBytes : 0);
}

__device__ __forceinline__ void bitonic_sort_desc(uint64_t* a, int n2) {
  for (int k = 2; k <= n2; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int i = threadIdx.x; i < n2; i += kThreads) {
        const int ixj = i ^ jj;
        if (ixj > i) {
          const uint64_t x = a[i], y = a[ixj];
          const bool up = (i & k) == 0;  // this half ends descending
          if (up ? (x < y) : (x > y)) {
            a[i] = y;
            a[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) topp_refine_kernel(const RefineJob j) {
  extern __shared__ __align__(16) uint64_t win[];  // [kRefineCap], then the histogram
  uint32_t* hist = reinterpret_cast<uint32_t*>(win + kRefineCap);
  constexpr bool kHist = sizeof(T) == 2;
  __shared__ Fx128 scr[kWarps];
  __shared__ int s_cnt, s_best, s_nabove, s_bad;
  __shared__ unsigned long long s_lo_above, s_hi_below;  // neighbours of the window
  __shared__ double s_cum;
  const RowJob& rj = j.r;
  const int V = rj.V;
  const long long nlist = *j.count;
  const double iT = 1.0 / double(rj.temp);
  for (long long li = blockIdx.x; li < nlist; li += gridDim.x) {
    const long long row = j.rows[li];
    const RowStats rs = rj.stats[row];
    if (rs.status != ROW_OK) continue;  // uniform
    const T* src = (row < rj.rows0) ? static_cast<const T*>(rj.base0) + size_t(row) * V
                                    : static_cast<const T*>(rj.base1) + size_t(row - rj.rows0) * V;
    int32_t* kids = rj.kept_ids ? rj.kept_ids + size_t(row) * kKeptCap : nullptr;
    const float c = rs.c, mc = rs.mc, m = rs.m;
    const int bsel = bin_of(key_value<T>(rs.thr_key), c, mc);
    if (threadIdx.x == 0) {
      s_cnt = 0;
      s_best = INT_MAX;
      s_nabove = 0;
      s_bad = 0;
      s_lo_above = ~0ull;
      s_hi_below = 0ull;
    }
    if (kHist) hist_clear(hist);
    __syncthreads();
    Fx128 zall = fx_zero(), above = fx_zero();
    unsigned long long lo_above = ~0ull, hi_below = 0ull;
    bool ok = true;  // no histogram counter overflowed
    auto visit = [&](float x, int v) {
      if (!(x > -INFINITY)) return;  // weight 0
      const uint32_t key = Elem<T>::key(x);
      const int b = bin_of(x, c, mc);
      const unsigned long long e = make_comp(key, v);
      if (kHist) {
        ok &= hist_count(hist, key);
      } else {
        const Fx128 fe = fx_from(weight_d(x, m, iT));
        zall = fx_add(zall, fe);
        if (b < bsel - 1) above = fx_add(above, fe);
      }
      if (b < bsel - 1) {
        lo_above = e < lo_above ? e : lo_above;
        if (kids) {
          const int slot = atomicAdd(&s_nabove, 1);
          if (slot < kKeptCap) kids[slot] = v;
        }
      } else if (b <= bsel + 1) {
        const int slot = atomicAdd(&s_cnt, 1);
        if (slot < kRefineCap) win[slot] = e;
      } else {
        hi_below = e > hi_below ? e : hi_below;
      }
    };
    const bool al = (reinterpret_cast<uintptr_t>(src) & 15u) == 0;
    // eight groups of 8 per thread in flight (one block per SM keeps 64 KB of loads going)
    for (int v0 = int(threadIdx.x) * 8; v0 < V; v0 += 8 * kThreads * 8) {
      float x[8][8];
#pragma unroll
      for (int g = 0; g < 8; ++g) load8<T>(src, v0 + g * kThreads * 8, V, al, x[g]);
#pragma unroll
      for (int g = 0; g < 8; ++g)
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int v = v0 + g * kThreads * 8 + k;
          if (v < V) visit(x[g][k], v);
        }
    }
    atomicMin(&s_lo_above, lo_above);
    atomicMax(&s_hi_below, hi_below);
    if (!ok) s_bad = 1;
    __syncthreads();
    if (kHist) {
      if (s_bad) {
        // a code held more than 65535 entries: weigh the counted entries one by one
        zall = fx_zero();
        above = fx_zero();
        for (int v = threadIdx.x; v < V; v += kThreads) {
          const float x = Elem<T>::load(src, size_t(v));
          if (!(x > -INFINITY)) continue;
          const Fx128 fe = fx_from(weight_d(x, m, iT));
          zall = fx_add(zall, fe);
          if (bin_of(x, c, mc) < bsel - 1) above = fx_add(above, fe);
        }
      } else {
        Fx128 ha;
        const Fx128 hz = hist_weigh(
            hist, m, iT,
            [&](uint32_t key) { return bin_of(key_value<T>(key), c, mc) < bsel - 1; }, &ha);
        zall = fx_add(zall, hz);
        above = fx_add(above, ha);
      }
    }
    zall = block_sum_fx(zall, scr);
    above = block_sum_fx(above, scr);
    const int n = s_cnt;
    const int nabove = s_nabove;
    if (n > kRefineCap) {
      // unresolved: the fp32 boundary stands, and the pass overwrote its kept list
      if (threadIdx.x == 0) {
        if (rj.kept_n) rj.kept_n[row] = 0;
        if (j.unresolved) atomicAdd(j.unresolved, 1);
      }
      __syncthreads();
      continue;
    }
    int n2 = 1;
    while (n2 < n) n2 <<= 1;
    for (int i = n + int(threadIdx.x); i < n2; i += kThreads) win[i] = 0ull;
    __syncthreads();
    bitonic_sort_desc(win, n2);
    // masses in sorted order: thread t scans its contiguous range of the window
    const int per = (n2 + kThreads - 1) / kThreads;
    const int wlo = int(threadIdx.x) * per;
    Fx128 own = fx_zero();
    for (int i = wlo; i < wlo + per && i < n; ++i)
      own = fx_add(own, fx_from(weight_d(key_value<T>(comp_key(win[i])), m, iT)));
    Fx128 wtot;
    const Fx128 ex = block_exclusive_scan_fx(own, scr, &wtot);
    const double target = double(rj.top_p) * fx_to_double(zall);
    Fx128 cum = fx_add(above, ex);
    for (int i = wlo; i < wlo + per && i < n; ++i) {
      cum = fx_add(cum, fx_from(weight_d(key_value<T>(comp_key(win[i])), m, iT)));
      if (fx_to_double(cum) >= target) {
        atomicMin(&s_best, i);
        break;
      }
    }
    __syncthreads();
    const int best = s_best;
    if (best != INT_MAX && best >= wlo && best < wlo + per) s_cum = fx_to_double(cum);
    __syncthreads();
    // the new boundary: e (0 if none), and how many window entries it keeps
    uint64_t e = 0ull;
    double zkept = 0.0;
    int nwin = 0;
    bool below = false;  // the heaviest entry below the window is kept too
    {
      const double a = fx_to_double(above);
      if (a >= target) {
        // the crossing lies above the window: the lightest entry above it, if that alone
        // holds the excess
        const double wl = weight_d(key_value<T>(comp_key(s_lo_above)), m, iT);
        if (s_lo_above != ~0ull && a - wl < target) {
          e = s_lo_above;
          zkept = a;
        }
      } else if (best != INT_MAX) {
        e = win[best];
        zkept = s_cum;
        nwin = best + 1;
      } else if (s_hi_below != 0ull) {
        // below the window: the heaviest entry after it, if it reaches the target
        const double through = fx_to_double(fx_add(above, wtot));
        const double wh = weight_d(key_value<T>(comp_key(s_hi_below)), m, iT);
        if (through + wh >= target) {
          e = s_hi_below;
          zkept = through + wh;
          nwin = n;
          below = true;
        }
      }
    }
    if (e != 0ull) {
      // kept ids: those above the window (listed in the pass), then the window's kept ones
      const int total = nabove + nwin + (below ? 1 : 0);
      const bool fits = kids && total <= kKeptCap;
      if (fits) {
        for (int i = threadIdx.x; i < nwin; i += kThreads) kids[nabove + i] = comp_id(win[i]);
        if (below && threadIdx.x == 0) kids[nabove + nwin] = comp_id(s_hi_below);
      }
      if (threadIdx.x == 0) {
        RowStats out = rs;
        out.thr_key = comp_key(e);
        out.cutoff = comp_id(e);
        out.zd = zkept;
        out.z = float(zkept);
        rj.stats[row] = out;
        if (rj.kept_n) rj.kept_n[row] = fits ? total : 0;
      }
    } else if (threadIdx.x == 0) {
      // the fp32 boundary stands, and with it the streaming kernel's list, which the pass
      // above overwrote: drop it
      if (rj.kept_n) rj.kept_n[row] = 0;
      if (j.unresolved) atomicAdd(j.unresolved, 1);
    }
    __syncthreads();
  }
}

}  // namespace sv
