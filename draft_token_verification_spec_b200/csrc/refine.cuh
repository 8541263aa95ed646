// Double-precision placement of top-p boundaries ("Speculative Sampling", spec-decoding-i
// notes: the probabilities are transformed, here truncated to the nucleus, before the
// rejection scheme; the nucleus is the shortest prefix in (probability desc, id asc) order
// whose mass reaches top_p, the crossing token kept).
//
// The streaming kernel places the boundary with fp32 masses. Rows where that placement lies
// within its error guard of the target, and rows the exact finisher settled, are listed;
// here one thread block per listed row places the boundary again with double weights
// exp((l - m) / T) summed exactly (Fx128):
//   - one pass over the row sums the total mass Z, the mass of the entries in log-weight
//     bins above a window of three bins around the listed boundary's bin (the same fp32 bin
//     function the streaming kernel used, so the classification is identical), and collects
//     the window's entries as (key << 32 | ~id) composites; it also notes the lightest entry
//     above the window and the heaviest below it;
//   - the window is sorted (bitonic, descending composite = descending probability, then
//     ascending id) and scanned: the first entry whose cumulative mass reaches top_p * Z is
//     the boundary. A crossing just outside the window is taken from the noted neighbours.
// The row statistics get the new boundary and the double normaliser of the kept set. A row
// whose window overflows, or whose crossing lies further out, keeps its fp32 boundary and is
// counted in *unresolved.
#pragma once

#include "draw.cuh"
#include "stream.cuh"

namespace sv {

constexpr int kRefineCap = 4096;  // window entries one block sorts

struct RefineJob {
  RowJob r;                 // rows, element type, temperature, top_p, statistics
  const int32_t* rows;      // listed rows
  const int32_t* count;     // number of listed rows
  int32_t* unresolved;      // rows left at their fp32 boundary (may be NULL)
};

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
  extern __shared__ __align__(16) uint64_t win[];  // [kRefineCap]
  __shared__ Fx128 scr[kWarps];
  __shared__ int s_cnt, s_best;
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
    const float c = rs.c, mc = rs.mc, m = rs.m;
    const int bsel = bin_of(key_value<T>(rs.thr_key), c, mc);
    if (threadIdx.x == 0) {
      s_cnt = 0;
      s_best = INT_MAX;
      s_lo_above = ~0ull;
      s_hi_below = 0ull;
    }
    __syncthreads();
    Fx128 zall = fx_zero(), above = fx_zero();
    unsigned long long lo_above = ~0ull, hi_below = 0ull;
    const bool al = (reinterpret_cast<uintptr_t>(src) & 15u) == 0;
    for (int v0 = int(threadIdx.x) * 8; v0 < V; v0 += kThreads * 8) {
      float x[8];
      load8<T>(src, v0, V, al, x);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int v = v0 + k;
        if (v >= V || !(x[k] > -INFINITY)) continue;  // past the row, or weight 0
        const Fx128 fe = fx_from(weight_d(x[k], m, iT));
        zall = fx_add(zall, fe);
        const int b = bin_of(x[k], c, mc);
        const unsigned long long e = make_comp(Elem<T>::key(x[k]), v);
        if (b < bsel - 1) {
          above = fx_add(above, fe);
          lo_above = e < lo_above ? e : lo_above;
        } else if (b <= bsel + 1) {
          const int slot = atomicAdd(&s_cnt, 1);
          if (slot < kRefineCap) win[slot] = e;
        } else {
          hi_below = e > hi_below ? e : hi_below;
        }
      }
    }
    atomicMin(&s_lo_above, lo_above);
    atomicMax(&s_hi_below, hi_below);
    zall = block_sum_fx(zall, scr);
    above = block_sum_fx(above, scr);
    const int n = s_cnt;
    if (n > kRefineCap) {
      if (threadIdx.x == 0 && j.unresolved) atomicAdd(j.unresolved, 1);
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
    const int lo = int(threadIdx.x) * per;
    Fx128 own = fx_zero();
    for (int i = lo; i < lo + per && i < n; ++i)
      own = fx_add(own, fx_from(weight_d(key_value<T>(comp_key(win[i])), m, iT)));
    Fx128 wtot;
    const Fx128 ex = block_exclusive_scan_fx(own, scr, &wtot);
    const double target = double(rj.top_p) * fx_to_double(zall);
    Fx128 cum = fx_add(above, ex);
    for (int i = lo; i < lo + per && i < n; ++i) {
      cum = fx_add(cum, fx_from(weight_d(key_value<T>(comp_key(win[i])), m, iT)));
      if (fx_to_double(cum) >= target) {
        atomicMin(&s_best, i);
        break;
      }
    }
    __syncthreads();
    const int best = s_best;
    if (best != INT_MAX && best >= lo && best < lo + per) s_cum = fx_to_double(cum);
    __syncthreads();
    if (threadIdx.x == 0) {
      uint64_t e = 0ull;
      double zkept = 0.0;
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
      } else if (s_hi_below != 0ull) {
        // below the window: the heaviest entry after it, if it reaches the target
        const double through = fx_to_double(fx_add(above, wtot));
        const double wh = weight_d(key_value<T>(comp_key(s_hi_below)), m, iT);
        if (through + wh >= target) {
          e = s_hi_below;
          zkept = through + wh;
        }
      }
      if (e != 0ull) {
        RowStats out = rs;
        out.thr_key = comp_key(e);
        out.cutoff = comp_id(e);
        out.zd = zkept;
        out.z = float(zkept);
        rj.stats[row] = out;
      } else if (j.unresolved) {
        atomicAdd(j.unresolved, 1);
      }
    }
    __syncthreads();
  }
}

}  // namespace sv
