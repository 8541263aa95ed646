// Double-precision placement of top-p boundaries ("Speculative Sampling", spec-decoding-i
// notes: the probabilities are transformed, here truncated to the nucleus, before the
// rejection scheme; the nucleus is the shortest prefix in (probability desc, id asc) order
// whose mass reaches top_p, the crossing token kept).
//
// Rows whose boundary was placed within the error bound of an fp32 sum (the streaming
// kernel's sum of the entries below its threshold), and top-p rows the exact finisher
// settled with fp32 masses, are listed; here the boundary is placed again exactly.
//
// bfloat16 rows, two kernels:
//   - topp_zexact_kernel: the row's normaliser Z = sum of exp((l - m) / T) in double, summed
//     exactly (Fx128) by kZSlices blocks per listed row, each over a slice, into the row's
//     accumulator (128-bit atomic adds with carry, so the total does not depend on order);
//   - topp_finalize_kernel: one block per listed row collects every entry within two log2
//     units of weight of the listed boundary or above it (a histogram of their codes and
//     their 32-bit composites, as the streaming kernel keeps them) and runs the same
//     selection with the exact Z: the code where the mass from the top reaches top_p * Z,
//     how many of its entries (in id order) are kept, their ids.
// float32 rows, topp_refine_kernel, one block per listed row:
//   - one pass over the row collects, as (key << 32 | ~id) composites, the entries of a
//     window of three log-weight bins around the listed boundary's bin (the same fp32 bin
//     function the streaming kernel used), notes the lightest entry above the window and
//     the heaviest below it, and lists the ids above the window. It also sums the total
//     mass Z and the mass above the window entry by entry;
//   - the window is sorted (bitonic, descending composite = descending probability, then
//     ascending id) and scanned: the first entry whose cumulative mass reaches top_p * Z is
//     the boundary. A crossing just outside the window is taken from the noted neighbours.
// The row statistics get the new boundary and the double normaliser of the kept set, and
// the row's kept-id list is rewritten for the new boundary (emptied when it does not fit).
// A row whose crossing lies outside what was collected keeps its fp32 boundary and is
// counted in *unresolved.
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

// Dynamic shared memory of topp_refine_kernel: the window.
template <typename T>
__host__ __device__ constexpr size_t refine_smem() {
  return size_t(kRefineCap) * 8 + (sizeof(T) == 2 ? kHistBytes : 0);
}

constexpr int kZSlices = 64;  // blocks per listed row summing its exact normaliser

// 128-bit atomic add with carry: concurrent adds of exact terms give the exact total.
__device__ __forceinline__ void fx_atomic_add(unsigned long long* p, Fx128 a) {
  const unsigned long long old = atomicAdd(p, a.lo);
  const unsigned long long carry = (old + a.lo < old) ? 1ull : 0ull;
  if (a.hi + carry) atomicAdd(p + 1, a.hi + carry);
}

template <typename T>
__device__ __forceinline__ const T* refine_row_ptr(const RowJob& rj, long long row) {
  return (row < rj.rows0) ? static_cast<const T*>(rj.base0) + size_t(row) * rj.V
                          : static_cast<const T*>(rj.base1) + size_t(row - rj.rows0) * rj.V;
}

// Exact normalisers of the listed rows: work item (li, s) adds the Fx128 sum of exp((l - m)
// / T) over slice s of listed row li to rj.refine_z[li] (zeroed when the row was listed).
template <typename T>
__global__ void __launch_bounds__(kThreads) topp_zexact_kernel(const RefineJob j) {
  __shared__ Fx128 scr[kWarps];
  const RowJob& rj = j.r;
  const int V = rj.V;
  const long long items = (long long)*j.count * kZSlices;
  const int slice = ((V + kZSlices - 1) / kZSlices + 7) / 8 * 8;
  const double iT = 1.0 / double(rj.temp);
  for (long long it = blockIdx.x; it < items; it += gridDim.x) {
    const long long li = it / kZSlices;
    const int sl = int(it % kZSlices);
    const long long row = j.rows[li];
    const RowStats rs = rj.stats[row];
    if (rs.status != ROW_OK) continue;  // uniform
    const T* src = refine_row_ptr<T>(rj, row);
    const bool al = (reinterpret_cast<uintptr_t>(src) & 15u) == 0;
    const int v1 = min(V, (sl + 1) * slice);
    Fx128 acc = fx_zero();
    // four groups of 8 per thread in flight
    for (int v00 = sl * slice + int(threadIdx.x) * 8; v00 < v1; v00 += 8 * kThreads * 4) {
      float x[4][8];
      load8xG<T, 4>(src, v00, kThreads * 8, v1, al, x);
#pragma unroll
      for (int g = 0; g < 4; ++g)
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (x[g][k] > -INFINITY) acc = fx_add(acc, fx_from(weight_d(x[g][k], rs.m, iT)));
    }
    acc = block_sum_fx(acc, scr);
    if (threadIdx.x == 0) fx_atomic_add(rj.refine_z + 2 * li, acc);
  }
}

// One block of kFinThreads per listed bfloat16 row: the boundary again, from the exact
// normaliser.
constexpr int kFinThreads = 1024;
template <typename T>
__global__ void __launch_bounds__(kFinThreads) topp_finalize_kernel(const RefineJob j) {
  static_assert(sizeof(T) == 2, "bfloat16 rows");
  __shared__ StreamAux aux;
  __shared__ uint32_t plist[kCapP];
  __shared__ uint32_t hcnt[kPBins];
  __shared__ uint32_t pmem[kPMem];
  __shared__ unsigned long long zred[kFinThreads / 32];
  __shared__ long long s1red[kFinThreads / 32];
  CandSet<T> cs;
  cs.cand = nullptr;
  cs.ranked = nullptr;
  cs.plist = plist;
  cs.hcnt = hcnt;
  cs.pmem = pmem;
  cs.aux = &aux;
  const RowJob& rj = j.r;
  const int V = rj.V;
  const long long nlist = *j.count;
  const double iT = 1.0 / double(rj.temp);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (long long li = blockIdx.x; li < nlist; li += gridDim.x) {
    const long long row = j.rows[li];
    const RowStats rs = rj.stats[row];
    if (rs.status != ROW_OK) continue;  // uniform
    const T* src = refine_row_ptr<T>(rj, row);
    const bool al = (reinterpret_cast<uintptr_t>(src) & 15u) == 0;
    const double zt = fx_to_double(Fx128{rj.refine_z[2 * li], rj.refine_z[2 * li + 1]});
    // collect the codes from two log2 units of weight below the listed boundary up, in a
    // window of kPBins codes that reaches the row maximum
    const float xlo = key_value<T>(rs.thr_key) - 1.3862944f * rj.temp;
    uint32_t base = Elem<T>::key(xlo);
    const uint32_t kmax = Elem<T>::key(rs.m);
    if (kmax > base + uint32_t(kPBins - 1)) base = kmax - uint32_t(kPBins - 1);
    const float t = key_value<T>(base);
    for (int i = threadIdx.x; i < kPBins; i += kFinThreads) hcnt[i] = 0u;
    if (threadIdx.x == 0) aux.ccount = 0;
    __syncthreads();
    // two groups of 8 per thread in flight; every thread takes the same number of rounds
    // (the warp-level appends below need all lanes)
    for (int r0 = 0; r0 < V; r0 += 2 * kFinThreads * 8) {
      const int v00 = r0 + int(threadIdx.x) * 8;
      float x[2][8];
      load8xG<T, 2>(src, v00, kFinThreads * 8, V, al, x);
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const int v0 = v00 + g * kFinThreads * 8;
        uint32_t mk = 0u;
#pragma unroll
        for (int k = 0; k < 8; ++k) mk |= (x[g][k] >= t && v0 + k < V) ? 1u << k : 0u;
        // one shared atomic per warp for the list slots
        const int my = __popc(mk);
        int inc = my;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int up = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += up;
        }
        const int wtot = __shfl_sync(0xffffffffu, inc, 31);
        if (wtot == 0) continue;  // (uniform in the warp)
        int wb = 0;
        if (lane == 31) wb = atomicAdd(&aux.ccount, wtot);
        int pos = __shfl_sync(0xffffffffu, wb, 31) + inc - my;
        for (uint32_t m2 = mk; m2 != 0u; m2 &= m2 - 1u, ++pos) {
          const int k = __ffs(m2) - 1;
          const uint32_t h = Elem<T>::key(__uint_as_float(
              uint32_t(reinterpret_cast<const unsigned short*>(src)[v0 + k]) << 16));
          const uint32_t rel = h - base;  // < kPBins: the entry is at most the maximum
          if (pos < kCapP) plist[pos] = pcomp(rel, v0 + k);
          atomicAdd(&hcnt[rel], 1u);
        }
      }
    }
    __syncthreads();
    const int nall = aux.ccount;
    // the crossing code with the exact normaliser (warp 0), over the occupied codes
    if (warp == 0) {
      int jj = 0, stable = 0, bsel = -1;
      double above = 0.0, wc = 0.0;
      if (nall <= kCapP)
        bsel = cs.p_cross_warp(int(kmax - base), base, rs.m, iT, rj.top_p, 0.0, zt, 0.0, &jj,
                               &above, &wc, &stable);
      if (bsel >= 0 && hcnt[bsel] > uint32_t(kPMem)) bsel = -1;
      if (lane == 0) {
        aux.sel_bin = bsel;
        aux.sel_j = jj;
        aux.sel_above = above + double(jj) * wc;
        aux.sel_cnt = 0u;
        aux.mcount = 0;
      }
    }
    __syncthreads();
    const int bsel = aux.sel_bin;
    if (bsel < 0) {
      // unresolved: the listed boundary stands, with its kept list
      if (threadIdx.x == 0 && j.unresolved) atomicAdd(j.unresolved, 1);
      __syncthreads();
      continue;
    }
    // kept ids and the fp32 normaliser: the codes above the crossing code by every thread,
    // the crossing code's entries gathered, then the j with the lowest ids by warp 0
    int32_t* kids = rj.kept_ids ? rj.kept_ids + size_t(row) * kKeptCap : nullptr;
    const bool want_ent = (rj.flags & RS_ENTROPY) != 0;
    unsigned long long z = 0;
    long long s1 = 0;
    auto keep = [&](uint32_t e) {
      const float zx = wexp(key_value<T>(base + pcomp_rel(e)), rs.c, rs.mc);
      const float ex = ex2(zx);
      z += to_fx(ex);
      if (want_ent) s1 += __float2ll_rn(ent_term(ex, zx) * kS1Fx);
      const int slot = atomicAdd(&aux.mcount, 1);
      if (kids && slot < kKeptCap) kids[slot] = pcomp_id(e);
    };
    for (int i = threadIdx.x; i < nall; i += kFinThreads) {
      const uint32_t e = plist[i];
      const int r = int(pcomp_rel(e));
      if (r > bsel) {
        keep(e);
      } else if (r == bsel) {
        const uint32_t slot = atomicAdd(&aux.sel_cnt, 1u);
        if (slot < uint32_t(kPMem)) pmem[slot] = e;
      }
    }
    __syncthreads();
    if (warp == 0) {
      const int nm = min(int(aux.sel_cnt), kPMem);
      const int jj = aux.sel_j;
      uint32_t cst = 0u;
      bool got = false;
      for (int i = lane; i < nm; i += 32) {
        const uint32_t e = pmem[i];
        int ab = 0;
        for (int q = 0; q < nm; ++q) ab += pmem[q] > e ? 1 : 0;
        if (ab < jj) keep(e);
        if (ab == jj - 1) {
          cst = e;
          got = true;
        }
      }
      const unsigned g = __ballot_sync(0xffffffffu, got);
      if (lane == 0) aux.sel_found = g ? 1 : 0;
      if (g && lane == __ffs(g) - 1) aux.sel_c32 = cst;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      z += __shfl_xor_sync(0xffffffffu, z, o);
      s1 += __shfl_xor_sync(0xffffffffu, s1, o);
    }
    if (lane == 0) {
      zred[warp] = z;
      s1red[warp] = s1;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned long long zf = 0;
      long long s1a = 0;
      for (int w = 0; w < kFinThreads / 32; ++w) {
        zf += zred[w];
        s1a += s1red[w];
      }
      if (aux.sel_found) {
        const uint32_t cstar = aux.sel_c32;
        RowStats out = rs;
        out.thr_key = base + pcomp_rel(cstar);
        out.cutoff = pcomp_id(cstar);
        out.zd = aux.sel_above;
        const double Z = double(zf) * kFxInv;
        out.z = float(Z);
        if (want_ent)
          out.entropy = float(log(Z) - 0.6931471805599453 * (double(s1a) / double(kS1Fx)) / Z);
        rj.stats[row] = out;
        if (rj.kept_n) rj.kept_n[row] = (kids && aux.mcount <= kKeptCap) ? aux.mcount : 0;
      } else {
        // the list was partly rewritten: drop it, the listed boundary stands
        if (rj.kept_n) rj.kept_n[row] = 0;
        if (j.unresolved) atomicAdd(j.unresolved, 1);
      }
    }
    __syncthreads();
  }
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
