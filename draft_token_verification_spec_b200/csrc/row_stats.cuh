// Row statistics kernel: persistent thread-block clusters, one logit row per cluster
// at a time. It computes spec_logits_to_probs, finishes the rows the streaming kernel
// (stream.cuh) lists as unsettled, and takes top-k above the streaming kernel's limit.
//
// A cluster of C CTAs walks rows cid, cid + G, cid + 2G, ... (G clusters resident). Each
// CTA owns a contiguous slice of every row and keeps a ring of kNBuf slice buffers in
// shared memory: while it works on one row, 1-D bulk copies (cp.async.bulk, completion
// on an mbarrier per buffer) bring in the next rows' slices. Per row the cluster
// combines partial results through distributed shared memory (DSMEM):
//   - the row maximum (packed bf16x2 max with NaN propagation), validity and, in greedy
//     mode, the lowest index holding the maximum — one exchange;
//   - no truncation: the softmax normaliser (and entropy term) in one exp pass;
//   - top-k (fast path, k <= 256): every warp takes the ceil(k/8)-th largest of its
//     per-thread maxima by a ballot radix select; the smallest of a CTA's warp values
//     is a value that k of its entries reach, and the largest over the cluster (t0)
//     rides in the maximum exchange. A filter pass keeps the few entries >= t0, every
//     CTA gathers them and selects the top k exactly — no exp over the row;
//   - otherwise (top-p, or a fast path that does not fit): exact selection by radix
//     select over order-preserving keys, 8 bits per level, with fixed-point masses.
// It stores a RowStats record (and the kept ids of top-k rows) or writes the
// transformed probabilities.
//
// This is the sampling transform of "Speculative Sampling" (spec-decoding-i notes, last
// bullet: transform the probabilities first, then apply the rejection scheme) and the
// entropy that MEDUSA typical acceptance uses ("Key Components").
#pragma once

#include <climits>

#include "common.cuh"

namespace sv {

enum : int { RS_GREEDY = 1, RS_ENTROPY = 2, RS_WRITE_PROBS = 4 };

#ifndef SV_NBUF
#define SV_NBUF 2
#endif
constexpr int kNBuf = SV_NBUF;     // slice buffers per CTA (ring)
constexpr int kBulkChunk = 16384;
constexpr int kCandCap = 512;      // candidates one CTA may hold in the top-k filter
constexpr int kGatherCap = 1024;   // candidates a cluster may hold for exact selection
constexpr int kMaxCluster = 16;
constexpr int kKeptCap = 2048;     // kept ids listed per row: top-k rows, top-p nuclei this small
constexpr float kS1Fx = 4294967296.0f;  // 2^32: signed fixed point for entropy terms

struct RowJob {
  const void* base0;   // rows [0, rows0)
  const void* base1;   // rows [rows0, rows)
  long long rows0;
  long long rows;
  int V;
  int slice;           // elements per CTA slice (multiple of 16)
  int slice_bytes;     // bytes reserved per slice buffer (multiple of 128)
  float c;             // log2(e) / T   (unused in greedy mode)
  float inv_t;         // 1 / T
  float temp;          // T as given (the double-precision view uses it)
  int top_k;           // 1 <= top_k < V, else off
  float top_p;         // < 1: on
  int flags;
  RowStats* stats;     // [rows] or NULL
  int32_t* kept_n;     // [rows] or NULL: number of ids in kept_ids (0: no list)
  int32_t* kept_ids;   // [rows][kKeptCap] or NULL: the kept set of top-k rows
  float* probs;        // RS_WRITE_PROBS: [rows][V]
  float* entropy;      // RS_WRITE_PROBS: [rows] or NULL
  int32_t* dev_status; // set to 1 on a copy timeout (may be NULL)
  const int32_t* row_list;   // if set: process rows row_list[0 .. *row_count) only
  const int32_t* row_count;
  int32_t* refine_rows;      // if set: top-p rows whose boundary is re-decided in double
  int32_t* refine_count;
  unsigned long long* refine_z;  // [rows][2]: their exact normalisers (Fx128), zeroed on listing
};

struct __align__(16) RowAux {
  uint64_t bar[kNBuf];
  // exchange slots, double-buffered by phase
  float xm[2];
  int xi[2];
  int xbad[2];
  float xt[2];
  unsigned long long xu64[2];
  double xf64[2];
  uint32_t xcnt[2];
  int xid[2];
  union {
    struct {  // radix select
      uint32_t hcnt[2][256];
      uint32_t hlimb[2][3 * 256];  // masses as 15-bit limbs (limb_add)
      uint32_t tot_cnt[256];
      unsigned long long tot_mass[256];
    } g;
    struct {  // top-k filter: this CTA's candidates, then the cluster's
      float cval[kCandCap];
      int cid[kCandCap];
      float gval[kGatherCap];
      int gid[kGatherCap];
    } f;
  } u;
  unsigned long long scr_u64[kWarps];
  double scr_f64[kWarps];
  uint32_t scr_u32[kWarps];
  float scr_m[kWarps];
  int scr_i[kWarps];
  float scr_t[kWarps];
  long long scr_s64[kWarps];
  int cnt_off[kMaxCluster + 1];
  uint32_t lh[256];  // CTA-local histogram
  int found_bin;
  int found;
  unsigned long long found_above;
  int ccount;
  int sel_id;
  int broken;        // a copy wait timed out: no further copies are issued
  int pending;       // bit b: a copy into buffer b was issued and not yet waited for
};

// Where one CTA's slice of a row lives and how it is split: the 16-byte-aligned middle
// moves by bulk copy, the unaligned head and tail (< 16 bytes each) by plain loads.
// Element j of the slice lands at byte pad + j * E of the buffer.
struct SliceLoc {
  const unsigned char* g;
  int n, pad, head, mid, tail;
};

template <typename T>
__device__ __forceinline__ SliceLoc slice_loc(const RowJob& job, long long row, int rank) {
  constexpr int E = Elem<T>::kBytes;
  const int V = job.V;
  const T* src = (row < job.rows0)
                     ? static_cast<const T*>(job.base0) + size_t(row) * V
                     : static_cast<const T*>(job.base1) + size_t(row - job.rows0) * V;
  SliceLoc s;
  const int s0 = rank * job.slice;
  s.n = max(0, min(V - s0, job.slice));
  s.g = reinterpret_cast<const unsigned char*>(src + s0);
  s.pad = int(reinterpret_cast<uintptr_t>(s.g) & 15u);
  const int bytes = s.n * E;
  s.head = min(bytes, (16 - s.pad) & 15);
  s.mid = ((bytes - s.head) >> 4) << 4;
  s.tail = bytes - s.head - s.mid;
  return s;
}

// Thread 0: starts the bulk copy of a slice into buf.
__device__ __forceinline__ void issue_slice(const SliceLoc& s, unsigned char* buf, uint64_t* bar) {
  mbar_arrive_expect_tx(bar, uint32_t(s.mid));
  unsigned char* d = buf + s.pad + s.head;
  for (int off = 0; off < s.mid; off += kBulkChunk)
    bulk_g2s(d + off, s.g + s.head + off, uint32_t(min(kBulkChunk, s.mid - off)), bar);
}

// All threads: plain loads of the head and tail, then wait for the bulk copy. Returns
// false if the copy did not complete within the wait limit.
template <typename T>
__device__ __forceinline__ bool finish_slice(const SliceLoc& s, unsigned char* buf,
                                             uint64_t* bar, uint32_t parity) {
  constexpr int E = Elem<T>::kBytes;
  const int hE = s.head / E, tE = s.tail / E;
  for (int j = threadIdx.x; j < hE + tE; j += kThreads) {
    const int e = (j < hE) ? j : (s.n - tE + (j - hE));
    if (E == 2)
      reinterpret_cast<uint16_t*>(buf + s.pad)[e] = reinterpret_cast<const uint16_t*>(s.g)[e];
    else
      reinterpret_cast<uint32_t*>(buf + s.pad)[e] = reinterpret_cast<const uint32_t*>(s.g)[e];
  }
  const bool ok = mbar_wait(bar, parity);
  __syncthreads();
  return ok;
}

template <typename T>
struct RowCtx {
  const unsigned char* buf;
  int pad, n, s0, nvec;
  RowAux* aux;
  cg::cluster_group cl;
  int C;
  int ph;

  __device__ __forceinline__ bool full(int j0) const {
    return j0 >= 0 && j0 + Elem<T>::kPerVec <= n;
  }
  __device__ __forceinline__ int first_elem(int v) const {
    return (v * 16 - pad) / Elem<T>::kBytes;
  }

  // Calls f(global id, value) for every element of this CTA's slice; each thread
  // visits its elements in ascending id order.
  template <typename F>
  __device__ __forceinline__ void each(F&& f) const {
    constexpr int P = Elem<T>::kPerVec;
    for (int v = threadIdx.x; v < nvec; v += kThreads) {
      const uint4 w = reinterpret_cast<const uint4*>(buf)[v];
      float x[P];
      Elem<T>::unpack(w, x);
      const int j0 = first_elem(v);
      if (full(j0)) {
#pragma unroll
        for (int k = 0; k < P; ++k) f(s0 + j0 + k, x[k]);
      } else {
#pragma unroll
        for (int k = 0; k < P; ++k) {
          const int j = j0 + k;
          if (j >= 0 && j < n) f(s0 + j, x[k]);
        }
      }
    }
  }

  // This thread's largest value (NaN if any of its entries is NaN, -inf if it has none)
  // and the first of its vectors that holds it.
  __device__ __forceinline__ float thread_max(int* vbest) const {
    float mt = -INFINITY;
    int vb = -1;
    bool nan = false;
    for (int v = threadIdx.x; v < nvec; v += kThreads) {
      const uint4 w = reinterpret_cast<const uint4*>(buf)[v];
      const int j0 = first_elem(v);
      float vm;
      if (full(j0)) {
        vm = Elem<T>::vmax_nan(w);
      } else {
        float x[Elem<T>::kPerVec];
        Elem<T>::unpack(w, x);
        vm = -INFINITY;
#pragma unroll
        for (int k = 0; k < Elem<T>::kPerVec; ++k) {
          const int j = j0 + k;
          if (j >= 0 && j < n) vm = fmax_nan(vm, x[k]);
        }
      }
      if (vm != vm) {
        nan = true;
      } else if (vm > mt) {
        mt = vm;
        vb = v;
      }
    }
    *vbest = vb;
    return nan ? __int_as_float(0x7fc00000) : mt;
  }

  // Lowest id of an entry equal to value m inside vector v of this slice (INT_MAX if none).
  __device__ __forceinline__ int first_equal(int v, float m) const {
    if (v < 0) return INT_MAX;
    const uint4 w = reinterpret_cast<const uint4*>(buf)[v];
    float x[Elem<T>::kPerVec];
    Elem<T>::unpack(w, x);
    const int j0 = first_elem(v);
    int id = INT_MAX;
#pragma unroll
    for (int k = Elem<T>::kPerVec - 1; k >= 0; --k) {
      const int j = j0 + k;
      if (j >= 0 && j < n && x[k] == m) id = s0 + j;
    }
    return id;
  }

  // Appends every entry >= t to this CTA's candidate list (warp-aggregated: one shared
  // atomic per warp and vector round; entries beyond kCandCap are counted, not stored).
  // Returns the number of entries >= t in the slice. The row holds no NaN.
  __device__ int collect_at_least(float t) {
    constexpr int P = Elem<T>::kPerVec;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) aux->ccount = 0;
    __syncthreads();
    for (int base = 0; base < nvec; base += kThreads) {
      const int v = base + threadIdx.x;
      uint32_t mask = 0;
      float x[P];
      int j0 = 0;
      if (v < nvec) {
        const uint4 w = reinterpret_cast<const uint4*>(buf)[v];
        j0 = first_elem(v);
        const bool fv = full(j0);
        if (!(fv && Elem<T>::vmax(w) < t)) {
          Elem<T>::unpack(w, x);
#pragma unroll
          for (int k = 0; k < P; ++k) {
            const int j = j0 + k;
            if ((fv || (j >= 0 && j < n)) && x[k] >= t) mask |= 1u << k;
          }
        }
      }
      const int cnt = __popc(mask);
      if (__any_sync(0xffffffffu, cnt != 0)) {
        int inc = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += u;
        }
        int wbase = 0;
        if (lane == 31) wbase = atomicAdd(&aux->ccount, inc);
        int pos = __shfl_sync(0xffffffffu, wbase, 31) + inc - cnt;
#pragma unroll
        for (int k = 0; k < P; ++k) {
          if (mask & (1u << k)) {
            if (pos < kCandCap) {
              aux->u.f.cval[pos] = x[k];
              aux->u.f.cid[pos] = s0 + j0 + k;
            }
            ++pos;
          }
        }
      }
    }
    __syncthreads();
    return aux->ccount;
  }

  template <typename U>
  __device__ __forceinline__ U* remote(U* p, int r) const {
    return cl.map_shared_rank(p, r);
  }

  // Row exchange: cluster-wide (max, lowest index on ties, OR of flags, max of t), where
  // t enters per warp and is reduced by its minimum within each CTA. Lanes 0..C-1 of
  // every warp read the C ranks' slots in parallel; no block barrier follows.
  __device__ void xchg_row(float& m, int& i, int& bad, float& t) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
      const int i2 = __shfl_xor_sync(0xffffffffu, i, o);
      maxloc_combine(m, i, m2, i2);
    }
    bad = __syncthreads_or(bad);
    if (lane == 0) {
      aux->scr_m[warp] = m;
      aux->scr_i[warp] = i;
      aux->scr_t[warp] = t;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float M = aux->scr_m[0], Tm = aux->scr_t[0];
      int I = aux->scr_i[0];
      for (int w = 1; w < kWarps; ++w) {
        maxloc_combine(M, I, aux->scr_m[w], aux->scr_i[w]);
        Tm = fminf(Tm, aux->scr_t[w]);
      }
      aux->xm[ph] = M;
      aux->xi[ph] = I;
      aux->xbad[ph] = bad;
      aux->xt[ph] = Tm;
    }
    cl.sync();
    float M = -INFINITY, Tm = -INFINITY;
    int I = INT_MAX, Bd = 0;
    if (lane < C) {
      const RowAux* ra = remote(aux, lane);
      M = ra->xm[ph];
      I = ra->xi[ph];
      Bd = ra->xbad[ph];
      Tm = ra->xt[ph];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, M, o);
      const int i2 = __shfl_xor_sync(0xffffffffu, I, o);
      maxloc_combine(M, I, m2, i2);
      Bd |= __shfl_xor_sync(0xffffffffu, Bd, o);
      Tm = fmaxf(Tm, __shfl_xor_sync(0xffffffffu, Tm, o));
    }
    m = M;
    i = I;
    bad = Bd;
    t = Tm;
    ph ^= 1;
  }

  // Cluster sums of a fixed-point mass and a float term (parallel remote reads; the
  // shuffle tree fixes the summation order).
  __device__ void xchg_sum_u64_f64(unsigned long long& a, double& b) {
    a = block_sum_u64(a, aux->scr_u64);
    b = block_sum_f64(b, aux->scr_f64);
    if (threadIdx.x == 0) {
      aux->xu64[ph] = a;
      aux->xf64[ph] = b;
    }
    cl.sync();
    const int lane = threadIdx.x & 31;
    unsigned long long s = 0;
    double t = 0.0;
    if (lane < C) {
      s = remote(aux, lane)->xu64[ph];
      t = remote(aux, lane)->xf64[ph];
    }
    a = warp_sum_u64(s);
    b = warp_sum_f64(t);
    ph ^= 1;
  }

  __device__ unsigned long long xchg_sum_u64(unsigned long long v) {
    double unused = 0.0;
    xchg_sum_u64_f64(v, unused);
    return v;
  }

  __device__ double xchg_sum_f64(double v) {
    unsigned long long unused = 0;
    xchg_sum_u64_f64(unused, v);
    return v;
  }

  __device__ long long block_sum_s64(long long v) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if (lane == 0) aux->scr_s64[warp] = v;
    __syncthreads();
    long long t = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) t += aux->scr_s64[w];
    return t;
  }

  // Warp 0 finds, over bins 255..0, the first bin b with above(b) + h[b] >= need where
  // above(b) sums the bins above b. Sets aux->found / found_bin / found_above.
  template <typename U>
  __device__ void find_desc_bin(const U* h, U need) {
    const int lane = threadIdx.x & 31;
    if (threadIdx.x >= 32) return;
    U s = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) s += h[255 - 8 * lane - k];
    U inc = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const U t = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += t;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, inc >= need);
    if (hit == 0) {
      if (lane == 0) aux->found = 0;
      return;
    }
    const int L = __ffs(hit) - 1;
    if (lane == L) {
      U acc = inc - s;
      for (int k = 0; k < 8; ++k) {
        const int b = 255 - 8 * lane - k;
        if (acc + h[b] >= need) {
          aux->found_bin = b;
          aux->found_above = (unsigned long long)acc;
          aux->found = 1;
          break;
        }
        acc += h[b];
      }
    }
  }

  // Global id of the t-th (1-based, ascending id) entry of the row with key == key0
  // and id <= id_cap. The caller guarantees it exists.
  __device__ int nth_match(uint32_t key0, int id_cap, uint32_t t) {
    constexpr int P = Elem<T>::kPerVec;
    uint32_t cnt = 0;
    each([&](int id, float x) { cnt += (Elem<T>::key(x) == key0 && id <= id_cap) ? 1u : 0u; });
    cnt = block_sum_u32(cnt, aux->scr_u32);
    if (threadIdx.x == 0) aux->xcnt[ph] = cnt;
    cl.sync();
    uint32_t before = 0;
    int owner = -1;
    for (int r = 0; r < C; ++r) {
      const uint32_t cr = remote(aux, r)->xcnt[ph];
      if (owner < 0 && before + cr >= t) owner = r;
      if (owner < 0) before += cr;
    }
    const int me = int(cl.block_rank());
    const int slot = ph;
    ph ^= 1;
    if (owner < 0) {  // unreachable when the caller's count is right: keep every tie
      cl.sync();
      ph ^= 1;
      return id_cap;
    }
    if (me == owner) {
      const uint32_t want = t - before;
      uint32_t base = 0;
      for (int v0 = 0; v0 < nvec; v0 += kThreads) {
        const int v = v0 + threadIdx.x;
        float x[P];
        int j0 = 0;
        uint32_t c = 0;
        if (v < nvec) {
          const uint4 w = reinterpret_cast<const uint4*>(buf)[v];
          Elem<T>::unpack(w, x);
          j0 = first_elem(v);
#pragma unroll
          for (int k = 0; k < P; ++k) {
            const int j = j0 + k;
            c += (j >= 0 && j < n && Elem<T>::key(x[k]) == key0 && s0 + j <= id_cap) ? 1u : 0u;
          }
        }
        uint32_t total;
        const uint32_t ex = block_exclusive_scan<uint32_t>(c, aux->scr_u32, &total);
        if (c > 0 && base + ex < want && want <= base + ex + c) {
          uint32_t seen = base + ex;
#pragma unroll
          for (int k = 0; k < P; ++k) {
            const int j = j0 + k;
            if (j >= 0 && j < n && Elem<T>::key(x[k]) == key0 && s0 + j <= id_cap) {
              if (++seen == want) aux->xid[slot] = s0 + j;
            }
          }
        }
        base += total;
        if (base >= want) break;
      }
    }
    cl.sync();
    const int id = remote(aux, owner)->xid[slot];
    ph ^= 1;
    return id;
  }

  // ---------------------------------------------------------------- generic selection
  // Top-k by count over the whole slice: boundary key and cutoff id of the k-th entry in
  // (value desc, id asc) order.
  __device__ void radix_topk(int k, uint32_t& thr, int& cut) {
    constexpr int KB = Elem<T>::kKeyBits;
    uint32_t prefix = 0, pmask = 0, need = uint32_t(k), cnt_eq = 0;
    for (int shift = KB - 8; shift >= 0; shift -= 8) {
      uint32_t* h = aux->u.g.hcnt[ph];
      for (int i = threadIdx.x; i < 256; i += kThreads) h[i] = 0;
      __syncthreads();
      each([&](int, float x) {
        const uint32_t key = Elem<T>::key(x);
        if ((key & pmask) == prefix) atomicAdd(&h[(key >> shift) & 255u], 1u);
      });
      __syncthreads();
      cl.sync();
      {
        uint32_t s = 0;
        for (int r = 0; r < C; ++r) s += remote(aux->u.g.hcnt[ph], r)[threadIdx.x];
        aux->u.g.tot_cnt[threadIdx.x] = s;
      }
      __syncthreads();
      find_desc_bin<uint32_t>(aux->u.g.tot_cnt, need);
      __syncthreads();
      const uint32_t b = uint32_t(aux->found_bin);
      need -= uint32_t(aux->found_above);
      prefix |= b << shift;
      pmask |= 255u << shift;
      cnt_eq = aux->u.g.tot_cnt[b];
      ph ^= 1;
    }
    thr = prefix;
    cut = (need == cnt_eq) ? INT_MAX : nth_match(prefix, INT_MAX, need);
  }

  // Exact fixed-point normaliser of the kept set (one rounding per entry).
  __device__ unsigned long long kept_mass(float c, float mc, uint32_t thr, int cut) {
    unsigned long long zs = 0;
    each([&](int id, float x) {
      if (kept(Elem<T>::key(x), id, thr, cut)) zs += to_fx(weight(x, c, mc));
    });
    return xchg_sum_u64(zs);
  }

  // Top-p by mass inside the kept set (thr, cut): updates thr, cut and the normaliser.
  __device__ void radix_topp(float top_p, float c, float mc, uint32_t& thr, int& cut,
                             unsigned long long& zfx) {
    constexpr int KB = Elem<T>::kKeyBits;
    unsigned long long target = (unsigned long long)ceil(double(top_p) * double(zfx));
    if (target < 1) target = 1;  // the top entry alone always reaches a tiny top_p
    const uint32_t thr_k = thr;
    const int cut_k = cut;
    uint32_t prefix = 0, pmask = 0, cnt_eq = 0;
    unsigned long long before = 0, mass_eq = 0;
    for (int shift = KB - 8; shift >= 0; shift -= 8) {
      uint32_t* hc = aux->u.g.hcnt[ph];
      uint32_t* hl = aux->u.g.hlimb[ph];
      for (int i = threadIdx.x; i < 256; i += kThreads) hc[i] = 0;
      for (int i = threadIdx.x; i < 3 * 256; i += kThreads) hl[i] = 0;
      __syncthreads();
      each([&](int id, float x) {
        const uint32_t key = Elem<T>::key(x);
        if ((key & pmask) == prefix && kept(key, id, thr_k, cut_k)) {
          const uint32_t bin = (key >> shift) & 255u;
          atomicAdd(&hc[bin], 1u);
          limb_add(hl, 256, int(bin), to_fx(weight(x, c, mc)));
        }
      });
      __syncthreads();
      cl.sync();
      {
        uint32_t sc = 0;
        unsigned long long sm = 0;
        for (int r = 0; r < C; ++r) {
          sc += remote(aux->u.g.hcnt[ph], r)[threadIdx.x];
          sm += limb_get(remote(aux->u.g.hlimb[ph], r), 256, int(threadIdx.x));
        }
        aux->u.g.tot_cnt[threadIdx.x] = sc;
        aux->u.g.tot_mass[threadIdx.x] = sm;
      }
      __syncthreads();
      find_desc_bin<unsigned long long>(aux->u.g.tot_mass, target - before);
      __syncthreads();
      ph ^= 1;
      if (!aux->found) return;  // rounding left the kept set short of top_p: keep it all
      const uint32_t b = uint32_t(aux->found_bin);
      before += aux->found_above;
      prefix |= b << shift;
      pmask |= 255u << shift;
      cnt_eq = aux->u.g.tot_cnt[b];
      mass_eq = aux->u.g.tot_mass[b];
    }
    const unsigned long long e_fx = mass_eq / cnt_eq;  // equal keys carry equal masses
    unsigned long long t = (target - before + e_fx - 1) / e_fx;
    t = t < 1 ? 1 : (t > cnt_eq ? cnt_eq : t);
    const int cap = (prefix == thr_k) ? cut_k : INT_MAX;
    thr = prefix;
    cut = (t == cnt_eq) ? cap : nth_match(prefix, cap, uint32_t(t));
    zfx = before + t * e_fx;
  }

  // ---------------------------------------------------------------- top-k fast path
  // t0 is a value that at least k entries of the row reach. Collects the entries >= t0,
  // gathers them in every CTA, and selects the top k among them exactly. Returns false
  // (uniformly across the cluster) when the candidates do not fit; the caller then runs
  // radix_topk. On success rank 0 of the cluster lists the kept ids.
  __device__ bool filter_topk(int k, float t0, float c, float mc, bool want_ent, uint32_t& thr,
                              int& cut, unsigned long long& zfx, double& S1, int32_t* ids_out,
                              int32_t* n_out) {
    constexpr int KB = Elem<T>::kKeyBits;
    const int lane = threadIdx.x & 31;
    const int mine = collect_at_least(t0);
    if (threadIdx.x == 0) aux->xcnt[ph] = uint32_t(mine);
    cl.sync();
    if (threadIdx.x < 32) {  // counts of every rank -> offsets
      const int cq = lane < C ? int(remote(aux, lane)->xcnt[ph]) : 0;
      int inc = cq;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += u;
      }
      const unsigned big = __ballot_sync(0xffffffffu, cq > kCandCap);
      if (lane <= C) aux->cnt_off[lane] = inc - cq;  // lane C holds the total
      if (lane == 0) aux->found = big ? 1 : 0;
    }
    ph ^= 1;
    __syncthreads();
    const int total = aux->cnt_off[C];
    if (aux->found || total < k || total > kGatherCap) return false;
    // every CTA gathers the cluster's candidates (one remote load per candidate)
    for (int i = threadIdx.x; i < total; i += kThreads) {
      int q = 0;
      while (i >= aux->cnt_off[q + 1]) ++q;
      const RowAux* ra = remote(aux, q);
      aux->u.f.gval[i] = ra->u.f.cval[i - aux->cnt_off[q]];
      aux->u.f.gid[i] = ra->u.f.cid[i - aux->cnt_off[q]];
    }
    __syncthreads();
    // k-th largest key among the candidates (every entry >= t0 is one, so this is the
    // row's k-th largest value)
    uint32_t prefix = 0, pmask = 0, need = uint32_t(k), cnt_eq = 0;
    for (int shift = KB - 8; shift >= 0; shift -= 8) {
      aux->lh[threadIdx.x] = 0;
      __syncthreads();
      for (int i = threadIdx.x; i < total; i += kThreads) {
        const uint32_t key = Elem<T>::key(aux->u.f.gval[i]);
        if ((key & pmask) == prefix) atomicAdd(&aux->lh[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      find_desc_bin<uint32_t>(aux->lh, need);
      __syncthreads();
      const uint32_t b = uint32_t(aux->found_bin);
      need -= uint32_t(aux->found_above);
      prefix |= b << shift;
      pmask |= 255u << shift;
      cnt_eq = aux->lh[b];
      __syncthreads();
    }
    thr = prefix;
    cut = INT_MAX;
    if (need < cnt_eq) {  // keep the `need` lowest ids among the entries equal to the k-th
      for (int i = threadIdx.x; i < total; i += kThreads) {
        if (Elem<T>::key(aux->u.f.gval[i]) != prefix) continue;
        const int ii = aux->u.f.gid[i];
        uint32_t below = 0;
        for (int q = 0; q < total; ++q)
          below += (Elem<T>::key(aux->u.f.gval[q]) == prefix && aux->u.f.gid[q] < ii) ? 1u : 0u;
        if (below == need - 1) aux->sel_id = ii;
      }
      __syncthreads();
      cut = aux->sel_id;
    }
    // normaliser and entropy term over the kept entries; fixed-point sums do not depend
    // on the order the candidates arrived in
    unsigned long long z = 0;
    long long s1 = 0;
    const bool list = ids_out != nullptr && cl.block_rank() == 0;
    if (threadIdx.x == 0) aux->ccount = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < total; i += kThreads) {
      const float xi = aux->u.f.gval[i];
      if (!kept(Elem<T>::key(xi), aux->u.f.gid[i], thr, cut)) continue;
      const float zx = wexp(xi, c, mc);
      const float e = ex2(zx);
      z += to_fx(e);
      if (want_ent) s1 += __float2ll_rn(ent_term(e, zx) * kS1Fx);
      if (list) ids_out[atomicAdd(&aux->ccount, 1)] = aux->u.f.gid[i];
    }
    zfx = block_sum_u64(z, aux->scr_u64);
    S1 = double(block_sum_s64(s1)) / double(kS1Fx);
    if (list && threadIdx.x == 0) *n_out = k;
    return true;
  }
};

// j-th largest (1 <= j <= 32) of the keys the 32 lanes pass in (ballot radix select).
template <int KB>
__device__ __forceinline__ uint32_t warp_kth_key(uint32_t key, int j) {
  uint32_t prefix = 0;
  int need = j;
#pragma unroll
  for (int b = KB - 1; b >= 0; --b) {
    const uint32_t cand = prefix | (1u << b);
    const int cnt = __popc(__ballot_sync(0xffffffffu, (key >> b) == (cand >> b)));
    if (cnt >= need)
      prefix = cand;
    else
      need -= cnt;
  }
  return prefix;
}

template <typename T>
__device__ __forceinline__ float key_value(uint32_t k) {
  if (Elem<T>::kKeyBits == 16)
    return __uint_as_float(((k & 0x8000u) ? (k & 0x7FFFu) : (~k & 0xFFFFu)) << 16);
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// One row: every CTA of the cluster holds its slice in ctx.buf.
template <typename T>
__device__ void process_row(RowCtx<T>& ctx, const RowJob& job, long long row, bool copied) {
  const int V = job.V;
  const int rank = int(ctx.cl.block_rank());
  const bool greedy = (job.flags & RS_GREEDY) != 0;
  const bool want_ent = (job.flags & RS_ENTROPY) != 0;
  const bool topk = !greedy && job.top_k >= 1 && job.top_k < V;
  const bool topp = !greedy && job.top_p < 1.0f;
  const int jw = (job.top_k + kWarps - 1) / kWarps;  // per-warp order statistic for t0
  const bool fast_topk = topk && !topp && jw <= 32;

  // ---- maximum (with its lowest index in greedy mode) and validity
  int vbest = -1;
  const float mt = copied ? ctx.thread_max(&vbest) : -INFINITY;  // NaN if this thread saw one
  int bad = copied ? ((mt != mt || mt == INFINITY) ? 1 : 0) : 2;
  float m = (mt != mt) ? -INFINITY : mt;
  int am = greedy ? ctx.first_equal(vbest, m) : INT_MAX;
  // top-k: each warp's jw-th largest per-thread maximum; a CTA's smallest warp value is
  // reached by >= 8 * jw >= k of its entries, so the cluster's largest such value is t0
  float t0 = -INFINITY;
  if (fast_topk) t0 = key_value<T>(warp_kth_key<Elem<T>::kKeyBits>(Elem<T>::key(m), jw));
  ctx.xchg_row(m, am, bad, t0);
  const int status = (bad & 2) ? ROW_TIMEOUT : ((bad & 1) || m == -INFINITY) ? ROW_INVALID : ROW_OK;
  if ((bad & 2) && job.dev_status && threadIdx.x == 0) atomicOr(job.dev_status, 1);

  const float c = job.c;
  const float mc = m * c;
  uint32_t thr = 0;
  int cut = INT_MAX;
  unsigned long long zfx = 0;
  double S1 = 0.0;  // sum over the kept set of weight * (l - m) * c  (log2 units)
  bool have_s1 = false;
  bool listed = false;

  if (status == ROW_OK && !greedy) {
    if (!topk && !topp) {
      // ---- no truncation: one exp pass for the normaliser (and the entropy term)
      float s_a = 0.0f, s_b = 0.0f, h = 0.0f;
      if (want_ent) {
        ctx.each([&](int, float x) {
          const float zx = wexp(x, c, mc);
          const float e = ex2(zx);
          s_a += e;
          h += ent_term(e, zx);
        });
      } else {
        constexpr int P = Elem<T>::kPerVec;
        for (int v = threadIdx.x; v < ctx.nvec; v += kThreads) {
          const uint4 w = reinterpret_cast<const uint4*>(ctx.buf)[v];
          float x[P];
          Elem<T>::unpack(w, x);
          const int j0 = ctx.first_elem(v);
          if (ctx.full(j0)) {
#pragma unroll
            for (int k = 0; k < P; k += 2) {
              s_a += weight(x[k], c, mc);
              s_b += weight(x[k + 1], c, mc);
            }
          } else {
#pragma unroll
            for (int k = 0; k < P; ++k) {
              const int j = j0 + k;
              if (j >= 0 && j < ctx.n) s_a += weight(x[k], c, mc);
            }
          }
        }
      }
      unsigned long long zt = to_fx(s_a + s_b);
      double ht = double(h);
      ctx.xchg_sum_u64_f64(zt, ht);
      zfx = zt;
      S1 = ht;
      have_s1 = true;
    } else {
      bool done = false;
      if (fast_topk) {
        int32_t* ids = (job.kept_ids && job.top_k <= kKeptCap)
                           ? job.kept_ids + size_t(row) * kKeptCap
                           : nullptr;
        done = ctx.filter_topk(job.top_k, t0, c, mc, want_ent, thr, cut, zfx, S1, ids,
                               job.kept_n ? job.kept_n + row : nullptr);
        listed = done && ids != nullptr;
      }
      if (done) {
        have_s1 = true;
      } else {
        if (topk) ctx.radix_topk(job.top_k, thr, cut);
        zfx = ctx.kept_mass(c, mc, thr, cut);
        if (topp) ctx.radix_topp(job.top_p, c, mc, thr, cut, zfx);
      }
    }
    if (want_ent && !have_s1) {
      float h = 0.0f;
      ctx.each([&](int id, float x) {
        if (kept(Elem<T>::key(x), id, thr, cut)) {
          const float zx = wexp(x, c, mc);
          h += ent_term(ex2(zx), zx);
        }
      });
      S1 = ctx.xchg_sum_f64(double(h));
    }
  }
  if (!listed && job.kept_n && rank == 0 && threadIdx.x == 0) job.kept_n[row] = 0;
  // a top-p boundary this kernel placed with fp32 masses: re-decided in double afterwards
  if (status == ROW_OK && topp && !topk && job.refine_rows && rank == 0 && threadIdx.x == 0) {
    const int li = atomicAdd(job.refine_count, 1);
    job.refine_rows[li] = int32_t(row);
    job.refine_z[2 * li] = 0ull;
    job.refine_z[2 * li + 1] = 0ull;
  }

  const double Z = double(zfx) * kFxInv;
  const double ent = (status == ROW_OK && !greedy && want_ent)
                         ? log(Z) - 0.6931471805599453 * S1 / Z
                         : 0.0;
  const float zf = float(Z);
  if (job.stats && rank == 0 && threadIdx.x == 0) {
    RowStats st;
    st.mc = mc;
    st.z = zf;
    st.entropy = float(ent);
    st.thr_key = thr;
    st.cutoff = cut;
    st.argmax = greedy ? am : -1;
    st.status = status;
    st.c = c;
    st.m = m;
    st.pad = 0;
    st.zd = -1.0;  // the consumer sums the double normaliser when it needs it
    job.stats[row] = st;
  }
  if (job.flags & RS_WRITE_PROBS) {
    float* out = job.probs + size_t(row) * V;
    if (status != ROW_OK) {
      for (int j = threadIdx.x; j < ctx.n; j += kThreads) out[ctx.s0 + j] = NAN;
    } else if (greedy) {
      for (int j = threadIdx.x; j < ctx.n; j += kThreads) out[ctx.s0 + j] = (ctx.s0 + j == am);
    } else {
      ctx.each([&](int id, float x) {
        out[id] = kept(Elem<T>::key(x), id, thr, cut) ? weight(x, c, mc) / zf : 0.0f;
      });
    }
    if (job.entropy && rank == 0 && threadIdx.x == 0)
      job.entropy[row] = status != ROW_OK ? NAN : (greedy ? 0.0f : float(ent));
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) row_stats_kernel(const RowJob job) {
  extern __shared__ __align__(128) unsigned char ring[];
  __shared__ RowAux aux;
  RowCtx<T> ctx{ring, 0, 0, 0, 0, &aux, cg::this_cluster(), 0, 0};
  ctx.C = int(ctx.cl.num_blocks());
  const int rank = int(ctx.cl.block_rank());
  const long long cid = blockIdx.x / ctx.C;
  const long long G = gridDim.x / ctx.C;
  if (threadIdx.x == 0) {
    for (int b = 0; b < kNBuf; ++b) mbar_init(&aux.bar[b], 1);
    aux.broken = 0;
    aux.pending = 0;
  }
  __syncthreads();
  auto buffer = [&](long long it) { return ring + size_t(it % kNBuf) * job.slice_bytes; };
  // rows: all of them, or the listed ones (rows another kernel could not settle)
  const long long nrows = job.row_list ? (long long)*job.row_count : job.rows;
  auto row_of = [&](long long li) { return job.row_list ? (long long)job.row_list[li] : li; };
  // prologue: the first kNBuf - 1 rows of this cluster
  if (threadIdx.x == 0) {
    for (int it = 0; it < kNBuf - 1; ++it) {
      const long long li = cid + it * G;
      if (li >= nrows) break;
      const SliceLoc s = slice_loc<T>(job, row_of(li), rank);
      if (s.n > 0) {
        issue_slice(s, buffer(it), &aux.bar[it % kNBuf]);
        aux.pending |= 1 << (it % kNBuf);
      }
    }
  }
  for (long long it = 0;; ++it) {
    const long long li = cid + it * G;
    if (li >= nrows) break;
    const long long row = row_of(li);
    // keep kNBuf - 1 rows in flight: the buffer refilled here was last read by
    // iteration it - 1, which every thread of this CTA has finished
    if (threadIdx.x == 0 && !aux.broken) {
      const long long ahead = it + kNBuf - 1;
      const long long ali = cid + ahead * G;
      if (ali < nrows) {
        const SliceLoc s = slice_loc<T>(job, row_of(ali), rank);
        if (s.n > 0) {
          issue_slice(s, buffer(ahead), &aux.bar[ahead % kNBuf]);
          aux.pending |= 1 << (ahead % kNBuf);
        }
      }
    }
    __syncthreads();
    const SliceLoc s = slice_loc<T>(job, row, rank);
    const int b = int(it % kNBuf);
    bool copied = true;
    if (s.n > 0) {
      if (!aux.broken && (aux.pending & (1 << b))) {
        copied = finish_slice<T>(s, buffer(it), &aux.bar[b], uint32_t((it / kNBuf) & 1));
        if (threadIdx.x == 0) {
          if (copied)
            aux.pending &= ~(1 << b);
          else
            aux.broken = 1;
        }
      } else {
        copied = false;  // an earlier copy timed out: this row is reported, not read
      }
    }
    ctx.buf = buffer(it);
    ctx.s0 = rank * job.slice;
    ctx.n = s.n;
    ctx.pad = s.pad;
    ctx.nvec = s.n > 0 ? (s.pad + s.n * Elem<T>::kBytes + 15) >> 4 : 0;
    process_row<T>(ctx, job, row, copied);
    __syncthreads();
  }
  // a copy that timed out may still land: give each one more bounded wait
  if (aux.broken && threadIdx.x == 0) {
    for (int b = 0; b < kNBuf; ++b)
      if (aux.pending & (1 << b)) {
        if (!mbar_wait(&aux.bar[b], 0)) mbar_wait(&aux.bar[b], 1);
      }
  }
  ctx.cl.sync();  // no CTA leaves while a peer may still read its shared memory
}

}  // namespace sv
