// Row statistics kernel: one thread-block cluster per logit row.
//
// Each CTA of the cluster stages a contiguous slice of the row in shared memory with
// 1-D bulk copies (cp.async.bulk, completion on an mbarrier); the cluster then combines
// its partial results through distributed shared memory (DSMEM):
//   - the row maximum (packed bf16x2 max with NaN propagation) and row validity;
//   - greedy: the lowest index holding the maximum;
//   - no truncation: the softmax normaliser (and entropy) in one exp pass;
//   - top-k (fast path, k <= 256): t0 = the largest over the cluster's CTAs of each
//     CTA's k-th largest per-thread maximum, so at least k entries reach t0; a filter
//     pass keeps the few entries >= t0, every CTA gathers them and selects the top k
//     exactly with a local radix select — no exp over the row;
//   - otherwise (top-p, or a fast path that does not apply): exact selection by radix
//     select over order-preserving keys, 8 bits per level, with fixed-point masses.
// It stores a RowStats record or writes the transformed probabilities.
//
// This is the sampling transform of "Speculative Sampling" (spec-decoding-i notes, last
// bullet: transform the probabilities first, then apply the rejection scheme) and the
// entropy that MEDUSA typical acceptance uses ("Key Components").
#pragma once

#include <climits>

#include "common.cuh"

namespace sv {

enum : int { RS_GREEDY = 1, RS_ENTROPY = 2, RS_WRITE_PROBS = 4 };

constexpr int kBulkChunk = 16384;
constexpr int kCandCap = 512;      // candidates one CTA may hold in the top-k filter
constexpr int kGatherCap = 1024;   // candidates a cluster may hold for exact selection
constexpr float kS1Fx = 4294967296.0f;  // 2^32: signed fixed point for entropy terms

struct RowJob {
  const void* base0;   // rows [0, rows0)
  const void* base1;   // rows [rows0, rows)
  long long rows0;
  long long rows;
  int V;
  int slice;           // elements per CTA slice (multiple of 16)
  float c;             // log2(e) / T   (unused in greedy mode)
  float inv_t;         // 1 / T
  int top_k;           // 1 <= top_k < V, else off
  float top_p;         // < 1: on
  int flags;
  RowStats* stats;     // [rows] or NULL
  float* probs;        // RS_WRITE_PROBS: [rows][V]
  float* entropy;      // RS_WRITE_PROBS: [rows] or NULL
  int32_t* dev_status; // set to 1 on a copy timeout (may be NULL)
};

struct __align__(16) RowAux {
  uint64_t bar;
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
      unsigned long long hmass[2][256];
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
  long long scr_s64[kWarps];
  uint32_t lh[256];  // CTA-local histogram
  int found_bin;
  int found;
  unsigned long long found_above;
  int ccount;
  uint32_t sel_key;
  int sel_id;
};

// Stages n elements starting at g into buf; element j lands at byte pad + j * E with
// pad = g mod 16, so the 16-byte-aligned middle of the slice moves by bulk copy and
// the unaligned head and tail (< 16 bytes each) by plain loads. Returns false if the
// copy did not complete within the wait limit.
template <typename T>
__device__ bool stage_slice(const T* g, int n, unsigned char* buf, uint64_t* bar, int* pad_out) {
  constexpr int E = Elem<T>::kBytes;
  const uintptr_t a = reinterpret_cast<uintptr_t>(g);
  const int pad = int(a & 15u);
  const int bytes = n * E;
  const int head = min(bytes, (16 - pad) & 15);
  const int mid = ((bytes - head) >> 4) << 4;
  const int tail = bytes - head - mid;
  *pad_out = pad;
  if (threadIdx.x == 0) mbar_init(bar, 1);
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar, uint32_t(mid));
    const char* gs = reinterpret_cast<const char*>(g) + head;
    unsigned char* d = buf + pad + head;
    for (int off = 0; off < mid; off += kBulkChunk)
      bulk_g2s(d + off, gs + off, uint32_t(min(kBulkChunk, mid - off)), bar);
  }
  const int hE = head / E, tE = tail / E;
  for (int j = threadIdx.x; j < hE + tE; j += kThreads) {
    const int e = (j < hE) ? j : (n - tE + (j - hE));
    if (E == 2)
      reinterpret_cast<uint16_t*>(buf + pad)[e] = reinterpret_cast<const uint16_t*>(g)[e];
    else
      reinterpret_cast<uint32_t*>(buf + pad)[e] = reinterpret_cast<const uint32_t*>(g)[e];
  }
  bool ok = mbar_wait(bar, 0);
  if (!ok) mbar_wait(bar, 0);  // give an in-flight copy one more bounded chance to land
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

  // k-th largest (1 <= k <= kThreads) of the keys the block's threads pass in, by an
  // 8-bit-per-level radix select over a CTA-local histogram.
  __device__ uint32_t block_kth_key(uint32_t key, int k) {
    constexpr int KB = Elem<T>::kKeyBits;
    uint32_t prefix = 0, pmask = 0, need = uint32_t(k);
    for (int shift = KB - 8; shift >= 0; shift -= 8) {
      aux->lh[threadIdx.x] = 0;
      __syncthreads();
      if ((key & pmask) == prefix) atomicAdd(&aux->lh[(key >> shift) & 255u], 1u);
      __syncthreads();
      find_desc_bin<uint32_t>(aux->lh, need);
      __syncthreads();
      need -= uint32_t(aux->found_above);
      prefix |= uint32_t(aux->found_bin) << shift;
      pmask |= 255u << shift;
      __syncthreads();
    }
    return prefix;
  }

  template <typename U>
  __device__ __forceinline__ U* remote(U* p, int r) const {
    return cl.map_shared_rank(p, r);
  }

  // Cluster-wide (max, lowest index, OR of flags, max of t).
  __device__ void xchg_maxloc(float& m, int& i, int& bad, float& t) {
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
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float M = aux->scr_m[0];
      int I = aux->scr_i[0];
      for (int w = 1; w < kWarps; ++w) maxloc_combine(M, I, aux->scr_m[w], aux->scr_i[w]);
      aux->xm[ph] = M;
      aux->xi[ph] = I;
      aux->xbad[ph] = bad;
      aux->xt[ph] = t;
    }
    cl.sync();
    float M = -INFINITY, Tm = -INFINITY;
    int I = INT_MAX, Bd = 0;
    for (int r = 0; r < C; ++r) {
      const RowAux* ra = remote(aux, r);
      maxloc_combine(M, I, ra->xm[ph], ra->xi[ph]);
      Bd |= ra->xbad[ph];
      Tm = fmaxf(Tm, ra->xt[ph]);
    }
    m = M;
    i = I;
    bad = Bd;
    t = Tm;
    ph ^= 1;
  }

  // Cluster-wide minimum (each thread passes a value; NaN never occurs here).
  __device__ float xchg_min(float v) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if (lane == 0) aux->scr_m[warp] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
      float M = aux->scr_m[0];
      for (int w = 1; w < kWarps; ++w) M = fminf(M, aux->scr_m[w]);
      aux->xm[ph] = M;
    }
    cl.sync();
    float M = INFINITY;
    for (int r = 0; r < C; ++r) M = fminf(M, remote(aux, r)->xm[ph]);
    ph ^= 1;
    return M;
  }

  // Cluster-wide minimum of an int (the lowest index of something).
  __device__ int xchg_min_int(int v) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if (lane == 0) aux->scr_i[warp] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
      int M = aux->scr_i[0];
      for (int w = 1; w < kWarps; ++w) M = min(M, aux->scr_i[w]);
      aux->xi[ph] = M;
    }
    cl.sync();
    int M = INT_MAX;
    for (int r = 0; r < C; ++r) M = min(M, remote(aux, r)->xi[ph]);
    ph ^= 1;
    return M;
  }

  __device__ unsigned long long xchg_sum_u64(unsigned long long v) {
    v = block_sum_u64(v, aux->scr_u64);
    if (threadIdx.x == 0) aux->xu64[ph] = v;
    cl.sync();
    unsigned long long s = 0;
    for (int r = 0; r < C; ++r) s += remote(aux, r)->xu64[ph];
    ph ^= 1;
    return s;
  }

  // Two sums in one exchange (fixed-point mass and float entropy term).
  __device__ void xchg_sum_u64_f64(unsigned long long& a, double& b) {
    a = block_sum_u64(a, aux->scr_u64);
    b = block_sum_f64(b, aux->scr_f64);
    if (threadIdx.x == 0) {
      aux->xu64[ph] = a;
      aux->xf64[ph] = b;
    }
    cl.sync();
    unsigned long long s = 0;
    double t = 0.0;
    for (int r = 0; r < C; ++r) {
      s += remote(aux, r)->xu64[ph];
      t += remote(aux, r)->xf64[ph];
    }
    a = s;
    b = t;
    ph ^= 1;
  }

  __device__ double xchg_sum_f64(double v) {
    v = block_sum_f64(v, aux->scr_f64);
    if (threadIdx.x == 0) aux->xf64[ph] = v;
    cl.sync();
    double s = 0.0;
    for (int r = 0; r < C; ++r) s += remote(aux, r)->xf64[ph];
    ph ^= 1;
    return s;
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
      unsigned long long* hm = aux->u.g.hmass[ph];
      for (int i = threadIdx.x; i < 256; i += kThreads) {
        hc[i] = 0;
        hm[i] = 0;
      }
      __syncthreads();
      each([&](int id, float x) {
        const uint32_t key = Elem<T>::key(x);
        if ((key & pmask) == prefix && kept(key, id, thr_k, cut_k)) {
          const uint32_t bin = (key >> shift) & 255u;
          atomicAdd(&hc[bin], 1u);
          atomicAdd(&hm[bin], to_fx(weight(x, c, mc)));
        }
      });
      __syncthreads();
      cl.sync();
      {
        uint32_t sc = 0;
        unsigned long long sm = 0;
        for (int r = 0; r < C; ++r) {
          sc += remote(aux->u.g.hcnt[ph], r)[threadIdx.x];
          sm += remote(aux->u.g.hmass[ph], r)[threadIdx.x];
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
  // t0 is a lower bound on the row's k-th largest value (some CTA holds k entries >= t0).
  // Collects the entries >= t0, gathers them in every CTA, and selects the top k among
  // them exactly. Returns false (uniformly across the cluster) when the candidates do not
  // fit; the caller then runs radix_topk.
  __device__ bool filter_topk(int k, float t0, float c, float mc, bool want_ent, uint32_t& thr,
                              int& cut, unsigned long long& zfx, double& S1) {
    constexpr int KB = Elem<T>::kKeyBits;
    const int mine = collect_at_least(t0);
    if (threadIdx.x == 0) aux->xcnt[ph] = uint32_t(mine);
    cl.sync();
    int total = 0, ovf = 0;
    for (int q = 0; q < C; ++q) {
      const int cq = int(remote(aux, q)->xcnt[ph]);
      ovf |= cq > kCandCap;
      total += cq;
    }
    const int slot = ph;
    ph ^= 1;
    if (ovf || total < k || total > kGatherCap) return false;
    // every CTA gathers the cluster's candidates
    for (int i = threadIdx.x; i < total; i += kThreads) {
      int q = 0, base = 0;
      for (;; ++q) {
        const int cq = int(remote(aux, q)->xcnt[slot]);
        if (i < base + cq) break;
        base += cq;
      }
      const RowAux* ra = remote(aux, q);
      aux->u.f.gval[i] = ra->u.f.cval[i - base];
      aux->u.f.gid[i] = ra->u.f.cid[i - base];
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
      if (threadIdx.x == 0) aux->sel_id = INT_MAX;
      __syncthreads();
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
    for (int i = threadIdx.x; i < total; i += kThreads) {
      const float xi = aux->u.f.gval[i];
      if (!kept(Elem<T>::key(xi), aux->u.f.gid[i], thr, cut)) continue;
      const float zx = wexp(xi, c, mc);
      const float e = ex2(zx);
      z += to_fx(e);
      if (want_ent) s1 += __float2ll_rn(e * zx * kS1Fx);
    }
    zfx = block_sum_u64(z, aux->scr_u64);
    S1 = double(block_sum_s64(s1)) / double(kS1Fx);
    return true;
  }
};

template <typename T>
__global__ void __launch_bounds__(kThreads) row_stats_kernel(const RowJob job) {
  extern __shared__ __align__(128) unsigned char slice_buf[];
  __shared__ RowAux aux;
  RowCtx<T> ctx{slice_buf, 0, 0, 0, 0, &aux, cg::this_cluster(), 0, 0};
  ctx.C = int(ctx.cl.num_blocks());
  const int rank = int(ctx.cl.block_rank());
  const long long row = blockIdx.x / ctx.C;
  const int V = job.V;
  const T* src = (row < job.rows0)
                     ? static_cast<const T*>(job.base0) + size_t(row) * V
                     : static_cast<const T*>(job.base1) + size_t(row - job.rows0) * V;
  ctx.s0 = rank * job.slice;
  ctx.n = max(0, min(V - ctx.s0, job.slice));
  bool copied = true;
  if (ctx.n > 0) {
    copied = stage_slice<T>(src + ctx.s0, ctx.n, slice_buf, &aux.bar, &ctx.pad);
    ctx.nvec = (ctx.pad + ctx.n * Elem<T>::kBytes + 15) >> 4;
  }

  const bool greedy = (job.flags & RS_GREEDY) != 0;
  const bool want_ent = (job.flags & RS_ENTROPY) != 0;
  const bool topk = !greedy && job.top_k >= 1 && job.top_k < V;
  const bool topp = !greedy && job.top_p < 1.0f;
  const bool fast_topk = topk && !topp && job.top_k <= kThreads;

  // ---- maximum (with its lowest index in greedy mode) and validity
  int vbest = -1;
  const float mt = copied ? ctx.thread_max(&vbest) : -INFINITY;  // NaN if this thread saw one
  int bad = copied ? ((mt != mt || mt == INFINITY) ? 1 : 0) : 2;
  float m = (mt != mt) ? -INFINITY : mt;
  int am = greedy ? ctx.first_equal(vbest, m) : INT_MAX;
  // top-k: this CTA's k-th largest per-thread maximum; the largest over the cluster is
  // a value that at least k entries reach
  float t0 = -INFINITY;
  if (fast_topk) {
    const uint32_t kk = ctx.block_kth_key(Elem<T>::key(m), job.top_k);
    t0 = (Elem<T>::kKeyBits == 16)
             ? __uint_as_float(((kk & 0x8000u) ? (kk & 0x7FFFu) : (~kk & 0xFFFFu)) << 16)
             : __uint_as_float((kk & 0x80000000u) ? (kk & 0x7FFFFFFFu) : ~kk);
  }
  ctx.xchg_maxloc(m, am, bad, t0);
  const int status = (bad & 2) ? ROW_TIMEOUT : ((bad & 1) || m == -INFINITY) ? ROW_INVALID : ROW_OK;
  if ((bad & 2) && job.dev_status && threadIdx.x == 0) atomicOr(job.dev_status, 1);

  const float c = job.c;
  const float mc = m * c;
  uint32_t thr = 0;
  int cut = INT_MAX;
  unsigned long long zfx = 0;
  double S1 = 0.0;  // sum over the kept set of weight * (l - m) * c  (log2 units)
  bool have_s1 = false;

  if (status == ROW_OK && greedy) {
    // the lowest index holding the maximum came with the exchange
  } else if (status == ROW_OK) {
    if (!topk && !topp) {
      // ---- no truncation: one exp pass for the normaliser (and the entropy term)
      float s_a = 0.0f, s_b = 0.0f, h = 0.0f;
      if (want_ent) {
        ctx.each([&](int, float x) {
          const float zx = wexp(x, c, mc);
          const float e = ex2(zx);
          s_a += e;
          h = fmaf(e, zx, h);
        });
      } else {
        constexpr int P = Elem<T>::kPerVec;
        for (int v = threadIdx.x; v < ctx.nvec; v += kThreads) {
          const uint4 w = reinterpret_cast<const uint4*>(slice_buf)[v];
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
      if (fast_topk) done = ctx.filter_topk(job.top_k, t0, c, mc, want_ent, thr, cut, zfx, S1);
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
          h = fmaf(ex2(zx), zx, h);
        }
      });
      S1 = ctx.xchg_sum_f64(double(h));
    }
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
    st.argmax = am;
    st.status = status;
    st.c = c;
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
  ctx.cl.sync();  // no CTA leaves while a peer may still read its shared memory
}

}  // namespace sv
