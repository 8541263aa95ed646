// Row statistics kernel: one thread-block cluster per logit row.
//
// Each CTA of the cluster stages a contiguous slice of the row in shared memory with
// 1-D bulk copies (cp.async.bulk, completion on an mbarrier), then the cluster
// computes, with exchanges through distributed shared memory:
//   - the row maximum and its lowest index (argmax), and row validity;
//   - top-k: the exact k-th entry in (value desc, id asc) order by a radix select
//     over order-preserving keys, 8 bits per level;
//   - the softmax normaliser over the kept set, as an exact fixed-point sum;
//   - top-p: the exact crossing entry by a mass-weighted radix select;
//   - the entropy of the transformed distribution (optional);
// and either stores a RowStats record or writes the transformed probabilities.
//
// This is the sampling transform of "Speculative Sampling" (spec-decoding-i notes,
// last bullet: transform the probabilities first, then apply the rejection scheme)
// and the entropy used by MEDUSA typical acceptance ("Key Components").
#pragma once

#include <climits>

#include "common.cuh"

namespace sv {

enum : int { RS_GREEDY = 1, RS_ENTROPY = 2, RS_WRITE_PROBS = 4 };

constexpr int kBulkChunk = 16384;

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
  float xm[2];
  int xi[2];
  int xbad[2];
  unsigned long long xu64[2];
  double xf64[2];
  uint32_t xcnt[2];
  int xid[2];
  uint32_t hcnt[2][256];
  unsigned long long hmass[2][256];
  uint32_t tot_cnt[256];
  unsigned long long tot_mass[256];
  unsigned long long scr_u64[kWarps];
  double scr_f64[kWarps];
  uint32_t scr_u32[kWarps];
  float scr_m[kWarps];
  int scr_i[kWarps];
  int found_bin;
  int found;
  unsigned long long found_above;
  int found_id;
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

  // Calls f(global id, value) for every element of this CTA's slice; each thread
  // visits its elements in ascending id order.
  template <typename F>
  __device__ __forceinline__ void each(F&& f) const {
    constexpr int P = Elem<T>::kPerVec, E = Elem<T>::kBytes;
    for (int v = threadIdx.x; v < nvec; v += kThreads) {
      const uint4 w = reinterpret_cast<const uint4*>(buf)[v];
      float x[P];
      Elem<T>::unpack(w, x);
      const int j0 = (v * 16 - pad) / E;
      if (j0 >= 0 && j0 + P <= n) {
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

  template <typename U>
  __device__ __forceinline__ U* remote(U* p, int r) const {
    return cl.map_shared_rank(p, r);
  }

  // Cluster-wide (max, lowest index, OR of flags).
  __device__ void xchg_maxloc(float& m, int& i, int& bad) {
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
    }
    cl.sync();
    float M = -INFINITY;
    int I = INT_MAX, Bd = 0;
    for (int r = 0; r < C; ++r) {
      const RowAux* ra = remote(aux, r);
      maxloc_combine(M, I, ra->xm[ph], ra->xi[ph]);
      Bd |= ra->xbad[ph];
    }
    m = M;
    i = I;
    bad = Bd;
    ph ^= 1;
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

  __device__ double xchg_sum_f64(double v) {
    v = block_sum_f64(v, aux->scr_f64);
    if (threadIdx.x == 0) aux->xf64[ph] = v;
    cl.sync();
    double s = 0.0;
    for (int r = 0; r < C; ++r) s += remote(aux, r)->xf64[ph];
    ph ^= 1;
    return s;
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
    constexpr int P = Elem<T>::kPerVec, E = Elem<T>::kBytes;
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
          j0 = (v * 16 - pad) / E;
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

  // ---- maximum, argmax and validity
  float m = -INFINITY;
  int am = INT_MAX, bad = copied ? 0 : 2;
  if (copied) {
    ctx.each([&](int id, float x) {
      if (!(x == x) || x == INFINITY) bad |= 1;
      if (x > m) {
        m = x;
        am = id;
      }
    });
  }
  ctx.xchg_maxloc(m, am, bad);
  const int status = (bad & 2) ? ROW_TIMEOUT : ((bad & 1) || m == -INFINITY) ? ROW_INVALID : ROW_OK;
  if ((bad & 2) && job.dev_status && threadIdx.x == 0) atomicOr(job.dev_status, 1);

  uint32_t thr = 0;
  int cut = INT_MAX;
  unsigned long long zfx = 0;
  double ent = 0.0;
  const bool greedy = (job.flags & RS_GREEDY) != 0;
  const float c = job.c;

  if (status == ROW_OK && !greedy) {
    constexpr int KB = Elem<T>::kKeyBits;
    // ---- top-k: k-th entry in (value desc, id asc) order, by count
    if (job.top_k >= 1 && job.top_k < V) {
      uint32_t prefix = 0, pmask = 0, need = uint32_t(job.top_k), cnt_eq = 0;
      for (int shift = KB - 8; shift >= 0; shift -= 8) {
        uint32_t* h = aux.hcnt[ctx.ph];
        for (int i = threadIdx.x; i < 256; i += kThreads) h[i] = 0;
        __syncthreads();
        ctx.each([&](int, float x) {
          const uint32_t key = Elem<T>::key(x);
          if ((key & pmask) == prefix) atomicAdd(&h[(key >> shift) & 255u], 1u);
        });
        __syncthreads();
        ctx.cl.sync();
        {
          uint32_t s = 0;
          for (int r = 0; r < ctx.C; ++r) s += ctx.remote(aux.hcnt[ctx.ph], r)[threadIdx.x];
          aux.tot_cnt[threadIdx.x] = s;
        }
        __syncthreads();
        ctx.template find_desc_bin<uint32_t>(aux.tot_cnt, need);
        __syncthreads();
        const uint32_t b = uint32_t(aux.found_bin);
        need -= uint32_t(aux.found_above);
        prefix |= b << shift;
        pmask |= 255u << shift;
        cnt_eq = aux.tot_cnt[b];
        ctx.ph ^= 1;
      }
      thr = prefix;
      cut = (need == cnt_eq) ? INT_MAX : ctx.nth_match(prefix, INT_MAX, need);
    }

    // ---- normaliser over the kept set (exact fixed-point sum of per-entry masses)
    {
      unsigned long long zs = 0;
      ctx.each([&](int id, float x) {
        if (kept(Elem<T>::key(x), id, thr, cut)) zs += to_fx(weight(x, m, c));
      });
      zfx = ctx.xchg_sum_u64(zs);
    }

    // ---- top-p: shortest prefix of the kept set whose mass reaches top_p * Z
    if (job.top_p < 1.0f) {
      unsigned long long target = (unsigned long long)ceil(double(job.top_p) * double(zfx));
      if (target < 1) target = 1;  // the top entry alone always reaches a tiny top_p
      const uint32_t thr_k = thr;
      const int cut_k = cut;
      uint32_t prefix = 0, pmask = 0;
      unsigned long long before = 0;
      bool reached = true;
      uint32_t cnt_eq = 0;
      unsigned long long mass_eq = 0;
      for (int shift = KB - 8; shift >= 0; shift -= 8) {
        uint32_t* hc = aux.hcnt[ctx.ph];
        unsigned long long* hm = aux.hmass[ctx.ph];
        for (int i = threadIdx.x; i < 256; i += kThreads) {
          hc[i] = 0;
          hm[i] = 0;
        }
        __syncthreads();
        ctx.each([&](int id, float x) {
          const uint32_t key = Elem<T>::key(x);
          if ((key & pmask) == prefix && kept(key, id, thr_k, cut_k)) {
            const uint32_t bin = (key >> shift) & 255u;
            atomicAdd(&hc[bin], 1u);
            atomicAdd(&hm[bin], to_fx(weight(x, m, c)));
          }
        });
        __syncthreads();
        ctx.cl.sync();
        {
          uint32_t sc = 0;
          unsigned long long sm = 0;
          for (int r = 0; r < ctx.C; ++r) {
            sc += ctx.remote(aux.hcnt[ctx.ph], r)[threadIdx.x];
            sm += ctx.remote(aux.hmass[ctx.ph], r)[threadIdx.x];
          }
          aux.tot_cnt[threadIdx.x] = sc;
          aux.tot_mass[threadIdx.x] = sm;
        }
        __syncthreads();
        ctx.template find_desc_bin<unsigned long long>(aux.tot_mass, target - before);
        __syncthreads();
        ctx.ph ^= 1;
        if (!aux.found) {  // rounding left the whole kept set short of top_p: keep it all
          reached = false;
          break;
        }
        const uint32_t b = uint32_t(aux.found_bin);
        before += aux.found_above;
        prefix |= b << shift;
        pmask |= 255u << shift;
        cnt_eq = aux.tot_cnt[b];
        mass_eq = aux.tot_mass[b];
      }
      if (reached) {
        const unsigned long long e_fx = mass_eq / cnt_eq;  // equal keys carry equal masses
        unsigned long long t = (target - before + e_fx - 1) / e_fx;
        t = t < 1 ? 1 : (t > cnt_eq ? cnt_eq : t);
        const int cap = (prefix == thr_k) ? cut_k : INT_MAX;
        thr = prefix;
        cut = (t == cnt_eq) ? cap : ctx.nth_match(prefix, cap, uint32_t(t));
        zfx = before + t * e_fx;
      }
    }

    // ---- entropy of the transformed distribution (nats)
    if (job.flags & RS_ENTROPY) {
      float s1 = 0.0f;
      ctx.each([&](int id, float x) {
        if (kept(Elem<T>::key(x), id, thr, cut)) s1 += weight(x, m, c) * (x - m);
      });
      const double S1 = ctx.xchg_sum_f64(double(s1));
      const double Z = double(zfx) * kFxInv;
      ent = log(Z) - double(job.inv_t) * S1 / Z;
    }
  }

  const float zf = float(double(zfx) * kFxInv);
  if (job.stats && rank == 0 && threadIdx.x == 0) {
    RowStats st;
    st.m = m;
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
        out[id] = kept(Elem<T>::key(x), id, thr, cut) ? weight(x, m, c) / zf : 0.0f;
      });
    }
    if (job.entropy && rank == 0 && threadIdx.x == 0)
      job.entropy[row] = status != ROW_OK ? NAN : (greedy ? 0.0f : float(ent));
  }
  ctx.cl.sync();  // no CTA leaves while a peer may still read its shared memory
}

}  // namespace sv
