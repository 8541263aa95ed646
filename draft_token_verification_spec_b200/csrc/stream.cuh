// Streaming row statistics kernel: one CTA per logit row at a time, persistent over rows.
//
// A CTA walks rows blockIdx.x, blockIdx.x + gridDim.x, ... and streams each row through
// a ring of kSBuf shared-memory chunk buffers with 1-D bulk copies (cp.async.bulk,
// completion on an mbarrier per buffer); the copies of the next chunks — across row
// boundaries — are in flight while a chunk is processed. Nothing is shared between
// CTAs, so a row costs no cluster or grid synchronisation.
//
// Per chunk, each thread updates its running maximum (packed bf16x2 max with NaN
// propagation) and, as the mode needs,
//   - greedy: the lowest index holding its maximum;
//   - no truncation / top-p: an online softmax sum (and entropy term), rescaled when
//     its maximum grows (one pass: online max / sum-exp);
//   - top-k / top-p (bfloat16): a warp-aggregated append of the entries >= a threshold
//     to the CTA's candidate list (4 bytes each: the entry's 16-bit key and its index
//     within the chunk; a boundary table gives each candidate's chunk). The threshold
//     only rises. Top-k starts from a value that k entries of the first chunk reach
//     (per-warp order statistics of per-thread maxima); top-p from (first-chunk
//     maximum - T ln(V / (1 - top_p))), below which the whole row holds less than
//     1 - top_p of the mass. When the list would overflow, the threshold is raised to
//     the k-th (top-k) or kKeep-th (top-p) largest candidate and the list compacted.
// At the end of a row the CTA selects exactly among its candidates — top-k by count,
// top-p by mass — over a histogram of exact bfloat16 keys counted down from the row
// maximum, and writes the RowStats record (and the kept ids of top-k rows). Rows the
// candidates cannot settle (float32 top-k/top-p, list overflow, a key range wider than
// the histogram, or candidates holding less than top_p of the mass) are marked
// ROW_FALLBACK and listed; the cluster kernel (row_stats.cuh) then finishes them
// exactly.
//
// This is the sampling transform of "Speculative Sampling" (spec-decoding-i notes, last
// bullet: transform the probabilities first, then apply the rejection scheme) and the
// entropy used by MEDUSA typical acceptance ("Key Components").
#pragma once

#include <climits>

#include "row_stats.cuh"

namespace sv {

#ifndef SV_SBUF
#define SV_SBUF 2
#endif
#ifndef SV_CHUNK_KB
#define SV_CHUNK_KB 32
#endif
constexpr int kSBuf = SV_SBUF;                 // chunk buffers per CTA (ring)
constexpr int kChunkBytes = SV_CHUNK_KB * 1024;  // bytes of logits per chunk
constexpr int kCap = 8192;                     // candidate list capacity (4 bytes each)
constexpr int kKeep = 4096;                    // top-p: candidates kept by a compaction
constexpr int kOffBins = 2048;                 // exact-key histogram: keys kM - 2047 .. kM
constexpr int kMaxChunks = 64;                 // chunks per row (bfloat16, V <= 2^20)
constexpr int kVecRound = 4;                   // 16-byte vectors a thread loads per round

enum : int { SEL_COUNT = 0, SEL_MASS = 1 };

struct StreamJob {
  RowJob r;             // rows, element type, transform, outputs
  int chunk;            // elements per chunk
  int nchunk;           // chunks per row
  int chunk_bytes;      // bytes reserved per ring buffer (multiple of 128)
  float topp_span;      // T * ln(V / (1 - top_p)) (top-p candidate window, in logit units)
  int32_t* fb_rows;     // [rows] rows the cluster kernel must finish
  int32_t* fb_count;    // number of entries in fb_rows
};

struct __align__(16) StreamAux {
  uint64_t bar[kSBuf];
  uint32_t cand[kCap];          // (key16 << 16) | index within the chunk
  uint32_t hist[kOffBins];
  int cbound[kMaxChunks + 1];   // candidates of chunk q: [cbound[q], cbound[q+1])
  int cbnew[kMaxChunks + 1];
  unsigned long long scr_u64[kWarps];
  double scr_f64[kWarps];
  uint32_t scr_u32[kWarps];
  float scr_f[kWarps];
  int scr_i[kWarps];
  int ccount;
  int overflow;
  float thr;          // candidates are the entries >= thr
  int sel_bin;
  unsigned long long sel_before;
  int sel_found;
  int sel_id;
  int broken;         // a copy wait timed out: no further copies are issued
  int pending;        // bit b: a copy into buffer b was issued and not yet waited for
};

// ------------------------------------------------------------------------- helpers

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block max / min (every thread gets the result).
__device__ __forceinline__ float block_max(float v, float* scr) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) scr[warp] = v;
  __syncthreads();
  float t = scr[0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) t = fmaxf(t, scr[w]);
  return t;
}
__device__ __forceinline__ float block_min(float v, float* scr) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_min(v);
  __syncthreads();
  if (lane == 0) scr[warp] = v;
  __syncthreads();
  float t = scr[0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) t = fminf(t, scr[w]);
  return t;
}
__device__ __forceinline__ int block_min_int(int v, int* scr) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) scr[warp] = v;
  __syncthreads();
  int t = scr[0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) t = min(t, scr[w]);
  return t;
}
__device__ __forceinline__ long long block_sum_s64(long long v, unsigned long long* scr) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) scr[warp] = (unsigned long long)v;
  __syncthreads();
  long long t = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) t += (long long)scr[w];
  return t;
}

// Counts into hist[bin] with one shared atomic per distinct bin per warp; every lane of
// the warp calls it.
__device__ __forceinline__ void hist_add(uint32_t* hist, int bin, bool valid) {
  const unsigned act = __ballot_sync(0xffffffffu, valid);
  if (!valid) return;
  const unsigned peers = __match_any_sync(act, bin);
  if ((threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], uint32_t(__popc(peers)));
}

template <typename T>
struct Streamer {
  StreamAux* aux;
  int chunk;
  // this thread's state for the current row
  float mt;            // running maximum (-inf: none yet)
  int am;              // greedy: lowest id holding mt
  float mct;           // fl(mt * c) (online sums are relative to it)
  float s, h;          // online weight sum and entropy term (log2 units)
  bool bad;            // saw NaN or +inf

  __device__ Streamer(StreamAux* a, int ch) : aux(a), chunk(ch) { reset(); }

  __device__ void reset() {
    mt = -INFINITY;
    am = INT_MAX;
    mct = 0.0f;
    s = 0.0f;
    h = 0.0f;
    bad = false;
  }

  // Raises this thread's running maximum to vm, rescaling the online sums.
  __device__ __forceinline__ void raise_max(float vm, float c) {
    const float nm = vm * c;
    if (s != 0.0f || h != 0.0f) {
      const float d = nm - mct;  // > 0
      const float scale = ex2(-d);
      h = scale * (h - d * s);
      s = scale * s;
    }
    mt = vm;
    mct = nm;
  }

  // ---------------------------------------------------------------- chunk pass
  // One pass over a chunk in rounds of kVecRound vectors per thread (loads first, then
  // work, for memory-level parallelism). Updates the running max (greedy: with its
  // lowest index), the online sums (kSum), and appends the entries >= thr (kFilter).
  // Every thread of a warp runs the same rounds (the append is warp-synchronous).
  template <bool kGreedy, bool kSum, bool kFilter>
  __device__ void pass(const unsigned char* buf, int pad, int n, int base, float c,
                       bool want_ent, float thr) {
    constexpr int P = Elem<T>::kPerVec, E = Elem<T>::kBytes;
    const int nvec = (pad + n * E + 15) >> 4;
    const int lane = threadIdx.x & 31;
    for (int r0 = 0; r0 < nvec; r0 += kVecRound * kThreads) {
      uint4 wv[kVecRound];
#pragma unroll
      for (int u = 0; u < kVecRound; ++u) {
        const int v = r0 + u * kThreads + threadIdx.x;
        wv[u] = v < nvec ? reinterpret_cast<const uint4*>(buf)[v] : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kVecRound; ++u) {
        const int v = r0 + u * kThreads + threadIdx.x;
        const int j0 = (v * 16 - pad) / E;
        uint32_t mask = 0;
        float x[P];
        if (v < nvec) {
          Elem<T>::unpack(wv[u], x);
          const bool fv = j0 >= 0 && j0 + P <= n;
          uint32_t inside = (1u << P) - 1u;  // lanes of this vector inside the chunk
          float vm;
          if (fv) {
            vm = Elem<T>::vmax_nan(wv[u]);
          } else {
            vm = -INFINITY;
            inside = 0;
#pragma unroll
            for (int k = 0; k < P; ++k) {
              if (j0 + k >= 0 && j0 + k < n) {
                vm = fmax_nan(vm, x[k]);
                inside |= 1u << k;
              } else {
                x[k] = -INFINITY;  // outside the chunk: weight 0, never a candidate
              }
            }
          }
          if (vm != vm || vm == INFINITY) {
            bad = true;
          } else {
            if (vm > mt) {
              if (kSum) {
                raise_max(vm, c);
              } else {
                mt = vm;
              }
              if (kGreedy) {
#pragma unroll
                for (int k = P - 1; k >= 0; --k)
                  if (x[k] == vm) am = base + j0 + k;
              }
            }
            if (kSum) {
              if (want_ent) {
#pragma unroll
                for (int k = 0; k < P; ++k) {
                  const float zx = wexp(x[k], c, mct);
                  const float e = ex2(zx);
                  s += e;
                  h += ent_term(e, zx);
                }
              } else {
                float s2 = 0.0f;
#pragma unroll
                for (int k = 0; k < P; k += 2) {
                  s += ex2(wexp(x[k], c, mct));
                  s2 += ex2(wexp(x[k + 1], c, mct));
                }
                s += s2;
              }
            }
            if (kFilter && vm >= thr) {
#pragma unroll
              for (int k = 0; k < P; ++k)
                if (((inside >> k) & 1u) && x[k] >= thr) mask |= 1u << k;
            }
          }
        }
        if (kFilter) {
          const int cnt = __popc(mask);
          if (__any_sync(0xffffffffu, cnt != 0)) {
            int inc = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const int w = __shfl_up_sync(0xffffffffu, inc, o);
              if (lane >= o) inc += w;
            }
            int wbase = 0;
            if (lane == 31) wbase = atomicAdd(&aux->ccount, inc);
            int pos = __shfl_sync(0xffffffffu, wbase, 31) + inc - cnt;
#pragma unroll
            for (int k = 0; k < P; ++k) {
              if (mask & (1u << k)) {
                if (pos < kCap) aux->cand[pos] = (Elem<T>::key(x[k]) << 16) | uint32_t(j0 + k);
                ++pos;
              }
            }
          }
        }
      }
    }
  }

  // ---------------------------------------------------------------- candidates
  __device__ __forceinline__ uint32_t ckey(int i) const { return aux->cand[i] >> 16; }
  __device__ __forceinline__ int cid(int i, int nq) const {
    int q = 0;
    while (q + 1 < nq && aux->cbound[q + 1] <= i) ++q;
    return q * chunk + int(aux->cand[i] & 0xFFFFu);
  }

  // The need-th largest candidate key (by count, or by fixed-point mass with weights
  // relative to mc) over an exact histogram of keys counted down from kmax. Returns
  // false when a candidate lies more than kOffBins keys below kmax. On success
  // aux->sel_found says whether the candidates reach need, aux->sel_bin is the offset of
  // the selected key and aux->sel_before the count or mass of the candidates above it.
  __device__ bool select_offsets(int n, uint32_t kmax, unsigned long long need, int mode,
                                 float c, float mc) {
    for (int i = threadIdx.x; i < kOffBins; i += kThreads) aux->hist[i] = 0;
    __syncthreads();
    int wide = 0;
    for (int i0 = 0; i0 < n; i0 += kThreads) {
      const int i = i0 + threadIdx.x;
      int off = 0;
      bool ok = false;
      if (i < n) {
        const uint32_t k = ckey(i);
        off = k <= kmax ? int(kmax - k) : kOffBins;
        ok = off < kOffBins;
        wide |= !ok;
      }
      hist_add(aux->hist, ok ? off : 0, ok);
    }
    wide = __syncthreads_or(wide);
    if (wide) return false;
    constexpr int kPer = kOffBins / kThreads;
    unsigned long long part[kPer];
    unsigned long long tsum = 0;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int bin = threadIdx.x * kPer + q;
      const uint32_t cnt = aux->hist[bin];
      unsigned long long mass = cnt;
      if (mode == SEL_MASS && cnt) mass = cnt * to_fx(weight(key_value<T>(kmax - bin), c, mc));
      part[q] = mass;
      tsum += mass;
    }
    unsigned long long total;
    const unsigned long long ex =
        block_exclusive_scan<unsigned long long>(tsum, aux->scr_u64, &total);
    if (threadIdx.x == 0) aux->sel_found = 0;
    __syncthreads();
    if (ex < need && need <= ex + tsum) {
      unsigned long long acc = ex;
#pragma unroll
      for (int q = 0; q < kPer; ++q) {
        if (acc + part[q] >= need) {
          aux->sel_bin = threadIdx.x * kPer + q;
          aux->sel_before = acc;
          aux->sel_found = 1;
          break;
        }
        acc += part[q];
      }
    }
    __syncthreads();
    return true;
  }

  // The need-th largest candidate key by count, by 8-bit radix levels (any key range).
  // Returns the key; *eq = candidates equal to it, aux->sel_before = how many of those
  // are needed.
  __device__ uint32_t select_radix(int n, uint32_t need, uint32_t* eq) {
    uint32_t prefix = 0, pmask = 0, cnt_eq = 0;
    for (int shift = 8; shift >= 0; shift -= 8) {
      for (int i = threadIdx.x; i < 256; i += kThreads) aux->hist[i] = 0;
      __syncthreads();
      for (int i0 = 0; i0 < n; i0 += kThreads) {
        const int i = i0 + threadIdx.x;
        uint32_t key = 0;
        bool ok = false;
        if (i < n) {
          key = ckey(i);
          ok = (key & pmask) == prefix;
        }
        hist_add(aux->hist, int((key >> shift) & 255u), ok);
      }
      __syncthreads();
      if (threadIdx.x < 32) {  // first bin from the top whose cumulative count reaches need
        const int lane = threadIdx.x;
        uint32_t sl = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) sl += aux->hist[255 - 8 * lane - k];
        uint32_t inc = sl;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += t;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, inc >= need);
        const int L = hit ? __ffs(hit) - 1 : 31;
        if (lane == L) {
          uint32_t acc = inc - sl;
          int b = 255 - 8 * lane - 7;
          for (int k = 0; k < 8; ++k) {
            const int bb = 255 - 8 * lane - k;
            if (acc + aux->hist[bb] >= need || k == 7) {
              b = bb;
              break;
            }
            acc += aux->hist[bb];
          }
          aux->sel_bin = b;
          aux->sel_before = acc;
        }
      }
      __syncthreads();
      need -= uint32_t(aux->sel_before);
      prefix |= uint32_t(aux->sel_bin) << shift;
      pmask |= 255u << shift;
      cnt_eq = aux->hist[aux->sel_bin];
      __syncthreads();
    }
    *eq = cnt_eq;
    aux->sel_before = need;
    return prefix;
  }

  // The need-th largest candidate key by count (exact-key histogram when the keys fit it).
  __device__ uint32_t kth_key(int n, uint32_t kmax, uint32_t need, uint32_t* eq, uint32_t* take) {
    if (select_offsets(n, kmax, need, SEL_COUNT, 0.0f, 0.0f) && aux->sel_found) {
      const uint32_t key = kmax - uint32_t(aux->sel_bin);
      *eq = aux->hist[aux->sel_bin];
      *take = need - uint32_t(aux->sel_before);
      __syncthreads();
      return key;
    }
    const uint32_t key = select_radix(n, need, eq);
    *take = uint32_t(aux->sel_before);
    __syncthreads();
    return key;
  }

  // The t-th smallest id (1-based) among the candidates whose key equals key0 and whose
  // id is at most cap.
  __device__ int nth_id(int n, int nq, uint32_t key0, uint32_t t, int cap) {
    if (threadIdx.x == 0) aux->sel_id = INT_MAX;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kThreads) {
      if (ckey(i) != key0) continue;
      const int ii = cid(i, nq);
      if (ii > cap) continue;
      uint32_t below = 0;
      for (int q = 0; q < n; ++q) {
        if (ckey(q) != key0) continue;
        const int iq = cid(q, nq);
        below += (iq < ii) ? 1u : 0u;
      }
      if (below == t - 1) aux->sel_id = ii;
    }
    __syncthreads();
    return aux->sel_id;
  }

  // Keeps the candidates with key > tkey, or key == tkey and id <= tcut (order-preserving
  // block compaction over nq chunks; updates the chunk boundaries).
  __device__ void compact(uint32_t tkey, int tcut, int nq) {
    const int n = min(aux->ccount, kCap);
    constexpr int kPer = kCap / kThreads;
    uint32_t v[kPer];
    uint32_t keep = 0;
    const int lo = threadIdx.x * kPer;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int i = lo + q;
      v[q] = i < n ? aux->cand[i] : 0u;
      if (i < n) {
        const uint32_t k = v[q] >> 16;
        if (k > tkey || (k == tkey && (tcut == INT_MAX || cid(i, nq) <= tcut))) keep |= 1u << q;
      }
    }
    uint32_t total;
    const uint32_t pos0 =
        block_exclusive_scan<uint32_t>(uint32_t(__popc(keep)), aux->scr_u32, &total);
    // new chunk boundaries: survivors before each old boundary
    for (int q = 0; q <= nq; ++q) {
      const int b = aux->cbound[q];
      if (b >= lo && b < lo + kPer && b < n)
        aux->cbnew[q] = int(pos0 + __popc(keep & ((1u << (b - lo)) - 1u)));
      else if (b >= n && threadIdx.x == 0)
        aux->cbnew[q] = int(total);
    }
    __syncthreads();
    uint32_t pos = pos0;
#pragma unroll
    for (int q = 0; q < kPer; ++q)
      if (keep & (1u << q)) aux->cand[pos++] = v[q];
    if (threadIdx.x <= nq) aux->cbound[threadIdx.x] = aux->cbnew[threadIdx.x];
    if (threadIdx.x == 0) aux->ccount = int(total);
    __syncthreads();
  }
};

// One chunk's location: element j of chunk q of the row lands at byte pad + j * E of its
// buffer; the aligned middle moves by bulk copy, head and tail by plain loads.
template <typename T>
__device__ __forceinline__ SliceLoc chunk_loc(const StreamJob& job, long long row, int q) {
  constexpr int E = Elem<T>::kBytes;
  const RowJob& rj = job.r;
  const int V = rj.V;
  const T* src = (row < rj.rows0) ? static_cast<const T*>(rj.base0) + size_t(row) * V
                                  : static_cast<const T*>(rj.base1) + size_t(row - rj.rows0) * V;
  SliceLoc s;
  const int s0 = q * job.chunk;
  s.n = max(0, min(V - s0, job.chunk));
  s.g = reinterpret_cast<const unsigned char*>(src + s0);
  s.pad = int(reinterpret_cast<uintptr_t>(s.g) & 15u);
  const int bytes = s.n * E;
  s.head = min(bytes, (16 - s.pad) & 15);
  s.mid = ((bytes - s.head) >> 4) << 4;
  s.tail = bytes - s.head - s.mid;
  return s;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) stream_rows_kernel(const StreamJob job) {
  extern __shared__ __align__(128) unsigned char ring[];
  __shared__ StreamAux aux;
  const RowJob& rj = job.r;
  const int V = rj.V;
  const bool greedy = (rj.flags & RS_GREEDY) != 0;
  const bool want_ent = (rj.flags & RS_ENTROPY) != 0;
  const bool topk = !greedy && rj.top_k >= 1 && rj.top_k < V;
  const bool topp = !greedy && rj.top_p < 1.0f;
  // candidates need 16-bit keys and chunk-relative ids below 2^16
  const bool cands = (topk || topp) && Elem<T>::kKeyBits == 16 && job.chunk <= 65536 &&
                     job.nchunk <= kMaxChunks;
  const bool sums = !greedy && !topk;  // online sums: no truncation, or top-p only
  const float c = rj.c;
  const int per_row = job.nchunk;
  const long long nrows_mine =
      rj.rows > blockIdx.x ? (rj.rows - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const long long items = nrows_mine * per_row;

  if (threadIdx.x == 0) {
    for (int b = 0; b < kSBuf; ++b) mbar_init(&aux.bar[b], 1);
    aux.broken = 0;
    aux.pending = 0;
    aux.ccount = 0;
    aux.overflow = 0;
    aux.thr = -INFINITY;
    aux.cbound[0] = 0;
  }
  __syncthreads();
  auto buffer = [&](long long g) { return ring + size_t(g % kSBuf) * job.chunk_bytes; };
  auto item_row = [&](long long g) { return blockIdx.x + (g / per_row) * (long long)gridDim.x; };
  auto issue = [&](long long g) {  // thread 0
    if (g >= items || aux.broken) return;
    const SliceLoc s = chunk_loc<T>(job, item_row(g), int(g % per_row));
    if (s.n > 0) {
      issue_slice(s, buffer(g), &aux.bar[g % kSBuf]);
      aux.pending |= 1 << (g % kSBuf);
    }
  };
  if (threadIdx.x == 0)
    for (int g = 0; g < kSBuf - 1; ++g) issue(g);

  Streamer<T> st(&aux, job.chunk);
  int last_added = 0;  // candidates the previous chunk appended

  for (long long g = 0; g < items; ++g) {
    // every thread is done with item g - 1, whose buffer the next copy refills
    __syncthreads();
    if (threadIdx.x == 0) issue(g + kSBuf - 1);
    const long long row = item_row(g);
    const int q = int(g % per_row);
    const SliceLoc s = chunk_loc<T>(job, row, q);
    const int b = int(g % kSBuf);
    bool copied = true;
    if (s.n > 0) {
      if (!aux.broken && (aux.pending & (1 << b))) {
        copied = finish_slice<T>(s, buffer(g), &aux.bar[b], uint32_t((g / kSBuf) & 1));
        if (threadIdx.x == 0) {
          if (copied)
            aux.pending &= ~(1 << b);
          else
            aux.broken = 1;
        }
      } else {
        copied = false;
      }
    }
    const unsigned char* buf = buffer(g);
    const int base = q * job.chunk;
    if (q == 0) {
      st.reset();
      last_added = 0;
    }
    if (!copied) st.bad = true;  // reported as a timeout below

    // ---- chunk pass
    if (copied && s.n > 0) {
      if (greedy) {
        st.template pass<true, false, false>(buf, s.pad, s.n, base, c, false, 0.0f);
      } else if (!cands) {
        if (sums)
          st.template pass<false, true, false>(buf, s.pad, s.n, base, c, want_ent, 0.0f);
        else
          st.template pass<false, false, false>(buf, s.pad, s.n, base, c, false, 0.0f);
      } else {
        if (q == 0) {  // the first threshold, from this chunk's per-thread maxima
          st.template pass<false, false, false>(buf, s.pad, s.n, base, c, false, 0.0f);
          float t0;
          if (topk) {
            const int jw = (rj.top_k + kWarps - 1) / kWarps;
            float tw = -INFINITY;
            if (jw <= 32)
              tw = key_value<T>(warp_kth_key<Elem<T>::kKeyBits>(Elem<T>::key(st.mt), jw));
            t0 = block_min(tw, aux.scr_f);
          } else {
            t0 = block_max(st.mt, aux.scr_f) - job.topp_span;
          }
          if (threadIdx.x == 0) aux.thr = t0;
          st.mt = -INFINITY;  // recomputed by the pass below (with the online sums)
          __syncthreads();
        }
        const int before = aux.ccount;
        const float thr = aux.thr;
        if (sums)
          st.template pass<false, true, true>(buf, s.pad, s.n, base, c, want_ent, thr);
        else
          st.template pass<false, false, true>(buf, s.pad, s.n, base, c, false, thr);
        __syncthreads();
        if (threadIdx.x == 0) aux.cbound[q + 1] = min(aux.ccount, kCap);
        if (topp) {  // follow the running maximum
          const float mrow = block_max(st.mt, aux.scr_f);
          if (threadIdx.x == 0 && mrow - job.topp_span > aux.thr) aux.thr = mrow - job.topp_span;
        }
        __syncthreads();
        const int cnt = aux.ccount;
        last_added = cnt - before;
        if (cnt > kCap) {
          if (threadIdx.x == 0) aux.overflow = 1;
          __syncthreads();
        } else if (q + 1 < job.nchunk && cnt + (3 * last_added) / 2 > kCap) {
          // the next chunk could overflow the list: raise the threshold and compact
          const int keep = topk ? rj.top_k : kKeep;
          if (keep < cnt) {
            const uint32_t kmax = Elem<T>::key(block_max(st.mt, aux.scr_f));
            uint32_t eq, take;
            const uint32_t key = st.kth_key(cnt, kmax, uint32_t(keep), &eq, &take);
            st.compact(key, INT_MAX, q + 1);
            if (threadIdx.x == 0) aux.thr = fmaxf(aux.thr, key_value<T>(key));
            __syncthreads();
          }
        }
      }
    }

    // ---- row end
    if (q != job.nchunk - 1) continue;
    const bool bad = __syncthreads_or(st.bad ? 1 : 0) != 0;
    const bool timeout = __syncthreads_or(copied ? 0 : 1) != 0;
    const float m = block_max(st.mt, aux.scr_f);
    int status = timeout ? ROW_TIMEOUT : ((bad || m == -INFINITY) ? ROW_INVALID : ROW_OK);
    if (timeout && rj.dev_status && threadIdx.x == 0) atomicOr(rj.dev_status, 1);
    const float mc = m * c;
    uint32_t thr = 0;
    int cut = INT_MAX, am = -1;
    unsigned long long zfx = 0;
    double S1 = 0.0;
    bool listed = false;
    if (status == ROW_OK && greedy) {
      am = block_min_int(st.mt == m ? st.am : INT_MAX, aux.scr_i);
    } else if (status == ROW_OK && !topk && !topp) {
      // combine the per-thread online sums relative to the row maximum
      float sc = 0.0f, hc = 0.0f;
      if (st.s != 0.0f) {
        const float d = mc - st.mct;  // >= 0
        const float scale = ex2(-d);
        sc = scale * st.s;
        hc = scale * (st.h - d * st.s);
      }
      zfx = block_sum_u64(to_fx(sc), aux.scr_u64);
      S1 = block_sum_f64(double(hc), aux.scr_f64);
    } else if (status == ROW_OK) {
      const int nq = job.nchunk;
      const int n = min(aux.ccount, kCap);
      const uint32_t kmax = Elem<T>::key(m);
      bool ok = cands && !aux.overflow;
      unsigned long long zall = 0;
      if (topp && !topk) {
        float sc = 0.0f;
        if (st.s != 0.0f) sc = ex2(-(mc - st.mct)) * st.s;
        zall = block_sum_u64(to_fx(sc), aux.scr_u64);
      }
      if (ok && topk) {  // exact k-th candidate by count; the list becomes the kept set
        if (n < rj.top_k) {
          ok = false;
        } else {
          uint32_t eq, take;
          const uint32_t key = st.kth_key(n, kmax, uint32_t(rj.top_k), &eq, &take);
          thr = key;
          cut = take < eq ? st.nth_id(n, nq, key, take, INT_MAX) : INT_MAX;
          st.compact(key, cut, nq);
        }
      }
      if (ok && topp) {  // crossing by mass over exact keys
        const int nk = aux.ccount;
        unsigned long long zk = zall;
        if (topk) {
          unsigned long long zz = 0;
          for (int i = threadIdx.x; i < nk; i += kThreads)
            zz += to_fx(weight(key_value<T>(st.ckey(i)), c, mc));
          zk = block_sum_u64(zz, aux.scr_u64);
        }
        unsigned long long target = (unsigned long long)ceil(double(rj.top_p) * double(zk));
        if (target < 1) target = 1;
        ok = st.select_offsets(nk, kmax, target, SEL_MASS, c, mc);
        if (ok && aux.sel_found) {
          const uint32_t key = kmax - uint32_t(aux.sel_bin);
          const unsigned long long before = aux.sel_before;
          const uint32_t cnt_eq = aux.hist[aux.sel_bin];
          const unsigned long long e_fx = to_fx(weight(key_value<T>(key), c, mc));
          unsigned long long t = e_fx ? (target - before + e_fx - 1) / e_fx : cnt_eq;
          t = t < 1 ? 1 : (t > cnt_eq ? cnt_eq : t);
          const int cap = (topk && key == thr) ? cut : INT_MAX;
          __syncthreads();
          cut = (t == cnt_eq) ? cap : st.nth_id(nk, nq, key, uint32_t(t), cap);
          thr = key;
        } else if (ok && !topk) {
          ok = false;  // the candidates hold less than top_p of the mass
        }
      }
      if (!ok) {
        status = ROW_FALLBACK;
      } else {
        // normaliser, entropy term and kept-id list over the kept candidates
        const int nk = aux.ccount;
        const bool list = topk && !topp && rj.kept_ids && rj.top_k <= kKeptCap;
        unsigned long long z = 0;
        long long s1 = 0;
        if (threadIdx.x == 0) aux.sel_id = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < nk; i += kThreads) {
          const uint32_t key = st.ckey(i);
          if (key < thr) continue;
          int id = -1;
          if (key == thr && cut != INT_MAX) {
            id = st.cid(i, nq);
            if (id > cut) continue;
          }
          const float xi = key_value<T>(key);
          const float zx = wexp(xi, c, mc);
          const float e = ex2(zx);
          z += to_fx(e);
          if (want_ent) s1 += __float2ll_rn(ent_term(e, zx) * kS1Fx);
          if (list) {
            if (id < 0) id = st.cid(i, nq);
            const int slot = atomicAdd(&aux.sel_id, 1);
            if (slot < kKeptCap) rj.kept_ids[size_t(row) * kKeptCap + slot] = id;
          }
        }
        zfx = block_sum_u64(z, aux.scr_u64);
        S1 = double(block_sum_s64(s1, aux.scr_u64)) / double(kS1Fx);
        listed = list;
      }
    }
    if (status == ROW_FALLBACK && threadIdx.x == 0)
      job.fb_rows[atomicAdd(job.fb_count, 1)] = int32_t(row);
    if (rj.kept_n && threadIdx.x == 0) rj.kept_n[row] = listed ? rj.top_k : 0;
    const double Z = double(zfx) * kFxInv;
    const double ent = (status == ROW_OK && !greedy && want_ent)
                           ? log(Z) - 0.6931471805599453 * S1 / Z
                           : 0.0;
    if (rj.stats && threadIdx.x == 0) {
      RowStats rs;
      rs.mc = mc;
      rs.z = float(Z);
      rs.entropy = float(ent);
      rs.thr_key = thr;
      rs.cutoff = cut;
      rs.argmax = greedy ? am : -1;
      rs.status = status;
      rs.c = c;
      rj.stats[row] = rs;
    }
    // the next row starts clean
    if (threadIdx.x == 0) {
      aux.ccount = 0;
      aux.overflow = 0;
      aux.thr = -INFINITY;
      aux.cbound[0] = 0;
    }
  }
  // a copy that timed out may still land: give each one more bounded wait
  if (aux.broken && threadIdx.x == 0) {
    for (int b = 0; b < kSBuf; ++b)
      if (aux.pending & (1 << b)) {
        if (!mbar_wait(&aux.bar[b], 0)) mbar_wait(&aux.bar[b], 1);
      }
  }
}

}  // namespace sv
