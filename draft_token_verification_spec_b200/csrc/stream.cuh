// Streaming row statistics kernel: one CTA per logit row at a time, persistent over rows,
// with a producer warp feeding eight consumer warps.
//
// A CTA walks rows blockIdx.x, blockIdx.x + gridDim.x, ... cut into chunks (Ring<mode>).
// Warp 8 (the producer, one elected lane) keeps a ring of chunk buffers in shared memory
// full with 1-D bulk copies (cp.async.bulk; a "full" mbarrier per buffer completes when
// the bytes land) and runs ahead across row boundaries; it reuses a buffer once the eight
// consumer warps have arrived on its "empty" mbarrier. Consumers synchronise among
// themselves only with named barrier 1, so the producer is never held up by their row-end
// work. Nothing is shared between CTAs.
//
// Per chunk each consumer thread takes eight 16-byte vectors and updates, as the mode
// needs:
//   SM_GREEDY  its running maximum (packed bf16x2 max, NaN propagating) and the lowest index
//              holding it;
//   SM_SUMS    an online softmax sum (and entropy term), rescaled when its maximum grows;
//   SM_TOPK    the running maximum, and appends the entries >= a threshold to the CTA's
//              candidate list (warp-aggregated: one shared atomic per warp, then each lane
//              writes only the set bits of its vectors' masks);
//   SM_TOPP    the online sum and the candidate list.
// Candidates are 64-bit composites (key << 32 | ~id): the order of composites is the order
// (value desc, id asc) that top-k and top-p use, so the k-th candidate is unique.
//
// Top-k: the first threshold is a value that k entries of the first chunk reach (per-warp
// order statistics of per-thread maxima; of vector maxima for k > 128). After the first
// chunk the consumer warps exchange their counts, and a list of more than k entries sets the
// threshold to the exact k-th seen so far (ranked directly, the list kept as it is). Further
// exchanges run every (kCapTopK / 2) / k chunks, so about half the list can fill between
// two even if every chunk brings k new entries; one past half the capacity is cut to its top
// k. Rows whose values do not grow along the vocabulary rarely reach the threshold again, and
// a list that still outgrows kCapTopK sends the row to the exact finisher. The short list
// keeps a top-k CTA small enough for three per SM.
//
// Top-p: the threshold starts at (first-chunk maximum - T ln(V / (1 - top_p))), below
// which the whole row holds less than 1 - top_p of the mass, raised to the smallest of
// the largest kChunk0Vecs vector maxima of the first chunk (so at most 8 x that many
// entries pass) if that is higher. The warps exchange counts and the row maximum after the
// first chunk and then every kXchgTopP chunks: the threshold follows the maximum, and the
// list is cut by count when it is about to overflow or its projected size at the row end
// exceeds the capacity, to the top max(kKeepFloor, kKeepTarget * seen / V) entries seen so
// far (about kKeepTarget candidates at the row end for rows whose values do not drift
// along the vocabulary).
//
// At the end of a row the CTA selects among the candidates. Top-k lists are ranked directly
// (each candidate counts the larger composites); with top-p as well, the top k go to their
// rank slots and a block scan of their weights finds the crossing. Top-p lists go over a
// histogram of log-weight bins (1/32 of a log2 unit each, relative to the row maximum; bins
// only coarsen the order, they never reorder it): the bin where the mass crosses the
// target, then the exact crossing candidate among that bin's members. It writes the
// RowStats record (and the kept ids of top-k rows). Rows the candidates cannot settle (list
// overflow, too many members in the crossing bin, or candidates holding less than top_p of
// the mass) are marked ROW_FALLBACK and listed; the cluster kernel (row_stats.cuh) then
// finishes them exactly.
//
// This is the sampling transform of "Speculative Sampling" (spec-decoding-i notes, last
// bullet: transform the probabilities first, then apply the rejection scheme), the argmax
// of the greedy forms and the entropy used by MEDUSA typical acceptance ("Key
// Components").
#pragma once

#include <climits>
#include <cstddef>

#include "draw.cuh"
#include "row_stats.cuh"

namespace sv {

// Ring of chunk buffers per CTA: two 32 KB chunks in every mode. Greedy, plain sums and
// top-k run three CTAs per SM (top-k adds its list of kCapTopK candidates and the top k in
// rank order, which just fits); top-p two (its larger list and the log-weight histogram
// take the rest). The depth and chunk size of each kind are build-time knobs.
#ifndef SV_RING_NBUF_PLAIN
#define SV_RING_NBUF_PLAIN 2
#endif
#ifndef SV_RING_KB_PLAIN
#define SV_RING_KB_PLAIN 32
#endif
#ifndef SV_RING_NBUF_CAND
#define SV_RING_NBUF_CAND 2
#endif
#ifndef SV_RING_KB_CAND
#define SV_RING_KB_CAND 32
#endif
#ifndef SV_RING_KB_TOPK
#define SV_RING_KB_TOPK 32
#endif
#ifndef SV_TOPK_CTAS
#define SV_TOPK_CTAS 3        // top-k CTAs resident per SM (2 or 3)
#endif
#ifndef SV_RING_NBUF_TOPK
#define SV_RING_NBUF_TOPK 2
#endif
constexpr int kMaxRing = 4;

enum : int { SM_GREEDY = 0, SM_SUMS = 1, SM_TOPK = 2, SM_TOPP = 3 };

template <int kMode>
struct Ring {
  static constexpr int kBuf = kMode <= SM_SUMS ? SV_RING_NBUF_PLAIN
                              : (kMode == SM_TOPK ? SV_RING_NBUF_TOPK : SV_RING_NBUF_CAND);
  static constexpr int kBytes =
      (kMode <= SM_SUMS ? SV_RING_KB_PLAIN : (kMode == SM_TOPK ? SV_RING_KB_TOPK : SV_RING_KB_CAND)) *
      1024;
  static constexpr int kBufBytes = kBytes + 128;  // a chunk starts up to 15 bytes in
  static constexpr int kVec = kBytes / (16 * kThreads);  // vectors per consumer thread
  static_assert(kBytes % (16 * kThreads) == 0, "chunk = whole vectors per consumer");
  static_assert(kBuf >= 2 && kBuf <= kMaxRing, "ring depth");
};

__host__ __device__ constexpr int stream_chunk_bytes(int mode) {
  return mode <= SM_SUMS ? Ring<SM_SUMS>::kBytes
                         : (mode == SM_TOPK ? Ring<SM_TOPK>::kBytes : Ring<SM_TOPP>::kBytes);
}

constexpr int kStreamThreads = kThreads + 32;   // eight consumer warps + the producer
constexpr int kCap = 4096;                      // top-p: candidates per row
constexpr int kCapTopK = 1024;                  // top-k: candidates per row
constexpr int kKeepFloor = 512;                 // top-p: a cut keeps at least this many
constexpr int kKeepTarget = 3 * kCap / 8;       // top-p: candidates a cut aims at by row end
constexpr int kXchgTopP = 4;                    // top-p: chunks between count exchanges
constexpr int kChunk0Vecs = 384;                // top-p: vectors of the first chunk kept
constexpr int kBins = 1024;                     // log-weight bins
constexpr float kBinScale = 32.0f;              // bins per log2 unit of weight
constexpr int kMemberCap = 512;                 // members of the crossing bin
constexpr int kRankMax = 1024;                  // lists this short are ranked directly
constexpr int kStreamMaxTopK = 256;             // top-k the candidate path takes
// Top-p: a bound on the error, relative to the row's total mass, of the fp32 masses that
// place the nucleus boundary (each weight: the exponent's rounding and the rounding of
// log2(e)/T, ex2.approx, the per-vector fp32 sum; the tail below 2^-24 of the maximum holds
// at most V * 2^-24 of it). A boundary within it is re-decided in double precision.
constexpr float kToppGuard = 6e-6f;

// Dynamic shared memory of one CTA: the ring, then top-k: the candidate list and the top k
// in rank order; top-p: the candidate list, the bin counts and the bin masses as 15-bit
// limbs (whose space the crossing bin's members reuse).
__host__ __device__ constexpr size_t stream_dyn_bytes(int mode) {
  return mode <= SM_SUMS ? size_t(Ring<SM_SUMS>::kBuf) * Ring<SM_SUMS>::kBufBytes
         : mode == SM_TOPK
             ? size_t(Ring<SM_TOPK>::kBuf) * Ring<SM_TOPK>::kBufBytes + size_t(kCapTopK) * 8 +
                   size_t(kStreamMaxTopK) * 8
             : size_t(Ring<SM_TOPP>::kBuf) * Ring<SM_TOPP>::kBufBytes + size_t(kCap) * 8 +
                   size_t(kBins) * 4 + size_t(kBins) * 12;
}
static_assert(2 * kMemberCap * 8 <= 3 * kBins * 4, "members and their weights fit the masses");
static_assert(kCapTopK <= kRankMax, "every top-k list is ranked directly");
static_assert(kStreamMaxTopK <= kThreads, "the top k in rank order: one per thread");

struct StreamJob {
  RowJob r;             // rows, element type, transform, outputs
  int chunk;            // elements per chunk
  int nchunk;           // chunks per row
  float topp_span;      // T * ln(V / (1 - top_p)) (top-p candidate window, in logit units)
  int32_t* fb_rows;     // [rows] rows the cluster kernel must finish
  int32_t* fb_count;    // number of entries in fb_rows
};

struct __align__(16) StreamAux {
  uint64_t full[kMaxRing];   // completes when a chunk's bytes have landed
  uint64_t empty[kMaxRing];  // completes when the eight consumer warps are done with it
  float red_f[2][kWarps];  // count exchange, double-buffered by exchange parity
  int red_i[2][kWarps];
  unsigned long long scr_u64[kWarps];  // scr_u64 and scr_s64 together also hold kWarps Fx128
  long long scr_s64[kWarps];
  double scr_f64[kWarps];
  float scr_f[kWarps];
  int scr_i[kWarps];
  uint32_t scr_u32[kWarps];
  unsigned long long sel_before;
  unsigned long long sel_comp;
  unsigned long long sel_mabove;  // resolve: mass of the crossing bin's members above it
  unsigned long long sel_mw;      // resolve: the crossing member's own mass
  uint32_t sel_cnt;
  int sel_bin;
  int sel_found;
  int ccount;   // next free slot of the candidate list
  int mcount;
  int broken;   // a copy or buffer wait timed out: the CTA stops reading rows
};

__device__ __forceinline__ Fx128* scr_fx(StreamAux& a) { return reinterpret_cast<Fx128*>(a.scr_u64); }
static_assert(offsetof(StreamAux, scr_s64) == offsetof(StreamAux, scr_u64) + 8 * kWarps,
              "scr_u64 and scr_s64 are adjacent");

// SV_TOPK_CTAS top-k CTAs per SM: ring, list, ranked top k, this record and the 1 KB the
// hardware reserves per CTA, within the SM's 228 KB.
static_assert(SV_TOPK_CTAS >= 2 && SV_TOPK_CTAS <= 3, "top-k CTAs per SM");
static_assert(SV_TOPK_CTAS * (stream_dyn_bytes(SM_TOPK) + sizeof(StreamAux) + 1024) <= 228 * 1024,
              "the top-k CTAs of an SM fit its shared memory");
static_assert(2 * (stream_dyn_bytes(SM_TOPP) + sizeof(StreamAux) + 1024) <= 228 * 1024,
              "two top-p CTAs per SM");

// ------------------------------------------------------------------ consumer barriers
// Named barrier 1 over the 256 consumer threads (the producer warp never joins it).
__device__ __forceinline__ void csync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory");
}
__device__ __forceinline__ bool csync_or(bool p) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred a, b;\n setp.ne.u32 a, %1, 0;\n bar.red.or.pred b, 1, %2, a;\n"
      " selp.u32 %0, 1, 0, b;\n}"
      : "=r"(r)
      : "r"(uint32_t(p)), "n"(kThreads)
      : "memory");
  return r != 0;
}

struct OpMaxNan {
  __device__ float operator()(float a, float b) const { return fmax_nan(a, b); }
};
struct OpMin {
  template <typename U>
  __device__ U operator()(U a, U b) const { return a < b ? a : b; }
};
struct OpSum {
  template <typename U>
  __device__ U operator()(U a, U b) const { return a + b; }
};

// Reduction over the consumer threads (all of them get the result).
template <typename U, typename Op>
__device__ __forceinline__ U creduce(U v, U* scr, Op op) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  csync();
  if (lane == 0) scr[warp] = v;
  csync();
  U t = scr[0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) t = op(t, scr[w]);
  return t;
}

// Exclusive prefix sum over the consumer threads in thread order; *total = the sum.
template <typename U>
__device__ __forceinline__ U cscan(U v, U* scr, U* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  U inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const U n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  csync();
  if (lane == 31) scr[warp] = inc;
  csync();
  U before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    if (w < warp) before += scr[w];
    all += scr[w];
  }
  *total = all;
  return before + inc - v;
}

// Fx128 sum over the consumer threads (all of them get it).
__device__ __forceinline__ Fx128 creduce_fx(Fx128 v, Fx128* scr) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum_fx(v);
  csync();
  if (lane == 0) scr[warp] = v;
  csync();
  Fx128 t = scr[0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) t = fx_add(t, scr[w]);
  return t;
}

// Exclusive Fx128 prefix sum over the consumer threads in thread order; *total = the sum.
__device__ __forceinline__ Fx128 cscan_fx(Fx128 v, Fx128* scr, Fx128* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  Fx128 inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const Fx128 n = fx_shfl_up(inc, o);
    if (lane >= o) inc = fx_add(inc, n);
  }
  csync();
  if (lane == 31) scr[warp] = inc;
  csync();
  Fx128 before = fx_zero(), all = fx_zero();
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    if (w < warp) before = fx_add(before, scr[w]);
    all = fx_add(all, scr[w]);
  }
  *total = all;
  Fx128 ex = fx_shfl_up(inc, 1);
  if (lane == 0) ex = fx_zero();
  return fx_add(before, ex);
}

// The double-precision work at a row's end, kept out of line so that its registers do not
// weigh on the streaming loop (the call is taken once per row): one entry's weight
// exp((x - m) / T) as Fx128, and a thread's share of the kept candidates' weights.
template <typename T>
__device__ __noinline__ Fx128 weight_fx(uint32_t key, float m, double iT) {
  return fx_from(weight_d(key_value<T>(key), m, iT));
}
template <typename T>
__device__ __noinline__ Fx128 kept_weights_fx(const uint64_t* cand, int n, uint64_t cstar, float m,
                                              double iT) {
  Fx128 acc = fx_zero();
  for (int i = threadIdx.x; i < n; i += kThreads) {
    const uint64_t e = cand[i];
    if (e >= cstar) acc = fx_add(acc, fx_from(weight_d(key_value<T>(uint32_t(e >> 32)), m, iT)));
  }
  return acc;
}

// Counts into hist[bin] with one shared atomic per distinct bin per warp; every lane of
// the warp calls it.
__device__ __forceinline__ void hist_add(uint32_t* hist, int bin, bool valid) {
  const unsigned act = __ballot_sync(0xffffffffu, valid);
  if (!valid) return;
  const unsigned peers = __match_any_sync(act, bin);
  if ((threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], uint32_t(__popc(peers)));
}


// The j-th largest (1 <= j <= 32 N) of the warp's 32 N keys (N per lane), by a radix walk
// from the top bit with warp-wide counts; every lane calls it.
template <int KB, int N>
__device__ __forceinline__ uint32_t warp_kth_key_n(const uint32_t (&key)[N], int j) {
  uint32_t prefix = 0;
  int need = j;
#pragma unroll 1
  for (int b = KB - 1; b >= 0; --b) {
    const uint32_t cand = prefix | (1u << b);
    uint32_t c = 0;
#pragma unroll
    for (int i = 0; i < N; ++i) c += (key[i] >> b) == (cand >> b) ? 1u : 0u;
    const int cnt = int(__reduce_add_sync(0xffffffffu, c));
    if (cnt >= need)
      prefix = cand;
    else
      need -= cnt;
  }
  return prefix;
}

// ------------------------------------------------------------------ chunks
// Chunk q of a row: element j lands at byte pad + j * E of its buffer (pad = the source
// address mod 16); the 16-byte-aligned middle [pad + head, pad + head + mid) moves by
// bulk copy, the < 16 bytes before and after it are read from global memory directly.
struct ChunkLoc {
  const unsigned char* g;  // first element
  int n;                   // elements
  int pad, head, mid;      // bytes
};

template <typename T>
__device__ __forceinline__ ChunkLoc chunk_at(const StreamJob& job, long long row, int q) {
  constexpr int E = Elem<T>::kBytes;
  const RowJob& rj = job.r;
  const int V = rj.V;
  const T* src = (row < rj.rows0) ? static_cast<const T*>(rj.base0) + size_t(row) * V
                                  : static_cast<const T*>(rj.base1) + size_t(row - rj.rows0) * V;
  ChunkLoc s;
  const int s0 = q * job.chunk;
  s.n = max(0, min(V - s0, job.chunk));
  s.g = reinterpret_cast<const unsigned char*>(src + s0);
  s.pad = int(reinterpret_cast<uintptr_t>(s.g) & 15u);
  const int bytes = s.n * E;
  s.head = min(bytes, (16 - s.pad) & 15);
  s.mid = ((bytes - s.head) >> 4) << 4;
  return s;
}

template <typename T>
__device__ __forceinline__ uint4 neg_inf_vec() {
  const uint32_t w = Elem<T>::kBytes == 2 ? 0xFF80FF80u : 0xFF800000u;
  return make_uint4(w, w, w, w);
}

// ------------------------------------------------------------------ candidates
__device__ __forceinline__ uint64_t make_comp(uint32_t key, int id) {
  return (uint64_t(key) << 32) | uint64_t(~uint32_t(id));
}
__device__ __forceinline__ uint32_t comp_key(uint64_t e) { return uint32_t(e >> 32); }
__device__ __forceinline__ int comp_id(uint64_t e) { return int(~uint32_t(e)); }

// Log-weight bin of a value: floor(((m - x) / T) in log2 units * kBinScale), clamped to
// [0, kBins - 1]. Non-increasing in x (one FMA, then a scaling by a power of two and a
// truncation), and equal for equal values.
__device__ __forceinline__ int bin_of(float x, float c, float mc) {
  const float d = fmaf(-x, c, mc) * kBinScale;
  return d < float(kBins - 1) ? max(0, int(d)) : kBins - 1;
}

template <typename T>
struct CandSet {
  uint64_t* cand;              // [kCap] (top-k: [kCapTopK])
  uint32_t* hcnt;              // [kBins] (top-p only)
  uint32_t* hlimb;             // [3][kBins]: bin masses as limbs; members and their weights
                               // reuse it (top-p only)
  uint64_t* ranked;            // [kStreamMaxTopK]: the top k in rank order (top-k only)
  StreamAux* aux;

  // Histogram of the candidates i < n with composite >= lim over log-weight bins relative to
  // mc: counts, and (mass) the sum of their fixed-point weights 2^(x c - wref).
  __device__ void hist_build(int n, uint64_t lim, float c, float mc, bool mass, float wref) {
    for (int i = threadIdx.x; i < kBins; i += kThreads) hcnt[i] = 0;
    if (mass)
      for (int i = threadIdx.x; i < 3 * kBins; i += kThreads) hlimb[i] = 0;
    csync();
    for (int i0 = 0; i0 < n; i0 += kThreads) {
      const int i = i0 + threadIdx.x;
      bool ok = false;
      int b = 0;
      float x = 0.0f;
      if (i < n) {
        const uint64_t e = cand[i];
        ok = e >= lim;
        if (ok) {
          x = key_value<T>(comp_key(e));
          b = bin_of(x, c, mc);
        }
      }
      hist_add(hcnt, b, ok);
      if (mass && ok) {
        const unsigned long long w = to_fx(weight(x, c, wref));
        limb_add(hlimb, kBins, b, w);
      }
    }
    csync();
  }

  // The bin where the count (or mass) accumulated from bin 0 first reaches need:
  // aux->sel_found, sel_bin, sel_before (the count or mass of the bins before it) and
  // sel_cnt (its count).
  __device__ void hist_find(unsigned long long need, bool mass) {
    constexpr int kPer = kBins / kThreads;
    unsigned long long part[kPer];
    unsigned long long tsum = 0;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int b = threadIdx.x * kPer + q;
      part[q] = mass ? limb_get(hlimb, kBins, b) : (unsigned long long)hcnt[b];
      tsum += part[q];
    }
    unsigned long long total;
    const unsigned long long ex = cscan<unsigned long long>(tsum, aux->scr_u64, &total);
    if (threadIdx.x == 0) aux->sel_found = 0;
    csync();
    if (ex < need && need <= ex + tsum) {
      unsigned long long acc = ex;
#pragma unroll
      for (int q = 0; q < kPer; ++q) {
        if (acc + part[q] >= need) {
          const int b = threadIdx.x * kPer + q;
          aux->sel_bin = b;
          aux->sel_before = acc;
          aux->sel_cnt = hcnt[b];
          aux->sel_found = 1;
          break;
        }
        acc += part[q];
      }
    }
    csync();
  }

  // Among the members of bin aux->sel_bin (composite >= lim), in composite order, the one
  // where the count (or mass) accumulated within the bin reaches need -> aux->sel_comp.
  // Returns false if the bin has more than kMemberCap members.
  __device__ bool resolve(int n, uint64_t lim, float c, float mc, bool mass,
                          unsigned long long need, float wref) {
    if (aux->sel_cnt > uint32_t(kMemberCap)) return false;  // uniform
    const int bsel = aux->sel_bin;
    uint64_t* mem = reinterpret_cast<uint64_t*>(hlimb);
    unsigned long long* mw = reinterpret_cast<unsigned long long*>(hlimb) + kMemberCap;
    if (threadIdx.x == 0) {
      aux->mcount = 0;
      aux->sel_comp = 0;
    }
    csync();
    for (int i = threadIdx.x; i < n; i += kThreads) {
      const uint64_t e = cand[i];
      if (e < lim) continue;
      const float x = key_value<T>(comp_key(e));
      if (bin_of(x, c, mc) != bsel) continue;
      const int slot = atomicAdd(&aux->mcount, 1);
      if (slot < kMemberCap) {
        mem[slot] = e;
        mw[slot] = mass ? to_fx(weight(x, c, wref)) : 1ull;
      }
    }
    csync();
    const int m = min(aux->mcount, kMemberCap);
    for (int i = threadIdx.x; i < m; i += kThreads) {
      const uint64_t ei = mem[i];
      unsigned long long above = 0;
      for (int j = 0; j < m; ++j)
        if (mem[j] > ei) above += mw[j];
      if (above < need && need <= above + mw[i]) {
        aux->sel_comp = ei;
        aux->sel_mabove = above;
        aux->sel_mw = mw[i];
      }
    }
    csync();
    return aux->sel_comp != 0;
  }

  // Cuts the list cand[0..n) to the candidates in the bins (relative to mc) up to the one
  // where the count reaches keep; returns the new count and sets *thr to the smallest kept
  // value, so the list stays "every entry seen so far that is >= thr".
  __device__ int cut(int n, int keep, float c, float mc, float* thr) {
    hist_build(n, 0, c, mc, false, mc);
    hist_find((unsigned long long)keep, false);
    const int bsel = aux->sel_found ? aux->sel_bin : kBins - 1;
    constexpr int kPer = kCap / kThreads;
    uint64_t v[kPer];
    uint32_t keepm = 0;
    uint32_t kmin = 0xFFFFFFFFu;
    const int lo = threadIdx.x * kPer;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int i = lo + q;
      v[q] = i < n ? cand[i] : 0ull;
      if (i < n) {
        const uint32_t key = comp_key(v[q]);
        if (bin_of(key_value<T>(key), c, mc) <= bsel) {
          keepm |= 1u << q;
          kmin = min(kmin, key);
        }
      }
    }
    uint32_t total;
    uint32_t pos = cscan<uint32_t>(uint32_t(__popc(keepm)), aux->scr_u32, &total);
#pragma unroll
    for (int q = 0; q < kPer; ++q)
      if (keepm & (1u << q)) cand[pos++] = v[q];
    const uint32_t kmin_all = creduce<uint32_t>(kmin, aux->scr_u32, OpMin());
    if (threadIdx.x == 0) aux->ccount = int(total);
    csync();
    *thr = fmaxf(*thr, key_value<T>(kmin_all));
    return int(total);
  }

  // Top-k lists: keeps the candidates of cand[0..n) (n <= kCapTopK) whose composite is
  // >= lim, in place; returns their count (also the list's new fill count).
  __device__ int compact_ge(int n, uint64_t lim) {
    constexpr int kPer = kCapTopK / kThreads;
    uint64_t v[kPer];
    uint32_t keepm = 0;
    const int lo = threadIdx.x * kPer;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int i = lo + q;
      v[q] = i < n ? cand[i] : 0ull;
      if (i < n && v[q] >= lim) keepm |= 1u << q;
    }
    uint32_t total;
    uint32_t pos = cscan<uint32_t>(uint32_t(__popc(keepm)), aux->scr_u32, &total);
#pragma unroll
    for (int q = 0; q < kPer; ++q)
      if (keepm & (1u << q)) cand[pos++] = v[q];
    if (threadIdx.x == 0) aux->ccount = int(total);
    csync();
    return int(total);
  }

  // Short lists (n <= kRankMax, flat): the k-th largest composite among cand[0..n) that are
  // >= lim, by counting for each the larger ones (composites are distinct) ->
  // aux->sel_comp. The caller has synchronised the list. False if there is none.
  __device__ bool rank_select(int n, uint64_t lim, int k) {
    if (threadIdx.x == 0) aux->sel_comp = 0;
    csync();
    for (int i = threadIdx.x; i < n; i += kThreads) {
      const uint64_t e = cand[i];
      if (e < lim) continue;
      int above = 0;
      for (int j = 0; j < n; ++j) above += cand[j] > e ? 1 : 0;
      if (above == k - 1) aux->sel_comp = e;
    }
    csync();
    return aux->sel_comp != 0;
  }

  // Top-k lists (n <= kRankMax): the top k of cand[0..n) (k <= kThreads) in rank order, then
  // the one where the mass accumulated from the top first reaches top_p of their total ->
  // aux->sel_comp, with the weights exp((l - m) / T) in double summed exactly. The caller has
  // synchronised the list, and read aux->sel_comp if it needs it, before the call.
  __device__ bool rank_topp(int n, int k, float top_p, float m, double iT) {
    for (int i = threadIdx.x; i < n; i += kThreads) {
      const uint64_t e = cand[i];
      int above = 0;
      for (int j = 0; j < n; ++j) above += cand[j] > e ? 1 : 0;
      if (above < k) ranked[above] = e;
    }
    if (threadIdx.x == 0) aux->sel_comp = 0;
    csync();
    const bool mine = int(threadIdx.x) < k;
    const uint64_t e = mine ? ranked[threadIdx.x] : 0ull;
    const Fx128 w = mine ? weight_fx<T>(comp_key(e), m, iT) : fx_zero();
    Fx128 z;
    const Fx128 ex = cscan_fx(w, scr_fx(*aux), &z);
    const double target = double(top_p) * fx_to_double(z);
    if (mine && fx_to_double(ex) < target && target <= fx_to_double(fx_add(ex, w)))
      aux->sel_comp = e;
    csync();
    return aux->sel_comp != 0;
  }
};

// ------------------------------------------------------------------ per-thread row state
template <typename T, int kMode>
struct RowAcc {
  static constexpr bool kSums = kMode == SM_SUMS || kMode == SM_TOPP;
  float mt;   // running maximum (NaN once a NaN was seen)
  int am;     // greedy: lowest index holding mt
  float mct;  // the online sums are relative to it: fl(mt * c); top-p: ceil(fl(mt * c))
  float s, h; // online weight sum and entropy term (log2 units)
  // top-p: the online weight sum as 42-bit fixed point, relative to the integer reference
  // mct. Each vector's eight weights are summed in fp32 and added exactly; a reference that
  // rises by d shifts the sum right by d bits (the exact power of two, truncated below
  // 2^-42), so the sum's error stays within a few fp32 roundings per weight (the bound the
  // top-p decision's guard relies on) with no floating-point rescale in the loop.
  unsigned long long sfx;

  __device__ void reset() {
    mt = -INFINITY;
    am = INT_MAX;
    mct = 0.0f;
    s = 0.0f;
    h = 0.0f;
    sfx = 0ull;
  }

  // Raises the running maximum to vm (> mt), rescaling the online sums.
  __device__ __forceinline__ void raise_max(float vm, float c) {
    const float nm = vm * c;
    if constexpr (kMode == SM_TOPP) {
      const float nr = ceilf(nm);
      if (sfx == 0ull) {
        mct = nr;
      } else if (nr > mct) {
        const float d = nr - mct;
        sfx = d < 64.0f ? sfx >> int(d) : 0ull;
        mct = nr;
      }
      return;
    } else if (s != 0.0f || h != 0.0f) {
      const float d = nm - mct;  // > 0
      const float scale = ex2(-d);
      h = scale * (h - d * s);
      s = scale * s;
    }
    mct = nm;
  }

  __device__ __forceinline__ void add(float x, float c, bool want_ent) {
    const float zx = wexp(x, c, mct);
    const float e = ex2(zx);
    if constexpr (kMode == SM_TOPP) {
      sfx += to_fx(e);
    } else {
      s += e;
      if (want_ent) h += ent_term(e, zx);
    }
  }

  // One 16-byte vector whose first element has row index j0 (entries outside the chunk
  // hold -inf). vm = its largest value. Top-p: returns the mask of its entries >= t, from
  // the values the sums unpacked (0 in the other modes).
  __device__ __forceinline__ uint32_t vec(const uint4& w, float vm, int j0, float c,
                                          bool want_ent, float t) {
    constexpr int P = Elem<T>::kPerVec;
    uint32_t cm = 0;
    if (!(vm > -INFINITY)) {  // all -inf (weight 0), or a NaN
      mt = fmax_nan(mt, vm);
      if (kMode == SM_TOPP && vm >= t) cm = (1u << P) - 1u;  // all -inf, and t = -inf
      return cm;
    }
    if constexpr (kMode == SM_GREEDY) {
      if (vm > mt) {  // later vectors hold higher indices: strict > keeps the lowest
        float x[P];
        Elem<T>::unpack(w, x);
#pragma unroll
        for (int k = P - 1; k >= 0; --k)
          if (x[k] == vm) am = j0 + k;
      }
    } else if constexpr (kSums) {
      if (vm > mt) raise_max(vm, c);
      float x[P];
      Elem<T>::unpack(w, x);
      if (kMode == SM_TOPP) {
        float s1 = 0.0f, s2 = 0.0f;
#pragma unroll
        for (int k = 0; k < P; k += 2) {
          s1 += ex2(wexp(x[k], c, mct));
          s2 += ex2(wexp(x[k + 1], c, mct));
        }
        sfx += to_fx(s1 + s2);
      } else if (want_ent) {
#pragma unroll
        for (int k = 0; k < P; ++k) add(x[k], c, true);
      } else {
        float s2 = 0.0f;
#pragma unroll
        for (int k = 0; k < P; k += 2) {
          s += ex2(wexp(x[k], c, mct));
          s2 += ex2(wexp(x[k + 1], c, mct));
        }
        s += s2;
      }
      if (kMode == SM_TOPP && vm >= t) {
#pragma unroll
        for (int k = 0; k < P; ++k)
          if (x[k] >= t) cm |= 1u << k;
      }
    }
    mt = fmax_nan(mt, vm);
    return cm;
  }

  // One element outside the vector path (chunk head or tail), row index j.
  __device__ __forceinline__ void scalar(float x, int j, float c, bool want_ent) {
    if constexpr (kMode == SM_GREEDY) {
      if (x > mt || (x == mt && j < am)) am = j;
    } else if constexpr (kSums) {
      if (x > mt) raise_max(x, c);
      add(x, c, want_ent);
    }
    mt = fmax_nan(mt, x);
  }
};


// ------------------------------------------------------------------ kernel
// Greedy and plain-sum CTAs need no candidate list and fit three to an SM.
template <typename T, int kMode>
__global__ void __launch_bounds__(kStreamThreads,
                                  (kMode == SM_TOPP ? 2 : (kMode == SM_TOPK ? SV_TOPK_CTAS : 3)))
    stream_rows_kernel(const StreamJob job) {
  constexpr bool kCand = kMode == SM_TOPK || kMode == SM_TOPP;
  constexpr int kCapM = kMode == SM_TOPK ? kCapTopK : kCap;  // candidates per row
  constexpr int E = Elem<T>::kBytes, P = Elem<T>::kPerVec;
  using RG = Ring<kMode>;
  constexpr int kRing = RG::kBuf, kRingBufBytes = RG::kBufBytes, kVecPerThread = RG::kVec;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ StreamAux aux;
  unsigned char* ring = smem;
  const RowJob& rj = job.r;
  const int nchunk = job.nchunk;
  // top-k: chunks between count exchanges, so that about kCapTopK / 2 entries can arrive
  // between two even when every chunk brings k new ones
  const int xchg_k = kMode == SM_TOPK ? max(1, (kCapTopK / 2) / max(1, rj.top_k)) : 0;
  // rows [0, rows), or the rows row_list[0 .. *row_count) when a list is given (logical index
  // lr -> row row_of(lr); statistics and outputs are indexed by the row itself)
  const long long nrows = rj.row_list ? (long long)*rj.row_count : rj.rows;
  auto row_of = [&](long long lr) { return rj.row_list ? (long long)rj.row_list[lr] : lr; };
  const long long nrows_mine =
      nrows > blockIdx.x ? (nrows - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const long long items = nrows_mine * nchunk;

  if (threadIdx.x == 0) {
    for (int b = 0; b < kRing; ++b) {
      mbar_init(&aux.full[b], 1);
      mbar_init(&aux.empty[b], kWarps);
    }
    aux.broken = 0;
    aux.ccount = 0;
  }
  __syncthreads();

  // ---------------------------------------------------------------- producer
  if (threadIdx.x >= kThreads) {
    if (threadIdx.x == kThreads) {
      uint32_t issued = 0, lastpar = 0;
      long long lr = blockIdx.x, row = nrows_mine > 0 ? row_of(lr) : 0;
      int q = 0, b = 0;
      for (long long g = 0; g < items; ++g) {
        // buffer b last held item g - kRing: wait until every consumer warp is done with it
        if (g >= kRing && !mbar_wait(&aux.empty[b], uint32_t((g / kRing - 1) & 1))) {
          atomicExch(&aux.broken, 1);
          break;
        }
        if (*reinterpret_cast<volatile int*>(&aux.broken)) break;
        const ChunkLoc s = chunk_at<T>(job, row, q);
        mbar_arrive_expect_tx(&aux.full[b], uint32_t(s.mid));
        unsigned char* dst = ring + size_t(b) * kRingBufBytes + s.pad + s.head;
        for (int off = 0; off < s.mid; off += kBulkChunk)
          bulk_g2s(dst + off, s.g + s.head + off, uint32_t(min(kBulkChunk, s.mid - off)),
                   &aux.full[b]);
        issued |= 1u << b;
        lastpar = (lastpar & ~(1u << b)) | (uint32_t((g / kRing) & 1) << b);
        if (++q == nchunk) {
          q = 0;
          lr += gridDim.x;
          if (g + 1 < items) row = row_of(lr);
        }
        if (++b == kRing) b = 0;
      }
      // no copy may still be landing when the CTA exits
      for (int bb = 0; bb < kRing; ++bb)
        if ((issued >> bb) & 1u) mbar_wait(&aux.full[bb], (lastpar >> bb) & 1u);
    }
    return;
  }

  // ---------------------------------------------------------------- consumers
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool want_ent = (rj.flags & RS_ENTROPY) != 0;
  const float c = rj.c;
  const double iT = rj.temp > 0.0f ? 1.0 / double(rj.temp) : 0.0;
  CandSet<T> cs;
  cs.cand = reinterpret_cast<uint64_t*>(smem + size_t(kRing) * kRingBufBytes);
  if (kMode == SM_TOPK) {
    cs.ranked = cs.cand + kCapTopK;
    cs.hcnt = nullptr;
    cs.hlimb = nullptr;
  } else {
    cs.ranked = nullptr;
    cs.hcnt = reinterpret_cast<uint32_t*>(cs.cand + kCap);
    cs.hlimb = cs.hcnt + kBins;
  }
  cs.aux = &aux;
  RowAcc<T, kMode> st;
  st.reset();
  float thr = -INFINITY;  // candidates: every entry seen this row that is >= thr (uniform)
  int cnt = 0;            // candidates appended this row (uniform)
  bool overflow = false;  // (uniform)
  bool row_timeout = false;
  int wacc = 0, wlen = 0, xpar = 0;  // count exchange: this warp's appends, chunks, parity
  int single = 0;                    // entries this thread appended one by one
  long long lr = blockIdx.x, row = nrows_mine > 0 ? row_of(lr) : 0;
  int q = 0, b = 0;

  for (long long g = 0; g < items; ++g) {
    const ChunkLoc s = chunk_at<T>(job, row, q);
    bool copied = false;
    if (!*reinterpret_cast<volatile int*>(&aux.broken)) {
      copied = mbar_wait(&aux.full[b], uint32_t((g / kRing) & 1));
      if (!copied) atomicExch(&aux.broken, 1);
    }
    if (!copied) row_timeout = true;
    const uint4* vb = reinterpret_cast<const uint4*>(ring + size_t(b) * kRingBufBytes);
    const int base = q * job.chunk;
    const int v_lo = (s.pad + s.head) >> 4, v_hi = (s.pad + s.head + s.mid) >> 4;
    // the chunk's vectors of this thread; top-k keeps only their maxima in registers and
    // reads a vector again from the ring in the rare case that it holds a candidate (the
    // buffer is released after the appends)
    auto load_vec = [&](int v) {
      return (copied && v >= v_lo && v < v_hi) ? vb[v] : neg_inf_vec<T>();
    };
    uint4 w[kMode == SM_TOPK ? 1 : kVecPerThread];
    float vm[kVecPerThread];
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
      const uint4 wu = load_vec(u * kThreads + int(threadIdx.x));
      vm[u] = Elem<T>::vmax_nan(wu);
      if constexpr (kMode != SM_TOPK) w[u] = wu;
    }
    auto vec_at = [&](int u) -> uint4 {
      if constexpr (kMode == SM_TOPK) return load_vec(u * kThreads + int(threadIdx.x));
      else return w[u];
    };
    // elements outside the bulk-copied middle (< 16 bytes at each end): thread 0 takes the
    // head, thread 32 the tail, from global memory
    const int head_e = s.head / E, tail_e0 = (s.head + s.mid) / E;
    const int e_lo = threadIdx.x == 0 ? 0 : tail_e0;
    const int e_hi = threadIdx.x == 0 ? head_e : (threadIdx.x == 32 ? s.n : 0);
    const bool edge = copied && e_lo < e_hi;

    if constexpr (kCand) {
      if (q == 0) {  // the row's first threshold, from this chunk's per-thread maxima
        float pm = -INFINITY;
#pragma unroll
        for (int u = 0; u < kVecPerThread; ++u) pm = fmax_nan(pm, vm[u]);
        if (edge)
          for (int j = e_lo; j < e_hi; ++j) pm = fmax_nan(pm, Elem<T>::load(s.g, j));
        if constexpr (kMode == SM_TOPK) {
          const int jw = (rj.top_k + kWarps - 1) / kWarps;  // <= 32: top_k <= 256
          uint32_t kw;
          if (jw <= 16) {  // a value that jw of the warp's per-thread maxima reach
            kw = warp_kth_key<Elem<T>::kKeyBits>(Elem<T>::key(pm), jw);
          } else {
            // large k: a per-thread maximum stands for eight vectors, too coarse a step;
            // a value that jw of the warp's vector maxima reach (vectors outside the
            // chunk hold -inf)
            uint32_t kv[kVecPerThread];
#pragma unroll
            for (int u = 0; u < kVecPerThread; ++u) kv[u] = Elem<T>::key(vm[u]);
            kw = warp_kth_key_n<Elem<T>::kKeyBits, kVecPerThread>(kv, jw);
          }
          thr = creduce<float>(key_value<T>(kw), aux.scr_f, OpMin());
        } else {
          const float m0 = creduce<float>(pm, aux.scr_f, OpMaxNan());
          float t0 = m0 - job.topp_span;
          if (m0 > -INFINITY && m0 < INFINITY) {
            // the vectors whose maxima fall in the bins up to the one where kChunk0Vecs of
            // them are reached; the smallest such maximum bounds what this chunk appends
            const float mc0 = m0 * c;
            for (int i = threadIdx.x; i < kBins; i += kThreads) cs.hcnt[i] = 0;
            csync();
#pragma unroll
            for (int u = 0; u < kVecPerThread; ++u) {
              const int v = u * kThreads + int(threadIdx.x);
              const bool ok = v >= v_lo && v < v_hi && vm[u] > -INFINITY;
              hist_add(cs.hcnt, ok ? bin_of(vm[u], c, mc0) : 0, ok);
            }
            csync();
            cs.hist_find((unsigned long long)kChunk0Vecs, false);
            const int bsel = aux.sel_found ? aux.sel_bin : kBins - 1;
            float tv = INFINITY;
#pragma unroll
            for (int u = 0; u < kVecPerThread; ++u) {
              const int v = u * kThreads + int(threadIdx.x);
              if (v >= v_lo && v < v_hi && vm[u] > -INFINITY && bin_of(vm[u], c, mc0) <= bsel)
                tv = fminf(tv, vm[u]);
            }
            tv = creduce<float>(tv, aux.scr_f, OpMin());
            if (tv < INFINITY) t0 = fmaxf(t0, tv);
          }
          thr = t0;
        }
      }
    }

    // ---- the chunk pass
    uint32_t cm[kVecPerThread];
    float vmax4 = -INFINITY;
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
      const int v = u * kThreads + int(threadIdx.x);
      const int j0 = base + (16 * v - s.pad) / E;
      cm[u] = st.vec(kMode == SM_TOPK ? uint4{} : vec_at(u), vm[u], j0, c, want_ent,
                     (v >= v_lo && v < v_hi) ? thr : INFINITY);
      vmax4 = fmaxf(vmax4, vm[u]);  // pad vectors hold -inf; NaN never passes a filter
    }
    if constexpr (kMode == SM_TOPK) {
      if (vmax4 >= thr) {
#pragma unroll
        for (int u = 0; u < kVecPerThread; ++u) {
          const int v = u * kThreads + int(threadIdx.x);
          if (v >= v_lo && v < v_hi && vm[u] >= thr) {
            float x[P];
            Elem<T>::unpack(vec_at(u), x);
#pragma unroll
            for (int k = 0; k < P; ++k)
              if (x[k] >= thr) cm[u] |= 1u << k;
          }
        }
      }
    }
    int wadd = 0;  // entries this warp appended in this chunk (uniform in the warp)
    if constexpr (kCand) {
      int my = 0;
#pragma unroll
      for (int u = 0; u < kVecPerThread; ++u) my += __popc(cm[u]);
      if (__any_sync(0xffffffffu, my != 0)) {  // one shared atomic for the warp
        int inc = my;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += t;
        }
        int wbase = 0;
        if (lane == 31) wbase = atomicAdd(&aux.ccount, inc);
        wadd = __shfl_sync(0xffffffffu, inc, 31);
        int pos = __shfl_sync(0xffffffffu, wbase, 31) + inc - my;
#pragma unroll
        for (int u = 0; u < kVecPerThread; ++u) {
          const int j0 = base + (16 * (u * kThreads + int(threadIdx.x)) - s.pad) / E;
          if (cm[u] == 0) continue;
          const uint4 wu = vec_at(u);
          for (uint32_t m = cm[u]; m != 0; m &= m - 1) {  // the set bits only
            const int k = __ffs(m) - 1;
            if (pos < kCapM) cs.cand[pos] = make_comp(Elem<T>::key_at(wu, k), j0 + k);
            ++pos;
          }
        }
      }
    }
    if (edge) {
      for (int j = e_lo; j < e_hi; ++j) {
        const float x = Elem<T>::load(s.g, j);
        st.scalar(x, base + j, c, want_ent);
        if (kCand && x >= thr) {
          const int pos = atomicAdd(&aux.ccount, 1);
          if (pos < kCapM) cs.cand[pos] = make_comp(Elem<T>::key(x), base + j);
          ++single;  // entries this thread appended one by one (edge elements)
        }
      }
    }
    // the buffer is free once every lane of the warp is done with it
    __syncwarp();
    if (lane == 0) mbar_arrive(&aux.empty[b]);

    if constexpr (kCand) {
      wacc += wadd;
      ++wlen;
      if ((kMode == SM_TOPP && wlen == kXchgTopP && q != nchunk - 1) ||
          (kMode == SM_TOPK && wlen == xchg_k && q != nchunk - 1) || q == 0) {
        // exchange: the row maximum so far and the entries appended since the last one
        float wm = st.mt;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) wm = fmax_nan(wm, __shfl_xor_sync(0xffffffffu, wm, o));
        const int wsingle = __reduce_add_sync(0xffffffffu, single);
        if (lane == 0) {
          aux.red_f[xpar][warp] = wm;
          aux.red_i[xpar][warp] = wacc + wsingle;
        }
        csync();
        float mrow = aux.red_f[xpar][0];
        int added = aux.red_i[xpar][0];
#pragma unroll
        for (int ww = 1; ww < kWarps; ++ww) {
          mrow = fmax_nan(mrow, aux.red_f[xpar][ww]);
          added += aux.red_i[xpar][ww];
        }
        xpar ^= 1;
        cnt += added;
        if (kMode == SM_TOPP) thr = fmaxf(thr, mrow - job.topp_span);
        const int rem = nchunk - 1 - q;  // chunks of this row still to come
        if (cnt > kCapM) {
          overflow = true;
        } else if (rem > 0 && ((kMode == SM_TOPK && cnt > rj.top_k) ||
                               cnt + added + added / 2 > kCapM ||
                               (cnt >= kCapM / 4 &&
                                cnt + (long long)added * rem / wlen > kCapM))) {
          // top-k: more than 2k candidates; or about to overflow, or projected to: cut
          // the list by count (top-k: to the exact k-th of the entries seen so far)
          int keep = rj.top_k;
          if (kMode == SM_TOPP) {
            const long long seen = min((long long)(q + 1) * job.chunk, (long long)rj.V);
            keep = max(kKeepFloor, int((long long)kKeepTarget * seen / rj.V));
          }
          if constexpr (kMode == SM_TOPK) {
            // the exact k-th of the entries seen so far becomes the threshold; a short list
            // keeps the entries below it (the row-end selection ranks past them), one past
            // half the capacity drops them
            if (cnt >= keep && cs.rank_select(cnt, 0, keep)) {
              const uint64_t kth = aux.sel_comp;
              thr = fmaxf(thr, key_value<T>(comp_key(kth)));
              if (cnt > kCapTopK / 2) cnt = cs.compact_ge(cnt, kth);
            }
          } else if (keep < cnt && mrow > -INFINITY && mrow < INFINITY) {
            cnt = cs.cut(cnt, keep, c, mrow * c, &thr);
          }
        }
        wacc = 0;
        single = 0;
        wlen = 0;
      }
    }

    if (q == nchunk - 1) {
      // ---------------------------------------------------------------- row end
      const bool tmo = csync_or(row_timeout);
      const int nall = aux.ccount;  // every append of the row is done (candidate modes)
      const float m = creduce<float>(st.mt, aux.scr_f, OpMaxNan());
      int status = tmo ? ROW_TIMEOUT
                       : ((m != m || m == INFINITY || m == -INFINITY) ? ROW_INVALID : ROW_OK);
      if (tmo && rj.dev_status && threadIdx.x == 0) atomicOr(rj.dev_status, 1);
      const float mc = m * c;
      uint32_t thr_key = 0;
      int cutoff = INT_MAX, am = -1;
      unsigned long long zfx = 0;
      double S1 = 0.0;
      double zd = -1.0;  // the double normaliser, where the kept set is in the list
      bool listed = false;
      if constexpr (kMode == SM_GREEDY) {
        if (status == ROW_OK)
          am = creduce<int>(st.mt == m ? st.am : INT_MAX, aux.scr_i, OpMin());
      } else if constexpr (kMode == SM_SUMS) {
        if (status == ROW_OK) {  // the per-thread online sums, relative to the row maximum
          float sc = 0.0f, hc = 0.0f;
          if (st.s != 0.0f) {
            const float d = mc - st.mct;  // >= 0
            const float scale = ex2(-d);
            sc = scale * st.s;
            hc = scale * (st.h - d * st.s);
          }
          zfx = creduce<unsigned long long>(to_fx(sc), aux.scr_u64, OpSum());
          S1 = creduce<double>(double(hc), aux.scr_f64, OpSum());
        }
      } else {
        if (status == ROW_OK) {
          const int n = min(nall, kCapM);
          bool ok = !overflow && nall <= kCapM;
          uint64_t cstar = 0;
          if constexpr (kMode == SM_TOPK) {
            ok = ok && n >= rj.top_k;
            if (ok) {  // every list is short (kCapTopK <= kRankMax): rank directly
              if (rj.top_p < 1.0f) {  // the top-p crossing within the top k
                ok = cs.rank_topp(n, rj.top_k, rj.top_p, m, iT);
              } else {
                ok = cs.rank_select(n, 0, rj.top_k);
              }
              cstar = aux.sel_comp;
            }
          } else {  // top-p over the whole row: the mass target from the online sums,
                    // relative to the row's integer reference rref = ceil(mc)
            const float rref = ceilf(mc);
            const float dsh = rref - st.mct;  // >= 0 for every thread with a sum
            const unsigned long long zt = (st.sfx && dsh < 64.0f) ? st.sfx >> int(dsh) : 0ull;
            const unsigned long long zall = creduce<unsigned long long>(zt, aux.scr_u64, OpSum());
            unsigned long long target =
                (unsigned long long)ceil(double(rj.top_p) * double(zall));
            if (target < 1) target = 1;
            if (ok) {
              cs.hist_build(n, 0, c, mc, true, rref);
              cs.hist_find(target, true);  // not found: the candidates hold too little mass
              ok = aux.sel_found && cs.resolve(n, 0, c, mc, true, target - aux.sel_before, rref);
              cstar = aux.sel_comp;
              if (ok && rj.refine_rows) {
                // the fp32 masses before and through the crossing; within the guard of the
                // target the decision goes to the double-precision refinement
                const unsigned long long before = aux.sel_before + aux.sel_mabove;
                const unsigned long long through = before + aux.sel_mw;
                const unsigned long long g =
                    (unsigned long long)ceil(double(kToppGuard) * double(zall)) + 1ull;
                if ((target - before <= g || through - target <= g) && threadIdx.x == 0)
                  rj.refine_rows[atomicAdd(rj.refine_count, 1)] = int32_t(row);
              }
            }
          }
          if (!ok) {
            status = ROW_FALLBACK;
          } else {
            // normaliser, entropy term and kept-id list over the kept candidates. Rows list
            // their kept ids (a nucleus of more than kKeptCap entries is not listed); top-k
            // rows leave the double normaliser to the consumer, which sums it over the list
            // if it needs it, and top-p rows get it here.
            const bool list = rj.kept_ids != nullptr;
            if (threadIdx.x == 0) aux.mcount = 0;
            csync();
            unsigned long long z = 0;
            long long s1 = 0;
            Fx128 zdx = fx_zero();
            if constexpr (kMode == SM_TOPP) zdx = kept_weights_fx<T>(cs.cand, n, cstar, m, iT);
            for (int i = threadIdx.x; i < n; i += kThreads) {
              const uint64_t e = cs.cand[i];
              if (e < cstar) continue;
              const float xv = key_value<T>(comp_key(e));
              const float zx = wexp(xv, c, mc);
              const float ex = ex2(zx);
              z += to_fx(ex);
              if (want_ent) s1 += __float2ll_rn(ent_term(ex, zx) * kS1Fx);
              if (list) {
                const int slot = atomicAdd(&aux.mcount, 1);
                if (slot < kKeptCap) rj.kept_ids[size_t(row) * kKeptCap + slot] = comp_id(e);
              }
            }
            if constexpr (kMode == SM_TOPP) zd = fx_to_double(creduce_fx(zdx, scr_fx(aux)));
            zfx = creduce<unsigned long long>(z, aux.scr_u64, OpSum());
            S1 = double(creduce<long long>(s1, aux.scr_s64, OpSum())) / double(kS1Fx);
            thr_key = comp_key(cstar);
            cutoff = comp_id(cstar);
            listed = list;
          }
        }
      }
      if (status == ROW_FALLBACK && threadIdx.x == 0)
        job.fb_rows[atomicAdd(job.fb_count, 1)] = int32_t(row);
      if (rj.kept_n && threadIdx.x == 0)
        rj.kept_n[row] = (listed && aux.mcount <= kKeptCap) ? aux.mcount : 0;
      const double Z = double(zfx) * kFxInv;
      const double ent = (status == ROW_OK && kMode != SM_GREEDY && want_ent)
                             ? log(Z) - 0.6931471805599453 * S1 / Z
                             : 0.0;
      if (rj.stats && threadIdx.x == 0) {
        RowStats rs;
        rs.mc = mc;
        rs.z = float(Z);
        rs.entropy = float(ent);
        rs.thr_key = thr_key;
        rs.cutoff = cutoff;
        rs.argmax = am;
        rs.status = status;
        rs.c = c;
        rs.m = m;
        rs.pad = 0;
        rs.zd = status == ROW_OK ? zd : -1.0;
        rj.stats[row] = rs;
      }
      // the next row starts clean
      st.reset();
      thr = -INFINITY;
      cnt = 0;
      wacc = 0;  // appends since the last exchange belong to this row
      single = 0;
      wlen = 0;
      overflow = false;
      row_timeout = false;
      if constexpr (kCand) {
        if (threadIdx.x == 0) aux.ccount = 0;
        csync();
      }
    }
    if (++b == kRing) b = 0;
    if (++q == nchunk) {
      q = 0;
      lr += gridDim.x;
      if (g + 1 < items) row = row_of(lr);
    }
  }
}

}  // namespace sv
