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
//   SM_TOPP    the online sum of the entries below the threshold and the candidate list.
// Top-k candidates are 64-bit composites (key << 32 | ~id): the order of composites is the
// order (value desc, id asc) that top-k and top-p use, so the k-th candidate is unique.
//
// Top-k: the first threshold is a value that k entries of the first chunk reach (per-warp
// order statistics of per-thread maxima; of vector maxima for k > 128). After the first
// chunk the consumer warps exchange their counts, and a list of more than k entries sets the
// threshold to the exact k-th seen so far (ranked directly) and drops the entries below it.
// Further exchanges run every (kCapTopK / 2) / k chunks, so about half the list can fill
// between two even if every chunk brings k new entries. Rows whose values do not grow along the vocabulary rarely reach the threshold again, and
// a list that still outgrows kCapTopK sends the row to the exact finisher. The short list
// keeps a top-k CTA small enough for three per SM.
//
// Top-p (bfloat16 rows): the threshold starts at (first-chunk maximum - T ln(V / (1 -
// top_p))), below which the whole row holds less than 1 - top_p of the mass, raised to the
// smallest of the largest kChunk0Vecs vector maxima of the first chunk if that is higher,
// and is always an exact bfloat16 value. A candidate is a 32-bit composite of its code
// (relative to the row's base code, the code of the first threshold) and its id, and is
// also counted in a histogram of codes. Candidates are left out of the online fp32 sums
// (their weight is replaced by 0 before the exponentials), so the sums hold only the
// entries below the threshold. The warps exchange counts and the row maximum after the
// first chunk and then every kXchgTopP chunks: the threshold follows the maximum, and a list
// about to overflow is cut to the codes holding its top max(kKeepFloor, kKeepTarget * seen /
// V) entries (the histogram keeps the counts of the entries cut).
//
// At the end of a row the CTA selects among the candidates. Top-k lists are ranked directly
// (each candidate counts the larger composites); with top-p as well, the top k go to their
// rank slots and a block scan of their weights finds the crossing. Top-p rows weigh the
// histogram's codes once each in double (exp((l - m) / T)); the total plus the fp32 sum of
// the entries below the threshold gives the mass target, a suffix scan over the codes finds
// the code where the mass crosses it and how many of its entries (in id order) are kept,
// and the list gives their ids. Only the sum below the threshold carries fp32 error: a
// crossing within its error bound of the target is listed for the exact placement
// (refine.cuh). The CTA writes the RowStats record and the kept ids. Rows the candidates
// cannot settle (list overflow, a code outside the histogram's window, a crossing among
// entries cut from the list or below the threshold) are marked ROW_FALLBACK and listed; the
// cluster kernel (row_stats.cuh) then finishes them.
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

// Ring of chunk buffers per CTA: two 32 KB chunks (24 KB for top-p). Every mode runs three
// CTAs per SM: top-k adds its list of kCapTopK candidates and the top k in rank order,
// top-p its list of 32-bit candidates, the code histogram and the crossing code's members.
// The depth and chunk size of each kind are build-time knobs.
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
#define SV_RING_KB_CAND 24
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
constexpr int kCapTopK = 1024;                  // top-k: candidates per row
constexpr int kCapP = 4096;                     // top-p: candidates per row (32-bit)
constexpr int kPBins = 1024;                    // top-p: codes of the histogram's window
constexpr int kPMem = 256;                      // top-p: entries of the crossing code
constexpr int kKeepFloor = 512;                 // top-p: a cut keeps at least this many
constexpr int kKeepTarget = 3 * kCapP / 8;      // top-p: candidates a cut aims at by row end
constexpr int kXchgTopP = 5;                    // top-p: chunks between count exchanges
constexpr int kBins = 1024;                     // log-weight bins
constexpr float kBinScale = 32.0f;              // bins per log2 unit of weight
constexpr int kRankMax = 1024;                  // lists this short are ranked directly
constexpr int kStreamMaxTopK = 256;             // top-k the candidate path takes
// Top-p: a bound on the error of the fp32 sum of the entries below the threshold, relative
// to that sum, in weights exp((l - m) / T) (max 1). Per entry of depth d = (m - l) log2(e) /
// T log2 units: c = fl(log2(e) / T) is off by 3 * 2^-24 at most (d * 3 * 2^-24 in the
// exponent), the exponent fl(l c - r) by 2^-24 of (d + 1), ex2.approx by 2^-22 relative,
// and the fp32 sum of a thread's share of a chunk (4 roundings within a vector, one per
// further vector: at most 10) by 10 * 2^-24; entries with d <= 32 are thus within
// ln2 * 2^-24 * (4 * 32 + 1) + 2^-22 + 10 * 2^-24 = 6.17e-6 of their weight, and the rest
// (each below 2^-32, at most 2^20 of them) are off by under 1.5e-9 in all. The fixed-point
// sums add at most 2^-42 per conversion (one per chunk and thread with a sum, and one per
// reference shift: fewer than one per vector) and per shift (kPGuardFxUnit).
constexpr double kPGuardRel = 6.2e-6;
constexpr double kPGuardAbs = 2.0e-9;
constexpr double kPGuardFxUnit = 2.2737367544323206e-13;  // 2^-42

// Dynamic shared memory of one CTA: the ring, then top-k: the candidate list and the top k
// in rank order; top-p: the candidate list, the code histogram and the crossing code's
// members.
__host__ __device__ constexpr size_t stream_dyn_bytes(int mode) {
  return mode <= SM_SUMS ? size_t(Ring<SM_SUMS>::kBuf) * Ring<SM_SUMS>::kBufBytes
         : mode == SM_TOPK
             ? size_t(Ring<SM_TOPK>::kBuf) * Ring<SM_TOPK>::kBufBytes + size_t(kCapTopK) * 8 +
                   size_t(kStreamMaxTopK) * 8
             : size_t(Ring<SM_TOPP>::kBuf) * Ring<SM_TOPP>::kBufBytes + size_t(kCapP) * 4 +
                   size_t(kPBins) * 4 + size_t(kPMem) * 4;
}
// top-p: per warp, the vectors of the first chunk whose maxima set its threshold (1 in 12)
constexpr int kChunk0WarpVecs = Ring<SM_TOPP>::kVec * 32 / 12;
static_assert(kPBins % kThreads == 0, "whole histogram bins per consumer thread");
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
  unsigned long long sel_x[2];  // top-k: the exchange's k-th, by exchange parity
  double sel_above;  // top-p: mass of the codes above the crossing code
  double sel_w;      // top-p: weight of the crossing code
  int sel_j;         // top-p: entries of the crossing code kept
  int sel_stable;    // top-p: the crossing lies outside the guard
  uint32_t sel_c32;  // top-p: the crossing composite
  int pover;         // top-p: a candidate's code fell outside the histogram's window
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
// hardware reserves per CTA, within the SM's 228 KB; likewise three top-p CTAs.
static_assert(SV_TOPK_CTAS >= 2 && SV_TOPK_CTAS <= 3, "top-k CTAs per SM");
static_assert(SV_TOPK_CTAS * (stream_dyn_bytes(SM_TOPK) + sizeof(StreamAux) + 1024) <= 228 * 1024,
              "the top-k CTAs of an SM fit its shared memory");
static_assert(3 * (stream_dyn_bytes(SM_TOPP) + sizeof(StreamAux) + 1024) <= 228 * 1024,
              "three top-p CTAs per SM");

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
// exp((x - m) / T) as Fx128.
template <typename T>
__device__ __noinline__ Fx128 weight_fx(uint32_t key, float m, double iT) {
  return fx_from(weight_d(key_value<T>(key), m, iT));
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

// Top-p candidates: 32-bit composites (rel << 20) | (2^20 - 1 - id), rel = the entry's code
// key minus the row's base key (rel < kPBins, id < 2^20): larger composite = larger value,
// then lower id.
__device__ __forceinline__ uint32_t pcomp(uint32_t rel, int id) {
  return (rel << 20) | (0xFFFFFu - uint32_t(id));
}
__device__ __forceinline__ uint32_t pcomp_rel(uint32_t e) { return e >> 20; }
__device__ __forceinline__ int pcomp_id(uint32_t e) { return int(0xFFFFFu - (e & 0xFFFFFu)); }

template <typename T>
struct CandSet {
  uint64_t* cand;              // top-k: [kCapTopK]
  uint64_t* ranked;            // top-k: [kStreamMaxTopK], the top k in rank order
  uint32_t* plist;             // top-p: [kCapP] candidates
  uint32_t* hcnt;              // top-p: [kPBins] code histogram (first chunk: vector-maxima bins)
  uint32_t* pmem;              // top-p: [kPMem] entries of the crossing code
  StreamAux* aux;

  // The bin of hcnt[0 .. kBins) where the count accumulated from bin 0 first reaches need:
  // aux->sel_found, sel_bin, sel_before (the count of the bins before it) and sel_cnt (its
  // count).
  __device__ void hist_find(unsigned long long need) {
    constexpr int kPer = kBins / kThreads;
    unsigned long long part[kPer];
    unsigned long long tsum = 0;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int b = threadIdx.x * kPer + q;
      part[q] = (unsigned long long)hcnt[b];
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

  // Top-p cut: the highest code c >= *lfloor whose entries and those above number at least
  // keep becomes the list's floor; the list plist[0..n) keeps the candidates of codes >= c
  // (all of them: every entry of a code at or above the floor is listed), *thr becomes
  // that code's value. The histogram keeps every count. Returns the new count. Thread t
  // holds the codes kPBins - 1 - kPer t down to kPBins - kPer (t + 1).
  __device__ int p_cut(int n, int keep, uint32_t base, int* lfloor, float* thr) {
    constexpr int kPer = kPBins / kThreads;
    const int top = kPBins - 1 - kPer * int(threadIdx.x);
    uint32_t part[kPer];
    uint32_t tsum = 0;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int bb = top - q;
      part[q] = bb >= *lfloor ? hcnt[bb] : 0u;
      tsum += part[q];
    }
    uint32_t total;
    const uint32_t ex = cscan<uint32_t>(tsum, aux->scr_u32, &total);
    if (threadIdx.x == 0) aux->sel_found = 0;
    csync();
    if (ex < uint32_t(keep) && uint32_t(keep) <= ex + tsum) {
      uint32_t acc = ex;
#pragma unroll
      for (int q = 0; q < kPer; ++q) {
        acc += part[q];
        if (acc >= uint32_t(keep)) {
          aux->sel_bin = top - q;
          aux->sel_found = 1;
          break;
        }
      }
    }
    csync();
    if (!aux->sel_found) return n;  // uniform: the list holds fewer than keep
    const int cf = aux->sel_bin;
    constexpr int kPerL = kCapP / kThreads;
    uint32_t v[kPerL];
    uint32_t keepm = 0;
    const int lo = threadIdx.x * kPerL;
#pragma unroll
    for (int q = 0; q < kPerL; ++q) {
      const int i = lo + q;
      v[q] = i < n ? plist[i] : 0u;
      if (i < n && int(pcomp_rel(v[q])) >= cf) keepm |= 1u << q;
    }
    uint32_t kept;
    uint32_t pos = cscan<uint32_t>(uint32_t(__popc(keepm)), aux->scr_u32, &kept);
#pragma unroll
    for (int q = 0; q < kPerL; ++q)
      if (keepm & (1u << q)) plist[pos++] = v[q];
    if (threadIdx.x == 0) aux->ccount = int(kept);
    csync();
    *lfloor = cf;
    *thr = fmaxf(*thr, key_value<T>(base + uint32_t(cf)));
    return int(kept);
  }

  // Top-p crossing over the code histogram's occupied bins 0..btop (relative to base), by
  // one warp (all 32 lanes call it; no block barrier): the codes are weighed once each in
  // double, exp((l - m) / T); Z is ztot if that is >= 0, else their total plus zrest. Lane L
  // holds per = ceil((btop + 1) / 32) codes from btop - per L down. Returns the code where
  // the mass accumulated from the top reaches top_p * Z (-1: none), with how many of its
  // entries are kept (*j, in id order), the mass above it (*above), its weight (*w) and
  // whether the crossing stays put when the target moves by guard either way (*stable).
  __device__ int p_cross_warp(int btop, uint32_t base, float m, double iT, float top_p,
                              double zrest, double ztot, double guard, int* j, double* above,
                              double* w, int* stable) const {
    const int lane = threadIdx.x & 31;
    const int per = (btop + 32) / 32;
    const int top = btop - per * lane;
    Fx128 tsum = fx_zero();
#pragma unroll 4
    for (int q = 0; q < per; ++q) {
      const int bb = top - q;
      const uint32_t cnt = bb >= 0 ? hcnt[bb] : 0u;
      if (cnt)
        tsum = fx_add(tsum, fx_mul_u32(fx_from(weight_d(key_value<T>(base + uint32_t(bb)), m, iT)),
                                       cnt));
    }
    Fx128 incl = tsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const Fx128 nb = fx_shfl_up(incl, o);
      if (lane >= o) incl = fx_add(incl, nb);
    }
    const Fx128 zh{__shfl_sync(0xffffffffu, incl.lo, 31), __shfl_sync(0xffffffffu, incl.hi, 31)};
    Fx128 ex = fx_shfl_up(incl, 1);
    if (lane == 0) ex = fx_zero();
    const double target = double(top_p) * (ztot >= 0.0 ? ztot : fx_to_double(zh) + zrest);
    const unsigned hit = __ballot_sync(
        0xffffffffu, fx_to_double(ex) < target && target <= fx_to_double(incl));
    if (!hit) return -1;  // the histogram holds less than the target
    const int cl = __ffs(hit) - 1;
    int bsel = -1, jj = 0, stb = 0;
    double ab = 0.0, wc = 0.0;
    if (lane == cl) {
      Fx128 acc = ex;
      for (int q = 0; q < per; ++q) {
        const int bb = top - q;
        const uint32_t cnt = bb >= 0 ? hcnt[bb] : 0u;
        if (!cnt) continue;
        const double wq = weight_d(key_value<T>(base + uint32_t(bb)), m, iT);
        const Fx128 nacc = fx_add(acc, fx_mul_u32(fx_from(wq), cnt));
        const double a = fx_to_double(acc), t = fx_to_double(nacc);
        if (a < target && target <= t) {
          // the fewest entries of the code that reach the target
          int k = int(ceil((target - a) / wq));
          k = max(1, min(int(cnt), k));
          while (k > 1 && a + double(k - 1) * wq >= target) --k;
          while (k < int(cnt) && a + double(k) * wq < target) ++k;
          bsel = bb;
          jj = k;
          ab = a;
          wc = wq;
          stb = (a + double(k - 1) * wq < target - guard && a + double(k) * wq >= target + guard)
                    ? 1 : 0;
          break;
        }
        acc = nacc;
      }
    }
    *j = __shfl_sync(0xffffffffu, jj, cl);
    *stable = __shfl_sync(0xffffffffu, stb, cl);
    *above = __shfl_sync(0xffffffffu, ab, cl);
    *w = __shfl_sync(0xffffffffu, wc, cl);
    return __shfl_sync(0xffffffffu, bsel, cl);
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
  // >= lim, by counting for each the larger ones (composites are distinct) -> *out, which
  // the caller zeroed before a barrier that precedes the call; a barrier must follow before
  // *out is read. No barrier inside.
  __device__ void rank_into(int n, uint64_t lim, int k, unsigned long long* out) const {
    for (int i = threadIdx.x; i < n; i += kThreads) {
      const uint64_t e = cand[i];
      if (e < lim) continue;
      int above = 0;
      for (int j = 0; j < n; ++j) above += cand[j] > e ? 1 : 0;  // (a fixed trip count)
      if (above == k - 1) *out = e;
    }
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
  // top-p: the online weight sum of the entries below the candidate threshold as 42-bit
  // fixed point, relative to the integer reference mct. A thread's weights of one chunk are
  // summed in fp32 (sp) and added exactly; a reference that rises by d shifts the sum right by
  // d bits (the
  // exact power of two, truncated below 2^-42), so the sum's error stays within a few fp32
  // roundings per weight (the bound kPGuardRel states) with no floating-point rescale in the
  // loop.
  unsigned long long sfx;
  float sp;  // top-p: the fp32 sum not yet added to sfx

  __device__ __forceinline__ void flush() {
    sfx += to_fx(sp);
    sp = 0.0f;
  }

  __device__ void reset() {
    mt = -INFINITY;
    am = INT_MAX;
    mct = 0.0f;
    s = 0.0f;
    h = 0.0f;
    sfx = 0ull;
    sp = 0.0f;
  }

  // Raises the running maximum to vm (> mt), rescaling the online sums.
  __device__ __forceinline__ void raise_max(float vm, float c) {
    const float nm = vm * c;
    if constexpr (kMode == SM_TOPP) {
      const float nr = ceilf(nm);
      flush();
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
  // hold -inf). vm = its largest value; the sums' reference already covers it (the caller
  // raises it to the chunk's maximum first, so the vectors of a chunk carry no dependence
  // through it). Top-p: returns the mask of its entries >= t (the candidates, bit k for
  // entry k), which the sums leave out; 0 in the other modes.
  __device__ __forceinline__ uint32_t vec(const uint4& w, float vm, int j0, float c,
                                          bool want_ent, float t) {
    constexpr int P = Elem<T>::kPerVec;
    uint32_t cm = 0u;
    if (!(vm > -INFINITY)) {  // all -inf (weight 0), or a NaN
      mt = fmax_nan(mt, vm);
      return (kMode == SM_TOPP && vm >= t) ? (1u << P) - 1u : 0u;  // all -inf, t = -inf
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
      float x[P];
      if constexpr (kMode == SM_TOPP) {
        // candidates become -inf (weight 0) in the copy the sums read; bfloat16 vectors take
        // the packed compares whether or not they hold one (four compares and selects cost
        // less than a branch between the vectors of a chunk)
        uint4 ws = w;
        if (sizeof(T) == 2 || vm >= t) {
          if constexpr (sizeof(T) == 2) {
            const __nv_bfloat162 tt = __float2bfloat162_rn(t);  // t is a bfloat16 value
            uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint32_t mk = __hge2_mask(Elem<T>::pair(a[i]), tt);
              a[i] = (a[i] & ~mk) | (mk & 0xFF80FF80u);
              cm |= ((mk & 1u) | ((mk >> 15) & 2u)) << (2 * i);  // entries 2i, 2i + 1
            }
            ws = make_uint4(a[0], a[1], a[2], a[3]);
          } else {
            uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
              if (__uint_as_float(a[i]) >= t) {
                a[i] = 0xFF800000u;
                cm |= 1u << i;
              }
            ws = make_uint4(a[0], a[1], a[2], a[3]);
          }
        }
        Elem<T>::unpack(ws, x);
        // two chains, their exponents and additions in packed pairs
        float2 s12 = make_float2(0.0f, 0.0f);
        const float2 c2 = make_float2(c, c), m2 = make_float2(-mct, -mct);
#pragma unroll
        for (int k = 0; k < P; k += 2) {
          const float2 z = ffma2(make_float2(x[k], x[k + 1]), c2, m2);
          s12 = fadd2(s12, make_float2(ex2(z.x), ex2(z.y)));
        }
        sp += s12.x + s12.y;
      } else if (want_ent) {
        Elem<T>::unpack(w, x);
#pragma unroll
        for (int k = 0; k < P; ++k) add(x[k], c, true);
      } else {
        Elem<T>::unpack(w, x);
        // two chains (s and s2), their exponents and additions in packed pairs
        float2 ss = make_float2(s, 0.0f);
        const float2 c2 = make_float2(c, c), m2 = make_float2(-mct, -mct);
#pragma unroll
        for (int k = 0; k < P; k += 2) {
          const float2 z = ffma2(make_float2(x[k], x[k + 1]), c2, m2);
          ss = fadd2(ss, make_float2(ex2(z.x), ex2(z.y)));
        }
        s = ss.x + ss.y;
      }
    }
    mt = fmax_nan(mt, vm);
    return cm;
  }

  // One element outside the vector path (chunk head or tail), row index j; top-p sums
  // only the entries that are not candidates (sum).
  __device__ __forceinline__ void scalar(float x, int j, float c, bool want_ent, bool sum) {
    if constexpr (kMode == SM_GREEDY) {
      if (x > mt || (x == mt && j < am)) am = j;
    } else if constexpr (kSums) {
      if (x > mt) raise_max(x, c);
      if (sum) add(x, c, want_ent);
    }
    mt = fmax_nan(mt, x);
  }
};


// ------------------------------------------------------------------ kernel
// Greedy and plain-sum CTAs need no candidate list and fit three to an SM.
template <typename T, int kMode>
__global__ void __launch_bounds__(kStreamThreads, (kMode == SM_TOPK ? SV_TOPK_CTAS : 3))
    stream_rows_kernel(const StreamJob job) {
  constexpr bool kCand = kMode == SM_TOPK || kMode == SM_TOPP;
  constexpr int kCapM = kMode == SM_TOPK ? kCapTopK : kCapP;  // candidates per row
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
    aux.pover = 0;
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
  unsigned char* const cand_area = smem + size_t(kRing) * kRingBufBytes;
  if (kMode == SM_TOPK) {
    cs.cand = reinterpret_cast<uint64_t*>(cand_area);
    cs.ranked = cs.cand + kCapTopK;
    cs.plist = nullptr;
    cs.hcnt = nullptr;
    cs.pmem = nullptr;
  } else {
    cs.cand = nullptr;
    cs.ranked = nullptr;
    cs.plist = reinterpret_cast<uint32_t*>(cand_area);
    cs.hcnt = cs.plist + kCapP;
    cs.pmem = cs.hcnt + kPBins;
  }
  cs.aux = &aux;
  RowAcc<T, kMode> st;
  st.reset();
  float thr = -INFINITY;  // candidates: every entry seen this row that is >= thr (uniform)
  uint32_t pbase = 0;     // top-p: the key of the row's histogram bin 0 (uniform)
  int lfloor = 0;         // top-p: every entry of a code >= pbase + lfloor is listed (uniform)
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
    // the chunk's vectors of this thread; the candidate modes keep only their maxima in
    // registers and read a vector again from the ring when they need it (top-k: in the rare
    // case that it holds a candidate; top-p: for the sums; the buffer is released after the
    // appends)
    constexpr bool kReload = kMode == SM_TOPK || kMode == SM_TOPP;
    auto load_vec = [&](int v) {
      return (copied && v >= v_lo && v < v_hi) ? vb[v] : neg_inf_vec<T>();
    };
    uint4 w[kReload ? 1 : kVecPerThread];
    float vm[kVecPerThread];
    uint32_t cm[kVecPerThread];
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
      const uint4 wu = load_vec(u * kThreads + int(threadIdx.x));
      vm[u] = Elem<T>::vmax_nan(wu);
      if constexpr (!kReload) w[u] = wu;
    }
    auto vec_at = [&](int u) -> uint4 {
      if constexpr (kReload) return load_vec(u * kThreads + int(threadIdx.x));
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
          // top-p: each warp takes the maximum of its share of the chunk and a value that
          // kChunk0WarpVecs of its vector maxima reach; one exchange combines them (the
          // smallest such value: every warp has that many vectors at or above it)
          float wm0 = pm;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) wm0 = fmax_nan(wm0, __shfl_xor_sync(0xffffffffu, wm0, o));
          uint32_t kv[kVecPerThread];
#pragma unroll
          for (int u = 0; u < kVecPerThread; ++u) {
            const int v = u * kThreads + int(threadIdx.x);
            kv[u] = (v >= v_lo && v < v_hi && vm[u] == vm[u]) ? Elem<T>::key(vm[u]) : 0u;
          }
          const uint32_t kw =
              warp_kth_key_n<Elem<T>::kKeyBits, kVecPerThread>(kv, kChunk0WarpVecs);
          for (int i = threadIdx.x; i < kPBins; i += kThreads) cs.hcnt[i] = 0;  // starts empty
          if (lane == 0) {
            aux.red_f[xpar][warp] = wm0;
            aux.red_i[xpar][warp] = int(kw);
          }
          csync();
          float m0 = aux.red_f[xpar][0];
          uint32_t kmin = uint32_t(aux.red_i[xpar][0]);
#pragma unroll
          for (int ww = 1; ww < kWarps; ++ww) {
            m0 = fmax_nan(m0, aux.red_f[xpar][ww]);
            kmin = min(kmin, uint32_t(aux.red_i[xpar][ww]));
          }
          xpar ^= 1;
          float t0 = m0 - job.topp_span;
          if (m0 > -INFINITY && m0 < INFINITY) {
            t0 = fmaxf(t0, key_value<T>(kmin));
            // the window of kPBins codes starts at the threshold's code, and at most
            // kPBins - 256 codes below the first chunk's maximum
            uint32_t kb = Elem<T>::key(t0);
            const uint32_t ktop = Elem<T>::key(m0) + 256u;
            if (ktop > kb + uint32_t(kPBins - 1)) kb = ktop - uint32_t(kPBins - 1);
            pbase = kb;
            t0 = key_value<T>(kb);  // an exact value: entries of code >= kb are candidates
          } else {
            // an empty first chunk (-inf: every entry is appended, the list overflows and
            // the cluster kernel finishes the row) or a NaN (invalid: nothing is appended)
            if (!(m0 == m0)) t0 = INFINITY;
            pbase = Elem<T>::key(t0);
          }
          lfloor = 0;
          thr = t0;
        }
      }
    }

    // ---- the chunk pass
    if constexpr (RowAcc<T, kMode>::kSums) {
      // the sums' reference rises once per chunk, to the largest value of this thread's
      // vectors (fmaxf passes over a NaN; such a row is invalid)
      float cmax = -INFINITY;
#pragma unroll
      for (int u = 0; u < kVecPerThread; ++u) cmax = fmaxf(cmax, vm[u]);
      if (cmax > st.mt) st.raise_max(cmax, c);
    }
    float vmax4 = -INFINITY;
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
      const int v = u * kThreads + int(threadIdx.x);
      const int j0 = base + (16 * v - s.pad) / E;
      cm[u] = st.vec(kMode == SM_TOPK ? uint4{} : vec_at(u), vm[u], j0, c, want_ent,
                     (v >= v_lo && v < v_hi) ? thr : INFINITY);
      vmax4 = fmaxf(vmax4, vm[u]);  // pad vectors hold -inf; NaN never passes a filter
    }
    if constexpr (kMode == SM_TOPP) st.flush();
    int wadd = 0;  // entries this warp appended in this chunk (uniform in the warp)
    if constexpr (kMode == SM_TOPK) {
      // the candidates' bits, from the ring again (most vectors hold none)
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
    } else if constexpr (kMode == SM_TOPP) {
      // the candidates' bits from the sums pass, 8 per vector slot u (bit 8 (u % 4) + k of
      // mb[u / 4])
      static_assert(kVecPerThread <= 8, "two words of candidate bits per thread");
      uint32_t mb[2] = {0u, 0u};
#pragma unroll
      for (int u = 0; u < kVecPerThread; ++u) mb[u >> 2] |= cm[u] << (8 * (u & 3));
      // warp-cooperative appends: the warp's candidates in (lane, slot, element) order,
      // one per lane per round, each lane reading its entry from the ring
      const int my = __popc(mb[0]) + __popc(mb[1]);
      int inc = my;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
      }
      wadd = __shfl_sync(0xffffffffu, inc, 31);
      if (wadd) {
        int wbase = 0;
        if (lane == 31) wbase = atomicAdd(&aux.ccount, wadd);
        wbase = __shfl_sync(0xffffffffu, wbase, 31);
        const unsigned char* rb = ring + size_t(b) * kRingBufBytes;
        for (int j0 = 0; j0 < wadd; j0 += 32) {
          const int j = j0 + lane;
          // the lane holding candidate j: the number of lanes whose inclusive count is <= j
          int src = 0;
#pragma unroll
          for (int st = 16; st > 0; st >>= 1) {
            const int c_in = __shfl_sync(0xffffffffu, inc, src + st - 1);
            if (c_in <= j) src += st;
          }
          src = min(src, 31);
          const int ex_s = __shfl_sync(0xffffffffu, inc - my, src);
          const uint32_t m0s = __shfl_sync(0xffffffffu, mb[0], src);
          const uint32_t m1s = __shfl_sync(0xffffffffu, mb[1], src);
          if (j < wadd) {
            int r = j - ex_s;  // its rank among that lane's candidates
            const int c0 = __popc(m0s);
            const int word = r < c0 ? 0 : 1;
            if (word) r -= c0;
            const int bit = int(__fns(word ? m1s : m0s, 0u, r + 1));
            const int u = 4 * word + (bit >> 3), k = bit & 7;
            const int v = u * kThreads + warp * 32 + src;
            uint32_t key;
            if constexpr (E == 2) {
              const uint32_t h = *reinterpret_cast<const unsigned short*>(rb + 16 * v + 2 * k);
              key = Elem<T>::key(__uint_as_float(h << 16));
            } else {
              key = Elem<T>::key(*reinterpret_cast<const float*>(rb + 16 * v + 4 * k));
            }
            const int id = base + (16 * v - s.pad) / E + k;
            const int pos = wbase + j;
            const uint32_t rel = key - pbase;
            if (rel < uint32_t(kPBins)) {
              if (pos < kCapM) cs.plist[pos] = pcomp(rel, id);
              atomicAdd(&cs.hcnt[rel], 1u);
            } else {
              aux.pover = 1;
            }
          }
        }
      }
    }
    if (edge) {
      for (int j = e_lo; j < e_hi; ++j) {
        const float x = Elem<T>::load(s.g, j);
        const bool is_cand = kCand && x >= thr;
        st.scalar(x, base + j, c, want_ent, !is_cand);
        if (is_cand) {
          const int pos = atomicAdd(&aux.ccount, 1);
          if constexpr (kMode == SM_TOPK) {
            if (pos < kCapM) cs.cand[pos] = make_comp(Elem<T>::key(x), base + j);
          } else {
            const uint32_t rel = Elem<T>::key(x) - pbase;
            if (rel < uint32_t(kPBins)) {
              if (pos < kCapM) cs.plist[pos] = pcomp(rel, base + j);
              atomicAdd(&cs.hcnt[rel], 1u);
            } else {
              aux.pover = 1;
            }
          }
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
          (kMode == SM_TOPK && ((wlen == xchg_k && q != nchunk - 1) || q == 0))) {
        // exchange: the row maximum so far and the entries appended since the last one
        float wm = st.mt;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) wm = fmax_nan(wm, __shfl_xor_sync(0xffffffffu, wm, o));
        const int wsingle = __reduce_add_sync(0xffffffffu, single);
        if (lane == 0) {
          aux.red_f[xpar][warp] = wm;
          aux.red_i[xpar][warp] = wacc + wsingle;
        }
        if (kMode == SM_TOPK && threadIdx.x == 0) aux.sel_x[xpar] = 0ull;
        const int xp = xpar;
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
        if (kMode == SM_TOPP) {
          // the threshold follows the maximum, as an exact value (the code at or below it)
          const float tn = mrow - job.topp_span;
          if (tn > thr) thr = key_value<T>(Elem<T>::key(tn));
        }
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
            // the exact k-th of the entries seen so far becomes the threshold, and the list
            // drops the entries below it
            bool have = false;
            if (cnt >= keep) {  // (uniform)
              cs.rank_into(cnt, 0, keep, &aux.sel_x[xp]);
              csync();
              have = aux.sel_x[xp] != 0ull;
            }
            if (have) {
              const uint64_t kth = aux.sel_x[xp];
              thr = fmaxf(thr, key_value<T>(comp_key(kth)));
              cnt = cs.compact_ge(cnt, kth);  // the row end then ranks a short list
            }
          } else if (keep < cnt) {
            cnt = cs.p_cut(cnt, keep, pbase, &lfloor, &thr);
          }
        }
        wacc = 0;
        single = 0;
        wlen = 0;
      }
    }

    if (kMode == SM_TOPP && q == nchunk - 1) {
      // ---------------------------------------------------------------- top-p row end
      // one exchange: per warp the timeout flag, the maximum and the sum below the
      // threshold, relative to the warp's integer reference ceil(fl(max * c))
      float wmx = st.mt;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) wmx = fmax_nan(wmx, __shfl_xor_sync(0xffffffffu, wmx, o));
      const float wref = ceilf(wmx * c);
      const float dsw = wref - st.mct;  // >= 0 for every thread with a sum
      unsigned long long zw = (st.sfx && dsw < 64.0f) ? st.sfx >> int(dsw) : 0ull;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) zw += __shfl_xor_sync(0xffffffffu, zw, o);
      const bool wtmo = __any_sync(0xffffffffu, row_timeout);
      if (lane == 0) {
        aux.red_f[xpar][warp] = wmx;
        aux.red_i[xpar][warp] = wtmo ? 1 : 0;
        aux.scr_u64[warp] = zw;
      }
      csync();
      const int nall = aux.ccount;  // every append of the row is done
      float m = aux.red_f[xpar][0];
      bool tmo = aux.red_i[xpar][0] != 0;
#pragma unroll
      for (int ww = 1; ww < kWarps; ++ww) {
        m = fmax_nan(m, aux.red_f[xpar][ww]);
        tmo = tmo || aux.red_i[xpar][ww] != 0;
      }
      int status = tmo ? ROW_TIMEOUT
                       : ((m != m || m == INFINITY || m == -INFINITY) ? ROW_INVALID : ROW_OK);
      const float mc = m * c;
      // the sum of the entries below the threshold, relative to the row's integer reference
      // rref = ceil(mc), then in weights exp((l - m) / T)
      const float rref = ceilf(mc);
      unsigned long long zb = 0ull;
#pragma unroll
      for (int ww = 0; ww < kWarps; ++ww) {
        const float d = rref - ceilf(aux.red_f[xpar][ww] * c);
        const unsigned long long z = aux.scr_u64[ww];
        zb += (z && d < 64.0f) ? z >> int(d) : 0ull;
      }
      const double fxw = kFxInv * exp2(double(rref) - double(m) * double(c));
      const double sbelow = double(zb) * fxw;
      // its error bound: the weights' fp32 error, the fixed-point roundings (one per
      // vector, per reference shift and per warp's and thread's final shift)
      const double guard = kPGuardRel * sbelow + kPGuardAbs +
                           (double(rj.V) / 8.0 + 66.0 * kThreads) * kPGuardFxUnit * (fxw / kFxInv);
      const int n = min(nall, kCapM);
      const bool go = status == ROW_OK && !overflow && nall <= kCapM && !aux.pover;
      // warp 0: the crossing code over the histogram's occupied bins
      if (warp == 0) {
        int j = 0, stable = 0, bsel = -1;
        double above = 0.0, wc = 0.0;
        if (go) {
          const int km = int(Elem<T>::key(m)) - int(pbase);
          if (km >= 0)
            bsel = cs.p_cross_warp(min(km, kPBins - 1), pbase, m, iT, rj.top_p, sbelow, -1.0,
                                   double(rj.top_p) * guard, &j, &above, &wc, &stable);
          // a crossing below the list's floor, or with too many entries at its code
          if (bsel < lfloor || cs.hcnt[bsel >= 0 ? bsel : 0] > uint32_t(kPMem)) bsel = -1;
        }
        if (lane == 0) {
          aux.sel_bin = bsel;
          aux.sel_j = j;
          aux.sel_stable = stable;
          aux.sel_above = above + double(j) * wc;  // the kept mass
          aux.mcount = 0;  // kept ids listed
          aux.sel_cnt = 0u;  // entries of the crossing code gathered
        }
      }
      csync();
      const int bsel = aux.sel_bin;
      if (status == ROW_OK && bsel < 0) status = ROW_FALLBACK;
      const bool ok = status == ROW_OK;
      const bool list = ok && rj.kept_ids != nullptr;
      // the fp32 normaliser, entropy term and kept-id list: every warp takes the entries of
      // the codes above the crossing code and gathers those of the crossing code; then warp
      // 0 keeps the j of them with the lowest ids
      unsigned long long z = 0;
      long long s1 = 0;
      auto keep = [&](uint32_t e) {
        const float xv = key_value<T>(pbase + pcomp_rel(e));
        const float zx = wexp(xv, c, mc);
        const float ex = ex2(zx);
        z += to_fx(ex);
        if (want_ent) s1 += __float2ll_rn(ent_term(ex, zx) * kS1Fx);
        if (list) {
          const int slot = atomicAdd(&aux.mcount, 1);
          if (slot < kKeptCap) rj.kept_ids[size_t(row) * kKeptCap + slot] = pcomp_id(e);
        }
      };
      if (ok) {
        for (int i = threadIdx.x; i < n; i += kThreads) {
          const uint32_t e = cs.plist[i];
          const int r = int(pcomp_rel(e));
          if (r > bsel) {
            keep(e);
          } else if (r == bsel) {
            const uint32_t slot = atomicAdd(&aux.sel_cnt, 1u);
            if (slot < uint32_t(kPMem)) cs.pmem[slot] = e;
          }
        }
      }
      csync();
      if (ok && warp == 0) {
        const int nm = min(int(aux.sel_cnt), kPMem);
        const int j = aux.sel_j;
        uint32_t cst = 0u;
        bool got = false;
        for (int i = lane; i < nm; i += 32) {
          const uint32_t e = cs.pmem[i];
          int ab = 0;
          for (int q = 0; q < nm; ++q) ab += cs.pmem[q] > e ? 1 : 0;
          if (ab < j) keep(e);  // one of the j largest composites: the j lowest ids
          if (ab == j - 1) {
            cst = e;
            got = true;
          }
        }
        const unsigned g = __ballot_sync(0xffffffffu, got);
        if (lane == 0) aux.sel_c32 = g ? 0u : 1u;  // (1: not found)
        if (g && lane == __ffs(g) - 1) aux.sel_comp = cst;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        z += __shfl_xor_sync(0xffffffffu, z, o);
        s1 += __shfl_xor_sync(0xffffffffu, s1, o);
      }
      if (lane == 0) {
        aux.scr_u64[warp] = z;
        aux.scr_s64[warp] = s1;
      }
      csync();
      const uint32_t cstar = uint32_t(aux.sel_comp);
      if (ok && aux.sel_c32 != 0u) status = ROW_FALLBACK;
      if (threadIdx.x == 0) {
        unsigned long long zfx = 0;
        long long s1a = 0;
#pragma unroll
        for (int ww = 0; ww < kWarps; ++ww) {
          zfx += aux.scr_u64[ww];
          s1a += aux.scr_s64[ww];
        }
        if (tmo && rj.dev_status) atomicOr(rj.dev_status, 1);
        const bool settled = status == ROW_OK;
        if (settled && !aux.sel_stable && rj.refine_rows) {
          const int li = atomicAdd(rj.refine_count, 1);
          rj.refine_rows[li] = int32_t(row);
          rj.refine_z[2 * li] = 0ull;  // the exact normaliser's accumulator
          rj.refine_z[2 * li + 1] = 0ull;
        }
        if (status == ROW_FALLBACK) job.fb_rows[atomicAdd(job.fb_count, 1)] = int32_t(row);
        if (rj.kept_n)
          rj.kept_n[row] = (settled && list && aux.mcount <= kKeptCap) ? aux.mcount : 0;
        const double Z = double(zfx) * kFxInv;
        const double S1 = double(s1a) / double(kS1Fx);
        if (rj.stats) {
          RowStats rs;
          rs.mc = mc;
          rs.z = float(Z);
          rs.entropy = (settled && want_ent) ? float(log(Z) - 0.6931471805599453 * S1 / Z) : 0.0f;
          rs.thr_key = settled ? pbase + pcomp_rel(cstar) : 0u;
          rs.cutoff = settled ? pcomp_id(cstar) : INT_MAX;
          rs.argmax = -1;
          rs.status = status;
          rs.c = c;
          rs.m = m;
          rs.pad = 0;
          rs.zd = settled ? aux.sel_above : -1.0;
          rj.stats[row] = rs;
        }
        // the next row starts clean (its first exchange orders this before its appends)
        aux.ccount = 0;
        aux.pover = 0;
      }
      st.reset();
      thr = -INFINITY;
      cnt = 0;
      wacc = 0;
      single = 0;
      wlen = 0;
      overflow = false;
      row_timeout = false;
    } else if (kMode == SM_TOPK && q == nchunk - 1) {
      // ---------------------------------------------------------------- top-k row end
      // one exchange: per warp the timeout flag and the maximum
      float wmx = st.mt;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) wmx = fmax_nan(wmx, __shfl_xor_sync(0xffffffffu, wmx, o));
      const bool wtmo = __any_sync(0xffffffffu, row_timeout);
      if (lane == 0) {
        aux.red_f[xpar][warp] = wmx;
        aux.red_i[xpar][warp] = wtmo ? 1 : 0;
      }
      if (threadIdx.x == 0) {
        aux.sel_comp = 0ull;
        aux.mcount = 0;
      }
      csync();
      const int nall = aux.ccount;  // every append of the row is done
      float m = aux.red_f[xpar][0];
      bool tmo = aux.red_i[xpar][0] != 0;
#pragma unroll
      for (int ww = 1; ww < kWarps; ++ww) {
        m = fmax_nan(m, aux.red_f[xpar][ww]);
        tmo = tmo || aux.red_i[xpar][ww] != 0;
      }
      int status = tmo ? ROW_TIMEOUT
                       : ((m != m || m == INFINITY || m == -INFINITY) ? ROW_INVALID : ROW_OK);
      const float mc = m * c;
      const int n = min(nall, kCapM);
      const bool go = status == ROW_OK && !overflow && nall <= kCapM && n >= rj.top_k;
      // the k-th composite (every list is short, kCapTopK <= kRankMax: ranked directly); with
      // top-p, the crossing within the top k
      if (go) {
        if (rj.top_p < 1.0f) {
          cs.rank_topp(n, rj.top_k, rj.top_p, m, iT);
        } else {
          cs.rank_into(n, 0, rj.top_k, &aux.sel_comp);
          csync();
        }
      } else {
        csync();
      }
      const uint64_t cstar = aux.sel_comp;
      if (status == ROW_OK && cstar == 0ull) status = ROW_FALLBACK;
      const bool ok = status == ROW_OK;
      const bool list = ok && rj.kept_ids != nullptr;
      // normaliser, entropy term and kept-id list over the kept candidates; the double
      // normaliser is left to the consumer, which sums it over the list if it needs it
      unsigned long long z = 0;
      long long s1 = 0;
      if (ok) {
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
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        z += __shfl_xor_sync(0xffffffffu, z, o);
        s1 += __shfl_xor_sync(0xffffffffu, s1, o);
      }
      if (lane == 0) {
        aux.scr_u64[warp] = z;
        aux.scr_s64[warp] = s1;
      }
      csync();
      if (threadIdx.x == 0) {
        unsigned long long zfx = 0;
        long long s1a = 0;
#pragma unroll
        for (int ww = 0; ww < kWarps; ++ww) {
          zfx += aux.scr_u64[ww];
          s1a += aux.scr_s64[ww];
        }
        if (tmo && rj.dev_status) atomicOr(rj.dev_status, 1);
        if (status == ROW_FALLBACK) job.fb_rows[atomicAdd(job.fb_count, 1)] = int32_t(row);
        if (rj.kept_n) rj.kept_n[row] = (list && aux.mcount <= kKeptCap) ? aux.mcount : 0;
        const double Z = double(zfx) * kFxInv;
        const double S1 = double(s1a) / double(kS1Fx);
        if (rj.stats) {
          RowStats rs;
          rs.mc = mc;
          rs.z = float(Z);
          rs.entropy = (ok && want_ent) ? float(log(Z) - 0.6931471805599453 * S1 / Z) : 0.0f;
          rs.thr_key = ok ? comp_key(cstar) : 0u;
          rs.cutoff = ok ? comp_id(cstar) : INT_MAX;
          rs.argmax = -1;
          rs.status = status;
          rs.c = c;
          rs.m = m;
          rs.pad = 0;
          rs.zd = -1.0;
          rj.stats[row] = rs;
        }
        aux.ccount = 0;  // the next row starts clean (its first exchange orders this)
      }
      st.reset();
      thr = -INFINITY;
      cnt = 0;
      wacc = 0;
      single = 0;
      wlen = 0;
      overflow = false;
      row_timeout = false;
    } else if (q == nchunk - 1) {
      // ---------------------------------------------------------------- row end (greedy, sums)
      const bool tmo = csync_or(row_timeout);
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
        if (threadIdx.x == 0) {
          aux.ccount = 0;
          aux.pover = 0;
        }
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
