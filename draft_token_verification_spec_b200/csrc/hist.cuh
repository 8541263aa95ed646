// Exact double-precision sums of exp((l - m) / T) over a bfloat16 logit row through a
// histogram of its 16-bit codes.
//
// The weight of an entry depends on its code alone, so a row of V entries has at most as
// many distinct weights as distinct codes: a few thousand for logit rows, against V up to
// 2^20. One pass counts the entries per code (16-bit counters in shared memory, two to a
// word, one for each of the 65536 codes); each occupied code is then weighed once in double
// and its weight, as 128-bit fixed point, multiplied by its count. Fixed-point sums are
// exact, so the total equals the entry-by-entry Fx128 sum bit for bit (the sum the rest of
// the library takes). A counter that would pass 65535 makes the caller sum the row entry by
// entry instead.
#pragma once

#include "draw.cuh"
#include "row_stats.cuh"

namespace sv {

constexpr int kHistCodes = 65536;                       // every bfloat16 code
constexpr int kHistWords = kHistCodes / 2;              // two 16-bit counters per word
constexpr size_t kHistBytes = size_t(kHistWords) * 4;   // 128 KB of shared memory

__device__ __forceinline__ void hist_clear(uint32_t* hist) {
  uint4* h4 = reinterpret_cast<uint4*>(hist);
  for (int i = threadIdx.x; i < kHistWords / 4; i += kThreads) h4[i] = make_uint4(0, 0, 0, 0);
}

// Counts an entry of key k (its code's 16-bit order key) in the histogram; returns false if
// its counter overflowed.
__device__ __forceinline__ bool hist_count(uint32_t* hist, uint32_t k) {
  const uint32_t sh = (k & 1u) << 4;
  const uint32_t old = atomicAdd(&hist[k >> 1], 1u << sh);
  return ((old >> sh) & 0xFFFFu) != 0xFFFFu;
}

// The Fx128 weight total of the histogram's codes (all of them), and of the codes whose key
// satisfies sel(key) into *sel_sum. Block-wide partial sums: the caller reduces them.
template <typename Sel>
__device__ __forceinline__ Fx128 hist_weigh(const uint32_t* hist, float m, double iT, Sel sel,
                                            Fx128* sel_sum) {
  Fx128 acc = fx_zero(), part = fx_zero();
  const uint4* h4 = reinterpret_cast<const uint4*>(hist);
  for (int i = threadIdx.x; i < kHistWords / 4; i += kThreads) {
    const uint4 q = h4[i];
    if ((q.x | q.y | q.z | q.w) == 0u) continue;
    const uint32_t word[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t n = (word[e >> 1] >> ((e & 1) << 4)) & 0xFFFFu;
      if (n == 0u) continue;
      const uint32_t key = uint32_t(8 * i + e);
      const Fx128 f =
          fx_mul_u32(fx_from(weight_d(key_value<__nv_bfloat16>(key), m, iT)), n);
      acc = fx_add(acc, f);
      if (sel(key)) part = fx_add(part, f);
    }
  }
  *sel_sum = part;
  return acc;
}

}  // namespace sv
