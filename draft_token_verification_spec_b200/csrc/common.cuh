// Shared device helpers for libspecverify (sm_100a).
#pragma once

#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cstdint>

namespace cg = cooperative_groups;

namespace sv {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
// Masses in [0, 1] are summed as unsigned 64-bit fixed point with 42 fraction bits:
// integer sums are exact and independent of summation order, so every reduction is
// deterministic; V <= 2^20 keeps any sum below 2^62.
constexpr float kFxF = 4398046511104.0f;  // 2^42
constexpr double kFxInv = 1.0 / 4398046511104.0;
constexpr float kLog2e = 1.4426950408889634f;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // bound on any copy wait

// ROW_FALLBACK: the streaming kernel could not settle the row from its candidates;
// the cluster kernel recomputes it (never seen by consumers).
enum : int32_t { ROW_OK = 0, ROW_INVALID = 1, ROW_TIMEOUT = 2, ROW_FALLBACK = 3 };

// Per-logit-row statistics that define the transformed distribution:
//   p(v) = kept(v) ? exp2(l_v * c - mc) / z : 0,
//   kept(v) = key(l_v) > thr_key || (key(l_v) == thr_key && v <= cutoff),
// with c = log2(e) / T and mc = fl(m * c), m the largest logit. thr_key = 0 keeps every
// row entry. The rounding of mc scales every weight of the row by the same factor, so
// it cancels in p.
//
// The decisions of the sampling rule (the ratio test, the residual and bonus draws) use the
// double-precision view of the same distribution: p(v) = kept(v) ? exp((l_v - m) / T) / zd : 0,
// with zd the double sum over the kept set (zd < 0: not computed here; the consumer sums it).
struct RowStats {
  float mc;          // fl(m * c), m the largest logit
  float z;           // sum over the kept set of exp2((l - m) * c)
  float entropy;     // entropy (nats) of the transformed distribution, if computed
  uint32_t thr_key;  // boundary key of the kept prefix in (value desc, id asc) order
  int32_t cutoff;    // largest kept id among entries whose key equals thr_key
  int32_t argmax;    // lowest id holding the largest logit
  int32_t status;    // ROW_OK / ROW_INVALID / ROW_TIMEOUT
  float c;           // log2(e) / T
  float m;           // the largest logit (exact)
  int32_t pad;
  double zd;         // sum over the kept set of exp((l - m) / T) in double, or -1
};
static_assert(sizeof(RowStats) == 48, "RowStats is 48 bytes");

// ------------------------------------------------------------------------- keys
// Order-preserving unsigned key of a float value (larger value -> larger key);
// -0 maps to the key of +0 so equal values have equal keys. A bfloat16 value's key
// is the top 16 bits of its float key.
__device__ __forceinline__ uint32_t f32_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// max with NaN propagation (PTX max.NaN).
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

template <typename T>
struct Elem;

template <>
struct Elem<float> {
  static constexpr int kBytes = 4;
  static constexpr int kPerVec = 4;     // elements per 16-byte vector
  static constexpr int kKeyBits = 32;
  __device__ static __forceinline__ void unpack(const uint4& w, float* x) {
    x[0] = __uint_as_float(w.x);
    x[1] = __uint_as_float(w.y);
    x[2] = __uint_as_float(w.z);
    x[3] = __uint_as_float(w.w);
  }
  __device__ static __forceinline__ float load(const void* base, size_t i) {
    return __ldg(static_cast<const float*>(base) + i);
  }
  __device__ static __forceinline__ uint32_t key(float x) { return f32_key(x); }
  // Key of entry k of a 16-byte vector, from its bits.
  __device__ static __forceinline__ uint32_t key_at(const uint4& w, int k) {
    const uint32_t b = k < 2 ? (k == 0 ? w.x : w.y) : (k == 2 ? w.z : w.w);
    return f32_key(__uint_as_float(b));
  }
  // Largest value of a 16-byte vector; NaN if any entry is NaN.
  __device__ static __forceinline__ float vmax_nan(const uint4& w) {
    return fmax_nan(fmax_nan(__uint_as_float(w.x), __uint_as_float(w.y)),
                    fmax_nan(__uint_as_float(w.z), __uint_as_float(w.w)));
  }
  // Largest value of a 16-byte vector (entries are not NaN).
  __device__ static __forceinline__ float vmax(const uint4& w) {
    return fmaxf(fmaxf(__uint_as_float(w.x), __uint_as_float(w.y)),
                 fmaxf(__uint_as_float(w.z), __uint_as_float(w.w)));
  }
};

template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kBytes = 2;
  static constexpr int kPerVec = 8;
  static constexpr int kKeyBits = 16;
  __device__ static __forceinline__ void unpack(const uint4& w, float* x) {
    const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x[2 * k] = __uint_as_float(a[k] << 16);
      x[2 * k + 1] = __uint_as_float(a[k] & 0xFFFF0000u);
    }
  }
  __device__ static __forceinline__ float load(const void* base, size_t i) {
    const unsigned short h = __ldg(static_cast<const unsigned short*>(base) + i);
    return __uint_as_float(uint32_t(h) << 16);
  }
  __device__ static __forceinline__ uint32_t key(float x) { return f32_key(x) >> 16; }
  // Key of entry k of a 16-byte vector, from its 16 bits (-0 maps to the key of +0).
  __device__ static __forceinline__ uint32_t key_at(const uint4& w, int k) {
    const int q = k >> 1;
    const uint32_t b = q < 2 ? (q == 0 ? w.x : w.y) : (q == 2 ? w.z : w.w);
    uint32_t h = (k & 1) ? (b >> 16) : (b & 0xFFFFu);
    if (h == 0x8000u) h = 0u;
    return (h & 0x8000u) ? (~h & 0xFFFFu) : (h | 0x8000u);
  }
  __device__ static __forceinline__ __nv_bfloat162 pair(uint32_t u) {
    return *reinterpret_cast<const __nv_bfloat162*>(&u);
  }
  // Largest value of a 16-byte vector (packed bf16x2 max); NaN if any entry is NaN.
  __device__ static __forceinline__ float vmax_nan(const uint4& w) {
    const __nv_bfloat162 r = __hmax2_nan(__hmax2_nan(pair(w.x), pair(w.y)),
                                         __hmax2_nan(pair(w.z), pair(w.w)));
    return fmax_nan(__low2float(r), __high2float(r));
  }
  __device__ static __forceinline__ float vmax(const uint4& w) {
    const __nv_bfloat162 r = __hmax2(__hmax2(pair(w.x), pair(w.y)), __hmax2(pair(w.z), pair(w.w)));
    return fmaxf(__low2float(r), __high2float(r));
  }
};

__device__ __forceinline__ bool kept(uint32_t key, int id, uint32_t thr_key, int cutoff) {
  return key > thr_key || (key == thr_key && id <= cutoff);
}

// 2^x with the SFU instruction (approximate, flushes denormal results to zero).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two fp32 lanes at once (the packed f32x2 forms of sm_100): each lane rounds as the scalar
// instruction does, so the results equal two fmaf / two additions bit for bit.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n .reg .b64 ra, rb, rc, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " mov.b64 rc, {%6, %7};\n fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0, %1}, rd;\n}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " add.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// Exponent l * c - mc = (l - m) / T in log2 units, with one rounding (FFMA).
__device__ __forceinline__ float wexp(float l, float c, float mc) { return fmaf(l, c, -mc); }

// Unnormalised weight exp((l - m) / T) of one logit.
__device__ __forceinline__ float weight(float l, float c, float mc) { return ex2(wexp(l, c, mc)); }

// Entropy term e * zx of one entry; an entry of weight 0 (a -inf logit) contributes 0,
// not 0 * -inf.
__device__ __forceinline__ float ent_term(float e, float zx) { return e > 0.0f ? e * zx : 0.0f; }

__device__ __forceinline__ unsigned long long to_fx(float mass01) {
  return __float2ull_rn(mass01 * kFxF);
}

// Fixed-point masses (< 2^45) summed in shared memory as three 15-bit limbs with 32-bit
// atomics: a 64-bit shared atomic add is many times slower, most of all when lanes collide
// on one address. A histogram of n bins keeps limb i of bin b at l[i * n + b]; up to 2^16
// adds per bin cannot overflow a limb, and the sum is exact.
__device__ __forceinline__ void limb_add(uint32_t* l, int n, int b, unsigned long long w) {
  const uint32_t w0 = uint32_t(w & 0x7FFFu), w1 = uint32_t((w >> 15) & 0x7FFFu),
                 w2 = uint32_t(w >> 30);
  if (w0) atomicAdd(&l[b], w0);
  if (w1) atomicAdd(&l[n + b], w1);
  if (w2) atomicAdd(&l[2 * n + b], w2);
}
__device__ __forceinline__ unsigned long long limb_get(const uint32_t* l, int n, int b) {
  return (unsigned long long)l[b] + ((unsigned long long)l[n + b] << 15) +
         ((unsigned long long)l[2 * n + b] << 30);
}

// ------------------------------------------------------------------------- exact wide sums
// Nonnegative doubles below 2^27 as unsigned 128-bit fixed point with 100 fraction bits.
// Conversion drops only what lies below 2^-100; sums of converted values are exact, so they
// do not depend on the order of the terms (deterministic reductions over lists that arrive
// in any order), and 2^20 terms below 1 each stay far below the range.
struct Fx128 {
  unsigned long long lo, hi;
};
__device__ __forceinline__ Fx128 fx_zero() { return Fx128{0ull, 0ull}; }
__device__ __forceinline__ Fx128 fx_add(Fx128 a, Fx128 b) {
  Fx128 r;
  r.lo = a.lo + b.lo;
  r.hi = a.hi + b.hi + (r.lo < a.lo ? 1ull : 0ull);
  return r;
}
// a * n exactly (a < 2^28 * 2^100 / n, true of any row sum here).
__device__ __forceinline__ Fx128 fx_mul_u32(Fx128 a, uint32_t n) {
  Fx128 r;
  r.lo = a.lo * n;
  r.hi = a.hi * n + __umul64hi(a.lo, uint64_t(n));
  return r;
}
__device__ __forceinline__ bool fx_is_zero(Fx128 a) { return (a.lo | a.hi) == 0ull; }
// x in [0, 2^27): x * 2^100 truncated to an integer.
__device__ __forceinline__ Fx128 fx_from(double x) {
  const unsigned long long bits = static_cast<unsigned long long>(__double_as_longlong(x));
  const int E = int((bits >> 52) & 0x7FFu);
  if (E == 0 || (bits >> 63)) return fx_zero();  // zero, subnormal (< 2^-1022) or negative
  const unsigned long long m = (bits & ((1ull << 52) - 1ull)) | (1ull << 52);
  const int sh = E - 975;  // x * 2^100 = m * 2^(E - 1075 + 100)
  Fx128 r;
  if (sh >= 64) {
    r.hi = m << (sh - 64);
    r.lo = 0ull;
  } else if (sh > 0) {
    r.hi = m >> (64 - sh);
    r.lo = m << sh;
  } else if (sh > -64) {
    r.hi = 0ull;
    r.lo = m >> (-sh);
  } else {
    r = fx_zero();
  }
  return r;
}
__device__ __forceinline__ double fx_to_double(Fx128 a) {
  // exact scalings by powers of two (both products are normal doubles)
  return double(a.hi) * 0x1.0p-36 + double(a.lo) * 0x1.0p-100;
}
__device__ __forceinline__ Fx128 fx_shfl_xor(Fx128 a, int o) {
  return Fx128{__shfl_xor_sync(0xffffffffu, a.lo, o), __shfl_xor_sync(0xffffffffu, a.hi, o)};
}
__device__ __forceinline__ Fx128 fx_shfl_up(Fx128 a, int o) {
  return Fx128{__shfl_up_sync(0xffffffffu, a.lo, o), __shfl_up_sync(0xffffffffu, a.hi, o)};
}
__device__ __forceinline__ Fx128 warp_sum_fx(Fx128 v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fx_add(v, fx_shfl_xor(v, o));
  return v;
}

// ------------------------------------------------------------------------- PTX: bulk copies
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// dst and src 16-byte aligned, bytes a multiple of 16. Streamed data: evict-first in L2.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  uint64_t policy;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// One wait on phase `parity` of `bar`: true once it has completed. While it has not, the
// thread is suspended for up to kWaitHintNs (it wakes when the phase completes), so a
// waiting warp takes no issue slots from the warps that share its scheduler.
constexpr uint32_t kWaitHintNs = 20000;
__device__ __forceinline__ bool mbar_try_wait(uint32_t addr, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(done)
      : "r"(addr), "r"(parity), "r"(kWaitHintNs)
      : "memory");
  return done != 0;
}

// Waits for phase `parity` of `bar` to complete; gives up after kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t addr = smem_u32(bar);
  if (mbar_try_wait(addr, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(addr, parity)) return true;
    if ((it & 15u) == 15u && global_timer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// ------------------------------------------------------------------------- reductions
__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ uint32_t warp_sum_u32(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Block-wide sums (all threads get the result). `scratch` holds kWarps entries.
__device__ __forceinline__ unsigned long long block_sum_u64(unsigned long long v,
                                                            unsigned long long* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum_u64(v);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  unsigned long long t = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) t += scratch[w];
  return t;
}
__device__ __forceinline__ double block_sum_f64(double v, double* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum_f64(v);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  double t = 0.0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) t += scratch[w];
  return t;
}
__device__ __forceinline__ uint32_t block_sum_u32(uint32_t v, uint32_t* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum_u32(v);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  uint32_t t = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) t += scratch[w];
  return t;
}

// Block-wide exclusive prefix sum in thread order; returns the exclusive prefix and
// writes the block total to *total.
template <typename U>
__device__ __forceinline__ U block_exclusive_scan(U v, U* scratch, U* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  U inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const U n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  __syncthreads();
  if (lane == 31) scratch[warp] = inc;
  __syncthreads();
  U before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    if (w < warp) before += scratch[w];
    all += scratch[w];
  }
  *total = all;
  return before + inc - v;
}

// Block-wide sum of Fx128 (all threads get it); scratch holds kWarps entries.
__device__ __forceinline__ Fx128 block_sum_fx(Fx128 v, Fx128* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum_fx(v);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  Fx128 t = fx_zero();
#pragma unroll
  for (int w = 0; w < kWarps; ++w) t = fx_add(t, scratch[w]);
  return t;
}

// Block-wide exclusive prefix sum of Fx128 in thread order; *total = the sum.
__device__ __forceinline__ Fx128 block_exclusive_scan_fx(Fx128 v, Fx128* scratch, Fx128* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  Fx128 inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const Fx128 n = fx_shfl_up(inc, o);
    if (lane >= o) inc = fx_add(inc, n);
  }
  __syncthreads();
  if (lane == 31) scratch[warp] = inc;
  __syncthreads();
  Fx128 before = fx_zero(), all = fx_zero();
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    if (w < warp) before = fx_add(before, scratch[w]);
    all = fx_add(all, scratch[w]);
  }
  *total = all;
  // inclusive - v, computed as before + (inc - v) without a subtraction: scan of the
  // exclusive within-warp prefix
  Fx128 ex = fx_shfl_up(inc, 1);
  if (lane == 0) ex = fx_zero();
  return fx_add(before, ex);
}

// (max value, lowest index) combine; NaN never reaches it (rows with NaN are invalid).
__device__ __forceinline__ void maxloc_combine(float& m, int& i, float m2, int i2) {
  if (m2 > m || (m2 == m && i2 < i)) {
    m = m2;
    i = i2;
  }
}

}  // namespace sv
