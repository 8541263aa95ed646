// Fused LM head + verification statistics on the 5th-generation tensor cores (sm_100a).
//
// The pages put the cost of a speculative round in the target's scoring forward ([SD]
// "Speculative Sampling": K drafts are scored for about the price of one token because the
// linear layers are bound by memory at small batch). Its last matrix product turns hidden
// states into logits, logits[r][v] = h_r . W_v, and the verification rule then needs only a
// few statistics of each logit row: here the top-k entries (k = 1: the argmax), from which
// the transformed distribution of a top-k row is fully known. This kernel computes the
// product tile by tile in tensor memory and keeps those statistics in the epilogue, so the
// logit rows (8,704 x 151,936 x 4 bytes on the largest workload) never reach HBM.
//
// Structure (one CTA per SM, persistent over work items; 192 threads):
//   warp 0   TMA producer: 128 x 64 tiles of the hidden states and 256 x 64 tiles of the
//            output embeddings (bf16, 128-byte swizzle) into a ring of kLmStages stages;
//   warp 1   MMA issuer: tcgen05.mma kind::f16 (bf16 x bf16 -> fp32), M = 128, N = 256,
//            K = 16, four per 64-wide stage, accumulating a 128 x 256 tile in one of two
//            tensor-memory buffers (512 columns), tcgen05.commit releasing stages and tiles;
//   warps 2-5 epilogue: one logit row per thread (its tensor-memory lane), 32 columns per
//            tcgen05.ld; the row's running top-k lives in shared memory as an unsorted list
//            of (value, id) composites whose weakest entry is the next to be replaced.
// A work item is one 128-row tile and a chunk of consecutive 256-column tiles; at its end the
// epilogue writes each row's top-k of that chunk, and lmhead_merge_kernel takes the exact
// top-k of a row from its chunks. Every wait is bounded (kWaitLimitNs); a wait that runs out
// sets the device status word, the CTA stops issuing work, waits for what it issued and
// frees its tensor memory.
#pragma once

#include <cuda.h>

#include <climits>

#include "chain.cuh"
#include "common.cuh"
#include "draw.cuh"

namespace sv {

constexpr int kLmBM = 128, kLmBN = 256, kLmBK = 64;
constexpr int kLmStages = 3;
constexpr int kLmKMax = 64;                        // top-k the fused path keeps per row
constexpr int kLmStageA = kLmBM * kLmBK * 2;       // 16 KB
constexpr int kLmStageB = kLmBN * kLmBK * 2;       // 32 KB
constexpr int kLmStageBytes = kLmStageA + kLmStageB;
constexpr int kLmThreads = 192;
constexpr int kLmMergeCap = 4096;                  // chunks x k a row's merge may hold
// dynamic shared memory: the ring (1024-byte aligned atoms), then the top-k lists
constexpr int kLmStageStride = 33;                 // floats per row of the epilogue's staging
// dynamic shared memory: the ring, the top-k lists, the staging of 32 logits per row
constexpr size_t kLmSmem = size_t(kLmStages) * kLmStageBytes + size_t(kLmKMax) * kLmBM * 8 +
                           size_t(kLmBM) * kLmStageStride * 4 + 1024;
static_assert(kLmSmem + 1024 <= 227 * 1024, "LM-head shared memory (dynamic and static)");

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, both K-major; one thread issues it.
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.u32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(uint32_t(accumulate))
      : "memory");
}

// Arrives once on bar when every tcgen05.mma this thread issued before it has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 consecutive 32-bit columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major tile written by TMA with the 128-byte
// swizzle: rows of 64 bf16 (128 bytes), 8-row atoms of 1024 bytes packed one after another
// (stride 1024 B), leading offset 16 B (unused by the swizzled layout), descriptor version 1,
// layout type 2 (128-byte swizzle). The address advances by 32 bytes per K = 16 step.
__device__ __forceinline__ uint64_t smem_desc_k128(uint32_t addr) {
  uint64_t d = 0;
  d |= uint64_t((addr >> 4) & 0x3FFFu);
  d |= uint64_t(1u) << 16;                 // leading byte offset: 16 B
  d |= uint64_t(1024u >> 4) << 32;         // stride byte offset: 1024 B
  d |= uint64_t(1u) << 46;                 // version
  d |= uint64_t(2u) << 61;                 // 128-byte swizzle
  return d;
}

// Instruction descriptor: kind::f16 with bf16 A and B, fp32 D, both K-major, M = 128, N = 256.
constexpr uint32_t kLmIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kLmBN >> 3) << 17) |
                              (uint32_t(kLmBM >> 4) << 24);

struct LmJob {
  int M, V, d;
  int k;                 // list length per row (1: the argmax)
  int nchunk;            // vocabulary chunks per row tile
  int tiles_per_chunk;   // 256-column tiles per chunk
  int n_tiles;           // ceil(V / 256)
  int m_tiles;           // ceil(M / 128)
  float* part_val;       // [M][nchunk][k]
  int32_t* part_id;      // [M][nchunk][k]
  float* logits_out;     // [M][V] or NULL: the fp32 logits as well (verification of the path)
  int32_t* dev_status;   // bit 0: a wait ran out
};

struct __align__(8) LmBars {
  uint64_t full[kLmStages];
  uint64_t empty[kLmStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t done;
  uint32_t tmem_base;
  int broken;
};

// Work item `it`: row tile it % m_tiles of vocabulary chunk it / m_tiles. CTAs running at the
// same time take neighbouring items, so they share a chunk of the output embeddings, which is
// then read from HBM about once and from L2 by the other row tiles.
struct LmItem {
  int m0, chunk, t0, t1;
};
__device__ __forceinline__ LmItem lm_item(const LmJob& j, int it) {
  LmItem w;
  w.m0 = (it % j.m_tiles) * kLmBM;
  w.chunk = it / j.m_tiles;
  w.t0 = w.chunk * j.tiles_per_chunk;
  w.t1 = min(j.n_tiles, w.t0 + j.tiles_per_chunk);
  return w;
}

// The float whose f32_key is `key` (-0 comes back as +0).
__device__ __forceinline__ float lm_key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

__device__ __forceinline__ bool lm_wait(uint64_t* bar, uint32_t parity, LmBars& s,
                                        int32_t* dev_status) {
  if (*reinterpret_cast<volatile int*>(&s.broken)) return false;
  if (mbar_wait(bar, parity)) return true;
  atomicExch(&s.broken, 1);
  if (dev_status) atomicOr(dev_status, 1);
  return false;
}

__global__ void __launch_bounds__(kLmThreads, 1)
    lmhead_topk_kernel(const __grid_constant__ CUtensorMap map_h,
                       const __grid_constant__ CUtensorMap map_w, const LmJob j) {
  extern __shared__ __align__(1024) unsigned char lm_raw[];
  __shared__ LmBars s;
  // the ring must start on a 1024-byte boundary (swizzle atoms)
  unsigned char* ring = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(lm_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* lc = reinterpret_cast<uint64_t*>(ring + size_t(kLmStages) * kLmStageBytes);  // [k][128]
  float* stg = reinterpret_cast<float*>(lc + kLmKMax * kLmBM);  // [128][kLmStageStride]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int items = j.m_tiles * j.nchunk;
  const int kblocks = j.d / kLmBK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kLmStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.acc_full[i], 1);
      mbar_init(&s.acc_empty[i], 128);
    }
    mbar_init(&s.done, 1);
    s.broken = 0;
  }
  if (warp == 0) {  // the whole warp allocates the 512 tensor-memory columns
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(&s.tmem_base))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      for (int it = blockIdx.x; it < items && !s.broken; it += gridDim.x) {
        const LmItem w = lm_item(j, it);
        for (int t = w.t0; t < w.t1; ++t) {
          for (int kb = 0; kb < kblocks; ++kb) {
            if (issued >= kLmStages && !lm_wait(&s.empty[stage], phase ^ 1u, s, j.dev_status))
              break;
            unsigned char* a = ring + size_t(stage) * kLmStageBytes;
            mbar_arrive_expect_tx(&s.full[stage], uint32_t(kLmStageBytes));
            tma_load_2d(a, &map_h, kb * kLmBK, w.m0, &s.full[stage]);
            tma_load_2d(a + kLmStageA, &map_w, kb * kLmBK, t * kLmBN, &s.full[stage]);
            ++issued;
            if (++stage == kLmStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (s.broken) break;
        }
      }
      // no copy may still be landing when the CTA exits: wait for the last ones issued
      for (int q = 0; q < kLmStages && q < issued; ++q) {
        long long n = issued - 1 - q;  // copy n went to stage n % S, phase (n / S) & 1
        mbar_wait(&s.full[n % kLmStages], uint32_t((n / kLmStages) & 1));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      long long tiles = 0;
      for (int it = blockIdx.x; it < items && !s.broken; it += gridDim.x) {
        const LmItem w = lm_item(j, it);
        for (int t = w.t0; t < w.t1 && !s.broken; ++t) {
          if (tiles >= 2 && !lm_wait(&s.acc_empty[acc], acc_phase ^ 1u, s, j.dev_status)) break;
          tc_fence_after();
          const uint32_t d_tmem = tmem + uint32_t(acc * kLmBN);
          for (int kb = 0; kb < kblocks; ++kb) {
            if (!lm_wait(&s.full[stage], phase, s, j.dev_status)) break;
            tc_fence_after();
            const uint32_t a = smem_u32(ring + size_t(stage) * kLmStageBytes);
            const uint64_t ad = smem_desc_k128(a), bd = smem_desc_k128(a + kLmStageA);
#pragma unroll
            for (int k = 0; k < kLmBK / 16; ++k)  // +32 bytes per K = 16 step (>> 4: +2)
              tc_mma(d_tmem, ad + uint64_t(2 * k), bd + uint64_t(2 * k), kLmIdesc, kb > 0 || k > 0);
            tc_commit(&s.empty[stage]);  // the stage is free once these MMAs have read it
            if (++stage == kLmStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
          tc_commit(&s.acc_full[acc]);
          ++tiles;
          if (++acc == 2) {
            acc = 0;
            acc_phase ^= 1u;
          }
        }
      }
      // every MMA issued has completed before the tensor memory is freed
      tc_commit(&s.done);
      mbar_wait(&s.done, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // the tensor-memory lane quadrant this warp reads
    const int r = q * 32 + lane;            // row within the tile
    const uint32_t lane_addr = uint32_t(q * 32) << 16;
    int acc = 0;
    uint32_t acc_phase = 0;
    const int k = j.k;
    for (int it = blockIdx.x; it < items && !s.broken; it += gridDim.x) {
      const LmItem w = lm_item(j, it);
      const int row = w.m0 + r;
      // The row's list holds the chunk's best k entries so far as composites
      // (key << 32 | ~id: larger is better, value desc then id asc), unsorted; once it is
      // full, `weak` is its smallest composite and `wslot` where that sits. A new entry
      // replaces the weakest, and one scan of the list (independent loads) finds the next.
      int n = 0;
      uint64_t weak = 0;
      int wslot = 0;
      float thr = -INFINITY;      // the weakest entry's value (a quick first test)
      bool bad = false;           // a NaN or +inf logit in this chunk of the row
      for (int t = w.t0; t < w.t1; ++t) {
        // warp-uniform, as the tensor-memory loads below are .sync.aligned
        if (!__all_sync(0xffffffffu, lm_wait(&s.acc_full[acc], acc_phase, s, j.dev_status)))
          break;
        tc_fence_after();
        for (int cc = 0; cc < kLmBN / 32; ++cc) {
          uint32_t v[32];
          tc_ld32(tmem + lane_addr + uint32_t(acc * kLmBN + cc * 32), v);
          const int c0 = t * kLmBN + cc * 32;
          if (j.logits_out && row < j.M) {
            for (int e = 0; e < 32; ++e)
              if (c0 + e < j.V) j.logits_out[size_t(row) * j.V + c0 + e] = __uint_as_float(v[e]);
          }
          // which of the 32 may enter (against the list as it stands: a superset); those few
          // go through this row's staging slot in shared memory, so the list code below
          // exists once (a small epilogue keeps the MMA warp's instructions cached)
          uint32_t want = 0;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float x = __uint_as_float(v[e]);
            const bool in = c0 + e < j.V;
            bad |= in && !(x < INFINITY);
            if (in && !(n == k && x < thr)) want |= 1u << e;
          }
          if (want) {
            float* sr = stg + r * kLmStageStride;
#pragma unroll
            for (int e = 0; e < 32; ++e) sr[e] = __uint_as_float(v[e]);
            while (want) {
              const int e = __ffs(int(want)) - 1;
              want &= want - 1u;
              const float x = sr[e];
              if (n == k && x < thr) continue;
              const uint64_t c = (uint64_t(f32_key(x)) << 32) | uint64_t(~uint32_t(c0 + e));
              if (n < k) {
                lc[n * kLmBM + r] = c;
                if (++n < k) continue;
              } else if (c > weak) {
                lc[wslot * kLmBM + r] = c;
              } else {
                continue;
              }
              weak = ~0ull;
              for (int i = 0; i < k; ++i) {
                const uint64_t q = lc[i * kLmBM + r];
                if (q < weak) {
                  weak = q;
                  wslot = i;
                }
              }
              thr = lm_key_value(uint32_t(weak >> 32));
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&s.acc_empty[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (row < j.M) {
        // the weakest entry goes to the last slot (the merge reads a chunk's k-th value
        // there); a NaN first entry tells the merge that the row holds a NaN or +inf logit
        const size_t o = (size_t(row) * j.nchunk + w.chunk) * k;
        for (int i = 0; i < k; ++i) {
          const int src = n < k ? i : (i == k - 1 ? wslot : (i == wslot ? k - 1 : i));
          const uint64_t c = lc[src * kLmBM + r];
          j.part_val[o + i] = (i == 0 && bad) ? __int_as_float(0x7fc00000)
                              : i < n      ? lm_key_value(uint32_t(c >> 32))
                                           : -INFINITY;
          j.part_id[o + i] = i < n ? int32_t(~uint32_t(c)) : INT_MAX;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

// ------------------------------------------------------------------ merge
// Per logit row: the exact top-k over its chunks' lists (value desc, id asc), the row maximum
// and its lowest id, and the double normaliser of the kept set at temperature T.
struct LmRow {
  float m;        // largest logit
  int32_t argmax; // lowest id holding it
  int32_t n;      // kept entries (k)
  int32_t status; // ROW_OK, or ROW_INVALID (a NaN or +inf logit, or none finite)
  double zd;      // sum over the kept set of exp((l - m) / T)
};

struct LmMergeJob {
  const float* part_val;   // [rows][nchunk][k]
  const int32_t* part_id;
  int rows, nchunk, k;
  float temp;              // 0: greedy (no normaliser)
  LmRow* out;              // [rows]
  float* kept_val;         // [rows][k]: the kept entries, (value desc, id asc)
  int32_t* kept_id;        // [rows][k]
};

__global__ void __launch_bounds__(kThreads) lmhead_merge_kernel(const LmMergeJob j) {
  __shared__ unsigned long long cand[kLmMergeCap];
  __shared__ float s_t0;
  __shared__ int s_n, s_bad;
  const int row = blockIdx.x, k = j.k, nc = j.nchunk;
  const float* pv = j.part_val + size_t(row) * nc * k;
  const int32_t* pi = j.part_id + size_t(row) * nc * k;
  if (threadIdx.x == 0) {
    s_n = 0;
    s_bad = 0;
    float t0 = -INFINITY;  // a chunk's k-th value is a lower bound on the row's k-th
    for (int c = 0; c < nc; ++c) t0 = fmaxf(t0, pv[size_t(c) * k + k - 1]);
    s_t0 = t0;
  }
  __syncthreads();
  const float t0 = s_t0;
  for (int i = threadIdx.x; i < nc * k; i += kThreads) {
    const float x = pv[i];
    if (x != x || x == INFINITY) s_bad = 1;
    if (pi[i] != INT_MAX && x >= t0) {
      const int slot = atomicAdd(&s_n, 1);
      if (slot < kLmMergeCap)
        cand[slot] = (uint64_t(f32_key(x)) << 32) | uint64_t(~uint32_t(pi[i]));
    }
  }
  __syncthreads();
  const int n = min(s_n, kLmMergeCap);
  // rank every candidate (composites are distinct); the top k go to their rank slots
  for (int i = threadIdx.x; i < n; i += kThreads) {
    const unsigned long long e = cand[i];
    int above = 0;
    for (int q = 0; q < n; ++q) above += cand[q] > e ? 1 : 0;
    if (above < k) {
      j.kept_val[size_t(row) * k + above] = lm_key_value(uint32_t(e >> 32));
      j.kept_id[size_t(row) * k + above] = int32_t(~uint32_t(e));
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    LmRow o;
    const float m = j.kept_val[size_t(row) * k];
    o.m = m;
    o.argmax = j.kept_id[size_t(row) * k];
    o.n = min(k, n);
    o.status = (s_bad || n < k || !(m > -INFINITY)) ? ROW_INVALID : ROW_OK;
    Fx128 z = fx_zero();  // exact, so it equals the same sum taken in any order
    if (j.temp > 0.0f)
      for (int i = 0; i < o.n; ++i)
        z = fx_add(z, fx_from(weight_d(j.kept_val[size_t(row) * k + i], m, 1.0 / double(j.temp))));
    o.zd = fx_to_double(z);
    j.out[row] = o;
  }
}

// ------------------------------------------------------------------ verification from lists
struct LmChainJob {
  int B, K, k;
  const LmRow* rows;        // target rows [B*(K+1)], then draft rows [B*K]
  const float* kept_val;    // [rows][k]
  const int32_t* kept_id;
  const int32_t* tokens;    // [B][K]
  const float* uniforms;    // [B][K+1]
  float temp;               // 0: greedy
  int V;
  int32_t* accepted_len;
  int32_t* out_tokens;
};

// 1 / T for sampling (greedy calls never use it).
__device__ __forceinline__ double greedy_temp_inverse(float temp) {
  return temp > 0.0f ? 1.0 / double(temp) : 0.0;
}

// The logit of token x in a row's kept list, or -inf when x is not kept.
__device__ __forceinline__ float lm_lookup(const float* vals, const int32_t* ids, int k, int x) {
  for (int i = 0; i < k; ++i)
    if (ids[i] == x) return vals[i];
  return -INFINITY;
}

__global__ void __launch_bounds__(kThreads) lmhead_chain_kernel(const LmChainJob j) {
  __shared__ DrawSmem sm;
  __shared__ int s_a, s_ev;
  const int b = blockIdx.x, K = j.K, k = j.k;
  const size_t trow0 = size_t(b) * (K + 1), drow0 = size_t(j.B) * (K + 1) + size_t(b) * K;
  const int32_t* x = j.tokens + size_t(b) * K;
  const float* u = j.uniforms + size_t(b) * (K + 1);
  const double iT = greedy_temp_inverse(j.temp);
  const bool greedy = j.temp == 0.0f;
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int a = -1, ev = EV_STOP;
    for (int base = 0; base <= K && a < 0; base += 32) {
      const int i = base + lane;
      int e = EV_ACCEPT;
      if (i <= K) {
        const LmRow sp = j.rows[trow0 + i];
        e = sp.status == ROW_OK ? EV_ACCEPT : EV_ERROR;
        if (e == EV_ACCEPT) {
          if (i == K) {
            e = EV_STOP;
          } else {
            const int xi = x[i];
            if (xi < 0 || xi >= j.V) {
              e = EV_ERROR;
            } else if (greedy) {
              e = xi == sp.argmax ? EV_ACCEPT : EV_STOP;
            } else {
              const LmRow sq = j.rows[drow0 + i];
              if (sq.status != ROW_OK) {
                e = EV_ERROR;
              } else {
                const float lp = lm_lookup(j.kept_val + (trow0 + i) * k, j.kept_id + (trow0 + i) * k, k, xi);
                const float lq = lm_lookup(j.kept_val + (drow0 + i) * k, j.kept_id + (drow0 + i) * k, k, xi);
                const double p = lp > -INFINITY ? weight_d(lp, sp.m, iT) / sp.zd : 0.0;
                const double q = lq > -INFINITY ? weight_d(lq, sq.m, iT) / sq.zd : 0.0;
                const double rr = q > 0.0 ? p / q : (p > 0.0 ? double(INFINITY) : 0.0);
                e = double(u[i]) < fmin(1.0, rr) ? EV_ACCEPT : EV_STOP;
              }
            }
          }
        }
      }
      const unsigned stop = __ballot_sync(0xffffffffu, i <= K && e != EV_ACCEPT);
      if (stop) {
        const int L = __ffs(stop) - 1;
        a = base + L;
        ev = __shfl_sync(0xffffffffu, e, L);
      }
    }
    if (lane == 0) {
      s_a = a;
      s_ev = ev;
    }
  }
  __syncthreads();
  const int a = s_a, ev = s_ev;
  int32_t* out = j.out_tokens + size_t(b) * (K + 1);
  if (ev != EV_STOP) {
    if (threadIdx.x == 0) j.accepted_len[b] = -1;
    for (int q = threadIdx.x; q <= K; q += kThreads) out[q] = -1;
    return;
  }
  int tok;
  if (greedy) {
    tok = j.rows[trow0 + a].argmax;
  } else {
    const LmRow sp = j.rows[trow0 + a];
    const float* pv = j.kept_val + (trow0 + a) * k;
    const int32_t* pid = j.kept_id + (trow0 + a) * k;
    tok = -1;
    if (a < K) {  // the residual max(0, p - q) over p's kept set
      const LmRow sq = j.rows[drow0 + a];
      const float* qv = j.kept_val + (drow0 + a) * k;
      const int32_t* qid = j.kept_id + (drow0 + a) * k;
      const double izp = 1.0 / sp.zd, izq = 1.0 / sq.zd;
      tok = sparse_draw(
          pid, k,
          [&](int v) {
            const float lp = lm_lookup(pv, pid, k, v), lq = lm_lookup(qv, qid, k, v);
            const double p = weight_d(lp, sp.m, iT) * izp;
            const double q = lq > -INFINITY ? weight_d(lq, sq.m, iT) * izq : 0.0;
            return fx_from(fmax(p - q, 0.0));
          },
          u[K], sm);
    }
    if (tok < 0)
      tok = sparse_draw(
          pid, k,
          [&](int v) { return fx_from(weight_d(lm_lookup(pv, pid, k, v), sp.m, iT)); }, u[K], sm);
  }
  if (threadIdx.x == 0) {
    j.accepted_len[b] = a;
    for (int q = 0; q < a; ++q) out[q] = x[q];
    out[a] = tok;
    for (int q = a + 1; q <= K; ++q) out[q] = -1;
  }
}

}  // namespace sv
