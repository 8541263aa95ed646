// Chain verification, after the row statistics: one thread block per batch row.
//
// Warp 0 evaluates every position at once — the ratio test u_i < min(1, p_i(x_i) /
// q_i(x_i)) (or x_i == argmax p_i in the greedy form) — and a ballot finds the first
// position that stops the scan: a rejection, the bonus position K, or a data error.
// The whole block then draws the emitted token: from norm(max(0, p_a - q_a)) after a
// rejection at a (p_a if that residual is empty), from p_K when all K drafts were
// accepted. When the row of p_a lists its kept ids (top-k rows), the draw runs over
// that support only: the residual and p both vanish outside it. "Speculative Decoding"
// and "Speculative Sampling" (spec-decoding-i notes); greedy longest-prefix verification
// from blockwise parallel decoding ("推测解码").
//
// The ratio tests and the draw are taken in double precision: p(v) = exp((l_v - m) / T) / zd
// over the kept set, zd the double normaliser of the row statistics. A row whose statistics
// carry no zd (untruncated rows, rows the exact finisher settled) has it summed here, by the
// whole block, the first time the scan reaches a test that needs it. For untruncated rows the
// test first uses the streaming kernel's fp32 normaliser with a bound on its error: only a
// ratio within that bound of u needs the double one (the decision is the same either way, as
// the true ratio lies inside the bound). The draw's masses are doubles summed as exact 128-bit
// fixed point, with double normalisers (summed here when the scan did not need them).
#pragma once

#include "draw.cuh"
#include "row_stats.cuh"

static_assert(sv::kSparseCap >= sv::kKeptCap, "a listed kept set fits one sparse draw");

namespace sv {

struct ChainJob {
  const void* target;     // [B][K+1][V]
  const void* draft;      // [B][K][V]
  int B, K, V;
  const int32_t* tokens;  // [B][K]
  const float* uniforms;  // [B][K+1]
  const RowStats* stats;  // target rows [B*(K+1)], then draft rows [B*K]
  const int32_t* kept_n;  // [rows] or NULL: ids listed per row (0: none)
  const int32_t* kept_ids;  // [rows][kKeptCap]
  int greedy;
  float temp;             // the temperature as given (sampling)
  // > 0: rows without a double normaliser carry an fp32 one (RowStats::z) whose relative
  // error is at most zguard + 2^-23 |m| log2(e) / T (untruncated rows of the streaming
  // kernel); a ratio test that clears that margin is decided with it. 0: never.
  float zguard;
  int32_t* accepted_len;  // [B]
  int32_t* out_tokens;    // [B][K+1]
};

// EV_NEEDZ: the test at this position needs a normaliser that the block must sum first.
enum : int { EV_ACCEPT = 0, EV_STOP = 1, EV_ERROR = 2, EV_TIMEOUT = 3, EV_NEEDZ = 4 };

__device__ __forceinline__ int row_event(const RowStats& s) {
  return s.status == ROW_OK ? EV_ACCEPT : (s.status == ROW_TIMEOUT ? EV_TIMEOUT : EV_ERROR);
}

constexpr int kZPos = 32;  // positions whose listed rows get their normalisers up front

// The ratio test at position i when a double normaliser is missing: each missing one is
// replaced by the row's fp32 normaliser z, whose relative error is at most
// e = zguard + 2^-23 |m| c (the summation and ex2 roundings of the streaming kernel, and the
// rounding of m c and c that shifts every exponent of the row). The true ratio then lies in
// [r (1 - g), r (1 + g)] with g twice the sum of the missing rows' e (a margin over the
// first-order bound); a u outside that interval is decided, one inside returns EV_NEEDZ. The
// token's own weights are doubles, and a zero weight decides exactly as the double test does.
template <typename T>
__device__ __forceinline__ int guarded_test(const ChainJob& j, const RowStats& sp,
                                            const RowStats& sq, double zp, double zq,
                                            const T* trow0, const T* drow0, int i, int xi,
                                            int V, double iT, float ui) {
  const float lp = Elem<T>::load(trow0, size_t(i) * V + xi);
  const float lq = Elem<T>::load(drow0, size_t(i) * V + xi);
  const double wp = kept_weight_d<T>(sp, iT, lp, xi);
  const double wq = kept_weight_d<T>(sq, iT, lq, xi);
  if (wq == 0.0) return wp > 0.0 ? EV_ACCEPT : EV_STOP;  // r = inf (u < 1) or r = 0
  if (wp == 0.0) return EV_STOP;
  double g = 0.0;
  if (zp < 0.0) {
    if (!(sp.z > 0.0f && sp.z < INFINITY)) return EV_NEEDZ;
    zp = double(sp.z);
    g += double(j.zguard) + 0x1p-23 * fabs(double(sp.m) * double(sp.c));
  }
  if (zq < 0.0) {
    if (!(sq.z > 0.0f && sq.z < INFINITY)) return EV_NEEDZ;
    zq = double(sq.z);
    g += double(j.zguard) + 0x1p-23 * fabs(double(sq.m) * double(sq.c));
  }
  g *= 2.0;
  const double r = (wp / zp) / (wq / zq);
  const double uu = double(ui);
  if (uu < fmin(1.0, r * (1.0 - g))) return EV_ACCEPT;
  if (uu >= r * (1.0 + g)) return EV_STOP;
  return EV_NEEDZ;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) chain_finish_kernel(const ChainJob j) {
  __shared__ DrawSmem sm;
  __shared__ int s_a, s_ev, s_zpos;
  __shared__ double s_z[2];  // zd of p and q at position s_zpos, summed by the block
  __shared__ double s_zl[2][kZPos];  // zd of p and q at positions < kZPos (< 0: unknown)
  const int b = blockIdx.x;
  const int K = j.K, V = j.V;
  const RowStats* ts = j.stats + size_t(b) * (K + 1);
  const RowStats* ds = j.stats + size_t(j.B) * (K + 1) + size_t(b) * K;
  const T* trow0 = static_cast<const T*>(j.target) + size_t(b) * (K + 1) * V;
  const T* drow0 = j.greedy ? nullptr : static_cast<const T*>(j.draft) + size_t(b) * K * V;
  const int32_t* x = j.tokens + size_t(b) * K;
  const float* u = j.uniforms + size_t(b) * (K + 1);
  const double iT = 1.0 / double(j.temp);  // greedy rows never use it
  if (threadIdx.x == 0) s_zpos = -1;
  const int npos = min(K + 1, kZPos);
  if (!j.greedy) {
    // rows that list their kept ids: the double normaliser over the list, eight lanes per
    // row (four rows per warp at a time), each lane's ids and logits loaded together
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = lane & 7;
    for (int r0 = warp * 4; r0 < 2 * npos; r0 += 4 * kWarps) {  // (uniform in the warp)
      const int r = r0 + (lane >> 3);
      const bool tgt = r < npos;
      const int i = tgt ? r : r - npos;
      const bool live = r < 2 * npos && (tgt || i < K);
      double z = -1.0;
      RowStats st;
      int nk = 0;
      size_t gr = 0;
      if (live) {
        st = tgt ? ts[i] : ds[i];
        gr = tgt ? size_t(b) * (K + 1) + i : size_t(j.B) * (K + 1) + size_t(b) * K + i;
        nk = j.kept_n ? j.kept_n[gr] : 0;
        z = st.zd;
      }
      const bool sum = live && z < 0.0 && st.status == ROW_OK && nk > 0;
      Fx128 acc = fx_zero();
      if (sum) {
        const T* row = tgt ? trow0 + size_t(i) * V : drow0 + size_t(i) * V;
        const int32_t* ids = j.kept_ids + gr * kKeptCap;
        for (int q0 = 0; q0 < nk; q0 += 8 * 8) {
          int v[8];
          float x[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int q = q0 + 8 * k + sub;
            v[k] = q < nk ? ids[q] : -1;
          }
#pragma unroll
          for (int k = 0; k < 8; ++k) x[k] = v[k] >= 0 ? Elem<T>::load(row, size_t(v[k])) : 0.0f;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if (v[k] >= 0) acc = fx_add(acc, fx_from(kept_weight_d<T>(st, iT, x[k], v[k])));
        }
      }
#pragma unroll
      for (int o = 4; o > 0; o >>= 1) acc = fx_add(acc, fx_shfl_xor(acc, o));
      if (sum) z = fx_to_double(acc);
      if (live && sub == 0) s_zl[tgt ? 0 : 1][i] = z;
    }
  }
  __syncthreads();

  for (int start = 0;;) {
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      const int zpos = s_zpos;
      int a = -1, ev = EV_STOP;
      for (int base = start; base <= K && a < 0; base += 32) {
        const int i = base + lane;
        int e = EV_ACCEPT;
        if (i <= K) {
          const RowStats sp = ts[i];
          e = row_event(sp);
          if (e == EV_ACCEPT) {
            if (i == K) {
              e = EV_STOP;
            } else {
              const int xi = x[i];
              if (xi < 0 || xi >= V) {
                e = EV_ERROR;
              } else if (j.greedy) {
                e = (xi == sp.argmax) ? EV_ACCEPT : EV_STOP;
              } else {
                const RowStats sq = ds[i];
                e = row_event(sq);
                if (e == EV_ACCEPT) {
                  const double zp = i == zpos ? s_z[0] : (i < npos ? s_zl[0][i] : sp.zd);
                  const double zq = i == zpos ? s_z[1] : (i < npos ? s_zl[1][i] : sq.zd);
                  if (zp < 0.0 || zq < 0.0) {
                    e = EV_NEEDZ;
                    if (j.zguard > 0.0f) e = guarded_test<T>(j, sp, sq, zp, zq, trow0, drow0, i, xi, V, iT, u[i]);
                  } else {
                    const float lp = Elem<T>::load(trow0, size_t(i) * V + xi);
                    const float lq = Elem<T>::load(drow0, size_t(i) * V + xi);
                    const double p = kept_weight_d<T>(sp, iT, lp, xi) / zp;
                    const double q = kept_weight_d<T>(sq, iT, lq, xi) / zq;
                    const double r = q > 0.0 ? p / q : (p > 0.0 ? double(INFINITY) : 0.0);
                    e = (double(u[i]) < fmin(1.0, r)) ? EV_ACCEPT : EV_STOP;
                  }
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
    if (s_ev != EV_NEEDZ) break;
    // the first position still to test lacks a normaliser: the block sums it, then the
    // scan resumes there (the positions before it are accepted)
    const int i = s_a;
    const size_t tr = size_t(b) * (K + 1) + i, dr = size_t(j.B) * (K + 1) + size_t(b) * K + i;
    const int ntk = j.kept_n ? j.kept_n[tr] : 0, ndk = j.kept_n ? j.kept_n[dr] : 0;
    const double zp = row_zd<T>(ts[i], trow0 + size_t(i) * V, V, iT, sm.scr,
                                j.kept_ids + tr * kKeptCap, ntk);
    const double zq = row_zd<T>(ds[i], drow0 + size_t(i) * V, V, iT, sm.scr,
                                j.kept_ids + dr * kKeptCap, ndk);
    if (threadIdx.x == 0) {
      s_z[0] = zp;
      s_z[1] = zq;
      s_zpos = i;
    }
    start = i;
    __syncthreads();
  }
  const int a = s_a, ev = s_ev;
  int32_t* out = j.out_tokens + size_t(b) * (K + 1);
  if (ev != EV_STOP) {
    if (threadIdx.x == 0) j.accepted_len[b] = ev == EV_TIMEOUT ? -2 : -1;
    for (int k = threadIdx.x; k <= K; k += kThreads) out[k] = ev == EV_TIMEOUT ? -2 : -1;
    return;
  }
  int tok;
  if (j.greedy) {
    tok = ts[a].argmax;
  } else {
    const RowStats sp = ts[a];
    const T* prow = trow0 + size_t(a) * V;
    const bool pal = (reinterpret_cast<uintptr_t>(prow) & 15u) == 0;
    const float w = u[K];
    const size_t prow_idx = size_t(b) * (K + 1) + a;
    const int nk = j.kept_n ? j.kept_n[prow_idx] : 0;
    // the double normalisers at a (the bonus draw needs none: it scales by its total); a
    // test the fp32 normalisers decided leaves them to be summed now
    if (a < K) {
      const size_t dr = size_t(j.B) * (K + 1) + size_t(b) * K + a;
      double zp = a == s_zpos ? s_z[0] : (a < npos ? s_zl[0][a] : sp.zd);
      double zq = a == s_zpos ? s_z[1] : (a < npos ? s_zl[1][a] : ds[a].zd);
      if (zp < 0.0)
        zp = row_zd<T>(sp, prow, V, iT, sm.scr, j.kept_ids + prow_idx * kKeptCap, nk);
      if (zq < 0.0)
        zq = row_zd<T>(ds[a], drow0 + size_t(a) * V, V, iT, sm.scr, j.kept_ids + dr * kKeptCap,
                       j.kept_n ? j.kept_n[dr] : 0);
      __syncthreads();
      if (threadIdx.x == 0) {
        s_z[0] = zp;
        s_z[1] = zq;
        s_zpos = a;
      }
      __syncthreads();
    }
    const double izp = a < K ? 1.0 / s_z[0] : 1.0;
    tok = -1;
    if (nk > 0 && nk <= kSparseCap) {
      const int32_t* ids = j.kept_ids + prow_idx * kKeptCap;
      if (a < K) {
        const RowStats sq = ds[a];
        const double izq = 1.0 / s_z[1];
        const T* qrow = drow0 + size_t(a) * V;
        tok = sparse_draw(
            ids, nk,
            [&](int v) {
              const double d = prob_d<T>(sp, izp, iT, Elem<T>::load(prow, size_t(v)), v) -
                               prob_d<T>(sq, izq, iT, Elem<T>::load(qrow, size_t(v)), v);
              return fx_from(fmax(d, 0.0));
            },
            w, sm, V);
      }
      if (tok < 0)
        tok = sparse_draw(
            ids, nk,
            [&](int v) {
              return fx_from(kept_weight_d<T>(sp, iT, Elem<T>::load(prow, size_t(v)), v));
            },
            w, sm, V);
    } else {
      if (a < K) {
        const RowStats sq = ds[a];
        const double izq = 1.0 / s_z[1];
        const T* qrow = drow0 + size_t(a) * V;
        const bool qal = (reinterpret_cast<uintptr_t>(qrow) & 15u) == 0;
        tok = inverse_cdf_draw(
            [&](int v0, Fx128* r) {
              float lp[8], lq[8];
              load8<T>(prow, v0, V, pal, lp);
              load8<T>(qrow, v0, V, qal, lq);
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const int v = v0 + k;
                const double d = (v < V) ? prob_d<T>(sp, izp, iT, lp[k], v) -
                                               prob_d<T>(sq, izq, iT, lq[k], v)
                                         : 0.0;
                r[k] = fx_from(fmax(d, 0.0));
              }
            },
            V, w, sm);
      }
      if (tok < 0) {  // bonus position, or an empty residual: draw from p
        tok = inverse_cdf_draw(
            [&](int v0, Fx128* r) {
              float lp[8];
              load8<T>(prow, v0, V, pal, lp);
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const int v = v0 + k;
                r[k] = (v < V) ? fx_from(kept_weight_d<T>(sp, iT, lp[k], v)) : fx_zero();
              }
            },
            V, w, sm);
      }
    }
  }
  if (threadIdx.x == 0) {
    j.accepted_len[b] = a;
    for (int k = 0; k < a; ++k) out[k] = x[k];
    out[a] = tok;
    for (int k = a + 1; k <= K; ++k) out[k] = -1;
  }
}

}  // namespace sv
