// Rejection sampling over a candidate tree, after the row statistics: one thread block per
// batch row ("Key Components", spec-decoding-i notes: MEDUSA's step (3) may reuse the
// rejection rule of speculative sampling, which keeps the target's output distribution).
//
// From the root, at the current node n the children are tried in index order: child c is
// accepted iff u[c] < min(1, r(x_c) / q_n(x_c)), r the current residual (p_n at first). A
// rejection replaces r by norm(max(0, r - q_n)) (unchanged when that is empty): the block
// sums max(0, r - q_n) over the row (over the kept ids when the row lists them, since r
// vanishes outside p_n's support) into the normaliser z_j, and r is carried as the
// recursion r_j(v) = max(0, r_(j-1)(v) - q_n(v)) / z_j. An accepted child becomes the current
// node; when none is accepted the emitted token is drawn from r by the inverse CDF with
// u[N]. In the greedy limit the first child whose token is the argmax of p_n is accepted and
// the emitted token is that argmax. The tests, the residual chain and the draw are taken in
// double precision (p(v) = exp((l_v - m) / T) / zd over the kept set, masses summed as exact
// 128-bit fixed point).
#pragma once

#include "chain.cuh"

namespace sv {

struct TreeSampleJob {
  const void* target;       // [B][N][V]
  const void* draft;        // [B][N][V] (unused when greedy)
  int B, N, V;
  const int32_t* tokens;    // [B][N]
  const int32_t* parent;    // [N]
  const float* uniforms;    // [B][N+1]
  const RowStats* stats;    // target rows [B*N], then draft rows [B*N]
  const int32_t* kept_n;    // [2*B*N] or NULL: ids listed per row (0: none)
  const int32_t* kept_ids;  // [rows][kKeptCap]
  int greedy;
  float temp;               // the temperature as given (sampling)
  int32_t* best_path;       // [B][path_cap]
  int path_cap;
  int32_t* accepted_len;    // [B]
  int32_t* next_token;      // [B] or NULL
};

template <typename T>
__global__ void __launch_bounds__(kThreads) tree_sample_kernel(const TreeSampleJob j) {
  extern __shared__ __align__(16) unsigned char tsm[];
  const int N = j.N, V = j.V, b = blockIdx.x;
  double* zs = reinterpret_cast<double*>(tsm);        // [N] normalisers of the residual chain
  int32_t* kstart = reinterpret_cast<int32_t*>(zs + N);  // [N+1] children of n: kids[kstart[n]..)
  int32_t* kids = kstart + N + 1;                      // [N]
  int32_t* path = kids + N;                            // [N] nodes on the accepted path
  const double iT = j.temp > 0.0f ? 1.0 / double(j.temp) : 0.0;
  __shared__ DrawSmem sm;
  __shared__ int s_bad;
  const int32_t* par = j.parent;
  if (threadIdx.x == 0) {  // children in index order (counting sort over parents)
    int bad = par[0] != -1;
    for (int n = 0; n <= N; ++n) kstart[n] = 0;
    for (int c = 1; c < N && !bad; ++c) {
      if (par[c] < 0 || par[c] >= c) bad = 1;
      else kstart[par[c] + 1] += 1;
    }
    for (int n = 0; n < N; ++n) kstart[n + 1] += kstart[n];
    if (!bad) {
      for (int n = 0; n < N; ++n) path[n] = kstart[n];  // fill cursors (path is free here)
      for (int c = 1; c < N; ++c) kids[path[par[c]]++] = c;
    }
    s_bad = bad;
  }
  __syncthreads();
  const RowStats* st = j.stats + size_t(b) * N;
  const RowStats* sd = j.stats + size_t(j.B) * N + size_t(b) * N;
  const T* trow0 = static_cast<const T*>(j.target) + size_t(b) * N * V;
  const T* drow0 = j.greedy ? nullptr : static_cast<const T*>(j.draft) + size_t(b) * N * V;
  const int32_t* tok = j.tokens + size_t(b) * N;
  const float* u = j.uniforms + size_t(b) * (N + 1);

  int err = s_bad ? EV_ERROR : 0;  // uniform over the block from here on
  int len = 1, emitted = -1;
  int cur = 0;
  if (threadIdx.x == 0) path[0] = 0;
  while (!err) {
    const RowStats sp = st[cur];
    if (sp.status != ROW_OK) {
      err = sp.status == ROW_TIMEOUT ? EV_TIMEOUT : EV_ERROR;
      break;
    }
    const int k0 = kstart[cur], k1 = kstart[cur + 1];
    int next = -1;
    if (j.greedy) {
      for (int i = k0; i < k1 && next < 0 && !err; ++i) {
        const int x = tok[kids[i]];
        if (x < 0 || x >= V) err = EV_ERROR;
        else if (x == sp.argmax) next = kids[i];
      }
      if (!err && next < 0) emitted = sp.argmax;
    } else {
      const T* prow = trow0 + size_t(cur) * V;
      const T* qrow = drow0 + size_t(cur) * V;
      const size_t prow_idx = size_t(b) * N + cur;
      const int nk = j.kept_n ? j.kept_n[prow_idx] : 0;
      const bool sparse = nk > 0 && nk <= kSparseCap;
      const int32_t* ids = sparse ? j.kept_ids + prow_idx * kKeptCap : nullptr;
      RowStats sq = sp;
      if (k1 > k0) {
        sq = sd[cur];
        if (sq.status != ROW_OK) {
          err = sq.status == ROW_TIMEOUT ? EV_TIMEOUT : EV_ERROR;
          break;
        }
      }
      // the double normalisers of p_n and (with children) q_n; every thread gets them
      const size_t qrow_idx = size_t(j.B) * N + size_t(b) * N + cur;
      const int nqk = (j.kept_n && k1 > k0) ? j.kept_n[qrow_idx] : 0;
      const double izp = 1.0 / row_zd<T>(sp, prow, V, iT, sm.scr, ids, sparse ? nk : 0);
      const double izq = k1 > k0 ? 1.0 / row_zd<T>(sq, qrow, V, iT, sm.scr,
                                                    j.kept_ids + qrow_idx * kKeptCap, nqk)
                                 : 1.0;
      int nrej = 0;
      // the current residual at v: the recursion over the rejections so far
      auto resid = [&](double pv, double qv) {
        double r = pv;
        for (int i = 0; i < nrej; ++i)
          if (zs[i] > 0.0) r = fmax(r - qv, 0.0) / zs[i];
        return r;
      };
      for (int i = k0; i < k1 && next < 0; ++i) {
        const int c = kids[i];
        const int x = tok[c];
        if (x < 0 || x >= V) {
          err = EV_ERROR;
          break;
        }
        const double px = prob_d<T>(sp, izp, iT, Elem<T>::load(prow, size_t(x)), x);
        const double qx = prob_d<T>(sq, izq, iT, Elem<T>::load(qrow, size_t(x)), x);
        const double rx = resid(px, qx);
        const double ratio = qx > 0.0 ? rx / qx : (rx > 0.0 ? double(INFINITY) : 0.0);
        if (double(u[c]) < fmin(1.0, ratio)) {
          next = c;
          break;
        }
        // rejected: the normaliser of max(0, r - q) over the row
        Fx128 zsum = fx_zero();
        if (sparse) {
          for (int t = threadIdx.x; t < nk; t += kThreads) {
            const int v = ids[t];
            const double pv = prob_d<T>(sp, izp, iT, Elem<T>::load(prow, size_t(v)), v);
            const double qv = prob_d<T>(sq, izq, iT, Elem<T>::load(qrow, size_t(v)), v);
            zsum = fx_add(zsum, fx_from(fmax(resid(pv, qv) - qv, 0.0)));
          }
        } else {
          for (int v = threadIdx.x; v < V; v += kThreads) {
            const double pv = prob_d<T>(sp, izp, iT, Elem<T>::load(prow, size_t(v)), v);
            const double qv = prob_d<T>(sq, izq, iT, Elem<T>::load(qrow, size_t(v)), v);
            zsum = fx_add(zsum, fx_from(fmax(resid(pv, qv) - qv, 0.0)));
          }
        }
        zsum = block_sum_fx(zsum, sm.scr);
        if (threadIdx.x == 0) zs[nrej] = fx_to_double(zsum);
        __syncthreads();
        ++nrej;
      }
      if (!err && next < 0) {  // no child accepted (or none): draw from the residual
        const float w = u[N];
        if (sparse) {
          emitted = sparse_draw(
              ids, nk,
              [&](int v) {
                const double pv = prob_d<T>(sp, izp, iT, Elem<T>::load(prow, size_t(v)), v);
                const double qv =
                    k1 > k0 ? prob_d<T>(sq, izq, iT, Elem<T>::load(qrow, size_t(v)), v) : 0.0;
                return fx_from(resid(pv, qv));
              },
              w, sm);
        } else {
          const bool pal = (reinterpret_cast<uintptr_t>(prow) & 15u) == 0;
          const bool qal = (reinterpret_cast<uintptr_t>(qrow) & 15u) == 0;
          emitted = inverse_cdf_draw(
              [&](int v0, Fx128* r) {
                float lp[8], lq[8];
                load8<T>(prow, v0, V, pal, lp);
                if (k1 > k0) load8<T>(qrow, v0, V, qal, lq);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                  const int v = v0 + k;
                  double mv = 0.0;
                  if (v < V) {
                    const double pv = prob_d<T>(sp, izp, iT, lp[k], v);
                    const double qv = k1 > k0 ? prob_d<T>(sq, izq, iT, lq[k], v) : 0.0;
                    mv = resid(pv, qv);
                  }
                  r[k] = fx_from(mv);
                }
              },
              V, w, sm);
        }
        if (emitted < 0) err = EV_ERROR;
      }
    }
    if (err || next < 0) break;
    if (threadIdx.x == 0) path[len] = next;
    ++len;
    cur = next;
  }
  __syncthreads();
  int32_t* out = j.best_path + size_t(b) * j.path_cap;
  if (!err && len > j.path_cap) err = EV_ERROR;
  const int fill = err == EV_TIMEOUT ? -2 : -1;
  for (int k = threadIdx.x; k < j.path_cap; k += kThreads)
    out[k] = (!err && k < len) ? path[k] : fill;
  if (threadIdx.x == 0) {
    j.accepted_len[b] = err ? fill : len;
    if (j.next_token) j.next_token[b] = err ? fill : emitted;
  }
}

}  // namespace sv
