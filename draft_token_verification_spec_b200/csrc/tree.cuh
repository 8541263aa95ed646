// Verification over a candidate tree, after the row statistics: one thread block per batch
// row. Typical acceptance (MEDUSA, "Key Components", spec-decoding-i notes; "推测解码"), or
// greedy acceptance (blockwise parallel decoding / Lookahead, "推测解码": several candidate
// branches checked against the target's argmax at once, the longest correct one kept).
//
// Threads test every non-root node in parallel: typical, p_parent(tok_c) > min(eps,
// delta * exp(-H(p_parent))), p the temperature-1 softmax of the parent's logits; greedy,
// tok_c == the argmax of the parent's logits (lowest id on ties). One thread
// then resolves ancestry in index order (parents precede children): a node is
// accepted iff its parent is and its own test passes; the root is accepted
// unconditionally. The deepest accepted node (lowest index on ties) and its
// root-first ancestor chain are written out; in greedy mode also the argmax of the deepest
// node's row, the token the round emits after the path.
//
// The typical test is taken with the fp32 row statistics. A test whose p lies within
// kTreeGuard (relative) of its threshold, a margin well above the fp32 statistics' error,
// is taken again in double precision: the block sums exp(l - m) and exp(l - m) * (m - l)
// over the parent's row exactly (Fx128), giving p and the entropy in double.
#pragma once

#include "draw.cuh"

namespace sv {

struct TreeJob {
  const void* target;        // [B][N][V]
  int B, N, V;
  const int32_t* tokens;     // [B][N]
  const int32_t* parent;     // [N]
  float eps, delta;
  const RowStats* stats;     // [B*N]
  int32_t* best_path;        // [B][path_cap]
  int path_cap;
  int32_t* accepted_len;     // [B]
  int greedy;                // greedy acceptance (stats hold each row's argmax)
  int32_t* next_token;       // [B] or NULL (greedy mode)
};

enum : int8_t { ND_REJECT = 0, ND_ACCEPT = 1, ND_ERROR = 2, ND_TIMEOUT = 3, ND_NEAR = 4 };

// Relative distance of p from the typical threshold below which the test is re-taken in
// double precision. The fp32 statistics err by less: per-thread fp32 sums of at most
// V / 256 + 16 terms (2^-24 each), ex2.approx and exponent roundings; they move p by under
// 3e-4 relative and the entropy by under 3e-3 (so the threshold by under 3e-3 relative) for
// V <= 2^20: the guard leaves a factor of three.
constexpr float kTreeGuard = 1e-2f;

constexpr int kTreeMaxNodes = 4096;  // SPEC_MAX_TREE_NODES

// Typical acceptance reads a node's row only to test the node's children, so only rows of
// nodes with a child are streamed. One block lists them for every batch row, parents in
// index order: map[b * P + j] = b * N + (j-th node with a child), *count = B * P. Malformed
// parent entries are skipped here (the finisher rejects the tree).
__global__ void __launch_bounds__(kThreads)
    tree_parent_rows_kernel(const int32_t* parent, int N, int B, int32_t* map, int32_t* count) {
  __shared__ uint8_t has_child[kTreeMaxNodes];
  __shared__ int32_t plist[kTreeMaxNodes];
  __shared__ uint32_t scr[kWarps];
  for (int c = threadIdx.x; c < N; c += kThreads) has_child[c] = 0;
  __syncthreads();
  for (int c = 1 + threadIdx.x; c < N; c += kThreads) {
    const int pa = parent[c];
    if (pa >= 0 && pa < c) has_child[pa] = 1;
  }
  __syncthreads();
  int P = 0;
  for (int base = 0; base < N; base += kThreads) {
    const int c = base + int(threadIdx.x);
    const uint32_t f = (c < N && has_child[c]) ? 1u : 0u;
    uint32_t total;
    const uint32_t pos = block_exclusive_scan<uint32_t>(f, scr, &total);
    if (f) plist[P + int(pos)] = c;
    P += int(total);
  }
  __syncthreads();
  const long long n = (long long)B * P;
  for (long long i = threadIdx.x; i < n; i += kThreads)
    map[i] = int32_t((i / P) * N + plist[i % P]);
  if (threadIdx.x == 0) *count = int32_t(n);
}

template <typename T>
__global__ void __launch_bounds__(kThreads) tree_finish_kernel(const TreeJob j) {
  extern __shared__ __align__(16) unsigned char tsm[];
  const int N = j.N, V = j.V, b = blockIdx.x;
  int32_t* par = reinterpret_cast<int32_t*>(tsm);           // [N]
  int32_t* depth = par + N;                                  // [N]
  int8_t* test = reinterpret_cast<int8_t*>(depth + N);       // [N]
  int8_t* acc = test + N;                                    // [N]
  __shared__ int s_bad_tree;
  if (threadIdx.x == 0) s_bad_tree = 0;
  __syncthreads();
  const RowStats* st = j.stats + size_t(b) * N;
  const T* rows = static_cast<const T*>(j.target) + size_t(b) * N * V;
  const int32_t* tok = j.tokens + size_t(b) * N;
  for (int c = threadIdx.x; c < N; c += kThreads) {
    const int pa = j.parent[c];
    par[c] = pa;
    const bool ok_edge = (c == 0) ? (pa == -1) : (pa >= 0 && pa < c);
    if (!ok_edge) s_bad_tree = 1;
    int8_t t = ND_ACCEPT;
    if (c > 0 && ok_edge) {
      const RowStats s = st[pa];
      if (s.status != ROW_OK) {
        t = s.status == ROW_TIMEOUT ? ND_TIMEOUT : ND_ERROR;
      } else {
        const int tk = tok[c];
        if (tk < 0 || tk >= V) {
          t = ND_ERROR;
        } else if (j.greedy) {
          t = tk == s.argmax ? ND_ACCEPT : ND_REJECT;
        } else {
          const float l = Elem<T>::load(rows, size_t(pa) * V + tk);
          const float p = prob<T>(s, l, tk);
          const float thr = fminf(j.eps, j.delta * expf(-s.entropy));
          t = fabsf(p - thr) <= kTreeGuard * thr ? ND_NEAR : (p > thr ? ND_ACCEPT : ND_REJECT);
        }
      }
    }
    test[c] = t;
  }
  __syncthreads();
  if (!j.greedy) {  // tests too close to call in fp32: again in double, one parent row at a
                    // time (its normaliser and entropy serve every child tested against it)
    __shared__ Fx128 zscr[kWarps];
    for (int c = 1; c < N; ++c) {
      if (test[c] != ND_NEAR) continue;  // uniform: test[] is in shared memory
      const int pa = par[c];
      const RowStats s = st[pa];
      const T* prow = rows + size_t(pa) * V;
      const bool al = (reinterpret_cast<uintptr_t>(prow) & 15u) == 0;
      Fx128 z = fx_zero(), h = fx_zero();
      // four groups of 8 per thread, all loaded before any is used
      for (int v00 = int(threadIdx.x) * 8; v00 < V; v00 += 4 * kThreads * 8) {
        float x[4][8];
        load8xG<T, 4>(prow, v00, kThreads * 8, V, al, x);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int v0 = v00 + g * kThreads * 8;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            if (v0 + k >= V || !(x[g][k] > -INFINITY)) continue;
            const double d = double(s.m) - double(x[g][k]);  // >= 0, exact
            const double e = exp_neg(-d);
            z = fx_add(z, fx_from(e));
            h = fx_add(h, fx_from(e * d));
          }
        }
      }
      const double zd = fx_to_double(block_sum_fx(z, zscr));
      const double hd = fx_to_double(block_sum_fx(h, zscr));
      if (threadIdx.x == 0) {
        const double H = log(zd) + hd / zd;  // -sum p ln p
        const double thr = fmin(double(j.eps), double(j.delta) * exp(-H));
        for (int c2 = c; c2 < N; ++c2) {  // this child and the later ones of the same parent
          if (test[c2] != ND_NEAR || par[c2] != pa) continue;
          const double p = exp(double(Elem<T>::load(prow, size_t(tok[c2]))) - double(s.m)) / zd;
          test[c2] = p > thr ? ND_ACCEPT : ND_REJECT;
        }
      }
      __syncthreads();
    }
  }
  int32_t* path = j.best_path + size_t(b) * j.path_cap;
  __shared__ int s_len, s_err;
  if (threadIdx.x == 0) {
    int err = s_bad_tree ? ND_ERROR : 0, best = 0;
    if (!err) {
      acc[0] = 1;
      depth[0] = 0;
      for (int c = 1; c < N && !err; ++c) {
        const int pa = par[c];
        depth[c] = depth[pa] + 1;
        acc[c] = 0;
        if (acc[pa]) {
          if (test[c] >= ND_ERROR) {
            err = test[c];
          } else {
            acc[c] = test[c];
            if (acc[c] && depth[c] > depth[best]) best = c;
          }
        }
      }
    }
    int len = err ? 0 : depth[best] + 1;
    if (!err && len > j.path_cap) err = ND_ERROR;
    int next = -1;
    if (!err && j.greedy) {  // the deepest node's own row is read for the next token
      const RowStats sb = st[best];
      if (sb.status != ROW_OK)
        err = sb.status == ROW_TIMEOUT ? ND_TIMEOUT : ND_ERROR;
      else
        next = sb.argmax;
    }
    if (j.next_token) j.next_token[b] = err ? (err == ND_TIMEOUT ? -2 : -1) : next;
    if (!err) {
      for (int n = best, k = len - 1; k >= 0; --k, n = (n > 0 ? par[n] : -1)) path[k] = n;
    }
    s_len = len;
    s_err = err;
    j.accepted_len[b] = err ? (err == ND_TIMEOUT ? -2 : -1) : len;
  }
  __syncthreads();
  const int fill_from = s_err ? 0 : s_len;
  const int fill = s_err == ND_TIMEOUT ? -2 : -1;
  for (int k = fill_from + threadIdx.x; k < j.path_cap; k += kThreads) path[k] = fill;
}

}  // namespace sv
