// Oracle for draft-token verification in speculative decoding.
//
// TEST INFRASTRUCTURE ONLY. This is a plain, slow, double-precision CPU
// statement of what the verification step computes. Only the test suite, the
// smoke check and the benchmark's CPU-baseline leg may load it; the library
// under test never does, and the two share no code, header or table.
//
// Sources (cited by page and section):
//   [SD]  taking-lying-flat.github.io/blog/posts/spec-decoding-i/ — notes on
//         "Fast Inference from Transformers via Speculative Decoding"
//         (section "Speculative Decoding"), "Accelerating Large Language Model
//         Decoding with Speculative Sampling" (section "Speculative Sampling")
//         and MEDUSA (section "Key Components").
//   [SV]  blog.csdn.net/yorkhunter/article/details/139214590 — survey
//         translation, section "推测解码" (blockwise parallel decoding,
//         MEDUSA typical acceptance).
// The pages lost their formulas in extraction; the surviving prose fixes the
// structure, and the formulas used here are the standard ones that prose
// describes: accept x with probability min(1, p(x)/q(x)), resample from
// norm(max(0, p - q)), bonus token from p after K acceptances, MEDUSA typical
// acceptance p(x) > min(eps, delta * exp(-H(p))).
//
// Readings where the pages are silent (each one is listed in the design notes):
//   * p is the target distribution, q the draft distribution.
//   * accept iff u < min(1, r), strict; r = +inf when q(x) = 0 < p(x), r = 0
//     when both are 0.
//   * uniforms per batch row: u[0..K-1] for the K accept tests, u[K] for the
//     single resample-or-bonus draw.
//   * transforms in the order temperature -> top-k -> softmax -> top-p ->
//     renormalise; ties broken by the lower token id; the top-p crossing token
//     is kept.
//   * inverse CDF in ascending token id: the smallest v with res[v] > 0 and
//     C_v > w * S; if rounding leaves none, the largest v with res[v] > 0.
//   * an empty residual (p == q) falls back to p.
//   * entropy in nats; tree: node 0 is accepted unconditionally, node c is
//     tested with p at its parent, the deepest accepted node wins with the
//     lowest index on ties.
//   * a row holding NaN or +inf, or whose logits are all -inf, is invalid;
//     a batch row that needs an invalid row, or an out-of-range token, is an
//     error row (accepted_len = -1, all outputs -1).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

const double kInf = std::numeric_limits<double>::infinity();

// Flag bits: decisions that fp32 and fp64 arithmetic may take differently.
enum : int32_t {
  FLAG_RATIO = 1,      // |u_i - r_i| < ratio window at a tested position
  FLAG_CDF = 2,        // inverse-CDF boundary within cdf_rel * S + cdf_abs of w * S
  FLAG_TOPP = 4,       // a top-p boundary within the top-p window of top_p, whose other
                       // side changes the row's output
  FLAG_TREE = 8,       // |p - thr| / thr < tree window at a tested tree node
  DIAG_Q_ZERO = 16,    // a tested draft token had q(x) = 0 (not a parity flag)
  FLAG_GAP = 32,       // a logit gap behind a decision (argmax, top-k boundary) within the
                       // gap window: for logits that the verifier computes itself
};

// Widths of the precision windows behind the flags. A flag marks a decision that another
// implementation, computing in lower precision, may take the other way; the defaults are
// the widest the acceptance criterion allows (1e-5 on the ratio, 1e-6 of S on the CDF; the
// same 1e-6 on a top-p boundary and a relative 1e-5 on a tree threshold). A caller whose
// arithmetic is more precise passes narrower windows. The windows change only the flags,
// never a result.
struct Windows {
  double ratio = 1e-5;
  double cdf_rel = 1e-6;
  double cdf_abs = 0.0;
  double topp = 1e-6;
  double tree = 1e-5;
  double gap = 0.0;  // logit-gap window (0: off; the logits are inputs, not computed)
};

// w = {ratio, cdf_rel, cdf_abs, topp, tree, gap}, or NULL for the defaults.
Windows windows_from(const double* w) {
  Windows x;
  if (w) {
    x.ratio = w[0];
    x.cdf_rel = w[1];
    x.cdf_abs = w[2];
    x.topp = w[3];
    x.tree = w[4];
    x.gap = w[5];
  }
  return x;
}

double bf16_bits_to_double(uint16_t h) {
  uint32_t u = uint32_t(h) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return double(f);
}

// dtype 0 = float32, 1 = bfloat16 (raw 16-bit patterns), 2 = float64.
void load_row(const void* base, int dtype, size_t row, int V, std::vector<double>& l) {
  l.resize(size_t(V));
  if (dtype == 2) {
    const double* p = static_cast<const double*>(base) + row * size_t(V);
    for (int v = 0; v < V; ++v) l[v] = p[v];
  } else if (dtype == 0) {
    const float* p = static_cast<const float*>(base) + row * size_t(V);
    for (int v = 0; v < V; ++v) l[v] = double(p[v]);
  } else {
    const uint16_t* p = static_cast<const uint16_t*>(base) + row * size_t(V);
    for (int v = 0; v < V; ++v) l[v] = bf16_bits_to_double(p[v]);
  }
}

bool row_valid(const std::vector<double>& l) {
  double mx = -kInf;
  for (double x : l) {
    if (std::isnan(x) || x == kInf) return false;
    if (x > mx) mx = x;
  }
  return mx > -kInf;
}

int argmax_lowest(const std::vector<double>& l) {
  int best = 0;
  for (int v = 1; v < int(l.size()); ++v)
    if (l[v] > l[best]) best = v;
  return best;
}

struct Dist {
  std::vector<double> p;
  double entropy = 0.0;
  // Distances to top_p of the cumulative mass that first reaches it (margin_reach)
  // and of the one just before (margin_prev): how close the nucleus is to one more
  // or one fewer token. Infinite when top-p is off.
  double margin_reach = kInf;
  double margin_prev = kInf;
  double topp_margin() const { return std::min(margin_reach, margin_prev); }
  // Logit gap at the decision the transform takes on logit order: between the k-th and the
  // (k+1)-th largest logits under top-k, between the largest and the next at T == 0.
  // Infinite when neither applies.
  double logit_gap = kInf;
};

// The sampling transform of [SD] "Speculative Sampling" (last bullet): the
// probabilities are transformed first, then the rejection scheme applies.
// Temperature T divides the logits; top-k keeps the k highest logits (lower id
// first on ties); softmax over the kept set; top-p keeps the shortest prefix of
// the probability-sorted kept tokens whose mass reaches top_p, then
// renormalises. T == 0 is the greedy limit: a one-hot at the argmax.
// alt = +1 / -1 keeps one token more / fewer than the nucleus (used only to decide
// whether a near-tie at the top-p boundary can change a verification outcome).
Dist transform(const std::vector<double>& l, double T, int top_k, double top_p, int alt = 0) {
  const int V = int(l.size());
  Dist d;
  d.p.assign(size_t(V), 0.0);
  if (T == 0.0) {
    const int g = argmax_lowest(l);
    d.p[g] = 1.0;
    double second = -kInf;
    for (int v = 0; v < V; ++v)
      if (v != g && l[v] > second) second = l[v];
    d.logit_gap = l[g] - second;
    return d;
  }
  std::vector<char> kept(static_cast<size_t>(V), 1);
  if (top_k >= 1 && top_k < V) {
    std::vector<int> order(static_cast<size_t>(V));
    for (int v = 0; v < V; ++v) order[v] = v;
    std::partial_sort(order.begin(), order.begin() + top_k, order.end(), [&](int a, int b) {
      if (l[a] != l[b]) return l[a] > l[b];
      return a < b;
    });
    std::fill(kept.begin(), kept.end(), 0);
    for (int j = 0; j < top_k; ++j) kept[order[j]] = 1;
    double next = -kInf;  // the largest logit left out
    for (int v = 0; v < V; ++v)
      if (!kept[v] && l[v] > next) next = l[v];
    d.logit_gap = l[order[top_k - 1]] - next;
  }
  double zmax = -kInf;
  for (int v = 0; v < V; ++v)
    if (kept[v] && l[v] / T > zmax) zmax = l[v] / T;
  std::vector<double> e(static_cast<size_t>(V), 0.0);
  double Z = 0.0;
  for (int v = 0; v < V; ++v)
    if (kept[v]) {
      e[v] = std::exp(l[v] / T - zmax);
      Z += e[v];
    }
  for (int v = 0; v < V; ++v) d.p[v] = e[v] / Z;

  if (top_p < 1.0) {
    std::vector<int> order;
    for (int v = 0; v < V; ++v)
      if (kept[v]) order.push_back(v);
    std::sort(order.begin(), order.end(), [&](int a, int b) {
      if (d.p[a] != d.p[b]) return d.p[a] > d.p[b];
      return a < b;
    });
    double cum = 0.0, prev = 0.0;
    size_t n_keep = order.size();
    for (size_t j = 0; j < order.size(); ++j) {
      prev = cum;
      cum += d.p[order[j]];
      if (cum >= top_p) {
        n_keep = j + 1;
        break;
      }
    }
    d.margin_reach = std::fabs(cum - top_p);
    d.margin_prev = std::fabs(prev - top_p);
    if (alt > 0) n_keep = std::min(n_keep + 1, order.size());
    if (alt < 0) n_keep = std::max<size_t>(n_keep - 1, 1);
    std::fill(kept.begin(), kept.end(), 0);
    for (size_t j = 0; j < n_keep; ++j) kept[order[j]] = 1;
    double Zp = 0.0;
    for (int v = 0; v < V; ++v)
      if (kept[v]) Zp += e[v];
    for (int v = 0; v < V; ++v) d.p[v] = kept[v] ? e[v] / Zp : 0.0;
  }
  double H = 0.0;
  for (int v = 0; v < V; ++v)
    if (d.p[v] > 0.0) H -= d.p[v] * std::log(d.p[v]);
  d.entropy = H;
  return d;
}

struct Draw {
  int token = -1;
  bool flag = false;
};

// Inverse-CDF draw in ascending token id: the smallest v with res[v] > 0 whose
// cumulative sum exceeds w * S. If rounding leaves none, the largest v with
// res[v] > 0 is taken (and the draw is flagged as sitting on an edge).
Draw inverse_cdf(const std::vector<double>& res, double w, const Windows& win) {
  Draw out;
  double S = 0.0;
  for (double r : res) S += r;
  const double target = w * S;
  double C = 0.0;
  for (int v = 0; v < int(res.size()); ++v) {
    const double before = C;
    C += res[v];
    if (res[v] > 0.0 && C > target) {
      out.token = v;
      const double band = win.cdf_rel * S + win.cdf_abs;
      out.flag = std::fabs(before - target) < band || std::fabs(C - target) < band;
      return out;
    }
  }
  for (int v = int(res.size()) - 1; v >= 0; --v)
    if (res[v] > 0.0) {
      out.token = v;
      out.flag = true;
      return out;
    }
  return out;
}

// Residual distribution of [SD] "Speculative Decoding": after rejecting x at
// position i, resample from norm(max(0, p_i - q_i)); an empty residual (only
// possible when p_i == q_i) falls back to p_i.
std::vector<double> residual(const std::vector<double>& p, const std::vector<double>& q) {
  std::vector<double> r(p.size());
  double S = 0.0;
  for (size_t v = 0; v < p.size(); ++v) {
    r[v] = std::max(0.0, p[v] - q[v]);
    S += r[v];
  }
  if (S == 0.0) return p;
  return r;
}

struct ChainArgs {
  const void* target;
  const void* draft;
  int dtype, B, K, V;
  const int32_t* draft_tokens;
  const double* uniforms;
  double T;
  int top_k;
  double top_p;
  int32_t* accepted_len;
  int32_t* out_tokens;
  int32_t* flags;
  Windows win;
};

void chain_error(const ChainArgs& a, int b) {
  a.accepted_len[b] = -1;
  for (int j = 0; j <= a.K; ++j) a.out_tokens[size_t(b) * (a.K + 1) + j] = -1;
  if (a.flags) a.flags[b] = 0;
}

// A transformed row to evaluate with one token more (alt = +1) or fewer (alt = -1) in
// its nucleus: kind 0 = target row, 1 = draft row, at position pos.
struct Override {
  int kind = -1, pos = -1, alt = 0;
};

struct Outcome {
  bool error = false;
  int acc = 0;
  std::vector<int32_t> out;
  int32_t flag = 0;
  std::vector<Override> near_ties;  // top-p boundaries within the window on decision rows
};

// One batch row of chain verification: [SD] "Speculative Decoding" (accept x_i left to
// right, stop at the first rejection and resample it, bonus token after K acceptances)
// and "Speculative Sampling" (the acceptance ratio and the residual). T == 0 is the
// greedy longest-prefix rule of blockwise parallel decoding ([SV], "推测解码").
Outcome chain_eval(const ChainArgs& a, int b, const Override& ov) {
  const int K = a.K, V = a.V;
  const int32_t* x = a.draft_tokens + size_t(b) * K;
  const double* u = a.uniforms + size_t(b) * (K + 1);
  Outcome o;
  o.out.assign(size_t(K + 1), -1);
  std::vector<double> lp, lq;
  int acc = K;
  int emitted = -1;
  auto note = [&](const Dist& d, int kind, int pos) {
    if (d.margin_reach < a.win.topp) o.near_ties.push_back({kind, pos, +1});
    if (d.margin_prev < a.win.topp) o.near_ties.push_back({kind, pos, -1});
  };
  auto alt_of = [&](int kind, int pos) { return (ov.kind == kind && ov.pos == pos) ? ov.alt : 0; };

  if (a.T == 0.0) {
    for (int i = 0; i <= K; ++i) {
      load_row(a.target, a.dtype, size_t(b) * (K + 1) + i, V, lp);
      if (!row_valid(lp)) return o.error = true, o;
      const int g = argmax_lowest(lp);
      if (a.win.gap > 0.0 && transform(lp, 0.0, 0, 1.0).logit_gap < a.win.gap) o.flag |= FLAG_GAP;
      if (i == K) {
        emitted = g;
        break;
      }
      if (x[i] < 0 || x[i] >= V) return o.error = true, o;
      if (x[i] != g) {
        acc = i;
        emitted = g;
        break;
      }
    }
  } else {
    for (int i = 0; i <= K; ++i) {
      load_row(a.target, a.dtype, size_t(b) * (K + 1) + i, V, lp);
      if (!row_valid(lp)) return o.error = true, o;
      const Dist P = transform(lp, a.T, a.top_k, a.top_p, alt_of(0, i));
      note(P, 0, i);
      if (P.logit_gap < a.win.gap) o.flag |= FLAG_GAP;
      if (i == K) {  // every draft accepted: bonus token from p at position K+1
        const Draw d = inverse_cdf(P.p, u[K], a.win);
        emitted = d.token;
        if (d.flag) o.flag |= FLAG_CDF;
        break;
      }
      if (x[i] < 0 || x[i] >= V) return o.error = true, o;
      load_row(a.draft, a.dtype, size_t(b) * K + i, V, lq);
      if (!row_valid(lq)) return o.error = true, o;
      const Dist Q = transform(lq, a.T, a.top_k, a.top_p, alt_of(1, i));
      note(Q, 1, i);
      if (Q.logit_gap < a.win.gap) o.flag |= FLAG_GAP;
      const double px = P.p[x[i]], qx = Q.p[x[i]];
      double r;
      if (qx > 0.0) {
        r = px / qx;
      } else {
        r = px > 0.0 ? kInf : 0.0;
        o.flag |= DIAG_Q_ZERO;
      }
      const double ui = u[i];
      if (std::isfinite(r) && std::fabs(ui - r) < a.win.ratio) o.flag |= FLAG_RATIO;
      if (ui < std::min(1.0, r)) continue;
      acc = i;
      const Draw d = inverse_cdf(residual(P.p, Q.p), u[K], a.win);
      emitted = d.token;
      if (d.flag) o.flag |= FLAG_CDF;
      break;
    }
  }
  o.acc = acc;
  for (int j = 0; j < acc; ++j) o.out[j] = x[j];
  o.out[acc] = emitted;
  return o;
}

// Evaluates a batch row and sets its flags. A top-p near-tie flags the row only when
// evaluating it with the other nucleus changes the row's output.
void chain_row(const ChainArgs& a, int b) {
  const Outcome base = chain_eval(a, b, Override{});
  if (base.error) return chain_error(a, b);
  int32_t flag = base.flag;
  for (const Override& t : base.near_ties) {
    const Outcome alt = chain_eval(a, b, t);
    if (alt.error || alt.acc != base.acc || alt.out != base.out) flag |= FLAG_TOPP;
  }
  a.accepted_len[b] = base.acc;
  std::copy(base.out.begin(), base.out.end(), a.out_tokens + size_t(b) * (a.K + 1));
  if (a.flags) a.flags[b] = flag;
}

template <class F>
void parallel_rows(int n, int threads, F&& f) {
  if (threads <= 1 || n <= 1) {
    for (int i = 0; i < n; ++i) f(i);
    return;
  }
  threads = std::min(threads, n);
  std::vector<std::thread> pool;
  for (int t = 0; t < threads; ++t)
    pool.emplace_back([&, t] {
      for (int i = t; i < n; i += threads) f(i);
    });
  for (auto& th : pool) th.join();
}

}  // namespace

extern "C" {

// Transform rows of logits into probabilities (double) and entropies (nats).
// valid[r] = 0 marks an invalid row (its probabilities are left at 0).
int oracle_transform_rows(const void* logits, int dtype, int rows, int V, double T, int top_k,
                          double top_p, double* probs, double* entropy, double* topp_margin,
                          int32_t* valid, int threads) {
  if (!logits || rows < 0 || V <= 0 || !(T >= 0.0)) return -1;
  parallel_rows(rows, threads, [&](int r) {
    std::vector<double> l;
    load_row(logits, dtype, size_t(r), V, l);
    double* pr = probs ? probs + size_t(r) * V : nullptr;
    if (!row_valid(l)) {
      if (pr) std::fill(pr, pr + V, 0.0);
      if (entropy) entropy[r] = 0.0;
      if (topp_margin) topp_margin[r] = kInf;
      if (valid) valid[r] = 0;
      return;
    }
    const Dist d = transform(l, T, top_k, top_p);
    if (pr) std::copy(d.p.begin(), d.p.end(), pr);
    if (entropy) entropy[r] = d.entropy;
    if (topp_margin) topp_margin[r] = d.topp_margin();
    if (valid) valid[r] = 1;
  });
  return 0;
}

// Chain verification over B batch rows (see chain_row), with the uniforms
// given in double precision. flags may be NULL.
int oracle_verify_chain_f64u(const void* target, const void* draft, int dtype, int B, int K,
                             int V, const int32_t* draft_tokens, const double* uniforms, double T,
                             int top_k, double top_p, int32_t* accepted_len, int32_t* out_tokens,
                             int32_t* flags, int threads, const double* windows) {
  if (!target || (T != 0.0 && !draft) || B < 0 || K < 0 || V <= 0 || !draft_tokens ||
      !uniforms || !accepted_len || !out_tokens || !(T >= 0.0))
    return -1;
  ChainArgs a{target, draft, dtype, B, K, V, draft_tokens, uniforms, T, top_k, top_p,
              accepted_len, out_tokens, flags, windows_from(windows)};
  parallel_rows(B, threads, [&](int b) { chain_row(a, b); });
  return 0;
}

// The same with float32 uniforms (the library's interface); each is widened
// exactly to double.
int oracle_verify_chain(const void* target, const void* draft, int dtype, int B, int K, int V,
                        const int32_t* draft_tokens, const float* uniforms, double T, int top_k,
                        double top_p, int32_t* accepted_len, int32_t* out_tokens, int32_t* flags,
                        int threads, const double* windows) {
  if (!uniforms || B < 0 || K < 0) return -1;
  std::vector<double> u(size_t(B) * size_t(K + 1));
  for (size_t j = 0; j < u.size(); ++j) u[j] = double(uniforms[j]);
  return oracle_verify_chain_f64u(target, draft, dtype, B, K, V, draft_tokens, u.data(), T, top_k,
                                  top_p, accepted_len, out_tokens, flags, threads, windows);
}

// MEDUSA typical acceptance over a candidate tree ([SD] "Key Components";
// [SV] "推测解码"). Node n's logits give the next-token distribution after n;
// node 0 (the greedy first token) is accepted unconditionally; node c >= 1 is
// accepted iff its parent is and p_parent(tok_c) > min(eps, delta *
// exp(-H(p_parent))). The deepest accepted node (lowest index on ties) and its
// root-first ancestor chain are returned. T is the softmax temperature (1 in
// the library's interface; 0 gives the greedy limit).
int oracle_verify_tree_typical(const void* target, int dtype, int B, int N, int V,
                               const int32_t* node_tokens, const int32_t* parent_idx, double eps,
                               double delta, double T, int32_t* best_path, int path_cap,
                               int32_t* accepted_len, int32_t* flags, int threads,
                               const double* windows) {
  const Windows win = windows_from(windows);
  if (!target || B < 0 || N <= 0 || V <= 0 || !node_tokens || !parent_idx || !best_path ||
      path_cap <= 0 || !accepted_len || !(T >= 0.0))
    return -1;
  bool tree_ok = parent_idx[0] == -1;
  std::vector<int> depth(static_cast<size_t>(N), 0);
  for (int c = 1; c < N && tree_ok; ++c) {
    const int pa = parent_idx[c];
    if (pa < 0 || pa >= c)
      tree_ok = false;
    else
      depth[c] = depth[pa] + 1;
  }
  parallel_rows(B, threads, [&](int b) {
    int32_t* path = best_path + size_t(b) * path_cap;
    auto fail = [&]() {
      accepted_len[b] = -1;
      for (int j = 0; j < path_cap; ++j) path[j] = -1;
      if (flags) flags[b] = 0;
    };
    if (!tree_ok) return fail();
    int32_t flag = 0;
    std::vector<char> acc(static_cast<size_t>(N), 0);
    std::vector<char> have(static_cast<size_t>(N), 0);
    std::vector<Dist> dist(static_cast<size_t>(N));
    acc[0] = 1;
    std::vector<double> l;
    for (int c = 1; c < N; ++c) {
      const int pa = parent_idx[c];
      if (!acc[pa]) continue;
      if (!have[pa]) {
        load_row(target, dtype, size_t(b) * N + pa, V, l);
        if (!row_valid(l)) return fail();
        dist[pa] = transform(l, T, 0, 1.0);
        have[pa] = 1;
      }
      const int tok = node_tokens[size_t(b) * N + c];
      if (tok < 0 || tok >= V) return fail();
      const double p = dist[pa].p[tok];
      const double thr = std::min(eps, delta * std::exp(-dist[pa].entropy));
      if (thr > 0.0 && std::fabs(p - thr) / thr < win.tree) flag |= FLAG_TREE;
      acc[c] = p > thr;
    }
    int best = 0;
    for (int c = 1; c < N; ++c)
      if (acc[c] && depth[c] > depth[best]) best = c;
    const int len = depth[best] + 1;
    if (len > path_cap) return fail();
    for (int j = 0; j < path_cap; ++j) path[j] = -1;
    for (int n = best, j = len - 1; j >= 0; --j, n = (n > 0 ? parent_idx[n] : -1)) path[j] = n;
    accepted_len[b] = len;
    if (flags) flags[b] = flag;
  });
  return 0;
}

// Greedy verification over a candidate tree: several draft continuations checked against
// the target at once, the longest correct one kept ([SV] "推测解码": blockwise parallel
// decoding accepts a draft token while it equals the target's argmax; Lookahead decoding
// verifies candidate branches in parallel and keeps the longest correct one). Node n's
// logits give the next-token distribution after n; node 0 is accepted; node c >= 1 is
// accepted iff its parent is and node_tokens[c] is the argmax of the parent's logits
// (lowest id on ties). The deepest accepted node (lowest index on ties) and its root-first
// ancestor chain are returned, and next_token = the argmax of that node's logits (the
// token the round emits after the path). Rows the rule reads must be valid.
int oracle_verify_tree_greedy(const void* target, int dtype, int B, int N, int V,
                              const int32_t* node_tokens, const int32_t* parent_idx,
                              int32_t* best_path, int path_cap, int32_t* accepted_len,
                              int32_t* next_token, int threads) {
  if (!target || B < 0 || N <= 0 || V <= 0 || !node_tokens || !parent_idx || !best_path ||
      path_cap <= 0 || !accepted_len)
    return -1;
  bool tree_ok = parent_idx[0] == -1;
  std::vector<int> depth(static_cast<size_t>(N), 0);
  for (int c = 1; c < N && tree_ok; ++c) {
    const int pa = parent_idx[c];
    if (pa < 0 || pa >= c)
      tree_ok = false;
    else
      depth[c] = depth[pa] + 1;
  }
  parallel_rows(B, threads, [&](int b) {
    int32_t* path = best_path + size_t(b) * path_cap;
    auto fail = [&]() {
      accepted_len[b] = -1;
      for (int j = 0; j < path_cap; ++j) path[j] = -1;
      if (next_token) next_token[b] = -1;
    };
    if (!tree_ok) return fail();
    std::vector<int> arg(static_cast<size_t>(N), -1);  // argmax of node n's row, once read
    std::vector<double> l;
    auto argmax_of = [&](int n) {
      if (arg[n] < 0) {
        load_row(target, dtype, size_t(b) * N + n, V, l);
        if (!row_valid(l)) return -1;
        arg[n] = argmax_lowest(l);
      }
      return arg[n];
    };
    std::vector<char> acc(static_cast<size_t>(N), 0);
    acc[0] = 1;
    for (int c = 1; c < N; ++c) {
      const int pa = parent_idx[c];
      if (!acc[pa]) continue;
      const int g = argmax_of(pa);
      if (g < 0) return fail();
      const int tok = node_tokens[size_t(b) * N + c];
      if (tok < 0 || tok >= V) return fail();
      acc[c] = tok == g;
    }
    int best = 0;
    for (int c = 1; c < N; ++c)
      if (acc[c] && depth[c] > depth[best]) best = c;
    const int len = depth[best] + 1;
    const int g = argmax_of(best);
    if (len > path_cap || g < 0) return fail();
    for (int j = 0; j < path_cap; ++j) path[j] = -1;
    for (int n = best, j = len - 1; j >= 0; --j, n = (n > 0 ? parent_idx[n] : -1)) path[j] = n;
    accepted_len[b] = len;
    if (next_token) next_token[b] = g;
  });
  return 0;
}

// Rejection sampling over a candidate tree ([SD] "Key Components": MEDUSA's step (3) may
// reuse the rejection rule of speculative sampling so that the output keeps the target
// distribution). Node n's target row gives p_n, its draft row q_n, the distribution its
// children's tokens were drawn from (independently). From the root: at the current node,
// the children are tried in index order; child c is accepted iff u[c] < min(1, p'(x_c) /
// q(x_c)), p' the current residual (p_n at first); a rejection replaces p' by
// norm(max(0, p' - q_n)) (unchanged if that is empty). An accepted child becomes the current
// node. When no child is accepted (or there is none) the emitted token is drawn from p' by
// the inverse CDF with u[N]. The accepted path (root first) and that token are returned.
// T == 0 is the greedy limit: the first child whose token is the argmax of p_n is accepted,
// and the emitted token is that argmax. uniforms [B][N + 1] (u[0] unused).
int oracle_verify_tree_sampling_f64u(const void* target, const void* draft, int dtype, int B,
                                     int N, int V, const int32_t* node_tokens,
                                     const int32_t* parent_idx, const double* uniforms, double T,
                                     int top_k, double top_p, int32_t* best_path, int path_cap,
                                     int32_t* accepted_len, int32_t* next_token, int32_t* flags,
                                     int threads, const double* windows) {
  const Windows win = windows_from(windows);
  if (!target || (T != 0.0 && !draft) || B < 0 || N <= 0 || V <= 0 || !node_tokens ||
      !parent_idx || !uniforms || !best_path || path_cap <= 0 || !accepted_len || !(T >= 0.0))
    return -1;
  bool tree_ok = parent_idx[0] == -1;
  std::vector<std::vector<int>> kids(static_cast<size_t>(N));
  for (int c = 1; c < N && tree_ok; ++c) {
    const int pa = parent_idx[c];
    if (pa < 0 || pa >= c)
      tree_ok = false;
    else
      kids[pa].push_back(c);  // index order
  }
  parallel_rows(B, threads, [&](int b) {
    int32_t* path = best_path + size_t(b) * path_cap;
    auto fail = [&]() {
      accepted_len[b] = -1;
      for (int j = 0; j < path_cap; ++j) path[j] = -1;
      if (next_token) next_token[b] = -1;
      if (flags) flags[b] = 0;
    };
    if (!tree_ok) return fail();
    const int32_t* tok = node_tokens + size_t(b) * N;
    const double* u = uniforms + size_t(b) * (N + 1);
    int32_t flag = 0;
    std::vector<int> nodes{0};
    std::vector<double> lp, lq;
    int cur = 0, emitted = -1;
    for (;;) {
      load_row(target, dtype, size_t(b) * N + cur, V, lp);
      if (!row_valid(lp)) return fail();
      const Dist pd = transform(lp, T, top_k, top_p);
      if (pd.topp_margin() < win.topp) flag |= FLAG_TOPP;
      int next = -1;
      if (T == 0.0) {
        const int g = argmax_lowest(lp);
        for (int c : kids[cur]) {
          if (tok[c] < 0 || tok[c] >= V) return fail();
          if (tok[c] == g) {
            next = c;
            break;
          }
        }
        if (next < 0) emitted = g;
      } else {
        std::vector<double> r = pd.p;  // the current residual, normalised
        if (!kids[cur].empty()) {
          load_row(draft, dtype, size_t(b) * N + cur, V, lq);
          if (!row_valid(lq)) return fail();
          const Dist qd = transform(lq, T, top_k, top_p);
          if (qd.topp_margin() < win.topp) flag |= FLAG_TOPP;
          for (int c : kids[cur]) {
            const int x = tok[c];
            if (x < 0 || x >= V) return fail();
            const double px = r[x], qx = qd.p[x];
            const double ratio = qx > 0.0 ? px / qx : (px > 0.0 ? kInf : 0.0);
            if (std::fabs(u[c] - ratio) < win.ratio) flag |= FLAG_RATIO;
            if (u[c] < std::min(1.0, ratio)) {
              next = c;
              break;
            }
            std::vector<double> rn(static_cast<size_t>(V));
            double S = 0.0;
            for (int v = 0; v < V; ++v) {
              rn[v] = std::max(0.0, r[v] - qd.p[v]);
              S += rn[v];
            }
            if (S > 0.0) {
              for (int v = 0; v < V; ++v) r[v] = rn[v] / S;
            }
          }
        }
        if (next < 0) {
          const Draw d = inverse_cdf(r, u[N], win);
          if (d.flag) flag |= FLAG_CDF;
          emitted = d.token;
        }
      }
      if (next < 0) break;
      nodes.push_back(next);
      cur = next;
    }
    const int len = int(nodes.size());
    if (len > path_cap || emitted < 0) return fail();
    for (int j = 0; j < path_cap; ++j) path[j] = j < len ? nodes[j] : -1;
    accepted_len[b] = len;
    if (next_token) next_token[b] = emitted;
    if (flags) flags[b] = flag;
  });
  return 0;
}

// The same with float32 uniforms (the library's interface), each widened exactly.
int oracle_verify_tree_sampling(const void* target, const void* draft, int dtype, int B, int N,
                                int V, const int32_t* node_tokens, const int32_t* parent_idx,
                                const float* uniforms, double T, int top_k, double top_p,
                                int32_t* best_path, int path_cap, int32_t* accepted_len,
                                int32_t* next_token, int32_t* flags, int threads,
                                const double* windows) {
  if (!uniforms || B < 0 || N <= 0) return -1;
  std::vector<double> u(size_t(B) * size_t(N + 1));
  for (size_t j = 0; j < u.size(); ++j) u[j] = double(uniforms[j]);
  return oracle_verify_tree_sampling_f64u(target, draft, dtype, B, N, V, node_tokens, parent_idx,
                                          u.data(), T, top_k, top_p, best_path, path_cap,
                                          accepted_len, next_token, flags, threads, windows);
}

// Inverse-CDF draw from norm(max(0, p - q)) (q == NULL: from p) for explicit
// probability rows. Entries are probabilities: a row holding an entry that is
// NaN or outside [0, 1], or whose p has no positive entry, gives token -1.
int oracle_residual_sample(const float* p, const float* q, int rows, int V, const float* uniforms,
                           int32_t* tokens, int32_t* flags, int threads, const double* windows) {
  const Windows win = windows_from(windows);
  if (!p || rows < 0 || V <= 0 || !uniforms || !tokens) return -1;
  parallel_rows(rows, threads, [&](int r) {
    std::vector<double> pr(static_cast<size_t>(V)), qr(size_t(V), 0.0);
    bool ok = true;
    for (int v = 0; v < V; ++v) {
      pr[v] = double(p[size_t(r) * V + v]);
      if (!(pr[v] >= 0.0 && pr[v] <= 1.0)) ok = false;
      if (q) {
        qr[v] = double(q[size_t(r) * V + v]);
        if (!(qr[v] >= 0.0 && qr[v] <= 1.0)) ok = false;
      }
    }
    double mass = 0.0;
    for (double x : pr) mass += x;
    if (!ok || !(mass > 0.0)) {
      tokens[r] = -1;
      if (flags) flags[r] = 0;
      return;
    }
    const Draw d = inverse_cdf(q ? residual(pr, qr) : pr, double(uniforms[r]), win);
    tokens[r] = d.token;
    if (flags) flags[r] = d.flag ? FLAG_CDF : 0;
  });
  return 0;
}

// Logits of the scoring forward's last layer: logits[r][v] = sum_j hidden[r][j] * weight[v][j]
// (the LM head, weight row v = token v's output embedding), in double from bfloat16 inputs.
// The pages put the bandwidth and compute of a round in the target's forward ([SD]
// "Speculative Sampling": scoring K drafts costs about one forward because the linear layers
// are memory-bound at small batch); this is its final matrix product, written as plain loops.
// hidden [rows][d], weight [V][d] bfloat16 bit patterns; out [rows][V] double.
int oracle_lmhead_logits(const uint16_t* hidden, const uint16_t* weight, int rows, int V, int d,
                         double* out, int threads) {
  if (!hidden || !weight || !out || rows < 0 || V <= 0 || d <= 0) return -1;
  parallel_rows(rows, threads, [&](int r) {
    std::vector<double> h(static_cast<size_t>(d));
    for (int j = 0; j < d; ++j) h[j] = bf16_bits_to_double(hidden[size_t(r) * d + j]);
    for (int v = 0; v < V; ++v) {
      const uint16_t* w = weight + size_t(v) * d;
      double acc = 0.0;
      for (int j = 0; j < d; ++j) acc += h[j] * bf16_bits_to_double(w[j]);
      out[size_t(r) * V + v] = acc;
    }
  });
  return 0;
}

// State commit after verification for a linear-attention target ([SpecLA] summary: the
// state is a dense summary updated with every token, and after the verdict it is brought to
// the accepted prefix; the summary names the gated-delta-rule model GDN). The recurrence,
// per sequence b and head h, with the state S in R^{dk x dv}:
//   S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,   t = 1 .. steps[b],
// replayed here one step at a time in double (the plain definition; no compact factors).
// state0 [B][H][dk][dv] float, alpha, beta [B][H][K], keys [B][H][K][dk], values
// [B][H][K][dv] float; out [B][H][dk][dv] double. steps[b] outside [0, K] leaves the state
// unchanged (an error row of the verification).
int oracle_linear_state_replay(const float* state0, int B, int H, int dk, int dv, int K,
                               const float* alpha, const float* beta, const float* keys,
                               const float* values, const int32_t* steps, double* out,
                               int threads) {
  if (!state0 || B < 0 || H <= 0 || dk <= 0 || dv <= 0 || K < 0 || !alpha || !beta || !keys ||
      !values || !steps || !out)
    return -1;
  parallel_rows(B * H, threads, [&](int bh) {
    const int b = bh / H;
    const size_t n = size_t(dk) * dv;
    double* S = out + size_t(bh) * n;
    for (size_t i = 0; i < n; ++i) S[i] = double(state0[size_t(bh) * n + i]);
    const int a = steps[b];
    if (a < 0 || a > K) return;
    std::vector<double> kS(static_cast<size_t>(dv));
    for (int t = 0; t < a; ++t) {
      const size_t st = size_t(bh) * K + t;
      const double al = alpha[st], be = beta[st];
      const float* k = keys + st * dk;
      const float* v = values + st * dv;
      // kS = k^T S_{t-1}
      for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += double(k[i]) * S[size_t(i) * dv + j];
        kS[j] = acc;
      }
      // S_t = alpha (S - beta k kS^T) + beta k v^T
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) {
          double& x = S[size_t(i) * dv + j];
          x = al * (x - be * double(k[i]) * kS[j]) + be * double(k[i]) * double(v[j]);
        }
    }
  });
  return 0;
}

}  // extern "C"
