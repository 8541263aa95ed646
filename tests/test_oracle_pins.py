"""Pins of the oracle to what the pages and the mathematics fix (no GPU).

Sources: taking-lying-flat.github.io/blog/posts/spec-decoding-i/ (sections
"Speculative Decoding", "Speculative Sampling", "Key Components") and
blog.csdn.net/yorkhunter/article/details/139214590 (section "推测解码").
Each test names the property it pins; none re-types the oracle's formula.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import pytest
from scipy.special import softmax
from scipy.stats import chisquare
from scipy.stats import entropy as scipy_entropy

import oracle
import specgen
from tests._helpers import chain_case, check_chain_invariants, draft_tokens, f32_logits, to_f64

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------- golden (hand-derived)

@pytest.mark.parametrize("case", _load("chain_handworked.json")["cases"], ids=lambda c: c["name"])
def test_golden_chain(case):
    target = f32_logits(case["target"])[None]
    K = target.shape[1] - 1
    draft = None if case["draft"] is None else f32_logits(case["draft"])[None]
    toks = np.array([case["tokens"]], np.int32)
    u = np.array([case["u"]], np.float32)
    acc, out, _ = oracle.verify_chain(target, draft, toks, u, case["temp"])
    assert int(acc[0]) == case["accepted_len"]
    assert out[0].tolist() == case["out"]
    assert K == len(case["tokens"])


@pytest.mark.parametrize("case", _load("transform_handworked.json")["cases"],
                         ids=lambda c: c["name"])
def test_golden_transform(case):
    logits = f32_logits([case["logits"]])
    probs, _, _, valid = oracle.transform_rows(logits, case["temp"], case["top_k"], case["top_p"])
    expect = np.array([eval(s, {"e": math.e}) for s in case["expect"]], np.float64)
    assert valid[0] == 1
    np.testing.assert_allclose(probs[0], expect, rtol=0, atol=case["tol"])


@pytest.mark.parametrize("case", _load("tree_handworked.json")["cases"], ids=lambda c: c["name"])
def test_golden_tree(case):
    logits = f32_logits(case["logits"])[None]
    toks = np.array([case["tokens"]], np.int32)
    par = np.array(case["parent"], np.int32)
    path, acc, _ = oracle.verify_tree_typical(logits, toks, par, case["eps"], case["delta"])
    assert int(acc[0]) == case["accepted_len"]
    n = case["accepted_len"]
    assert path[0, :n].tolist() == case["path"]
    assert np.all(path[0, n:] == -1)


# --------------------------------------------------------------------------- T1: exact enumeration

def _bisect(pred, n, iters=70):
    """Boundary t_j in [0,1] of n monotone predicates (False below t_j, True from t_j on)."""
    lo, hi = np.zeros(n), np.ones(n)
    at_zero = pred(np.zeros(n))
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        r = pred(mid)
        hi = np.where(r, mid, hi)
        lo = np.where(r, lo, mid)
    return np.where(at_zero, 0.0, hi)


def _enumerate_chain(V, temp, top_k, top_p, seed, ties=False):
    """Exact output law of one K=2 round, integrated over (u_0, u_1, w) by locating every
    decision boundary of the oracle (black box) to double precision."""
    g = np.random.default_rng(seed)

    def logits(*shape):
        x = g.normal(0.0, 1.5, size=shape)
        if ties:
            x = np.round(x * 2) / 2
        return x.astype(np.float32)

    t1, d1 = logits(V), logits(V)
    t2, d2 = logits(V, V), logits(V, V)          # indexed by x1
    t3 = logits(V, V, V)                        # indexed by (x1, x2)
    X1, X2 = np.meshgrid(np.arange(V), np.arange(V), indexing="ij")
    X1, X2 = X1.ravel(), X2.ravel()
    n = V * V
    target = np.stack([np.broadcast_to(t1, (n, V)), t2[X1], t3[X1, X2]], axis=1).copy()
    draft = np.stack([np.broadcast_to(d1, (n, V)), d2[X1]], axis=1).copy()
    toks = np.stack([X1, X2], axis=1).astype(np.int32)

    def run(u0, u1, w):
        u = np.stack([np.broadcast_to(u0, (n,)), np.broadcast_to(u1, (n,)),
                      np.broadcast_to(w, (n,))], axis=1).astype(np.float64)
        acc, out, _ = oracle.verify_chain(target, draft, toks, u, temp, top_k, top_p, threads=1)
        return acc, out

    below1 = 1.0 - 2.0 ** -53
    tau1 = _bisect(lambda u: run(u, 0.0, 0.5)[0] < 1, n)
    tau2 = _bisect(lambda u: run(0.0, u, 0.5)[0] < 2, n)

    def law(u0, u1, slot):
        b = np.zeros((n, V + 1))
        b[:, V] = 1.0
        for v in range(1, V):
            b[:, v] = _bisect(lambda w: run(u0, u1, w)[1][:, slot] >= v, n)
        return np.diff(b, axis=1)  # [n, V] probability of each token

    R1 = law(below1, 0.0, 0)
    R2 = law(0.0, below1, 1)
    BON = law(0.0, 0.0, 2)

    def tp(rows):
        return oracle.transform_rows(rows, temp, top_k, top_p)[0]

    P1, Q1 = tp(t1[None])[0], tp(d1[None])[0]
    P2, Q2, P3 = tp(t2), tp(d2), tp(t3.reshape(V * V, V)).reshape(V, V, V)
    return dict(V=V, X1=X1, X2=X2, tau1=tau1, tau2=tau2, R1=R1, R2=R2, BON=BON,
                P1=P1, Q1=Q1, P2=P2, Q2=Q2, P3=P3, t1=t1, t2=t2, t3=t3)


def _check_law(E, atol=1e-12):
    V, X1, X2 = E["V"], E["X1"], E["X2"]
    P1, Q1, P2, Q2, P3 = E["P1"], E["Q1"], E["P2"], E["Q2"], E["P3"]
    first = np.zeros(V)
    for x1 in range(V):
        j = x1 * V  # any x2: position-1 decisions do not depend on x2
        first[x1] += Q1[x1] * E["tau1"][j]
        first += Q1[x1] * (1.0 - E["tau1"][j]) * E["R1"][j]
    np.testing.assert_allclose(first, P1, rtol=0, atol=atol)
    for x1 in range(V):
        if Q1[x1] * E["tau1"][x1 * V] == 0.0:
            continue
        second = np.zeros(V)
        for x2 in range(V):
            j = x1 * V + x2
            second[x2] += Q2[x1, x2] * E["tau2"][j]
            second += Q2[x1, x2] * (1.0 - E["tau2"][j]) * E["R2"][j]
        np.testing.assert_allclose(second, P2[x1], rtol=0, atol=atol)
    for j in range(V * V):
        if E["tau1"][j] * E["tau2"][j] > 0.0:
            np.testing.assert_allclose(E["BON"][j], P3[X1[j], X2[j]], rtol=0, atol=atol)


def test_T1_exact_law_equals_target_no_transform():
    """Each emitted token follows p exactly, whatever q is (distribution preservation,
    'Speculative Decoding' / 'Speculative Sampling'); here p and q are plain softmaxes,
    checked against scipy's softmax."""
    E = _enumerate_chain(V=8, temp=1.0, top_k=0, top_p=1.0, seed=11)
    np.testing.assert_allclose(E["P1"], softmax(E["t1"].astype(np.float64)), rtol=1e-14)
    _check_law(E)


@pytest.mark.parametrize("temp,top_k,top_p,ties", [(0.7, 0, 1.0, False), (1.0, 3, 1.0, True),
                                                  (1.3, 0, 0.8, False), (0.9, 5, 0.7, True)])
def test_T1_exact_law_equals_transformed_target(temp, top_k, top_p, ties):
    """With temperature/top-k/top-p the emitted tokens follow the transformed p
    ('Speculative Sampling', last bullet)."""
    E = _enumerate_chain(V=8, temp=temp, top_k=top_k, top_p=top_p, seed=23, ties=ties)
    _check_law(E)


# --------------------------------------------------------------------------- T2: p == q

@pytest.mark.parametrize("temp,top_k,top_p", [(1.0, 0, 1.0), (0.8, 7, 1.0), (1.2, 0, 0.85)])
def test_T2_equal_distributions_always_accept(temp, top_k, top_p):
    """With identical target and draft distributions the ratio rule accepts with
    probability 1 ('Key Components', contrast with independent sampling)."""
    g = np.random.default_rng(5)
    B, K, V = 64, 4, 40
    target = g.normal(0, 2, size=(B, K + 1, V)).astype(np.float32)
    draft = target[:, :K].copy()
    toks = g.integers(0, V, size=(B, K)).astype(np.int32)
    probs = oracle.transform_rows(draft, temp, top_k, top_p)[0]
    for b in range(B):                       # keep draft tokens inside q's support
        for i in range(K):
            if probs[b, i, toks[b, i]] == 0.0:
                toks[b, i] = int(np.argmax(probs[b, i]))
    u = g.random((B, K + 1)).astype(np.float32)
    u[:, :K] = np.minimum(u[:, :K], np.float32(1.0 - 2 ** -24))
    acc, out, _ = oracle.verify_chain(target, draft, toks, u, temp, top_k, top_p)
    assert np.all(acc == K)
    assert np.array_equal(out[:, :K], toks)


# --------------------------------------------------------------------------- T3: emit count

@pytest.mark.parametrize("cfg", [specgen.CFG1, specgen.CFG2, specgen.CFG3, specgen.CFG5],
                         ids=lambda c: c.name)
def test_T3_emit_count_on_workloads(cfg):
    """Every round emits at least 1 and at most K+1 tokens ('Speculative Sampling')."""
    B = min(cfg.B, 3)
    target, draft, toks, u, temp = chain_case(cfg, B)
    acc, out, flags = oracle.verify_chain(target, draft, toks, u, temp, cfg.top_k, cfg.top_p)
    check_chain_invariants(acc, out, toks, cfg.K, cfg.V)


# --------------------------------------------------------------------------- T4: greedy

def test_T4_greedy_is_longest_argmax_prefix():
    """Temperature 0: keep the longest prefix equal to the target's greedy predictions
    (blockwise parallel decoding in '推测解码'), ties to the lowest id as numpy.argmax does."""
    g = np.random.default_rng(7)
    B, K, V = 200, 6, 30
    vals = np.round(g.normal(0, 1, size=(B, K + 1, V)) * 2) / 2   # many ties
    target = specgen.f32_to_bf16_bits(vals.astype(np.float32))
    am = np.argmax(to_f64(target), axis=2)
    toks = np.where(g.random((B, K)) < 0.8, am[:, :K], g.integers(0, V, (B, K))).astype(np.int32)
    u = g.random((B, K + 1)).astype(np.float32)
    acc, out, _ = oracle.verify_chain(target, None, toks, u, 0.0)
    for b in range(B):
        a = 0
        while a < K and toks[b, a] == am[b, a]:
            a += 1
        assert acc[b] == a
        assert out[b, :a].tolist() == toks[b, :a].tolist()
        assert out[b, a] == am[b, a]
        assert np.all(out[b, a + 1:] == -1)


# --------------------------------------------------------------------------- T5: transforms

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("temp", [0.3, 1.0, 2.5])
def test_T5_identity_transform_is_softmax(dtype, temp):
    g = np.random.default_rng(3)
    x = g.normal(0, 3, size=(20, 257)).astype(np.float32)
    logits = specgen.f32_to_bf16_bits(x) if dtype == "bf16" else x
    for k, p in [(0, 1.0), (257, 1.0), (-1, 1.0), (0, 1.5)]:
        probs, ent, _, valid = oracle.transform_rows(logits, temp, k, p)
        ref = softmax(to_f64(logits) / temp, axis=1)
        np.testing.assert_allclose(probs, ref, rtol=1e-13, atol=1e-300)
        np.testing.assert_allclose(probs.sum(1), 1.0, rtol=0, atol=1e-14)
        np.testing.assert_allclose(ent, scipy_entropy(ref, axis=1), rtol=1e-9, atol=1e-14)
        assert valid.all()


def test_T5_topk_is_renormalised_lexsort_prefix():
    g = np.random.default_rng(4)
    V = 64
    x = np.round(g.normal(0, 1, size=(50, V)) * 3) / 3          # ties
    logits = specgen.f32_to_bf16_bits(x.astype(np.float32))
    l = to_f64(logits)
    for k in (1, 2, 5, 17, 63):
        probs = oracle.transform_rows(logits, 0.8, k, 1.0)[0]
        for r in range(l.shape[0]):
            keep = np.lexsort((np.arange(V), -l[r]))[:k]
            ref = np.zeros(V)
            ref[keep] = softmax(l[r, keep] / 0.8)
            np.testing.assert_allclose(probs[r], ref, rtol=1e-13, atol=1e-300)


def test_T5_topp_keeps_tokens_whose_preceding_mass_is_below_top_p():
    """Nucleus = the tokens whose exclusive cumulative mass (in descending-probability,
    ascending-id order) is below top_p: the same set as 'shortest prefix reaching top_p'."""
    g = np.random.default_rng(9)
    V = 48
    x = np.round(g.normal(0, 1.2, size=(80, V)) * 4) / 4
    logits = x.astype(np.float32)
    l = logits.astype(np.float64)
    for top_p in (0.05, 0.5, 0.9, 0.999):
        probs, _, marg, _ = oracle.transform_rows(logits, 1.0, 0, top_p)
        for r in range(l.shape[0]):
            base = softmax(l[r])
            order = np.lexsort((np.arange(V), -base))
            excl = np.concatenate([[0.0], np.cumsum(base[order])[:-1]])
            keep = order[excl < top_p]
            ref = np.zeros(V)
            ref[keep] = base[keep] / base[keep].sum()
            if marg[r] > 1e-9:
                np.testing.assert_allclose(probs[r], ref, rtol=1e-12, atol=1e-300)


def test_T5_entropy_closed_forms():
    V = 1000
    uniform = np.zeros((1, V), np.float32)
    _, ent, _, _ = oracle.transform_rows(uniform, 1.0)
    assert abs(ent[0] - math.log(V)) < 1e-12
    onehot = np.full((1, V), -np.inf, np.float32)
    onehot[0, 17] = 3.0
    probs, ent, _, valid = oracle.transform_rows(onehot, 1.0)
    assert valid[0] == 1 and ent[0] == 0.0 and probs[0, 17] == 1.0
    _, ent_k, _, _ = oracle.transform_rows(uniform, 1.0, top_k=10)
    assert abs(ent_k[0] - math.log(10)) < 1e-12


def test_T5_bf16_decoding_and_invalid_rows():
    bits = np.array([[0x3F80, 0x0000, 0xC000, 0xFF80]], np.uint16)   # 1, 0, -2, -inf
    probs, _, _, valid = oracle.transform_rows(bits, 1.0)
    ref = softmax(np.array([1.0, 0.0, -2.0, -np.inf]))
    np.testing.assert_allclose(probs[0], ref, rtol=1e-15)
    bad = np.array([[0x7FC0, 0, 0, 0], [0x7F80, 0, 0, 0], [0xFF80] * 4, [0xFFC0, 0, 0, 0]],
                   np.uint16)                                      # NaN, +inf, all -inf, -NaN
    _, _, _, valid = oracle.transform_rows(bad, 1.0)
    assert valid.tolist() == [0, 0, 0, 0]


def test_T5_greedy_limit_is_onehot():
    logits = np.array([[1.0, 3.0, 3.0, 2.0]], np.float32)
    probs, ent, _, _ = oracle.transform_rows(logits, 0.0)
    assert probs[0].tolist() == [0.0, 1.0, 0.0, 0.0] and ent[0] == 0.0


# --------------------------------------------------------------------------- T6/T7: tree

def _random_tree(g, N):
    par = np.array([-1] + [int(g.integers(0, c)) for c in range(1, N)], np.int32)
    return par


def _tree_brute(l, toks, par, eps, delta, temp):
    """Evaluate the typical criterion on every edge of every root-to-node path."""
    N, V = l.shape
    def dist(n):
        if temp == 0.0:
            p = np.zeros(V)
            p[np.argmax(l[n])] = 1.0
            return p, 0.0
        p = softmax(l[n] / temp)
        return p, scipy_entropy(p)
    ok = np.zeros(N, bool)
    for c in range(1, N):
        p, H = dist(par[c])
        ok[c] = p[toks[c]] > min(eps, delta * math.exp(-H))
    best, best_depth = 0, 0
    for c in range(1, N):
        path, n = [], c
        while n > 0:
            path.append(n)
            n = par[n]
        if all(ok[m] for m in path) and len(path) > best_depth:
            best, best_depth = c, len(path)
    path, n = [best], best
    while n > 0:
        n = par[n]
        path.append(n)
    return path[::-1]


@pytest.mark.parametrize("seed", range(6))
def test_T6_tree_matches_path_enumeration(seed):
    g = np.random.default_rng(100 + seed)
    B, N, V = 6, 14, 16
    par = _random_tree(g, N)
    toks = g.integers(0, V, size=(B, N)).astype(np.int32)
    x = g.normal(0, 1.5, size=(B, N, V))
    for b in range(B):                    # favour children's tokens so paths get deep
        for c in range(1, N):
            if g.random() < 0.7:
                x[b, par[c], toks[b, c]] += 2.5
    logits = x.astype(np.float32)
    eps, delta = 0.09, 0.3
    path, acc, _ = oracle.verify_tree_typical(logits, toks, par, eps, delta)
    for b in range(B):
        ref = _tree_brute(logits[b].astype(np.float64), toks[b], par, eps, delta, 1.0)
        assert acc[b] == len(ref)
        assert path[b, :len(ref)].tolist() == ref


@pytest.mark.parametrize("seed", range(3))
def test_T7_tree_at_temperature_zero_is_greedy(seed):
    """At temperature 0 typical acceptance reduces to greedy matching ('Key Components')."""
    g = np.random.default_rng(200 + seed)
    B, N, V = 8, 12, 10
    par = _random_tree(g, N)
    l = g.permuted(np.tile(np.arange(V, dtype=np.float64), (B, N, 1)), axis=2)  # distinct
    am = np.argmax(l, axis=2)
    toks = np.where(g.random((B, N)) < 0.6, am[np.arange(B)[:, None], par[None, :].clip(0)],
                    g.integers(0, V, (B, N))).astype(np.int32)
    logits = l.astype(np.float32)
    for temp in (0.0, 1e-3):
        path, acc, _ = oracle.verify_tree_typical(logits, toks, par, 0.09, 0.3, temp=temp)
        for b in range(B):
            ref = _tree_brute(l[b], toks[b], par, 0.09, 0.3, 0.0)
            # greedy matching: accepted iff every token on the path equals its parent's argmax
            for n in ref[1:]:
                assert toks[b, n] == np.argmax(l[b, par[n]])
            assert path[b, :len(ref)].tolist() == ref and acc[b] == len(ref)


def _greedy_tree_brute(l, toks, par):
    """Every root-to-node path checked edge by edge against numpy's argmax (first index on
    ties); the deepest fully matching node, lowest index first; its row's argmax."""
    N = l.shape[0]
    best, best_depth = 0, 0
    for c in range(1, N):
        path, n = [], c
        while n > 0:
            path.append(n)
            n = par[n]
        if all(toks[m] == np.argmax(l[par[m]]) for m in path) and len(path) > best_depth:
            best, best_depth = c, len(path)
    path, n = [best], best
    while n > 0:
        n = par[n]
        path.append(n)
    return path[::-1], int(np.argmax(l[best]))


@pytest.mark.parametrize("seed", range(6))
def test_tree_greedy_matches_path_enumeration(seed):
    g = np.random.default_rng(300 + seed)
    B, N, V = 8, 14, 12
    par = _random_tree(g, N)
    l = np.round(g.normal(0, 1.0, size=(B, N, V)), 1)     # coarse values: ties occur
    am = np.argmax(l, axis=2)
    toks = np.where(g.random((B, N)) < 0.7, am[np.arange(B)[:, None], par[None, :].clip(0)],
                    g.integers(0, V, (B, N))).astype(np.int32)
    logits = l.astype(np.float32)
    assert np.array_equal(logits.astype(np.float64), l.astype(np.float32).astype(np.float64))
    path, acc, nxt = oracle.verify_tree_greedy(logits, toks, par)
    deep = 0
    for b in range(B):
        ref, ref_next = _greedy_tree_brute(logits[b].astype(np.float64), toks[b], par)
        assert acc[b] == len(ref) and path[b, :len(ref)].tolist() == ref
        assert np.all(path[b, len(ref):] == -1) and nxt[b] == ref_next
        deep = max(deep, len(ref))
    assert deep >= 3


def test_tree_greedy_is_typical_acceptance_at_temperature_zero():
    """Greedy tree verification is the T -> 0 limit of MEDUSA typical acceptance: the
    typical test against a one-hot distribution passes exactly for the argmax token."""
    g = np.random.default_rng(400)
    B, N, V = 10, 16, 9
    par = _random_tree(g, N)
    l = g.permuted(np.tile(np.arange(V, dtype=np.float64), (B, N, 1)), axis=2)
    am = np.argmax(l, axis=2)
    toks = np.where(g.random((B, N)) < 0.65, am[np.arange(B)[:, None], par[None, :].clip(0)],
                    g.integers(0, V, (B, N))).astype(np.int32)
    logits = l.astype(np.float32)
    p_g, a_g, _ = oracle.verify_tree_greedy(logits, toks, par)
    p_t, a_t, _ = oracle.verify_tree_typical(logits, toks, par, 0.5, 0.5, temp=0.0)
    assert np.array_equal(a_g, a_t) and np.array_equal(p_g, p_t)


def test_tree_greedy_on_a_path_is_chain_greedy():
    """A tree that is one path (parent = previous node) verifies like the greedy chain:
    node c's token is draft x_(c-1) against target row c-1; the emitted token after the
    accepted prefix is the chain's correction or bonus token."""
    g = np.random.default_rng(500)
    B, K, V = 12, 6, 20
    l = g.normal(0, 2.0, size=(B, K + 1, V)).astype(np.float32)
    am = np.argmax(l, axis=2)
    x = np.where(g.random((B, K)) < 0.75, am[:, :K], g.integers(0, V, (B, K))).astype(np.int32)
    acc_c, out_c, _ = oracle.verify_chain(l, None, x, np.zeros((B, K + 1), np.float32), 0.0)
    par = np.arange(-1, K, dtype=np.int32)
    toks = np.concatenate([np.zeros((B, 1), np.int32), x], axis=1)
    path, acc_t, nxt = oracle.verify_tree_greedy(l, toks, par)
    assert np.array_equal(acc_t, acc_c + 1)
    for b in range(B):
        assert path[b, :acc_t[b]].tolist() == list(range(acc_t[b]))
        assert nxt[b] == out_c[b, acc_c[b]]


def test_tree_greedy_errors_only_where_the_rule_reads():
    V = 6
    par = np.array([-1, 0, 0, 1], np.int32)
    l = np.zeros((2, 4, V), np.float32)
    l[:, 0, 2] = 1.0                 # root row argmax 2
    l[:, 1, 4] = 1.0                 # node 1 row argmax 4
    l[:, 2, :] = np.nan              # node 2's row: never read (no child of node 2)
    l[1, 1, 3] = np.inf              # batch row 1: node 1's row invalid, and it is read
    toks = np.array([[0, 2, 5, 4], [0, 2, 5, 4]], np.int32)
    path, acc, nxt = oracle.verify_tree_greedy(l, toks, par)
    assert acc.tolist() == [3, -1] and path[0, :3].tolist() == [0, 1, 3]
    assert nxt[0] == int(np.argmax(l[0, 3])) and nxt[1] == -1 and np.all(path[1] == -1)


# --------------------------------------------------------------------------- tree sampling

def _tree_sampling_first_token_law(V, m, temp, top_k, top_p, seed):
    """Exact law of the first token after the root of one round, the root holding m leaf
    children whose tokens are drawn independently from q_root: every tuple of child tokens
    is enumerated, and each acceptance threshold and the final draw's CDF are located by
    bisection on the oracle's decisions (black box)."""
    g = np.random.default_rng(seed)
    t_root = g.normal(0, 1.5, V).astype(np.float32)
    d_root = g.normal(0, 1.5, V).astype(np.float32)
    grids = np.meshgrid(*[np.arange(V)] * m, indexing="ij")
    X = np.stack([x.ravel() for x in grids], axis=1)           # [n, m] child tokens
    n, N = X.shape[0], m + 1
    target = np.zeros((n, N, V), np.float32)
    target[:, 0] = t_root
    target[:, 1:] = g.normal(0, 1.0, (n, m, V)).astype(np.float32)  # leaf rows (bonus only)
    draft = np.zeros((n, N, V), np.float32)
    draft[:, 0] = d_root
    draft[:, 1:] = 1.0
    toks = np.concatenate([np.zeros((n, 1), np.int32), X.astype(np.int32)], axis=1)
    par = np.array([-1] + [0] * m, np.int32)
    below1 = 1.0 - 2.0 ** -53

    def run(us, w):
        u = np.zeros((n, N + 1))
        for j, uj in enumerate(us):
            u[:, j + 1] = uj
        u[:, N] = w
        path, acc, nxt, _ = oracle.verify_tree_sampling(target, draft, toks, par, u, temp,
                                                        top_k, top_p, threads=1)
        return path, acc, nxt

    a = np.zeros((n, m))
    for j in range(m):
        def not_accepted_at_j(uj, j=j):
            us = [below1] * j + [uj] + [0.0] * (m - j - 1)
            path, acc, _ = run(us, 0.5)
            return ~((acc >= 2) & (path[:, 1] == j + 1))
        a[:, j] = _bisect(not_accepted_at_j, n)
    b = np.zeros((n, V + 1))
    b[:, V] = 1.0
    for v in range(1, V):
        b[:, v] = _bisect(lambda w: run([below1] * m, w)[2] >= v, n)
    draw = np.diff(b, axis=1)
    q = oracle.transform_rows(d_root[None], temp, top_k, top_p)[0][0]
    p = oracle.transform_rows(t_root[None], temp, top_k, top_p)[0][0]
    law = np.zeros(V)
    for t in range(n):
        w_t = np.prod(q[X[t]])
        if w_t == 0.0:
            continue
        reach = 1.0
        for j in range(m):
            law[X[t, j]] += w_t * reach * a[t, j]
            reach *= 1.0 - a[t, j]
        law += w_t * reach * draw[t]
    return law, p


@pytest.mark.parametrize("m,temp,top_k,top_p,seed", [
    (1, 1.0, 0, 1.0, 0), (2, 1.0, 0, 1.0, 1), (3, 1.0, 0, 1.0, 2), (2, 0.7, 3, 1.0, 3),
    (2, 1.3, 0, 0.8, 4), (3, 0.9, 3, 0.9, 5)])
def test_tree_sampling_keeps_the_target_distribution(m, temp, top_k, top_p, seed):
    """The first emitted token is distributed exactly as the transformed p_root, whatever
    the number of candidate children drawn from q_root ("Key Components": the rejection
    rule keeps the original model's output distribution)."""
    law, p = _tree_sampling_first_token_law(4, m, temp, top_k, top_p, seed)
    np.testing.assert_allclose(law, p, rtol=0, atol=1e-12)


def test_tree_sampling_with_p_equal_q_follows_first_children():
    g = np.random.default_rng(600)
    B, N, V = 6, 12, 9
    par = _random_tree(g, N)
    t = g.normal(0, 1.5, (B, N, V)).astype(np.float32)
    toks = g.integers(0, V, (B, N)).astype(np.int32)
    u = g.random((B, N + 1)).astype(np.float32) * np.float32(0.999)
    path, acc, nxt, _ = oracle.verify_tree_sampling(t, t, toks, par, u, 1.0)
    for b in range(B):
        ref, n_ = [0], 0
        while True:
            kids = [c for c in range(1, N) if par[c] == n_]
            if not kids:
                break
            n_ = kids[0]
            ref.append(n_)
        assert path[b, :acc[b]].tolist() == ref
        assert 0 <= nxt[b] < V


def test_tree_sampling_at_temperature_zero_is_greedy_tree():
    """With distinct sibling tokens, only one child can match the argmax: the T = 0 limit
    walks the same path as greedy tree verification and emits the same next token."""
    g = np.random.default_rng(700)
    B, N, V = 10, 16, 40
    par = _random_tree(g, N)
    l = g.normal(0, 2.0, (B, N, V)).astype(np.float32)
    am = np.argmax(l, axis=2)
    toks = np.zeros((B, N), np.int32)
    for b in range(B):
        for pa in range(N):
            kids = [c for c in range(1, N) if par[c] == pa]
            vals = g.permutation(V)[:len(kids)]
            if kids and g.random() < 0.8:
                vals[g.integers(0, len(kids))] = am[b, pa] if am[b, pa] not in vals else vals[0]
            for c, v in zip(kids, vals):
                toks[b, c] = v
    u = g.random((B, N + 1)).astype(np.float32)
    path_s, acc_s, nxt_s, _ = oracle.verify_tree_sampling(l, None, toks, par, u, 0.0)
    path_g, acc_g, nxt_g = oracle.verify_tree_greedy(l, toks, par)
    assert np.array_equal(acc_s, acc_g) and np.array_equal(path_s, path_g)
    assert np.array_equal(nxt_s, nxt_g)
    assert acc_g.max() >= 3


@pytest.mark.parametrize("temp,top_k,top_p", [(1.0, 0, 1.0), (0.8, 5, 1.0), (1.2, 0, 0.85)])
def test_tree_sampling_on_a_path_is_chain_sampling(temp, top_k, top_p):
    """A tree that is one path verifies like the chain: node c is draft x_(c-1) tested with
    uniform u[c] against target row c-1 and draft row c-1; the final draw uses u[N] like
    the chain's u[K]."""
    g = np.random.default_rng(800)
    B, K, V = 16, 5, 24
    target = g.normal(0, 2.0, (B, K + 1, V)).astype(np.float32)
    dk = (target[:, :K] + g.normal(0, 0.7, (B, K, V))).astype(np.float32)
    x = draft_tokens(dk, temp, top_k, top_p, g.random((B, K)).astype(np.float32))
    uc = g.random((B, K + 1)).astype(np.float32)
    acc_c, out_c, fl_c = oracle.verify_chain(target, dk, x, uc, temp, top_k, top_p)
    par = np.arange(-1, K, dtype=np.int32)
    draft = np.concatenate([dk, np.zeros((B, 1, V), np.float32)], axis=1)
    toks = np.concatenate([np.zeros((B, 1), np.int32), x], axis=1)
    ut = np.concatenate([np.zeros((B, 1), np.float32), uc], axis=1)   # u[c] = chain u[c-1]
    path, acc_t, nxt, fl_t = oracle.verify_tree_sampling(target, draft, toks, par, ut, temp,
                                                         top_k, top_p)
    assert np.array_equal(acc_t, acc_c + 1)
    for b in range(B):
        assert path[b, :acc_t[b]].tolist() == list(range(acc_t[b]))
        assert nxt[b] == out_c[b, acc_c[b]]
    assert acc_c.min() == 0 and acc_c.max() >= 2


def test_tree_sampling_errors_only_where_the_rule_reads():
    V = 6
    par = np.array([-1, 0, 0, 1], np.int32)
    t = np.zeros((2, 4, V), np.float32)
    d = np.zeros((2, 4, V), np.float32)
    t[:, 2, :] = np.nan              # node 2's target row: never read (node 2 has no child,
    d[:, 2, :] = np.nan              # and is not on an accepted path here)
    d[:, 3, :] = np.nan              # node 3 is a leaf: its draft row is never read
    toks = np.array([[0, 1, 2, 3], [0, 1, 2, 3]], np.int32)
    u = np.zeros((2, 5), np.float32)           # u = 0: every tested child is accepted
    d[1, 1, 0] = np.inf              # batch row 1: node 1's draft row is read (node 3 is its child)
    path, acc, nxt, _ = oracle.verify_tree_sampling(t, d, toks, par, u, 1.0)
    assert acc.tolist() == [3, -1] and path[0, :3].tolist() == [0, 1, 3]
    assert nxt[1] == -1 and np.all(path[1] == -1)


def test_tree_workload_structure_and_invalid_parent():
    par, depth, rank = specgen.tree_structure((4, 3, 2, 2), 64)
    assert np.bincount(depth).tolist() == [1, 4, 12, 24, 23]
    assert par[0] == -1 and np.all(par[1:] < np.arange(1, 64)) and np.all(par[1:] >= 0)
    logits = np.zeros((2, 3, 4), np.float32)
    toks = np.zeros((2, 3), np.int32)
    path, acc, _ = oracle.verify_tree_typical(logits, toks, np.array([-1, 2, 0], np.int32),
                                              0.09, 0.3)
    assert acc.tolist() == [-1, -1] and np.all(path == -1)


# --------------------------------------------------------------------------- errors

def test_chain_error_rows_are_procedural():
    """An invalid row or token only matters once the scan reaches it."""
    V, K = 6, 3
    target = np.zeros((3, K + 1, V), np.float32)
    draft = np.zeros((3, K, V), np.float32)
    draft[:, :, 0] = 5.0                      # q concentrated on token 0, p uniform
    toks = np.zeros((3, K), np.int32)         # r = (1/6)/q(0) < 1
    u = np.full((3, K + 1), 0.999, np.float32)  # reject at position 0
    target[1, 2, 0] = np.nan                  # after the stop: harmless
    toks[2, 0] = V                            # at the first test: error
    acc, out, _ = oracle.verify_chain(target, draft, toks, u, 1.0)
    assert acc.tolist() == [0, 0, -1]
    assert np.all(out[2] == -1)


# --------------------------------------------------------------------------- T8: Monte Carlo

def test_T8_monte_carlo_first_token_frequencies():
    """Sanity (not a pin): emitted first tokens over many seeded rounds follow p_1."""
    g = np.random.default_rng(12)
    B, K, V = 20000, 3, 20
    t = g.normal(0, 1.5, size=(K + 1, V)).astype(np.float32)
    d = (t[:K] + g.normal(0, 1.0, size=(K, V))).astype(np.float32)
    target = np.broadcast_to(t, (B, K + 1, V)).copy()
    draft = np.broadcast_to(d, (B, K, V)).copy()
    toks = draft_tokens(draft, 1.0, 0, 1.0, g.random((B, K)).astype(np.float32), 4096)
    u = g.random((B, K + 1)).astype(np.float32)
    acc, out, _ = oracle.verify_chain(target, draft, toks, u, 1.0)
    counts = np.bincount(out[:, 0], minlength=V)
    p1 = softmax(t[0].astype(np.float64))
    assert chisquare(counts, p1 * B).pvalue > 1e-4


# --------------------------------------------------------------------------- explicit-row draw

def _ln(x):
    return math.log(x) if x > 0 else None


def test_residual_sample_validity_rule():
    """The explicit-probability draw ("Speculative Sampling": resample from norm(max(0, p - q)))
    takes probabilities: an entry outside [0, 1] or NaN, in p or in q, or a p with no positive
    mass, gives token -1; every other row gives a token (hand-derived cases)."""
    V = 4
    good = [0.5, 0.25, 0.25, 0.0]
    rows_p = [good, [1.5, 0.0, 0.0, 0.0], [0.5, -0.25, 0.5, 0.25], [0.5, math.nan, 0.25, 0.25],
              [0.0, 0.0, 0.0, 0.0], good, good]
    rows_q = [good, good, good, good, good, [0.25, 1.25, 0.0, 0.0], [0.25, math.nan, 0.0, 0.0]]
    p = np.array(rows_p, np.float32)
    q = np.array(rows_q, np.float32)
    u = np.full(len(rows_p), 0.25, np.float32)
    tok, _ = oracle.residual_sample(p, q, u)
    # row 0: p == q, empty residual, falls back to p: w*S = 0.25 < C_0 = 0.5 -> token 0
    assert tok.tolist() == [0, -1, -1, -1, -1, -1, -1]
    tok_p, _ = oracle.residual_sample(p, None, u)          # q absent: only p is checked
    assert tok_p.tolist() == [0, -1, -1, -1, -1, 0, 0]


@pytest.mark.parametrize("w,expect", [(0.4, 0), (0.5, 2), (0.6, 2), (0.0, 0), (0.999, 2)])
def test_residual_sample_dyadic_golden(w, expect):
    """p = (1/2, 1/4, 1/4, 0), q = (1/4, 1/4, 0, 1/2): max(0, p - q) = (1/4, 0, 1/4, 0),
    S = 1/2. The smallest id whose cumulative mass exceeds w*S: C_0 = 1/4, C_2 = 1/2, so
    w*S < 1/4 (w < 1/2) gives token 0 and w >= 1/2 gives token 2 (strict '>' at the edge)."""
    p = np.array([[0.5, 0.25, 0.25, 0.0]], np.float32)
    q = np.array([[0.25, 0.25, 0.0, 0.5]], np.float32)
    tok, _ = oracle.residual_sample(p, q, np.array([w], np.float32))
    assert int(tok[0]) == expect


# --------------------------------------------------------------------------- top-p near ties

def _near_tie_case(x0, draft0):
    """K = 1, V = 4, top_p = 0.75. Target row 0 is p = (4, 2, 1, 1)/8: the two largest
    tokens hold exactly 0.75, so the nucleus {0, 1} sits on the top-p boundary (one more
    token, 2, on the other side). Target row 1 (the bonus) is (1, 2, 3, 10)/16, whose
    nucleus {3, 2} is far from the boundary (0.8125 and 0.625). u = (0, 0.3)."""
    target = f32_logits([[_ln(4), _ln(2), 0.0, 0.0], [0.0, _ln(2), _ln(3), _ln(10)]])[None]
    draft = f32_logits([draft0])[None]
    toks = np.array([[x0]], np.int32)
    u = np.array([[0.0, 0.3]], np.float32)
    return oracle.verify_chain(target, draft, toks, u, 1.0, 0, 0.75)


def test_topp_near_tie_flags_only_when_the_other_nucleus_changes_the_output():
    """A top-p boundary within the precision window flags a row only if evaluating the row
    with the other nucleus (one token more or fewer) changes its output ("Speculative
    Sampling": the transform decides p and q before the ratio test)."""
    # x = 2 lies outside {0, 1} but inside {0, 1, 2}; q = (1, 1, 14)/16 keeps {2}, q(2) = 1.
    # Nucleus {0, 1}: p(2) = 0, r = 0, u = 0 is not < 0 -> reject, redraw from p.
    # Nucleus {0, 1, 2}: p(2) = 1/7 > 0 -> accept, bonus token. Different outputs: flagged.
    acc, out, flags = _near_tie_case(2, [0.0, 0.0, _ln(14), None])
    assert int(flags[0]) & oracle.FLAG_TOPP
    assert int(acc[0]) == 0 and int(out[0, 0]) in (0, 1)
    # x = 0 lies inside both nuclei; q = (14, 1, 1)/16 keeps {0}, q(0) = 1, r = 2/3 or 4/7,
    # u = 0 accepts either way; the bonus draw from (3, 10)/13 at w = 0.3 gives token 3
    # (C_2 = 3/13 < 0.3). Same output: not flagged.
    acc, out, flags = _near_tie_case(0, [_ln(14), 0.0, 0.0, None])
    assert int(flags[0]) & oracle.PARITY_FLAGS == 0
    assert int(acc[0]) == 1 and out[0].tolist() == [0, 3]


def test_topp_near_tie_below_the_boundary_tries_one_token_fewer():
    """Cumulative mass just below top_p before the crossing token (p = (4, 2, 1, 1)/8,
    top_p = 0.75 + 5e-7: {0, 1} holds 0.75, so the nucleus is {0, 1, 2} with the boundary
    5e-7 away). The alternative nucleus {0, 1} drops token 2: a draft x = 2 accepted with
    {0, 1, 2} is rejected with {0, 1}, so the row is flagged; x = 0 is not."""
    target = f32_logits([[_ln(4), _ln(2), 0.0, 0.0], [0.0, _ln(2), _ln(3), _ln(10)]])[None]
    u = np.array([[0.0, 0.3]], np.float32)
    top_p = 0.75 + 5e-7
    d2 = f32_logits([[0.0, 0.0, _ln(14), None]])[None]
    acc, out, flags = oracle.verify_chain(target, d2, np.array([[2]], np.int32), u, 1.0, 0, top_p)
    assert int(acc[0]) == 1 and int(flags[0]) & oracle.FLAG_TOPP
    d0 = f32_logits([[_ln(14), 0.0, 0.0, None]])[None]
    acc, out, flags = oracle.verify_chain(target, d0, np.array([[0]], np.int32), u, 1.0, 0, top_p)
    assert int(acc[0]) == 1 and int(flags[0]) & oracle.PARITY_FLAGS == 0


# --------------------------------------------------------------------------- linear-state commit
# The recurrence S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T (the gated
# delta rule of the linear-attention model the SpecLA summary names); pins from its
# properties, none re-typing the update.

def _lstate(B=2, H=3, dk=8, dv=5, K=4, seed=0):
    g = np.random.default_rng(seed)
    S0 = g.normal(size=(B, H, dk, dv)).astype(np.float32)
    k = g.normal(size=(B, H, K, dk))
    k = (k / np.linalg.norm(k, axis=3, keepdims=True)).astype(np.float32)
    v = g.normal(size=(B, H, K, dv)).astype(np.float32)
    al = g.uniform(0.5, 1.0, (B, H, K)).astype(np.float32)
    be = g.uniform(0.0, 1.0, (B, H, K)).astype(np.float32)
    return S0, al, be, k, v


def test_linear_state_without_writes_only_decays():
    """beta = 0: no write; the state decays by the product of the gates."""
    S0, al, be, k, v = _lstate()
    steps = np.array([3, 4], np.int32)
    out = oracle.linear_state_replay(S0, al, np.zeros_like(be), k, v, steps)
    for b in range(2):
        g = np.prod(al[b, :, :steps[b]].astype(np.float64), axis=1)
        np.testing.assert_allclose(out[b], g[:, None, None] * S0[b], rtol=1e-12)


def test_linear_state_full_write_stores_the_value_at_its_key():
    """alpha = beta = 1 and a unit key: reading the state at k gives v (the delta rule
    replaces what k retrieved), and directions orthogonal to k are untouched."""
    S0, al, be, k, v = _lstate(B=1, H=1, dk=6, dv=4, K=1, seed=3)
    out = oracle.linear_state_replay(S0, np.ones_like(al), np.ones_like(be), k, v,
                                     np.array([1], np.int32))[0, 0]
    kk = k[0, 0, 0].astype(np.float64)
    n2 = kk @ kk                                   # 1 up to the key's float32 rounding
    np.testing.assert_allclose(kk @ out, (1 - n2) * (kk @ S0[0, 0]) + n2 * v[0, 0, 0],
                               rtol=1e-12, atol=1e-12)
    assert abs(n2 - 1) < 1e-6
    x = np.linalg.svd(kk[None])[2][1:]            # an orthonormal basis of k's complement
    np.testing.assert_allclose(x @ out, x @ S0[0, 0].astype(np.float64), atol=1e-12)


def test_linear_state_orthonormal_keys_keep_every_write():
    """Orthonormal keys, alpha = beta = 1: after a steps every k_t reads back its v_t."""
    dk, dv, K = 8, 3, 5
    g = np.random.default_rng(4)
    q, _ = np.linalg.qr(g.normal(size=(dk, dk)))
    keys = q[:, :K].T.astype(np.float32)[None, None]          # [1, 1, K, dk]
    S0 = g.normal(size=(1, 1, dk, dv)).astype(np.float32)
    v = g.normal(size=(1, 1, K, dv)).astype(np.float32)
    ones = np.ones((1, 1, K), np.float32)
    out = oracle.linear_state_replay(S0, ones, ones, keys, v, np.array([K], np.int32))[0, 0]
    np.testing.assert_allclose(keys[0, 0].astype(np.float64) @ out, v[0, 0], atol=1e-6)


def test_linear_state_partial_write_mixes_old_and_new():
    """A unit key with write strength beta and gate alpha: k^T S_1 = alpha (1 - beta) k^T S_0
    + beta v (the old content is reduced by beta before the decay, the new one is not
    decayed); with |k|^2 = n2 from the key's rounding, beta becomes beta * n2."""
    S0, al, be, k, v = _lstate(B=1, H=1, dk=7, dv=3, K=1, seed=5)
    out = oracle.linear_state_replay(S0, al, be, k, v, np.array([1], np.int32))[0, 0]
    kk = k[0, 0, 0].astype(np.float64)
    n2 = kk @ kk                                   # 1 up to the key's float32 rounding
    a, b = float(al[0, 0, 0]), float(be[0, 0, 0])
    np.testing.assert_allclose(kk @ out, a * (1 - b * n2) * (kk @ S0[0, 0]) + b * n2 * v[0, 0, 0],
                               rtol=1e-10, atol=1e-12)


def test_linear_state_prefixes_compose_and_bad_lengths_leave_the_state():
    """Committing a steps equals committing a - 1 and then one more step from that state;
    a length of 0 or outside [0, K] leaves the state as it was."""
    S0, al, be, k, v = _lstate(B=1, H=2, K=4, seed=6)
    full = oracle.linear_state_replay(S0, al, be, k, v, np.array([3], np.int32))
    part = oracle.linear_state_replay(S0, al, be, k, v, np.array([2], np.int32))
    step = oracle.linear_state_replay(part.astype(np.float32), al[:, :, 2:], be[:, :, 2:],
                                      k[:, :, 2:], v[:, :, 2:], np.array([1], np.int32))
    np.testing.assert_allclose(step, full, rtol=1e-6, atol=1e-6)   # part rounded to float32
    for a in (0, -1, 5):
        same = oracle.linear_state_replay(S0, al, be, k, v, np.array([a], np.int32))
        np.testing.assert_array_equal(same, S0.astype(np.float64))


# --------------------------------------------------------------------------- LM-head logits

def test_lmhead_logits_exact_on_small_integers():
    """Small integers are exact in bfloat16 and their products and sums are exact in double:
    the logits equal the integer matrix product exactly."""
    g = np.random.default_rng(21)
    h = g.integers(-8, 9, (5, 33)).astype(np.float32)
    w = g.integers(-8, 9, (70, 33)).astype(np.float32)
    got = oracle.lmhead_logits(specgen.f32_to_bf16_bits(h), specgen.f32_to_bf16_bits(w))
    exact = h.astype(np.int64) @ w.astype(np.int64).T
    np.testing.assert_array_equal(got, exact.astype(np.float64))


def test_lmhead_logits_match_numpy_matmul():
    """Random bfloat16 inputs: the loops agree with numpy's float64 matmul (a different
    summation order) to double rounding."""
    g = np.random.default_rng(22)
    hb = specgen.f32_to_bf16_bits(g.normal(size=(7, 256)).astype(np.float32))
    wb = specgen.f32_to_bf16_bits((g.normal(size=(300, 256)) / 16).astype(np.float32))
    got = oracle.lmhead_logits(hb, wb)
    ref = specgen.bf16_bits_to_f32(hb).astype(np.float64) @ \
        specgen.bf16_bits_to_f32(wb).astype(np.float64).T
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    # a transposed operand or a dropped row would not match
    assert not np.allclose(got[:, :7], (specgen.bf16_bits_to_f32(hb).astype(np.float64) @
                                        specgen.bf16_bits_to_f32(hb).astype(np.float64).T)[:, :7])


def test_double_logits_and_the_logit_gap_flag():
    """Logit rows given in double give what the same values in float32 give; the gap flag
    marks exactly the rows whose argmax or top-k boundary sits within the gap window."""
    g = np.random.default_rng(23)
    B, K, V = 6, 2, 40
    t32 = g.normal(0, 2, (B, K + 1, V)).astype(np.float32)
    d32 = (t32[:, :K] + g.normal(0, 1, (B, K, V))).astype(np.float32)
    toks = draft_tokens(d32, 1.0, 5, 1.0, g.random((B, K)).astype(np.float32))
    u = g.random((B, K + 1)).astype(np.float32)
    a32 = oracle.verify_chain(t32, d32, toks, u, 1.0, 5)
    a64 = oracle.verify_chain(t32.astype(np.float64), d32.astype(np.float64), toks, u, 1.0, 5)
    for x, y in zip(a32, a64):
        np.testing.assert_array_equal(x, y)
    # greedy: row 0's argmax leads the runner-up by 5e-4, row 1's by 0.5
    tg = np.zeros((2, 2, 8), np.float64)
    tg[:, :, 3] = 1.0
    tg[0, :, 5] = 1.0 - 5e-4
    tg[1, :, 5] = 0.5
    x = np.full((2, 1), 3, np.int32)
    _, _, fl = oracle.verify_chain(tg, None, x, np.zeros((2, 2), np.float32), 0.0,
                                   windows=oracle.FP32_LOGITS)
    assert fl[0] & oracle.FLAG_GAP and not fl[1] & oracle.FLAG_GAP
    _, _, fl = oracle.verify_chain(tg, None, x, np.zeros((2, 2), np.float32), 0.0,
                                   windows=oracle.FP64)
    assert not fl.any()
