"""Seeded synthetic inputs for draft-token verification.

This module only draws numbers: logits with the shapes, value distributions
and structure of the five verification workloads, uniforms, MEDUSA-style
candidate trees, and the recurrent state and per-step data of a linear-attention
target. It holds none of the verification arithmetic (no softmax,
no transform, no acceptance rule), and both the CUDA library's tests/bench and
the oracle's tests consume the same bytes from it.

Randomness: numpy's Philox-4x32 counter-based generator (Salmon et al., 2011),
one independent key per (seed, stream). Rows are drawn in batch order, so the
first B' batch rows of a size-B instance equal the size-B' instance.
bfloat16 values are rounded from float32 with round-to-nearest-even and are
returned as raw uint16 bit patterns.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# Independent streams (see module docstring).
S_TARGET, S_DRAFT, S_BOOST, S_UNIFORM, S_DRAFTPICK, S_HEADS, S_TREE = range(7)
S_STATE, S_KEYS, S_VALUES, S_GATES, S_ACCEPT = range(7, 12)


def rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=(int(seed) << 8) | int(stream)))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest even (inputs are finite)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(
        np.float32)


def dyadic_uniforms(g: np.random.Generator, shape) -> np.ndarray:
    """Uniforms k * 2^-24, k in [0, 2^24): exact in float32 and float64, in [0, 1)."""
    k = g.integers(0, 1 << 24, size=shape, dtype=np.int64)
    return (k.astype(np.float64) * 2.0 ** -24).astype(np.float32)


@dataclass(frozen=True)
class ChainConfig:
    name: str
    B: int
    K: int
    V: int
    dtype: str            # "f32" or "bf16"
    sigma: float          # target logit noise
    zipf: float           # Zipf log-prior exponent (0: none)
    boost: float          # +boost on one uniformly chosen token per target row (0: none)
    draft_sigma: float    # draft = target + N(0, draft_sigma^2)
    temp: float
    top_k: int = 0
    top_p: float = 1.0
    seed: int = 0


@dataclass(frozen=True)
class TreeConfig:
    name: str
    B: int
    V: int
    heads: tuple
    N: int
    sigma: float
    eps: float
    delta: float
    dtype: str = "bf16"
    seed: int = 3
    coverage_boost: float = 0.0   # +boost on each node's rank-0 child token (coverage variant)


# The five verification workloads (chain: 1, 2, 3, 5; tree: 4). Seeds 0..4.
CFG1 = ChainConfig("chain_B1_K4_V1000_f32_T1", 1, 4, 1000, "f32", 2.0, 0.0, 0.0, 0.5, 1.0,
                   seed=0)
CFG2 = ChainConfig("chain_B64_K5_V32000_bf16_T0.7_zipf1.1", 64, 5, 32000, "bf16", 3.0, 1.1, 0.0,
                   1.0, 0.7, seed=1)
CFG3 = ChainConfig("chain_B256_K7_V128256_bf16_T1_topp0.9", 256, 7, 128256, "bf16", 4.0, 0.0,
                   8.0, 1.5, 1.0, top_p=0.9, seed=2)
CFG4 = TreeConfig("tree_B32_N64_V32000_bf16_typical", 32, 32000, (4, 3, 2, 2), 64, 3.0, 0.09,
                  0.3, seed=3)
CFG5 = ChainConfig("chain_B512_K8_V151936_bf16_T0.8_topk50_zipf1.2", 512, 8, 151936, "bf16",
                   4.0, 1.2, 0.0, 2.0, 0.8, top_k=50, seed=4)
CHAIN_CONFIGS = {1: CFG1, 2: CFG2, 3: CFG3, 5: CFG5}


def _emit(x: np.ndarray, dtype: str) -> np.ndarray:
    return f32_to_bf16_bits(x) if dtype == "bf16" else x.astype(np.float32)


def chain_logits(cfg: ChainConfig, B: int | None = None):
    """Target logits [B, K+1, V] and draft logits [B, K, V] (float32, or bf16 bits in uint16).

    target = sigma * N(0,1) - zipf * ln(v+1) (+ boost on one uniform token per row);
    draft  = target + draft_sigma * N(0,1), both rounded independently to the storage type.
    """
    B = cfg.B if B is None else int(B)
    K, V = cfg.K, cfg.V
    gt, gd, gb = rng(cfg.seed, S_TARGET), rng(cfg.seed, S_DRAFT), rng(cfg.seed, S_BOOST)
    prior = (-cfg.zipf * np.log1p(np.arange(V, dtype=np.float64))).astype(np.float32) \
        if cfg.zipf else None
    st = np.uint16 if cfg.dtype == "bf16" else np.float32
    target = np.empty((B, K + 1, V), st)
    draft = np.empty((B, K, V), st)
    for b in range(B):
        t = gt.standard_normal((K + 1, V), dtype=np.float32) * np.float32(cfg.sigma)
        if prior is not None:
            t += prior
        if cfg.boost:
            idx = gb.integers(0, V, size=K + 1)
            t[np.arange(K + 1), idx] += np.float32(cfg.boost)
        d = t[:K] + gd.standard_normal((K, V), dtype=np.float32) * np.float32(cfg.draft_sigma)
        target[b] = _emit(t, cfg.dtype)
        draft[b] = _emit(d, cfg.dtype)
    return target, draft


def chain_uniforms(cfg: ChainConfig, B: int | None = None) -> np.ndarray:
    """uniforms [B, K+1]: u[:K] for the accept tests, u[K] for the resample/bonus draw."""
    B = cfg.B if B is None else int(B)
    return dyadic_uniforms(rng(cfg.seed, S_UNIFORM), (B, cfg.K + 1))


def drafter_uniforms(cfg: ChainConfig, B: int | None = None) -> np.ndarray:
    """uniforms [B, K] a drafter uses to pick its tokens x_i ~ q_i."""
    B = cfg.B if B is None else int(B)
    return dyadic_uniforms(rng(cfg.seed, S_DRAFTPICK), (B, cfg.K))


def tree_structure(heads=(4, 3, 2, 2), N: int | None = None):
    """Cartesian-product candidate tree of per-head top-s_d predictions, in BFS order with
    lexicographic rank order, truncated to N nodes (including the root).

    Returns (parent_idx int32 [N], depth int32 [N], rank int32 [N]) where rank is the node's
    rank among its head's top-s_d predictions (0 for the root)."""
    levels = [[()]]
    for s in heads:
        levels.append([p + (r,) for p in levels[-1] for r in range(s)])
    nodes = [n for lvl in levels for n in lvl]
    if N is not None:
        nodes = nodes[:N]
    index = {n: i for i, n in enumerate(nodes)}
    parent = np.array([-1] + [index[n[:-1]] for n in nodes[1:]], np.int32)
    depth = np.array([len(n) for n in nodes], np.int32)
    rank = np.array([n[-1] if n else 0 for n in nodes], np.int32)
    return parent, depth, rank


def tree_inputs(cfg: TreeConfig, B: int | None = None):
    """Node logits [B, N, V], node tokens [B, N] and parent_idx [N] for typical acceptance.

    Per batch row, head d's top-s_d tokens are the top-s_d entries of an independent
    N(0, sigma^2) head-logit vector; a depth-d node with rank r carries head d's rank-r token.
    Node logits are iid N(0, sigma^2); with coverage_boost > 0, each node's row gets
    +coverage_boost on the token of its rank-0 child (so deep paths get accepted)."""
    B = cfg.B if B is None else int(B)
    parent, depth, rank = tree_structure(cfg.heads, cfg.N)
    N, V, D = cfg.N, cfg.V, len(cfg.heads)
    gh, gl = rng(cfg.seed, S_HEADS), rng(cfg.seed, S_TARGET)
    head_tok = np.empty((B, D + 1, max(cfg.heads)), np.int32)
    for b in range(B):
        for d in range(D + 1):
            h = gh.standard_normal(V, dtype=np.float32)
            s = cfg.heads[d - 1] if d >= 1 else 1
            order = np.lexsort((np.arange(V), -h))  # descending value, lower id first
            head_tok[b, d, :s] = order[:s]
    tokens = np.ascontiguousarray(head_tok[:, depth, rank], dtype=np.int32)
    st = np.uint16 if cfg.dtype == "bf16" else np.float32
    logits = np.empty((B, N, V), st)
    child0 = {int(parent[c]): c for c in range(N - 1, 0, -1) if rank[c] == 0}
    for b in range(B):
        x = gl.standard_normal((N, V), dtype=np.float32) * np.float32(cfg.sigma)
        if cfg.coverage_boost:
            for n, c in child0.items():
                x[n, tokens[b, c]] += np.float32(cfg.coverage_boost)
        logits[b] = _emit(x, cfg.dtype)
    return logits, tokens, parent


@dataclass(frozen=True)
class LinearStateConfig:
    """A linear-attention target's recurrent state, per sequence and head, and the per-step
    data of one verified round: the previous round's emitted token (its update was deferred)
    plus K drafts, so K + 1 steps. A sequence whose first a drafts were accepted commits
    a + 1 steps."""
    name: str
    B: int
    H: int
    dk: int
    dv: int
    K: int                 # drafts; the round holds K + 1 steps
    accept: float          # per-draft acceptance probability (leading run of successes)
    alpha_lo: float = 0.9  # gates alpha ~ U(alpha_lo, 1)
    seed: int = 5


# Gated-delta-rule state of a 1.3B-parameter class model: 16 heads, 128-wide keys, 256-wide
# values, fp32 state (128 KiB per head); 512 sequences with 8 drafts each, acceptance 0.75.
LSTATE = LinearStateConfig("lstate_B512_H16_dk128_dv256_K8_f32", 512, 16, 128, 256, 8, 0.75)


def linear_state_inputs(cfg: LinearStateConfig, B: int | None = None):
    """state0 [B,H,dk,dv] float32 ~ N(0, 1); keys [B,H,K+1,dk] unit vectors (normalised
    N(0, I)); values [B,H,K+1,dv] ~ N(0, 1); alpha ~ U(alpha_lo, 1) and beta ~ U(0, 1)
    [B,H,K+1]; steps [B] int32 = 1 + the number of leading accepted drafts (each accepted
    with probability cfg.accept)."""
    B = cfg.B if B is None else int(B)
    H, dk, dv, S = cfg.H, cfg.dk, cfg.dv, cfg.K + 1
    gs, gk, gv, gg, ga = (rng(cfg.seed, x) for x in (S_STATE, S_KEYS, S_VALUES, S_GATES, S_ACCEPT))
    state = np.empty((B, H, dk, dv), np.float32)
    keys = np.empty((B, H, S, dk), np.float32)
    values = np.empty((B, H, S, dv), np.float32)
    for b in range(B):
        state[b] = gs.standard_normal((H, dk, dv), dtype=np.float32)
        k = gk.standard_normal((H, S, dk), dtype=np.float32)
        keys[b] = k / np.linalg.norm(k, axis=2, keepdims=True)
        values[b] = gv.standard_normal((H, S, dv), dtype=np.float32)
    alpha = gg.uniform(cfg.alpha_lo, 1.0, (B, H, S)).astype(np.float32)
    beta = gg.uniform(0.0, 1.0, (B, H, S)).astype(np.float32)
    ok = ga.random((B, cfg.K)) < cfg.accept
    lead = np.where(ok.all(axis=1), cfg.K, np.argmin(ok, axis=1))
    steps = (1 + lead).astype(np.int32)
    return state, alpha, beta, keys, values, steps


@dataclass(frozen=True)
class LmHeadConfig:
    """Hidden states and output embeddings of a target and a draft model: the inputs of the
    scoring forward's last matrix product. Hidden states ~ N(0, 1); target embeddings
    ~ N(0, (sigma / sqrt(d))^2), so target logits are ~ N(0, sigma^2); the draft model's
    hidden states and embeddings are the target's plus independent noise (scale h_noise,
    w_noise relative to each), so its logits follow the target's."""
    name: str
    B: int
    K: int
    V: int
    d: int
    sigma: float
    h_noise: float
    w_noise: float
    temp: float
    top_k: int
    seed: int = 6


LMHEAD = LmHeadConfig("lmhead_B512_K8_V151936_d4096_bf16_T0.8_topk50", 512, 8, 151936, 4096,
                      4.0, 0.5, 0.5, 0.8, 50)


def lmhead_inputs(cfg: LmHeadConfig, B: int | None = None, V: int | None = None):
    """(target_hidden [B, K+1, d], draft_hidden [B, K, d], target_weight [V, d],
    draft_weight [V, d]) as bfloat16 bit patterns."""
    B = cfg.B if B is None else int(B)
    V = cfg.V if V is None else int(V)
    K, d = cfg.K, cfg.d
    gh, gw, gn = rng(cfg.seed, S_STATE), rng(cfg.seed, S_KEYS), rng(cfg.seed, S_VALUES)
    ws = np.float32(cfg.sigma / np.sqrt(d))
    wt = np.empty((V, d), np.uint16)
    wd = np.empty((V, d), np.uint16)
    for v0 in range(0, V, 4096):
        n = min(4096, V - v0)
        w = gw.standard_normal((n, d), dtype=np.float32) * ws
        wt[v0:v0 + n] = f32_to_bf16_bits(w)
        wd[v0:v0 + n] = f32_to_bf16_bits(
            w + gn.standard_normal((n, d), dtype=np.float32) * (ws * np.float32(cfg.w_noise)))
    ht = np.empty((B, K + 1, d), np.uint16)
    hd = np.empty((B, K, d), np.uint16)
    for b in range(B):
        h = gh.standard_normal((K + 1, d), dtype=np.float32)
        ht[b] = f32_to_bf16_bits(h)
        hd[b] = f32_to_bf16_bits(
            h[:K] + gh.standard_normal((K, d), dtype=np.float32) * np.float32(cfg.h_noise))
    return ht, hd, wt, wd
