"""Shared test helpers: decoding of fixtures and a drafter that picks x_i ~ q_i.

The drafter stands in for the draft model (outside the verification step): it
draws each draft token from the transformed draft distribution with the
oracle's transform and inverse-CDF routines, so every parity input comes from
the generator or the oracle, never from the library under test.
"""
from __future__ import annotations

import math

import numpy as np

import oracle
import specgen


def f32_logits(rows):
    """Fixture rows -> float32 array; None -> -inf, "ln4"/"ln2" -> float32 logs."""
    def conv(x):
        if x is None:
            return -np.inf
        if isinstance(x, str):
            return {"ln4": math.log(4.0), "ln2": math.log(2.0)}[x]
        return float(x)
    return np.array([[conv(x) for x in r] for r in rows], dtype=np.float32)


def to_f64(logits: np.ndarray) -> np.ndarray:
    """float32 or bf16-bit logits -> float64 values."""
    if logits.dtype == np.uint16:
        return specgen.bf16_bits_to_f32(logits).astype(np.float64)
    return logits.astype(np.float64)


def draft_tokens(draft: np.ndarray, temp: float, top_k: int, top_p: float,
                 pick_uniforms: np.ndarray, chunk_rows: int = 64) -> np.ndarray:
    """x[b, i] ~ transformed q_i (temp 0: argmax of the draft logits)."""
    B, K, V = draft.shape
    flat = draft.reshape(B * K, V)
    u = None if temp == 0.0 else np.asarray(pick_uniforms, np.float32).reshape(B * K)
    out = np.empty(B * K, np.int32)
    for s in range(0, B * K, chunk_rows):
        rows = flat[s:s + chunk_rows]
        if temp == 0.0:
            out[s:s + len(rows)] = np.argmax(to_f64(rows), axis=1)
            continue
        probs, _, _, valid = oracle.transform_rows(rows, temp, top_k, top_p)
        assert valid.all()
        toks, _ = oracle.residual_sample(probs.astype(np.float32), None, u[s:s + len(rows)])
        out[s:s + len(rows)] = toks
    return out.reshape(B, K)


def chain_case(cfg: specgen.ChainConfig, B: int | None = None, greedy: bool = False):
    """Generator inputs for a chain workload plus drafter tokens.
    Returns (target, draft, tokens, uniforms, temp)."""
    target, draft = specgen.chain_logits(cfg, B)
    u = specgen.chain_uniforms(cfg, B)
    temp = 0.0 if greedy else cfg.temp
    toks = draft_tokens(draft, temp, cfg.top_k, cfg.top_p, specgen.drafter_uniforms(cfg, B))
    return target, draft, toks, u, temp


def check_chain_invariants(acc, out, toks, K, V):
    """Every round emits 1..K+1 tokens: the accepted drafts, one drawn token, then -1."""
    B = acc.shape[0]
    assert np.all((acc >= 0) & (acc <= K))
    for b in range(B):
        a = int(acc[b])
        assert np.array_equal(out[b, :a], toks[b, :a])
        assert 0 <= out[b, a] < V
        assert np.all(out[b, a + 1:] == -1)
