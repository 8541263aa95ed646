"""Oracle for draft-token verification (speculative decoding).

TEST INFRASTRUCTURE ONLY: a plain, slow, double-precision CPU statement of the
verification step, written from the pages' prose (see ``oracle.cpp`` for the
sources and readings). Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it. It shares no code with the
CUDA library and does not import it.

Every function takes numpy arrays and returns numpy arrays. Logits are either
float32 arrays or bfloat16 bit patterns held in uint16 arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

FLAG_RATIO = 1
FLAG_CDF = 2
FLAG_TOPP = 4
FLAG_TREE = 8
DIAG_Q_ZERO = 16
FLAG_GAP = 32
PARITY_FLAGS = FLAG_RATIO | FLAG_CDF | FLAG_TOPP | FLAG_TREE | FLAG_GAP

# Widths of the precision windows behind the flags (ratio, cdf_rel, cdf_abs, topp, tree, gap):
# a flag marks a decision that arithmetic of lower precision than the oracle's may take
# the other way. They change only the flags, never a result.
#   CRITERION: the widest the acceptance criterion allows: |u - r| < 1e-5, a CDF edge
#              within 1e-6 * S of w * S (and 1e-6 on a top-p boundary, relative 1e-5 on a
#              tree threshold, this build's extensions of the same idea).
#   FP64:      for a verifier that takes these decisions in double precision: double
#              rounding over up to 2^20 terms moves a sum by at most ~1.2e-10 of it.
#   FP32_LOGITS: for a verifier that computes the logits itself with fp32 accumulation
#              (the LM-head product): a logit gap under 1e-3 behind an argmax or top-k
#              decision, and ratios and CDF edges within 1e-4 (relative), are flagged.
CRITERION = (1e-5, 1e-6, 0.0, 1e-6, 1e-5, 0.0)
FP64 = (1e-9, 1e-9, 1e-10, 1e-10, 1e-9, 0.0)
FP32_LOGITS = (1e-4, 1e-4, 0.0, 1e-4, 1e-5, 1e-3)


def build(force: bool = False) -> str:
    """Compile the oracle into liboracle.so (plain g++, no GPU)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-shared", "-fPIC",
               "-pthread", _SRC, "-o", _LIB + ".tmp"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        _lib.oracle_transform_rows.argtypes = [P, I, I, I, D, I, D, P, P, P, P, I]
        _lib.oracle_verify_chain.argtypes = [P, P, I, I, I, I, P, P, D, I, D, P, P, P, I, P]
        _lib.oracle_verify_chain_f64u.argtypes = [P, P, I, I, I, I, P, P, D, I, D, P, P, P, I, P]
        _lib.oracle_verify_tree_typical.argtypes = [P, I, I, I, I, P, P, D, D, D, P, I, P, P, I,
                                                    P]
        _lib.oracle_residual_sample.argtypes = [P, P, I, I, P, P, P, I, P]
        _lib.oracle_verify_tree_greedy.argtypes = [P, I, I, I, I, P, P, P, I, P, P, I]
        _lib.oracle_verify_tree_sampling.argtypes = [P, P, I, I, I, I, P, P, P, D, I, D, P, I, P,
                                                     P, P, I, P]
        _lib.oracle_verify_tree_sampling_f64u.argtypes = \
            _lib.oracle_verify_tree_sampling.argtypes
        _lib.oracle_verify_tree_sampling.restype = I
        _lib.oracle_verify_tree_sampling_f64u.restype = I
        _lib.oracle_linear_state_replay.argtypes = [P, I, I, I, I, I, P, P, P, P, P, P, I]
        _lib.oracle_lmhead_logits.argtypes = [P, P, I, I, I, P, I]
        _lib.oracle_lmhead_logits.restype = I
        _lib.oracle_linear_state_replay.restype = I
        for f in (_lib.oracle_transform_rows, _lib.oracle_verify_chain,
                  _lib.oracle_verify_chain_f64u, _lib.oracle_verify_tree_greedy,
                  _lib.oracle_verify_tree_typical, _lib.oracle_residual_sample):
            f.restype = I
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(logits: np.ndarray) -> int:
    if logits.dtype == np.float32:
        return 0
    if logits.dtype == np.uint16:
        return 1
    if logits.dtype == np.float64:
        return 2
    raise TypeError("logits must be float32, float64 or uint16 (bfloat16 bit patterns)")


def _threads(threads):
    return (os.cpu_count() or 1) if threads is None else int(threads)


def _win(windows):
    w = np.ascontiguousarray(CRITERION if windows is None else windows, dtype=np.float64)
    assert w.shape == (6,)
    return w


def transform_rows(logits, temp, top_k=0, top_p=1.0, threads=None):
    """Rows of logits [..., V] -> (probs float64 [..., V], entropy, topp_margin, valid)."""
    logits = np.ascontiguousarray(logits)
    V = logits.shape[-1]
    rows = logits.size // V
    probs = np.zeros((rows, V), np.float64)
    ent = np.zeros(rows, np.float64)
    marg = np.zeros(rows, np.float64)
    valid = np.zeros(rows, np.int32)
    rc = _load().oracle_transform_rows(_ptr(logits), _dtype_code(logits), rows, V, float(temp),
                                       int(top_k), float(top_p), _ptr(probs), _ptr(ent),
                                       _ptr(marg), _ptr(valid), _threads(threads))
    if rc != 0:
        raise ValueError("oracle_transform_rows rejected its arguments")
    shp = logits.shape[:-1]
    return probs.reshape(*shp, V), ent.reshape(shp), marg.reshape(shp), valid.reshape(shp)


def verify_chain(target, draft, draft_tokens, uniforms, temp, top_k=0, top_p=1.0, threads=None,
                 windows=None):
    """Chain verification. target [B,K+1,V], draft [B,K,V] (unused when temp == 0),
    draft_tokens int32 [B,K], uniforms float32 [B,K+1] (float64 uniforms select the
    double-precision entry, used by the exact-integration tests).
    windows: the flag windows (CRITERION by default, see above).
    Returns (accepted_len int32 [B], out_tokens int32 [B,K+1], flags int32 [B])."""
    target = np.ascontiguousarray(target)
    B, K1, V = target.shape
    K = K1 - 1
    if draft is not None:
        draft = np.ascontiguousarray(draft)
        assert draft.shape == (B, K, V) and draft.dtype == target.dtype
    toks = np.ascontiguousarray(draft_tokens, dtype=np.int32).reshape(B, K)
    uniforms = np.asarray(uniforms)
    wide = uniforms.dtype == np.float64  # double uniforms: exact-integration pins only
    u = np.ascontiguousarray(uniforms, dtype=np.float64 if wide else np.float32).reshape(B, K + 1)
    acc = np.zeros(B, np.int32)
    out = np.zeros((B, K + 1), np.int32)
    flags = np.zeros(B, np.int32)
    w = _win(windows)
    fn = _load().oracle_verify_chain_f64u if wide else _load().oracle_verify_chain
    rc = fn(_ptr(target), _ptr(draft), _dtype_code(target), B, K, V,
            _ptr(toks), _ptr(u), float(temp), int(top_k), float(top_p),
            _ptr(acc), _ptr(out), _ptr(flags), _threads(threads), _ptr(w))
    if rc != 0:
        raise ValueError("oracle_verify_chain rejected its arguments")
    return acc, out, flags


def verify_tree_typical(target, node_tokens, parent_idx, eps, delta, temp=1.0, path_cap=None,
                        threads=None, windows=None):
    """Typical acceptance over a candidate tree. target [B,N,V], node_tokens int32 [B,N],
    parent_idx int32 [N]. Returns (best_path int32 [B,path_cap], accepted_len [B], flags [B])."""
    target = np.ascontiguousarray(target)
    B, N, V = target.shape
    cap = N if path_cap is None else int(path_cap)
    toks = np.ascontiguousarray(node_tokens, dtype=np.int32).reshape(B, N)
    par = np.ascontiguousarray(parent_idx, dtype=np.int32).reshape(N)
    path = np.zeros((B, cap), np.int32)
    acc = np.zeros(B, np.int32)
    flags = np.zeros(B, np.int32)
    rc = _load().oracle_verify_tree_typical(_ptr(target), _dtype_code(target), B, N, V,
                                            _ptr(toks), _ptr(par), float(eps), float(delta),
                                            float(temp), _ptr(path), cap, _ptr(acc),
                                            _ptr(flags), _threads(threads), _ptr(_win(windows)))
    if rc != 0:
        raise ValueError("oracle_verify_tree_typical rejected its arguments")
    return path, acc, flags


def verify_tree_greedy(target, node_tokens, parent_idx, path_cap=None, threads=None):
    """Greedy verification over a candidate tree. target [B,N,V], node_tokens int32 [B,N],
    parent_idx int32 [N]. Returns (best_path int32 [B,path_cap], accepted_len [B],
    next_token [B])."""
    target = np.ascontiguousarray(target)
    B, N, V = target.shape
    cap = N if path_cap is None else int(path_cap)
    toks = np.ascontiguousarray(node_tokens, dtype=np.int32).reshape(B, N)
    par = np.ascontiguousarray(parent_idx, dtype=np.int32).reshape(N)
    path = np.zeros((B, cap), np.int32)
    acc = np.zeros(B, np.int32)
    nxt = np.zeros(B, np.int32)
    rc = _load().oracle_verify_tree_greedy(_ptr(target), _dtype_code(target), B, N, V,
                                           _ptr(toks), _ptr(par), _ptr(path), cap, _ptr(acc),
                                           _ptr(nxt), _threads(threads))
    if rc != 0:
        raise ValueError("oracle_verify_tree_greedy rejected its arguments")
    return path, acc, nxt


def verify_tree_sampling(target, draft, node_tokens, parent_idx, uniforms, temp, top_k=0,
                         top_p=1.0, path_cap=None, threads=None, windows=None):
    """Rejection sampling over a candidate tree. target and draft [B,N,V] (draft unused
    when temp == 0), node_tokens int32 [B,N], parent_idx int32 [N], uniforms [B,N+1]
    (float64 uniforms select the double-precision entry). Returns (best_path [B,path_cap],
    accepted_len [B], next_token [B], flags [B])."""
    target = np.ascontiguousarray(target)
    B, N, V = target.shape
    if draft is not None:
        draft = np.ascontiguousarray(draft)
        assert draft.shape == target.shape and draft.dtype == target.dtype
    cap = N if path_cap is None else int(path_cap)
    toks = np.ascontiguousarray(node_tokens, dtype=np.int32).reshape(B, N)
    par = np.ascontiguousarray(parent_idx, dtype=np.int32).reshape(N)
    uniforms = np.asarray(uniforms)
    wide = uniforms.dtype == np.float64
    u = np.ascontiguousarray(uniforms, dtype=np.float64 if wide else np.float32).reshape(B, N + 1)
    path = np.zeros((B, cap), np.int32)
    acc = np.zeros(B, np.int32)
    nxt = np.zeros(B, np.int32)
    flags = np.zeros(B, np.int32)
    fn = _load().oracle_verify_tree_sampling_f64u if wide else _load().oracle_verify_tree_sampling
    rc = fn(_ptr(target), _ptr(draft), _dtype_code(target), B, N, V, _ptr(toks), _ptr(par),
            _ptr(u), float(temp), int(top_k), float(top_p), _ptr(path), cap, _ptr(acc),
            _ptr(nxt), _ptr(flags), _threads(threads), _ptr(_win(windows)))
    if rc != 0:
        raise ValueError("oracle_verify_tree_sampling rejected its arguments")
    return path, acc, nxt, flags


def residual_sample(p, q, uniforms, threads=None, windows=None):
    """Inverse-CDF draw per row from norm(max(0, p - q)) (q None: from p).
    p, q float32 [rows, V]; uniforms float32 [rows]. Returns (tokens int32, flags int32)."""
    p = np.ascontiguousarray(p, dtype=np.float32)
    rows, V = p.shape
    if q is not None:
        q = np.ascontiguousarray(q, dtype=np.float32)
        assert q.shape == p.shape
    u = np.ascontiguousarray(uniforms, dtype=np.float32).reshape(rows)
    toks = np.zeros(rows, np.int32)
    flags = np.zeros(rows, np.int32)
    rc = _load().oracle_residual_sample(_ptr(p), _ptr(q), rows, V, _ptr(u), _ptr(toks),
                                        _ptr(flags), _threads(threads), _ptr(_win(windows)))
    if rc != 0:
        raise ValueError("oracle_residual_sample rejected its arguments")
    return toks, flags


def linear_state_replay(state0, alpha, beta, keys, values, steps, threads=None):
    """Linear-attention state after each sequence's accepted prefix, replayed step by step
    (gated delta rule S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T).
    state0 float32 [B,H,dk,dv]; alpha, beta [B,H,K]; keys [B,H,K,dk]; values [B,H,K,dv];
    steps int32 [B] (outside [0, K]: unchanged). Returns float64 [B,H,dk,dv]."""
    state0 = np.ascontiguousarray(state0, np.float32)
    B, H, dk, dv = state0.shape
    alpha = np.ascontiguousarray(alpha, np.float32)
    K = alpha.shape[2]
    beta = np.ascontiguousarray(beta, np.float32)
    keys = np.ascontiguousarray(keys, np.float32)
    values = np.ascontiguousarray(values, np.float32)
    steps = np.ascontiguousarray(steps, np.int32)
    assert alpha.shape == beta.shape == (B, H, K)
    assert keys.shape == (B, H, K, dk) and values.shape == (B, H, K, dv) and steps.shape == (B,)
    out = np.zeros((B, H, dk, dv), np.float64)
    rc = _load().oracle_linear_state_replay(_ptr(state0), B, H, dk, dv, K, _ptr(alpha),
                                            _ptr(beta), _ptr(keys), _ptr(values), _ptr(steps),
                                            _ptr(out), _threads(threads))
    if rc != 0:
        raise ValueError("oracle_linear_state_replay rejected its arguments")
    return out


def lmhead_logits(hidden, weight, threads=None):
    """logits [rows, V] float64 = hidden [rows, d] @ weight[V, d]^T, both bfloat16 bit
    patterns (uint16), summed in double."""
    hidden = np.ascontiguousarray(hidden, np.uint16)
    weight = np.ascontiguousarray(weight, np.uint16)
    rows, d = hidden.shape
    V = weight.shape[0]
    assert weight.shape == (V, d)
    out = np.zeros((rows, V), np.float64)
    rc = _load().oracle_lmhead_logits(_ptr(hidden), _ptr(weight), rows, V, d, _ptr(out),
                                      _threads(threads))
    if rc != 0:
        raise ValueError("oracle_lmhead_logits rejected its arguments")
    return out
