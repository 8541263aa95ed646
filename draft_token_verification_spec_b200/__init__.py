"""Python binding of libspecverify (draft-token verification for speculative decoding).

Argument marshalling only: every step of verification runs in the CUDA library
(libspecverify.so, built in-tree for sm_100a). PyTorch supplies device memory and
streams. The functions carry the C ABI's names (include/specverify.h); each takes
torch CUDA tensors, allocates any output or workspace the caller did not pass, and
enqueues the work on the current CUDA stream (or `stream`). Calling any of them
without the built library raises; there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libspecverify.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "specverify.h")

SPEC_F32, SPEC_BF16 = 0, 1
SPEC_OK = 0
SPEC_ERR_INVALID_ARG, SPEC_ERR_UNSUPPORTED, SPEC_ERR_CUDA, SPEC_ERR_WORKSPACE = -1, -2, -3, -4
SPEC_ERR_DEVICE_TIMEOUT = -5
SPEC_MAX_VOCAB = 1 << 20
SPEC_MAX_TREE_NODES = 4096

_lib = None


class SpecError(RuntimeError):
    """A libspecverify call returned a non-zero spec_status."""

    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {status} ({status_string(status)})")
        self.status = status


def _declare(lib):
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sig = {
        "spec_status_string": ([I], ctypes.c_char_p),
        "spec_workspace_size": ([I, I, I], Z),
        "spec_verify_chain": ([P, P, I, I, I, I, P, P, F, I, F, P, P, P, Z, P], I),
        "spec_verify_chain_noalloc": ([P, P, I, I, I, I, P, P, F, I, F, P, P, P], I),
        "spec_verify_tree_typical": ([P, I, I, I, I, P, P, F, F, P, I, P, P, Z, P], I),
        "spec_verify_tree_greedy": ([P, I, I, I, I, P, P, P, I, P, P, P, Z, P], I),
        "spec_verify_tree_sampling": ([P, P, I, I, I, I, P, P, P, F, I, F, P, I, P, P, P, Z, P],
                                      I),
        "spec_logits_to_probs": ([P, I, I, I, F, I, F, P, P, P], I),
        "spec_residual_sample": ([P, P, I, I, P, P, P], I),
        "spec_get_device_status": ([P, P, P], I),
        "spec_linear_state_factors": ([P, P, P, P, I, I, I, I, I, P, P, P, P], I),
        "spec_lmhead_workspace_size": ([I, I, I, I, I], Z),
        "spec_verify_chain_lmhead": ([P, P, P, P, I, I, I, I, P, P, F, I, P, P, P, P, Z, P], I),
        "spec_commit_linear_state": ([P, I, I, I, I, I, P, P, P, P, P, P], I),
        "spec_set_row_kernel_events": ([P, P], None),
        "spec_kernels_per_call": ([ctypes.c_char_p], I),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res


def lib():
    """The loaded CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -c 'import __graft_entry__ as g; g.build()'`")
        l = ctypes.CDLL(LIB_PATH)
        _declare(l)
        _lib = l
    return _lib


def header_functions() -> list[str]:
    """Names of the functions declared in include/specverify.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b(spec_\w+)\s*\(", text, re.M)))


def status_string(status: int) -> str:
    return lib().spec_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != SPEC_OK:
        raise SpecError(fn, status)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SPEC_BF16
    if t.dtype == torch.float32:
        return SPEC_F32
    raise TypeError(f"logits must be bfloat16 or float32, got {t.dtype}")


def _dev(t: torch.Tensor, name: str, dtype=None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _on(device):
    """Makes `device` current for the call when it is not already (launches go to the
    tensors' device); a no-op context otherwise, so the common case costs nothing."""
    import contextlib
    if device.index is None or device.index == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(device)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def spec_workspace_size(B: int, K_or_N: int, V: int) -> int:
    return int(lib().spec_workspace_size(int(B), int(K_or_N), int(V)))


def spec_verify_chain(target_logits, draft_logits, draft_tokens, uniforms, temp, top_k=0,
                      top_p=1.0, accepted_len=None, out_tokens=None, workspace=None,
                      stream=None):
    """Chain verification. target [B,K+1,V], draft [B,K,V] (None when temp == 0),
    draft_tokens int32 [B,K], uniforms float32 [B,K+1]. Returns (accepted_len [B],
    out_tokens [B,K+1]) as int32 CUDA tensors."""
    t = _dev(target_logits, "target_logits")
    B, K1, V = t.shape
    K = K1 - 1
    d = None if draft_logits is None else _dev(draft_logits, "draft_logits", t.dtype)
    if d is not None and tuple(d.shape) != (B, K, V):
        raise ValueError("draft_logits must be [B, K, V]")
    x = _dev(draft_tokens, "draft_tokens", torch.int32)
    u = _dev(uniforms, "uniforms", torch.float32)
    if tuple(x.shape) != (B, K) or tuple(u.shape) != (B, K + 1):
        raise ValueError("draft_tokens must be [B, K] and uniforms [B, K+1]")
    if accepted_len is None:
        accepted_len = torch.empty(B, dtype=torch.int32, device=t.device)
    if out_tokens is None:
        out_tokens = torch.empty((B, K + 1), dtype=torch.int32, device=t.device)
    if workspace is None:
        workspace = torch.empty(spec_workspace_size(B, K, V), dtype=torch.uint8, device=t.device)
    with _on(t.device):
        _check("spec_verify_chain", lib().spec_verify_chain(
            _ptr(t), _ptr(d), _dtype(t), B, K, V, _ptr(x), _ptr(u), float(temp), int(top_k),
            float(top_p), _ptr(accepted_len), _ptr(out_tokens), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(stream, t.device)))
    return accepted_len, out_tokens


def spec_verify_chain_noalloc(target_logits, draft_logits, draft_tokens, uniforms, temp,
                              top_k=0, top_p=1.0, accepted_len=None, out_tokens=None,
                              stream=None):
    """spec_verify_chain with the library's static scratch instead of a workspace (calls on
    one device must not overlap). Returns (accepted_len [B], out_tokens [B,K+1])."""
    t = _dev(target_logits, "target_logits")
    B, K1, V = t.shape
    K = K1 - 1
    d = None if draft_logits is None else _dev(draft_logits, "draft_logits", t.dtype)
    if d is not None and tuple(d.shape) != (B, K, V):
        raise ValueError("draft_logits must be [B, K, V]")
    x = _dev(draft_tokens, "draft_tokens", torch.int32)
    u = _dev(uniforms, "uniforms", torch.float32)
    if tuple(x.shape) != (B, K) or tuple(u.shape) != (B, K + 1):
        raise ValueError("draft_tokens must be [B, K] and uniforms [B, K+1]")
    if accepted_len is None:
        accepted_len = torch.empty(B, dtype=torch.int32, device=t.device)
    if out_tokens is None:
        out_tokens = torch.empty((B, K + 1), dtype=torch.int32, device=t.device)
    with _on(t.device):
        _check("spec_verify_chain_noalloc", lib().spec_verify_chain_noalloc(
            _ptr(t), _ptr(d), _dtype(t), B, K, V, _ptr(x), _ptr(u), float(temp), int(top_k),
            float(top_p), _ptr(accepted_len), _ptr(out_tokens), _stream(stream, t.device)))
    return accepted_len, out_tokens


def spec_verify_tree_typical(target_logits, node_tokens, parent_idx, eps, delta,
                             path_cap=None, best_path=None, accepted_len=None, workspace=None,
                             stream=None):
    """Typical acceptance over a candidate tree. target [B,N,V], node_tokens int32 [B,N],
    parent_idx int32 [N]. Returns (best_path [B,path_cap], accepted_len [B])."""
    t = _dev(target_logits, "target_logits")
    B, N, V = t.shape
    nt = _dev(node_tokens, "node_tokens", torch.int32)
    par = _dev(parent_idx, "parent_idx", torch.int32)
    if tuple(nt.shape) != (B, N) or tuple(par.shape) != (N,):
        raise ValueError("node_tokens must be [B, N] and parent_idx [N]")
    cap = N if path_cap is None else int(path_cap)
    if best_path is None:
        best_path = torch.empty((B, cap), dtype=torch.int32, device=t.device)
    if accepted_len is None:
        accepted_len = torch.empty(B, dtype=torch.int32, device=t.device)
    if workspace is None:
        workspace = torch.empty(spec_workspace_size(B, N, V), dtype=torch.uint8, device=t.device)
    with _on(t.device):
        _check("spec_verify_tree_typical", lib().spec_verify_tree_typical(
            _ptr(t), _dtype(t), B, N, V, _ptr(nt), _ptr(par), float(eps), float(delta),
            _ptr(best_path), cap, _ptr(accepted_len), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(stream, t.device)))
    return best_path, accepted_len


def spec_verify_tree_greedy(target_logits, node_tokens, parent_idx, path_cap=None,
                            best_path=None, accepted_len=None, next_token=None, workspace=None,
                            stream=None):
    """Greedy (multi-branch) verification over a candidate tree. target [B,N,V],
    node_tokens int32 [B,N], parent_idx int32 [N]. Returns (best_path [B,path_cap],
    accepted_len [B], next_token [B])."""
    t = _dev(target_logits, "target_logits")
    B, N, V = t.shape
    nt = _dev(node_tokens, "node_tokens", torch.int32)
    par = _dev(parent_idx, "parent_idx", torch.int32)
    if tuple(nt.shape) != (B, N) or tuple(par.shape) != (N,):
        raise ValueError("node_tokens must be [B, N] and parent_idx [N]")
    cap = N if path_cap is None else int(path_cap)
    if best_path is None:
        best_path = torch.empty((B, cap), dtype=torch.int32, device=t.device)
    if accepted_len is None:
        accepted_len = torch.empty(B, dtype=torch.int32, device=t.device)
    if next_token is None:
        next_token = torch.empty(B, dtype=torch.int32, device=t.device)
    if workspace is None:
        workspace = torch.empty(spec_workspace_size(B, N, V), dtype=torch.uint8, device=t.device)
    with _on(t.device):
        _check("spec_verify_tree_greedy", lib().spec_verify_tree_greedy(
            _ptr(t), _dtype(t), B, N, V, _ptr(nt), _ptr(par), _ptr(best_path), cap,
            _ptr(accepted_len), _ptr(next_token), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(stream, t.device)))
    return best_path, accepted_len, next_token


def spec_verify_tree_sampling(target_logits, draft_logits, node_tokens, parent_idx, uniforms,
                              temp, top_k=0, top_p=1.0, path_cap=None, best_path=None,
                              accepted_len=None, next_token=None, workspace=None, stream=None):
    """Rejection sampling over a candidate tree. target and draft [B,N,V] (draft None when
    temp == 0), node_tokens int32 [B,N], parent_idx int32 [N], uniforms float32 [B,N+1].
    Returns (best_path [B,path_cap], accepted_len [B], next_token [B])."""
    t = _dev(target_logits, "target_logits")
    B, N, V = t.shape
    d = None if draft_logits is None else _dev(draft_logits, "draft_logits", t.dtype)
    if d is not None and tuple(d.shape) != (B, N, V):
        raise ValueError("draft_logits must be [B, N, V]")
    nt = _dev(node_tokens, "node_tokens", torch.int32)
    par = _dev(parent_idx, "parent_idx", torch.int32)
    u = _dev(uniforms, "uniforms", torch.float32)
    if tuple(nt.shape) != (B, N) or tuple(par.shape) != (N,) or tuple(u.shape) != (B, N + 1):
        raise ValueError("node_tokens must be [B, N], parent_idx [N] and uniforms [B, N+1]")
    cap = N if path_cap is None else int(path_cap)
    if best_path is None:
        best_path = torch.empty((B, cap), dtype=torch.int32, device=t.device)
    if accepted_len is None:
        accepted_len = torch.empty(B, dtype=torch.int32, device=t.device)
    if next_token is None:
        next_token = torch.empty(B, dtype=torch.int32, device=t.device)
    if workspace is None:
        workspace = torch.empty(spec_workspace_size(B, N, V), dtype=torch.uint8, device=t.device)
    with _on(t.device):
        _check("spec_verify_tree_sampling", lib().spec_verify_tree_sampling(
            _ptr(t), _ptr(d), _dtype(t), B, N, V, _ptr(nt), _ptr(par), _ptr(u), float(temp),
            int(top_k), float(top_p), _ptr(best_path), cap, _ptr(accepted_len), _ptr(next_token),
            _ptr(workspace), workspace.numel() * workspace.element_size(),
            _stream(stream, t.device)))
    return best_path, accepted_len, next_token


def spec_logits_to_probs(logits, temp, top_k=0, top_p=1.0, with_entropy=True, probs=None,
                         entropy=None, stream=None):
    """Transformed distribution of each row of logits [..., V]. Returns (probs float32
    [..., V], entropy float32 [...] or None)."""
    lg = _dev(logits, "logits")
    V = lg.shape[-1]
    rows = lg.numel() // V
    if probs is None:
        probs = torch.empty(lg.shape, dtype=torch.float32, device=lg.device)
    if with_entropy and entropy is None:
        entropy = torch.empty(lg.shape[:-1], dtype=torch.float32, device=lg.device)
    with _on(lg.device):
        _check("spec_logits_to_probs", lib().spec_logits_to_probs(
            _ptr(lg), _dtype(lg), rows, V, float(temp), int(top_k), float(top_p), _ptr(probs),
            _ptr(entropy), _stream(stream, lg.device)))
    return probs, entropy


def spec_residual_sample(p, q, uniforms, tokens=None, stream=None):
    """Draw per row from norm(max(0, p - q)) (q None: from p). p, q float32 [rows, V],
    uniforms float32 [rows]. Returns int32 tokens [rows]."""
    pp = _dev(p, "p", torch.float32)
    rows, V = pp.shape
    qq = None if q is None else _dev(q, "q", torch.float32)
    if qq is not None and qq.shape != pp.shape:
        raise ValueError("q must match p")
    u = _dev(uniforms, "uniforms", torch.float32)
    if tokens is None:
        tokens = torch.empty(rows, dtype=torch.int32, device=pp.device)
    with _on(pp.device):
        _check("spec_residual_sample", lib().spec_residual_sample(
            _ptr(pp), _ptr(qq), rows, V, _ptr(u), _ptr(tokens), _stream(stream, pp.device)))
    return tokens


def spec_lmhead_workspace_size(B: int, K: int, V: int, d: int, top_k: int) -> int:
    return int(lib().spec_lmhead_workspace_size(int(B), int(K), int(V), int(d), int(top_k)))


def spec_verify_chain_lmhead(target_hidden, draft_hidden, target_weight, draft_weight,
                             draft_tokens, uniforms, temp, top_k=0, logits_out=None,
                             accepted_len=None, out_tokens=None, workspace=None, stream=None):
    """Chain verification from hidden states: target_hidden bf16 [B,K+1,d], draft_hidden
    [B,K,d] (None when temp == 0), target_weight and draft_weight bf16 [V,d] (the LM heads).
    temp == 0 (greedy) or 1 <= top_k <= 64. logits_out: None, or float32 [B*(2K+1), V] to
    receive the logits as well (target rows, then draft rows). Returns (accepted_len [B],
    out_tokens [B,K+1])."""
    ht = _dev(target_hidden, "target_hidden", torch.bfloat16)
    B, K1, d = ht.shape
    K = K1 - 1
    wt = _dev(target_weight, "target_weight", torch.bfloat16)
    V = wt.shape[0]
    greedy = float(temp) == 0.0
    hd = None if draft_hidden is None else _dev(draft_hidden, "draft_hidden", torch.bfloat16)
    wd = None if draft_weight is None else _dev(draft_weight, "draft_weight", torch.bfloat16)
    if tuple(wt.shape) != (V, d) or (hd is not None and tuple(hd.shape) != (B, K, d)) or \
            (wd is not None and tuple(wd.shape) != (V, d)):
        raise ValueError("hidden [B,K+1,d] / [B,K,d], weights [V,d]")
    x = _dev(draft_tokens, "draft_tokens", torch.int32)
    u = _dev(uniforms, "uniforms", torch.float32)
    if accepted_len is None:
        accepted_len = torch.empty(B, dtype=torch.int32, device=ht.device)
    if out_tokens is None:
        out_tokens = torch.empty((B, K + 1), dtype=torch.int32, device=ht.device)
    if logits_out is not None:
        _dev(logits_out, "logits_out", torch.float32)
    if workspace is None:
        workspace = torch.empty(spec_lmhead_workspace_size(B, K, V, d, 0 if greedy else top_k),
                                dtype=torch.uint8, device=ht.device)
    with _on(ht.device):
        _check("spec_verify_chain_lmhead", lib().spec_verify_chain_lmhead(
            _ptr(ht), _ptr(hd), _ptr(wt), _ptr(wd), B, K, V, d, _ptr(x), _ptr(u), float(temp),
            int(top_k), _ptr(accepted_len), _ptr(out_tokens), _ptr(logits_out),
            _ptr(workspace), workspace.numel() * workspace.element_size(),
            _stream(stream, ht.device)))
    return accepted_len, out_tokens


def spec_linear_state_factors(alpha, beta, keys, values, w=None, u=None, gamma=None,
                              stream=None):
    """Compact factors of every prefix of a round's S steps (gated delta rule). alpha, beta
    float32 [B,H,S]; keys [B,H,S,dk]; values [B,H,S,dv]. Returns (w [B,H,S,dk], u [B,H,S,dv],
    gamma [B,H,S])."""
    al = _dev(alpha, "alpha", torch.float32)
    be = _dev(beta, "beta", torch.float32)
    k = _dev(keys, "keys", torch.float32)
    v = _dev(values, "values", torch.float32)
    B, H, S = al.shape
    dk, dv = k.shape[3], v.shape[3]
    if tuple(be.shape) != (B, H, S) or tuple(k.shape[:3]) != (B, H, S) or \
            tuple(v.shape[:3]) != (B, H, S):
        raise ValueError("alpha, beta [B,H,S], keys [B,H,S,dk], values [B,H,S,dv]")
    if w is None:
        w = torch.empty((B, H, S, dk), dtype=torch.float32, device=k.device)
    if u is None:
        u = torch.empty((B, H, S, dv), dtype=torch.float32, device=k.device)
    if gamma is None:
        gamma = torch.empty((B, H, S), dtype=torch.float32, device=k.device)
    with _on(k.device):
        _check("spec_linear_state_factors", lib().spec_linear_state_factors(
            _ptr(al), _ptr(be), _ptr(k), _ptr(v), B, H, S, dk, dv, _ptr(w), _ptr(u),
            _ptr(gamma), _stream(stream, k.device)))
    return w, u, gamma


def spec_commit_linear_state(state, keys, w, u, gamma, steps, stream=None):
    """In place: state float32 [B,H,dk,dv] becomes the state after steps[b] steps of its
    round (keys, w [B,H,S,dk]; u [B,H,S,dv]; gamma [B,H,S]; steps int32 [B])."""
    st = _dev(state, "state", torch.float32)
    B, H, dk, dv = st.shape
    k = _dev(keys, "keys", torch.float32)
    S = k.shape[2]
    ww = _dev(w, "w", torch.float32)
    uu = _dev(u, "u", torch.float32)
    g = _dev(gamma, "gamma", torch.float32)
    n = _dev(steps, "steps", torch.int32)
    if tuple(k.shape) != (B, H, S, dk) or tuple(ww.shape) != (B, H, S, dk) or \
            tuple(uu.shape) != (B, H, S, dv) or tuple(g.shape) != (B, H, S) or \
            tuple(n.shape) != (B,):
        raise ValueError("keys, w [B,H,S,dk]; u [B,H,S,dv]; gamma [B,H,S]; steps [B]")
    with _on(st.device):
        _check("spec_commit_linear_state", lib().spec_commit_linear_state(
            _ptr(st), B, H, dk, dv, S, _ptr(k), _ptr(ww), _ptr(uu), _ptr(g), _ptr(n),
            _stream(stream, st.device)))
    return st


def spec_get_device_status(workspace, stream=None) -> int:
    out = ctypes.c_int32(0)
    with _on(workspace.device):
        _check("spec_get_device_status", lib().spec_get_device_status(
            _ptr(workspace), ctypes.byref(out), _stream(stream, workspace.device)))
    return int(out.value)


def spec_set_row_kernel_events(before=None, after=None) -> None:
    """Record torch.cuda.Event `before`/`after` around every verify call's row kernel."""
    lib().spec_set_row_kernel_events(
        None if before is None else ctypes.c_void_p(before.cuda_event),
        None if after is None else ctypes.c_void_p(after.cuda_event))


def spec_kernels_per_call(entry_point: str) -> int:
    return int(lib().spec_kernels_per_call(entry_point.encode()))
