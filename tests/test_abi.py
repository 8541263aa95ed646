"""The C-ABI library loads, exports every declared symbol and rejects bad arguments on
the host before touching the GPU (no compute call runs here)."""
import ctypes

import pytest

import draft_token_verification_spec_b200 as sv
from draft_token_verification_spec_b200 import _build


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return sv.lib()


def test_every_declared_function_is_exported(lib):
    names = sv.header_functions()
    assert {"spec_verify_chain", "spec_verify_tree_typical", "spec_logits_to_probs",
            "spec_residual_sample", "spec_workspace_size"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings_and_kernel_counts(lib):
    assert sv.status_string(0) == "SPEC_OK"
    assert sv.status_string(-4) == "SPEC_ERR_WORKSPACE"
    assert sv.spec_kernels_per_call("spec_verify_chain") == 4
    assert sv.spec_kernels_per_call("spec_verify_tree_typical") == 3
    assert sv.spec_kernels_per_call("nope") == -1


def _ws(rows):
    up = lambda x: (x + 255) // 256 * 256
    return (256 + up(48 * rows) + up(4 * rows) + up(rows * 2048 * 4) + up(4 * rows) + up(4 * rows)
            + up(16 * rows))


def test_workspace_size(lib):
    """header, 48-byte row statistics, kept-id counts, up to 2048 kept ids per row, the list
    of rows the cluster kernel finishes, the list of refined rows and their exact
    normalisers (16 bytes each)"""
    assert sv.spec_workspace_size(0, 4, 10) == 0
    assert sv.spec_workspace_size(512, 8, 151936) == _ws(512 * 17)
    assert sv.spec_workspace_size(32, 64, 32000) == _ws(32 * 129)


P = ctypes.c_void_p


def _chain(lib, **kw):
    a = dict(t=P(16), d=P(16), dt=1, B=2, K=3, V=100, x=P(16), u=P(16), temp=1.0, k=0, p=1.0,
             acc=P(16), out=P(16), ws=P(256), wsb=1 << 20, s=None)
    a.update(kw)
    return lib.spec_verify_chain(a["t"], a["d"], a["dt"], a["B"], a["K"], a["V"], a["x"], a["u"],
                                 a["temp"], a["k"], a["p"], a["acc"], a["out"], a["ws"],
                                 a["wsb"], a["s"])


@pytest.mark.parametrize("bad", [dict(t=None), dict(x=None), dict(u=None), dict(acc=None),
                                 dict(out=None), dict(dt=7), dict(B=0), dict(K=0), dict(V=0),
                                 dict(temp=-1.0), dict(temp=float("nan")),
                                 dict(temp=float("inf")), dict(p=0.0), dict(p=float("nan")),
                                 dict(d=None)])
def test_chain_invalid_args(lib, bad):
    assert _chain(lib, **bad) == -1


def test_chain_greedy_needs_no_draft(lib):
    # greedy with a too-small workspace: argument check passes, workspace check fails
    assert _chain(lib, d=None, temp=0.0, wsb=16) == -4


@pytest.mark.parametrize("bad,code", [(dict(ws=None), -4), (dict(ws=P(258)), -4),
                                      (dict(wsb=100), -4), (dict(V=(1 << 20) + 1), -2)])
def test_chain_workspace_and_limits(lib, bad, code):
    assert _chain(lib, **bad) == code


def test_tree_invalid_args(lib):
    f = lib.spec_verify_tree_typical
    ok = [P(16), 1, 2, 8, 100, P(16), P(16), 0.09, 0.3, P(16), 8, P(16), P(256), 1 << 20, None]
    for i, v in [(0, None), (2, 0), (3, 0), (5, None), (6, None), (9, None), (10, 0),
                 (11, None), (7, float("nan")), (8, float("inf"))]:
        args = list(ok)
        args[i] = v
        assert f(*args) == -1, i
    args = list(ok)
    args[3] = 5000
    assert f(*args) == -2
    args = list(ok)
    args[13] = 10
    assert f(*args) == -4


def test_tree_greedy_invalid_args(lib):
    f = lib.spec_verify_tree_greedy
    ok = [P(16), 1, 2, 8, 100, P(16), P(16), P(16), 8, P(16), P(16), P(256), 1 << 20, None]
    for i, v in [(0, None), (1, 7), (2, 0), (3, 0), (4, 0), (5, None), (6, None), (7, None),
                 (8, 0), (9, None)]:
        args = list(ok)
        args[i] = v
        assert f(*args) == -1, i
    args = list(ok)
    args[3] = 5000
    assert f(*args) == -2
    args = list(ok)
    args[12] = 10
    assert f(*args) == -4


def test_tree_sampling_invalid_args(lib):
    f = lib.spec_verify_tree_sampling
    ok = [P(16), P(16), 1, 2, 8, 100, P(16), P(16), P(16), 1.0, 0, 1.0, P(16), 8, P(16), P(16),
          P(256), 1 << 20, None]
    for i, v in [(0, None), (1, None), (2, 7), (3, 0), (4, 0), (5, 0), (6, None), (7, None),
                 (8, None), (9, -1.0), (9, float("nan")), (11, 0.0), (12, None), (13, 0),
                 (14, None)]:
        args = list(ok)
        args[i] = v
        assert f(*args) == -1, i
    args = list(ok)
    args[1] = None
    args[9] = 0.0          # the greedy limit needs no draft logits: passes the host checks
    args[16] = None        # (and then stops at the missing workspace)
    assert f(*args) == -4
    args = list(ok)
    args[4] = 5000
    assert f(*args) == -2
    args = list(ok)
    args[17] = 10
    assert f(*args) == -4


def test_probs_and_residual_invalid_args(lib):
    assert lib.spec_logits_to_probs(None, 1, 4, 10, 1.0, 0, 1.0, P(16), None, None) == -1
    assert lib.spec_logits_to_probs(P(16), 1, 4, 10, 1.0, 0, 0.0, P(16), None, None) == -1
    assert lib.spec_logits_to_probs(P(16), 1, 4, 10, -2.0, 0, 1.0, P(16), None, None) == -1
    assert lib.spec_residual_sample(None, None, 4, 10, P(16), P(16), None) == -1
    assert lib.spec_residual_sample(P(16), None, 0, 10, P(16), P(16), None) == -1
    assert lib.spec_residual_sample(P(16), None, 4, 10, P(16), None, None) == -1


def test_noalloc_limits_on_the_host(lib):
    """The static-scratch call rejects sizes beyond its scratch before any CUDA call."""
    args = lambda B, K, V: (P(16), P(16), 1, B, K, V, P(16), P(16), 1.0, 0, 1.0, P(16), P(16), None)
    assert lib.spec_verify_chain_noalloc(*args(0, 8, 151936)) == -1
    assert lib.spec_verify_chain_noalloc(*args(4, 0, 151936)) == -1
    big = 1024  # 1024 * 17 rows need more than the 32 MiB scratch
    assert sv.spec_workspace_size(big, 8, 151936) > 32 << 20
    assert lib.spec_verify_chain_noalloc(*args(big, 8, 151936)) == -4
