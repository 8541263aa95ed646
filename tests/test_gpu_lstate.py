"""GPU parity of the linear-attention state commit (compact factors applied to the state)
against the oracle's step-by-step replay of the gated delta rule, through the C ABI.

Tolerance: the library works in float32. Each committed entry is
G_a (S_0 + sum_t k_t (u_t - S_0^T w_t)): sums of at most dk + S products of O(1) terms, with
the values scaled by 1 / G_t (G_t >= 0.9^S here); float32 rounding keeps every entry within
1e-5 of the oracle's double result, relative to the state's scale (|S| ~ 1), which the
tests assert as |gpu - oracle| <= 1e-5 * (1 + |oracle|) (and 3e-5 for 32 steps)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import draft_token_verification_spec_b200 as sv
import oracle
import specgen

pytestmark = pytest.mark.gpu


def _run(state, alpha, beta, keys, values, steps):
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    w, u, g = sv.spec_linear_state_factors(d(alpha), d(beta), d(keys), d(values))
    st = d(state)
    sv.spec_commit_linear_state(st, d(keys), w, u, g, d(steps))
    torch.cuda.synchronize()
    return st.cpu().numpy()


def _check(gpu, ref, tol=1e-5):
    err = np.abs(gpu.astype(np.float64) - ref) / (1.0 + np.abs(ref))
    assert err.max() <= tol, err.max()


@pytest.mark.parametrize("dk,dv,S", [(32, 48, 3), (64, 64, 5), (128, 256, 9), (256, 100, 4),
                                     (128, 4, 32), (64, 2056, 9)])
def test_commit_matches_replay(dk, dv, S):
    cfg = specgen.LinearStateConfig("t", 6, 3, dk, dv, S - 1, 0.75, seed=dk + dv + S)
    state, alpha, beta, keys, values, steps = specgen.linear_state_inputs(cfg)
    steps[0], steps[1] = 0, S          # nothing to commit, and every step
    ref = oracle.linear_state_replay(state, alpha, beta, keys, values, steps)
    _check(_run(state, alpha, beta, keys, values, steps), ref, 3e-5 if S > 16 else 1e-5)


def test_commit_leaves_untouched_sequences_bit_identical():
    """steps = 0 or outside [0, S]: the state is neither read nor written."""
    cfg = specgen.LinearStateConfig("t", 4, 2, 64, 64, 4, 0.75, seed=11)
    state, alpha, beta, keys, values, steps = specgen.linear_state_inputs(cfg)
    steps[:] = [0, -1, 6, 2]
    out = _run(state, alpha, beta, keys, values, steps)
    np.testing.assert_array_equal(out[:3], state[:3])
    ref = oracle.linear_state_replay(state, alpha, beta, keys, values, steps)
    _check(out, ref)


def test_commit_workload_full_size_sampled_sequences():
    """The 512-sequence, 16-head, 128 x 256 state workload (1 GiB of fp32 state) in the
    bench's launch shape; the oracle replays 24 sequences spread over the batch."""
    cfg = specgen.LSTATE
    state, alpha, beta, keys, values, steps = specgen.linear_state_inputs(cfg)
    out = _run(state, alpha, beta, keys, values, steps)
    rows = np.unique(np.linspace(0, cfg.B - 1, 24).astype(int))
    ref = oracle.linear_state_replay(state[rows], alpha[rows], beta[rows], keys[rows],
                                     values[rows], steps[rows])
    _check(out[rows], ref)


def test_commit_rejects_unsupported_shapes():
    t = torch.zeros((1, 1, 48, 8), dtype=torch.float32, device="cuda")
    k = torch.zeros((1, 1, 2, 48), dtype=torch.float32, device="cuda")
    u = torch.zeros((1, 1, 2, 8), dtype=torch.float32, device="cuda")
    g = torch.ones((1, 1, 2), dtype=torch.float32, device="cuda")
    n = torch.ones(1, dtype=torch.int32, device="cuda")
    with pytest.raises(sv.SpecError) as e:
        sv.spec_commit_linear_state(t, k, k, u, g, n)   # dk = 48 is not a supported width
    assert e.value.status == sv.SPEC_ERR_UNSUPPORTED
