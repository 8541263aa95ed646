"""GPU checks of verification from hidden states (the LM-head product on the tensor cores with
the verification statistics in its epilogue), through the C ABI.

The oracle computes the logits in double; the library accumulates bf16 products in fp32 on
the tensor cores, so its logits differ slightly, and an argmax or top-k decision whose logit
gap is that small can go either way. The checks are therefore:
  1. the library's logits (returned for checking) against the oracle's double product,
     elementwise: |gpu - oracle| <= 1e-3 + 1e-4 |oracle| (fp32 accumulation of d = 4096 bf16
     products moves a logit of size ~4 by ~1e-5; the bound leaves a wide margin);
  2. the fused decisions against the library's unfused verification of those same logits,
     bit for bit on every row (that path is itself checked against the oracle elsewhere):
     the epilogue's top-k, the merge and the list-based finisher change nothing;
  3. end to end against the oracle's verification of its double logits, identical except on
     rows the oracle flags with the FP32_LOGITS windows (a logit gap under 1e-3 behind an
     argmax or top-k decision; a ratio or CDF edge within 1e-4)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import draft_token_verification_spec_b200 as sv
import oracle
import specgen

pytestmark = pytest.mark.gpu


def _bf(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def _case(B, V, d, K=3, seed=6, temp=0.8, top_k=20):
    cfg = specgen.LmHeadConfig("t", B, K, V, d, 4.0, 0.5, 0.5, temp, top_k, seed=seed)
    ht, hd, wt, wd = specgen.lmhead_inputs(cfg)
    return cfg, ht, hd, wt, wd


def _oracle_logits(ht, hd, wt, wd):
    B, K1, d = ht.shape
    K = K1 - 1
    lt = oracle.lmhead_logits(ht.reshape(-1, d), wt).reshape(B, K1, -1)
    ld = oracle.lmhead_logits(hd.reshape(-1, d), wd).reshape(B, K, -1)
    return lt, ld


def _drafts(ld, temp, top_k, seed):
    """x_i ~ transformed q_i of the oracle's draft logits (the drafter's own choice)."""
    B, K, V = ld.shape
    g = np.random.default_rng(seed)
    if temp == 0.0:
        return np.argmax(ld, axis=2).astype(np.int32)
    q = oracle.transform_rows(ld, temp, top_k)[0].reshape(B * K, V)
    return oracle.residual_sample(q.astype(np.float32), None,
                                  g.random(B * K).astype(np.float32))[0].reshape(B, K)


def _fused(ht, hd, wt, wd, x, u, temp, top_k, want_logits=True):
    B, K1, d = ht.shape
    K, V = K1 - 1, wt.shape[0]
    rows = B * K1 + (0 if temp == 0.0 else B * (K1 - 1))
    lo = torch.full((rows, V), float("nan"), dtype=torch.float32, device="cuda") if want_logits \
        else None
    ws = torch.empty(sv.spec_lmhead_workspace_size(B, K, V, d, 0 if temp == 0.0 else top_k),
                     dtype=torch.uint8, device="cuda")
    acc, out = sv.spec_verify_chain_lmhead(
        _bf(ht), None if temp == 0.0 else _bf(hd), _bf(wt), None if temp == 0.0 else _bf(wd),
        torch.from_numpy(x).cuda(), torch.from_numpy(u).cuda(), temp, top_k, logits_out=lo,
        workspace=ws)
    torch.cuda.synchronize()
    assert sv.spec_get_device_status(ws) == sv.SPEC_OK  # no wait of the kernel ran out
    return acc.cpu().numpy(), out.cpu().numpy(), lo


@pytest.mark.parametrize("B,V,d", [(2, 1000, 128), (3, 2560, 256), (2, 4099, 64)])
def test_lmhead_logits_match_double_product(B, V, d):
    cfg, ht, hd, wt, wd = _case(B, V, d)
    lt, ld = _oracle_logits(ht, hd, wt, wd)
    x = _drafts(ld, cfg.temp, cfg.top_k, 1)
    u = np.random.default_rng(2).random((B, cfg.K + 1)).astype(np.float32)
    _, _, lo = _fused(ht, hd, wt, wd, x, u, cfg.temp, cfg.top_k)
    got = lo.cpu().numpy().astype(np.float64)
    ref = np.concatenate([lt.reshape(-1, V), ld.reshape(-1, V)])
    err = np.abs(got - ref)
    assert np.isfinite(got).all()
    assert (err <= 1e-3 + 1e-4 * np.abs(ref)).all(), err.max()


def _unfused_on(lo, B, K, V, x, u, temp, top_k):
    lt = lo[:B * (K + 1)].view(B, K + 1, V)
    ld = None if temp == 0.0 else lo[B * (K + 1):].view(B, K, V)
    acc, out = sv.spec_verify_chain(lt, ld, torch.from_numpy(x).cuda(),
                                    torch.from_numpy(u).cuda(), temp, top_k)
    torch.cuda.synchronize()
    return acc.cpu().numpy(), out.cpu().numpy()


@pytest.mark.parametrize("temp,top_k", [(0.8, 50), (1.0, 1), (0.7, 64), (0.0, 0)])
def test_lmhead_fusion_equals_unfused_verification_of_its_logits(temp, top_k):
    cfg, ht, hd, wt, wd = _case(8, 30000, 512, K=5, seed=7, temp=temp, top_k=top_k)
    ld = oracle.lmhead_logits(hd.reshape(-1, cfg.d), wd).reshape(8, 5, -1)
    x = _drafts(ld, temp, top_k, 3)
    u = np.random.default_rng(4).random((8, 6)).astype(np.float32)
    acc, out, lo = _fused(ht, hd, wt, wd, x, u, temp, top_k)
    acc_u, out_u = _unfused_on(lo, 8, 5, cfg.V, x, u, temp, top_k)
    assert np.array_equal(acc, acc_u) and np.array_equal(out, out_u)
    assert acc.min() >= 0


@pytest.mark.parametrize("temp,top_k", [(0.0, 0), (0.8, 50)])
def test_lmhead_persistent_ctas_over_many_tiles(temp, top_k):
    """More work items than SMs (5 row tiles x up to 118 vocabulary tiles): every CTA runs
    several items through the same stage ring and tensor-memory buffers. Logits against the
    oracle's double product on every row, decisions against the unfused verification."""
    cfg, ht, hd, wt, wd = _case(64, 30000, 256, K=8, seed=9, temp=temp, top_k=top_k)
    lt, ld = _oracle_logits(ht, hd, wt, wd)
    x = _drafts(ld, temp, top_k, 8)
    u = np.random.default_rng(10).random((64, 9)).astype(np.float32)
    acc, out, lo = _fused(ht, hd, wt, wd, x, u, temp, top_k)
    got = lo.cpu().numpy().astype(np.float64)
    ref = lt.reshape(-1, cfg.V) if temp == 0.0 else np.concatenate(
        [lt.reshape(-1, cfg.V), ld.reshape(-1, cfg.V)])
    assert (np.abs(got - ref) <= 1e-3 + 1e-4 * np.abs(ref)).all()
    acc_u, out_u = _unfused_on(lo, 64, 8, cfg.V, x, u, temp, top_k)
    assert np.array_equal(acc, acc_u) and np.array_equal(out, out_u)
    assert acc.min() >= 0


def test_lmhead_workload_shape_end_to_end():
    """The 151,936 x 4,096 LM heads of the workload at 12 sequences (K = 8, T = 0.8, top-k
    50): fused decisions equal the unfused verification of the same logits on every row, and
    the oracle's verification of its double logits wherever it flags nothing."""
    cfg = specgen.LMHEAD
    ht, hd, wt, wd = specgen.lmhead_inputs(cfg, 12)
    B, K, V = 12, cfg.K, cfg.V
    lt, ld = _oracle_logits(ht, hd, wt, wd)
    x = _drafts(ld, cfg.temp, cfg.top_k, 5)
    u = np.random.default_rng(6).random((B, K + 1)).astype(np.float32)
    acc, out, lo = _fused(ht, hd, wt, wd, x, u, cfg.temp, cfg.top_k)
    got = lo.cpu().numpy().astype(np.float64)
    ref = np.concatenate([lt.reshape(-1, V), ld.reshape(-1, V)])
    assert (np.abs(got - ref) <= 1e-3 + 1e-4 * np.abs(ref)).all()
    acc_u, out_u = _unfused_on(lo, B, K, V, x, u, cfg.temp, cfg.top_k)
    assert np.array_equal(acc, acc_u) and np.array_equal(out, out_u)
    acc_r, out_r, fl = oracle.verify_chain(lt, ld, x, u, float(np.float32(cfg.temp)), cfg.top_k,
                                           windows=oracle.FP32_LOGITS)
    ok = (fl & oracle.PARITY_FLAGS) == 0
    same = (acc == acc_r) & np.all(out == out_r, axis=1)
    assert np.all(same | ~ok), np.nonzero(~same & ok)
    print(f"\nflagged {int((~ok).sum())} of {B}; mean accepted {acc.mean():.2f}")


def test_lmhead_rejects_unsupported_transforms():
    cfg, ht, hd, wt, wd = _case(1, 512, 64)
    x = np.zeros((1, cfg.K), np.int32)
    u = np.zeros((1, cfg.K + 1), np.float32)
    for top_k in (0, 65):
        with pytest.raises(sv.SpecError) as e:
            sv.spec_verify_chain_lmhead(_bf(ht), _bf(hd), _bf(wt), _bf(wd),
                                        torch.from_numpy(x).cuda(), torch.from_numpy(u).cuda(),
                                        1.0, top_k)
        assert e.value.status == sv.SPEC_ERR_UNSUPPORTED
