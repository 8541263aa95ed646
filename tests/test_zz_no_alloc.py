"""spec_verify_chain_noalloc (static scratch) against spec_verify_chain (caller workspace):
identical outputs on two no-alloc calls in a row, so nothing carries over in the scratch from
one call into the next. The file is collected last on purpose; the test must pass both alone
and after every other test."""
import numpy as np
import pytest
import torch

import draft_token_verification_spec_b200 as sv
import specgen

pytestmark = pytest.mark.gpu


def _inputs(cfg, B, dev):
    t, d = specgen.chain_logits(cfg, B)
    u = specgen.chain_uniforms(cfg, B)

    def to(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)

    tg, dg = to(t), to(d)
    x = dg.float().argmax(-1).to(torch.int32).contiguous()  # valid draft tokens
    return tg, dg, x, to(u)


# (config, batch, greedy): top-k rows with kept-id lists and sparse draws, then top-p rows
# (candidate cuts, the exact finisher list); plain sampling, then greedy
PAIRS = [
    ((specgen.CFG5, 8, False), (specgen.CFG3, 8, False)),
    ((specgen.CFG2, 16, False), (specgen.CFG2, 16, True)),
]


@pytest.mark.parametrize("pair", PAIRS, ids=["topk_then_topp", "sampling_then_greedy"])
def test_noalloc_matches_workspace_call_on_two_calls_in_a_row(cuda_device, pair):
    runs = []
    for cfg, B, greedy in pair:
        tg, dg, x, u = _inputs(cfg, B, cuda_device)
        temp = 0.0 if greedy else cfg.temp
        d = None if greedy else dg
        ref = sv.spec_verify_chain(tg, d, x, u, temp, cfg.top_k, cfg.top_p)
        runs.append((tg, d, x, u, temp, cfg, ref))
    torch.cuda.synchronize()
    outs = [sv.spec_verify_chain_noalloc(tg, d, x, u, temp, cfg.top_k, cfg.top_p)
            for tg, d, x, u, temp, cfg, _ in runs]  # back to back on one stream
    torch.cuda.synchronize()
    for (tg, d, x, u, temp, cfg, (acc_r, out_r)), (acc, out) in zip(runs, outs):
        assert int(acc_r.min()) >= 0, cfg.name
        assert torch.equal(acc, acc_r), cfg.name
        assert torch.equal(out, out_r), cfg.name


def test_noalloc_rejects_a_batch_beyond_its_scratch(cuda_device):
    cfg = specgen.CFG5
    V = cfg.V
    assert sv.spec_workspace_size(64, cfg.K, V) <= 32 << 20
    assert sv.spec_workspace_size(1024, cfg.K, V) > 32 << 20
    t = torch.zeros((1024, cfg.K + 1, V), dtype=torch.bfloat16, device=cuda_device)
    d = torch.zeros((1024, cfg.K, V), dtype=torch.bfloat16, device=cuda_device)
    x = torch.zeros((1024, cfg.K), dtype=torch.int32, device=cuda_device)
    u = torch.zeros((1024, cfg.K + 1), dtype=torch.float32, device=cuda_device)
    with pytest.raises(sv.SpecError) as e:
        sv.spec_verify_chain_noalloc(t, d, x, u, 1.0)
    assert e.value.status == sv.SPEC_ERR_WORKSPACE


def test_noalloc_rejects_logits_off_the_current_device(cuda_device):
    """The scratch is the current device's, so logits that are not that device's memory
    (here: plain host memory) are refused before any launch."""
    import ctypes

    B, K, V = 2, 2, 64
    host = np.zeros((B, K + 1, V), np.float32)
    d = torch.zeros((B, K, V), dtype=torch.float32, device=cuda_device)
    x = torch.zeros((B, K), dtype=torch.int32, device=cuda_device)
    u = torch.zeros((B, K + 1), dtype=torch.float32, device=cuda_device)
    acc = torch.empty(B, dtype=torch.int32, device=cuda_device)
    out = torch.empty((B, K + 1), dtype=torch.int32, device=cuda_device)
    torch.cuda.synchronize()
    rc = sv.lib().spec_verify_chain_noalloc(
        host.ctypes.data_as(ctypes.c_void_p), ctypes.c_void_p(d.data_ptr()), sv.SPEC_F32, B, K,
        V, ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(u.data_ptr()), 1.0, 0, 1.0,
        ctypes.c_void_p(acc.data_ptr()), ctypes.c_void_p(out.data_ptr()), None)
    assert rc == sv.SPEC_ERR_INVALID_ARG
    torch.cuda.synchronize()  # nothing was launched, and the context is healthy


@pytest.mark.parametrize("cfg", [specgen.CFG5, specgen.CFG3], ids=["topk", "topp"])
def test_noalloc_call_captures_into_a_cuda_graph(cuda_device, cfg):
    """After one ordinary call, the no-alloc entry point records into a CUDA graph (global
    capture mode: an allocating or synchronising call inside would end the capture with an
    error), and every replay verifies the logits the buffers hold at that moment."""
    tg, dg, x, u = _inputs(cfg, 8, cuda_device)
    ref = sv.spec_verify_chain(tg, dg, x, u, cfg.temp, cfg.top_k, cfg.top_p)
    acc = torch.empty_like(ref[0])
    out = torch.empty_like(ref[1])
    sv.spec_verify_chain_noalloc(tg, dg, x, u, cfg.temp, cfg.top_k, cfg.top_p,
                                 accepted_len=acc, out_tokens=out)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        sv.spec_verify_chain_noalloc(tg, dg, x, u, cfg.temp, cfg.top_k, cfg.top_p,
                                     accepted_len=acc, out_tokens=out)
    acc.fill_(-7)
    out.fill_(-7)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(acc, ref[0]) and torch.equal(out, ref[1])
    # new inputs in the same buffers: the replay verifies them, not the captured values
    tg2, dg2, x2, u2 = _inputs(cfg, 8, cuda_device)
    u2.copy_(torch.flip(u2, dims=[0]))
    ref2 = sv.spec_verify_chain(tg2, dg2, x2, u2, cfg.temp, cfg.top_k, cfg.top_p)
    tg.copy_(tg2)
    dg.copy_(dg2)
    x.copy_(x2)
    u.copy_(u2)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(acc, ref2[0]) and torch.equal(out, ref2[1])
    del g
