"""The seeded input generator: determinism, shapes, storage rounding (no GPU)."""
import numpy as np
import torch

import specgen


def test_bf16_rounding_matches_torch_round_to_nearest_even():
    g = np.random.default_rng(0)
    x = np.concatenate([g.normal(0, 5, 100000), g.normal(0, 1e-3, 1000),
                        np.array([1.00390625, 1.01171875, -1.00390625])]).astype(np.float32)
    ours = specgen.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = specgen.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_uniforms_are_24bit_dyadics_in_unit_interval():
    u = specgen.chain_uniforms(specgen.CFG2)
    assert u.shape == (64, 6) and u.dtype == np.float32
    assert np.all((u >= 0) & (u < 1))
    k = u.astype(np.float64) * 2 ** 24
    assert np.array_equal(k, np.round(k))


def test_chain_logits_deterministic_and_prefix_stable():
    cfg = specgen.CFG2
    t1, d1 = specgen.chain_logits(cfg, 3)
    t2, d2 = specgen.chain_logits(cfg, 5)
    assert t1.shape == (3, 6, 32000) and d1.shape == (3, 5, 32000) and t1.dtype == np.uint16
    assert np.array_equal(t1, t2[:3]) and np.array_equal(d1, d2[:3])
    t3, _ = specgen.chain_logits(cfg, 3)
    assert np.array_equal(t1, t3)


def test_chain_logits_distribution():
    cfg = specgen.CFG1
    t, d = specgen.chain_logits(cfg)
    assert t.dtype == np.float32 and t.shape == (1, 5, 1000)
    assert abs(t.std() - 2.0) < 0.1 and abs((d - t[:, :4]).std() - 0.5) < 0.03
    cfg = specgen.CFG3
    t, _ = specgen.chain_logits(cfg, 1)
    tf = specgen.bf16_bits_to_f32(t)
    assert np.all(tf.max(axis=2) > 8.0)  # the boosted token sits at N(0,16) + 8


def test_tree_inputs_shapes():
    cfg = specgen.CFG4
    logits, toks, par = specgen.tree_inputs(cfg, 2)
    assert logits.shape == (2, 64, 32000) and toks.shape == (2, 64) and par.shape == (64,)
    assert np.all((toks >= 0) & (toks < 32000))
    _, depth, rank = specgen.tree_structure(cfg.heads, cfg.N)
    # nodes with the same depth and rank carry the same token within a batch row
    for b in range(2):
        for d in range(1, 5):
            for r in range(4):
                sel = (depth == d) & (rank == r)
                if sel.any():
                    assert len(set(toks[b, sel].tolist())) == 1
