"""The seeded input generators: reproducible, right shapes and recipes."""
import numpy as np
import torch

import synth


def test_deterministic_and_shapes():
    spec = synth.scaled(synth.WORKLOADS["attn4096"], 64, 96, 300)
    a = synth.layer(spec, 5)
    b = synth.layer(spec, 5)
    for x, y in zip(a[:3], b[:3]):
        assert torch.equal(x, y)
    W, X, G, Ti, To = a
    assert W.shape == (64, 96) and W.dtype == torch.float32
    assert X.shape == (300, 96) and X.dtype == torch.bfloat16
    assert G.shape == (300, 64) and G.dtype == torch.bfloat16
    assert torch.equal(W, W.to(torch.bfloat16).float())          # bf16-valued weights
    assert Ti.n == 96 and Ti.m == 3 and Ti.log2_p == 5 and Ti.Qm.shape == (3, 3)
    assert To.n == 64 and To.m == 1 and To.Qm is None
    assert set(Ti.signs.unique().tolist()) <= {-1.0, 1.0}
    assert np.max(np.abs(Ti.Qm64 @ Ti.Qm64.T - np.eye(3))) < 1e-12
    assert not torch.equal(synth.layer(spec, 6)[0], W)


def test_recipes():
    spec = synth.scaled(synth.WORKLOADS["layer512"], 128, 128, 4096)
    W = synth.weights(spec, 1)
    big = (W.abs() > 0.1).float().mean().item()          # 1% outliers x10 of N(0, 0.02^2)
    assert 0.004 < big < 0.02
    G = synth.gradients(spec, 1).float()
    r = G.pow(2).mean(0).sqrt()
    assert r.min() > 5e-4 and r.max() < 1.2                # log-uniform [1e-3, 1] scales
    for kind in ("silu_gated", "student_t3"):
        s2 = synth.scaled(synth.WORKLOADS["down28672"], 8, 16, 2000)
        s2 = synth.dataclasses.replace(s2, x_kind=kind)
        X = synth.activations(s2, 3).float()
        assert torch.isfinite(X).all() and X.std() > 0
    spec2 = synth.WORKLOADS["attn4096"]
    c = synth.channel_scales(synth.scaled(spec2, d_in=512), 2)
    assert (c > 50).sum() >= 8                              # the massive channels


def test_split_pow2():
    assert synth.split_pow2(4096) == (1, 12)
    assert synth.split_pow2(11008) == (43, 8)
    assert synth.split_pow2(28672) == (7, 12)
