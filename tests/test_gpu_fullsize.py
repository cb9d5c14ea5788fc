"""The full-size attention-projection layer (4096 x 4096, 262144 tokens), in
the launch configuration bench.py times, checked against the oracle on what
the oracle can afford: a sampled block of each covariance (every entry of the
block from the float64 dot products of the sampled channels), the whole
damped Cholesky factor, sampled rows of the solver (rows are independent
given Uc and W'), the rotation of W, and the whole Kronecker loss.
Tolerances as in test_gpu_parity.py.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from gpu_util import cov_close, device_rht, need_gpu, np64, oracle_T

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def layer():
    need_gpu()
    import post_weight_quantization_syrk_b200 as P
    from post_weight_quantization_syrk_b200.pipeline import LayerQuantizer
    P.load()
    spec = synth.WORKLOADS["attn4096"]
    seed = synth.layer_seed(2, 0)
    dev = torch.device("cuda")
    W = synth.weights(spec, seed, dev)
    X = synth.activations(spec, seed, dev)
    G = synth.gradients(spec, seed, dev)
    Ti, To = synth.rht_params(spec.d_in, seed * 2 + 11), synth.rht_params(spec.d_out, seed * 2 + 12)
    lq = LayerQuantizer(spec.d_out, spec.d_in, gemm_mode=P.KQ_GEMM_3XTF32)
    lq.statistics(X, G)
    HX0, HG0 = lq.H_X.clone(), lq.H_G.clone()
    res = lq.run(W, X, G, device_rht(Ti), device_rht(To), [(2, 0), (3, 0), (4, 0)])
    torch.cuda.synchronize()
    lq.check("full-size layer")
    return dict(P=P, spec=spec, W=W, X=X, G=G, Ti=Ti, To=To, lq=lq, res=res, HX0=HX0, HG0=HG0)


@pytest.mark.parametrize("which", ["X", "G"])
def test_covariance_sampled_block(layer, which):
    A = layer[which]
    H = layer["HX0"] if which == "X" else layer["HG0"]
    d = A.shape[1]
    rng = np.random.default_rng(0)
    idx = np.sort(rng.choice(d, 40, replace=False))
    if which == "X":   # include the massive channels (largest diagonal entries)
        big = torch.topk(torch.diagonal(H), 8).indices.cpu().numpy()
        idx = np.unique(np.concatenate([idx, big]))
    cols = A[:, torch.from_numpy(idx).cuda()].float().cpu().numpy().astype(np.float64)
    ref = cols.T @ cols / A.shape[0]
    got = np64(H[idx][:, idx])
    fro, ent = cov_close(got, ref)
    assert fro <= 1e-4 and ent <= 1e-4, (fro, ent)
    assert torch.equal(H, H.T)


def test_rotation_of_w(layer):
    lq = layer["lq"]
    Wp = oracle_T(layer["To"]) @ np64(layer["W"]) @ oracle_T(layer["Ti"]).T
    got = np64(lq.Wp)
    err = np.linalg.norm(got - Wp, axis=1) / np.linalg.norm(Wp, axis=1)
    assert err.max() <= 4e-6


def test_cholesky_factor_full(layer):
    lq = layer["lq"]
    ref, dead, _ = O.chol_inv(np64(lq.H_X), 0.01)
    got = np64(lq.Uc)
    rowmax = np.max(np.abs(ref), axis=1, keepdims=True)
    assert np.max(np.abs(got - ref) - (4e-7 * np.abs(ref) + 1e-8 * rowmax)) <= 0
    assert not dead.any() and not lq.dead.any()


@pytest.mark.parametrize("k", [0, 1, 2])
def test_solver_sampled_rows(layer, k):
    lq, r = layer["lq"], layer["res"][k]
    rng = np.random.default_rng(k)
    rows = np.sort(rng.choice(layer["spec"].d_out, 48, replace=False))
    ridx = torch.from_numpy(rows).cuda()
    codes = r.codes[ridx].cpu().numpy()
    ref = O.quantize_layer(np64(lq.Wp[ridx]), np64(lq.Uc), r.bits, 0, 128, force_codes=codes, excuse_tol=1e-5)
    assert ref.mismatches == [], ref.mismatches[:5]
    assert 1 - ref.excused / codes.size >= 0.999
    assert np.array_equal(r.scales[ridx].cpu().numpy(), ref.scales)
    assert np.array_equal(r.zeros[ridx].cpu().numpy(), ref.zeros)
    Wh = np64(r.W_hat[ridx])
    assert np.linalg.norm(Wh - ref.W_hat) / np.linalg.norm(ref.W_hat) <= 1e-3


@pytest.mark.parametrize("k", [0, 2])
def test_kron_loss_full(layer, k):
    lq, r = layer["lq"], layer["res"][k]
    ref = O.kron_loss(np64(lq.Wp), np64(r.W_hat), np64(lq.H_X), np64(lq.H_G))
    assert abs(r.loss.item() - ref) <= 1e-3 * ref, (r.loss.item(), ref)


def test_sensitivity_full(layer):
    lq = layer["lq"]
    ref = O.sensitivity(np64(layer["HX0"]), np64(layer["HG0"]))
    assert np.allclose(lq.sens.cpu().numpy(), ref, rtol=1e-10)
