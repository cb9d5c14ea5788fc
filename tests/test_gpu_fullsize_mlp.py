"""The Llama-2-7B MLP-shaped layers at full size (gate/up: 11008 x 4096,
down: 4096 x 11008 with SiLU-gated inputs; 262144 tokens; W3 group 128 and
W2 per-channel), in the launch configuration of the bench, checked against
the oracle on what it can afford: a sampled block of each covariance, the
whole damped Cholesky factor of the inverse, sampled solver rows (rows are
independent given Uc and W'), the whole Kronecker loss, and the sensitivity.
Each stage is compared on the GPU's own inputs to that stage.  Tolerances as
in test_gpu_parity.py.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from gpu_util import cov_close, device_rht, need_gpu, np64

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SETTINGS = [(3, 128), (2, 0)]


@pytest.fixture(scope="module", params=["mlp_up11008", "mlp_down11008"])
def layer(request):
    need_gpu()
    import post_weight_quantization_syrk_b200 as P
    from post_weight_quantization_syrk_b200.pipeline import LayerQuantizer
    P.load()
    spec = synth.WORKLOADS[request.param]
    seed = synth.layer_seed(2, 0 if request.param == "mlp_up11008" else 1)
    dev = torch.device("cuda")
    W = synth.weights(spec, seed, dev)
    X = synth.activations(spec, seed, dev)
    G = synth.gradients(spec, seed, dev)
    Ti, To = synth.rht_params(spec.d_in, seed * 2 + 11), synth.rht_params(spec.d_out, seed * 2 + 12)
    lq = LayerQuantizer(spec.d_out, spec.d_in, gemm_mode=P.KQ_GEMM_3XTF32)
    lq.statistics(X, G)
    HX0, HG0 = lq.H_X.clone(), lq.H_G.clone()
    res = lq.run(W, X, G, device_rht(Ti), device_rht(To), SETTINGS)
    torch.cuda.synchronize()
    lq.check(f"full-size {request.param}")
    yield dict(spec=spec, X=X, G=G, lq=lq, res=res, HX0=HX0, HG0=HG0)
    del X, G, lq, res
    torch.cuda.empty_cache()


@pytest.mark.parametrize("which", ["X", "G"])
def test_covariance_sampled_block(layer, which):
    A = layer[which]
    H = layer["HX0"] if which == "X" else layer["HG0"]
    d = A.shape[1]
    rng = np.random.default_rng(5)
    idx = np.sort(rng.choice(d, 40, replace=False))
    big = torch.topk(torch.diagonal(H), 8).indices.cpu().numpy()
    idx = np.unique(np.concatenate([idx, big]))
    cols = A[:, torch.from_numpy(idx).cuda()].float().cpu().numpy().astype(np.float64)
    ref = cols.T @ cols / A.shape[0]
    fro, ent = cov_close(np64(H[idx][:, idx]), ref)
    assert fro <= 1e-4 and ent <= 1e-4, (fro, ent)
    assert torch.equal(H, H.T)


def test_cholesky_factor_full(layer):
    lq = layer["lq"]
    ref, dead, _ = O.chol_inv(np64(lq.H_X), 0.01)
    got = np64(lq.Uc)
    rowmax = np.max(np.abs(ref), axis=1, keepdims=True)
    assert np.max(np.abs(got - ref) - (4e-7 * np.abs(ref) + 1e-8 * rowmax)) <= 0
    assert np.array_equal(lq.dead.cpu().numpy().astype(bool), dead)


def check_sampled_rows(lq, r, d_out, seed, n_rows=32):
    """Forced-code oracle replay of sampled rows, as in test_gpu_parity.py."""
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(d_out, n_rows, replace=False))
    ridx = torch.from_numpy(rows).cuda()
    codes = r.codes[ridx].cpu().numpy()
    scales, zeros = r.scales[ridx].cpu().numpy(), r.zeros[ridx].cpu().numpy()
    ref = O.quantize_layer(np64(lq.Wp[ridx]), np64(lq.Uc), r.bits, r.group, 128,
                           dead=lq.dead.cpu().numpy().astype(bool), force_codes=codes,
                           force_zeros=zeros if r.group else None, excuse_tol=excuse_tol(r.bits))
    assert ref.mismatches == [], ref.mismatches[:5]
    assert ref.zero_mismatches == [], ref.zero_mismatches[:5]
    assert 1 - ref.excused / codes.size >= 0.999
    if not r.group:
        assert np.array_equal(scales, ref.scales) and np.array_equal(zeros, ref.zeros)
    else:
        assert np.max(np.abs(scales / ref.scales - 1)) <= 1e-5
    Wh = np64(r.W_hat[ridx])
    assert np.linalg.norm(Wh - ref.W_hat) / np.linalg.norm(ref.W_hat) <= 1e-3


def excuse_tol(bits):
    return 1e-5 * max(1.0, (2 ** bits - 1) / 15.0)


@pytest.mark.parametrize("k", [0, 1])
def test_solver_sampled_rows(layer, k):
    check_sampled_rows(layer["lq"], layer["res"][k], layer["spec"].d_out, 10 + k)


@pytest.mark.parametrize("k", [0, 1])
def test_kron_loss_full(layer, k):
    lq, r = layer["lq"], layer["res"][k]
    ref = O.kron_loss(np64(lq.Wp), np64(r.W_hat), np64(lq.H_X), np64(lq.H_G))
    assert abs(r.loss.item() - ref) <= 1e-3 * ref, (r.loss.item(), ref)


def test_sensitivity_full(layer):
    lq = layer["lq"]
    ref = O.sensitivity(np64(layer["HX0"]), np64(layer["HG0"]))
    assert np.allclose(lq.sens.cpu().numpy(), ref, rtol=1e-10)
