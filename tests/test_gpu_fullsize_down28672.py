"""The Llama-70B-shaped down projection at full size (W 8192 x 28672,
65536 tokens of Student-t(3) activations, W2 per-channel), in the bench's
launch configuration, checked against the oracle where it can follow:
a sampled covariance block; the trailing 2048 x 2048 corner of the Cholesky
factor of the damped inverse, which depends only on the same corner of H_X'
and on lambda (for the reversed factorisation Uc = J L^-1 J, L = chol(J H J),
the leading block of L is the Cholesky factor of the leading block of J H J),
and a residual check of the whole factor on sampled columns;
sampled solver rows on the GPU's W' and Uc; the whole Kronecker loss; the
sensitivity.  Tolerances as in test_gpu_parity.py.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from gpu_util import cov_close, device_rht, need_gpu, np64
from test_gpu_fullsize_mlp import check_sampled_rows

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

CORNER = 2048


@pytest.fixture(scope="module")
def layer():
    need_gpu()
    import post_weight_quantization_syrk_b200 as P
    from post_weight_quantization_syrk_b200.pipeline import LayerQuantizer
    P.load()
    spec = synth.WORKLOADS["down28672"]
    seed = synth.layer_seed(3, 0)
    dev = torch.device("cuda")
    W = synth.weights(spec, seed, dev)
    X = synth.activations(spec, seed, dev)
    G = synth.gradients(spec, seed, dev)
    Ti, To = synth.rht_params(spec.d_in, seed * 2 + 11), synth.rht_params(spec.d_out, seed * 2 + 12)
    lq = LayerQuantizer(spec.d_out, spec.d_in, gemm_mode=P.KQ_GEMM_3XTF32)
    lq.statistics(X, G)
    HX0, HG0 = lq.H_X.clone(), lq.H_G.clone()
    res = lq.run(W, X, G, device_rht(Ti), device_rht(To), [(2, 0)])
    torch.cuda.synchronize()
    lq.check("full-size down28672")
    yield dict(spec=spec, X=X, G=G, lq=lq, res=res, HX0=HX0, HG0=HG0)
    del X, G, lq, res
    torch.cuda.empty_cache()


@pytest.mark.parametrize("which", ["X", "G"])
def test_covariance_sampled_block(layer, which):
    A = layer[which]
    H = layer["HX0"] if which == "X" else layer["HG0"]
    rng = np.random.default_rng(7)
    idx = np.sort(rng.choice(A.shape[1], 48, replace=False))
    cols = A[:, torch.from_numpy(idx).cuda()].float().cpu().numpy().astype(np.float64)
    ref = cols.T @ cols / A.shape[0]
    fro, ent = cov_close(np64(H[idx][:, idx]), ref)
    assert fro <= 1e-4 and ent <= 1e-4, (fro, ent)


def test_cholesky_trailing_corner(layer):
    lq = layer["lq"]
    n = layer["spec"].d_in
    Hfull = lq.H_X
    # damping and dead columns from the whole matrix, the factor from the corner
    diag = np64(torch.diagonal(Hfull))
    dead_all = diag == 0
    lam = 0.01 * float(np.mean(np.where(dead_all, 1.0, diag)))
    Hc = np64(Hfull[n - CORNER:, n - CORNER:])
    Hc = np.triu(Hc) + np.triu(Hc, 1).T
    idx = np.flatnonzero(np.diag(Hc) == 0)
    Hc[idx, idx] = 1.0
    Hc[np.diag_indices_from(Hc)] += lam
    # Oracle on the corner with the damping already applied (damp_frac = 0)
    ref, _, _ = O.chol_inv(Hc, 0.0)
    got = np64(lq.Uc[n - CORNER:, n - CORNER:])
    rowmax = np.max(np.abs(ref), axis=1, keepdims=True)
    assert np.max(np.abs(got - ref) - (4e-7 * np.abs(ref) + 1e-8 * rowmax)) <= 0
    assert np.array_equal(lq.dead.cpu().numpy().astype(bool), dead_all)
    # and Uc is upper triangular with a positive diagonal everywhere
    assert bool((torch.diagonal(lq.Uc) > 0).all())
    assert float(torch.tril(lq.Uc, -1).abs().max()) == 0.0


def test_cholesky_residual_sampled_columns(layer):
    """A residual pin of the WHOLE factor, leading rows included: for sampled
    columns j (the first 64, the last 64 and 64 at random),
    ||(Uc^T Uc (H_X' + lambda I) - I) e_j|| <= 2e-6, evaluated in fp64.  The
    exact factor of a Student-t layer of this shape, rounded to fp32, leaves
    1.4e-7 (1024 and 2048 channels) to 1.7e-7 (4096) here, so the bound
    catches any row of Uc off by more than about 1e-5 relative."""
    lq = layer["lq"]
    n = layer["spec"].d_in
    H = lq.H_X
    dev = H.device
    diag = torch.diagonal(H).double()
    dead = diag == 0
    lam = 0.01 * float(torch.where(dead, torch.ones_like(diag), diag).mean())
    rng = np.random.default_rng(29)
    S = np.unique(np.r_[np.arange(64), np.arange(n - 64, n), rng.choice(n, 64, replace=False)])
    St = torch.from_numpy(S).to(dev)
    # column j of the symmetric matrix the factor is defined from (its upper
    # triangle): rows i <= j from H[i, j], rows i > j from H[j, i]
    up = H[:, St].double()
    lo = H[St, :].double().T
    rows = torch.arange(n, device=dev)[:, None]
    Hs = torch.where(rows <= St[None, :], up, lo)
    k = torch.arange(len(S), device=dev)
    Hs[St, k] = torch.where(dead[St], torch.ones_like(diag[St]), diag[St]) + lam
    Uc = lq.Uc.double()
    R = Uc.T @ (Uc @ Hs)
    R[St, k] -= 1.0
    r = torch.linalg.vector_norm(R, dim=0).cpu().numpy()
    del Uc, R
    torch.cuda.empty_cache()
    assert r.max() <= 2e-6, (float(r.max()), int(S[int(np.argmax(r))]))


def test_solver_sampled_rows(layer):
    check_sampled_rows(layer["lq"], layer["res"][0], layer["spec"].d_out, 21, n_rows=16)


def test_kron_loss_full(layer):
    lq, r = layer["lq"], layer["res"][0]
    ref = O.kron_loss(np64(lq.Wp), np64(r.W_hat), np64(lq.H_X), np64(lq.H_G))
    assert abs(r.loss.item() - ref) <= 1e-3 * ref, (r.loss.item(), ref)


def test_sensitivity_full(layer):
    lq = layer["lq"]
    ref = O.sensitivity(np64(layer["HX0"]), np64(layer["HG0"]))
    assert np.allclose(lq.sens.cpu().numpy(), ref, rtol=1e-10)
