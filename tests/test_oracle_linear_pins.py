"""Pins of the composed oracle path ``oracle.quantize_linear`` (CPU only).

quantize_linear chains covariances -> sensitivity -> BiIP -> damped Cholesky
factor of the inverse -> blocked OBS -> Kronecker loss.  These tests check
what it returns against quantities computed here by other routes, in the
ORIGINAL (unrotated) coordinates where possible, so that a wrong link in the
chain fails: the factor taken from the unrotated H_X, the loss taken against
the unrotated W or with the rotations swapped, the dead-column mask dropped.

Sources: KronQ review, Background (H ~ H_X kron H_G, the loss is the
Kronecker-weighted norm of the weight error) and Method (1) (W' = V W U^T
keeps the layer's function, H_X' = U H_X U^T, H_G' = V H_G V^T); "A Unified
Hessian-Guided Framework for Post-Training Quantization", Appendix A.1 (the
Kronecker-weighted norm as a trace).
"""
import numpy as np
import pytest

import oracle as O


def _rht(rng, n, log2_p):
    """Random rotation parameters: signs and (for odd m > 1) an orthogonal Q_m."""
    m = n >> log2_p
    signs = np.where(rng.random(n) < 0.5, -1.0, 1.0)
    Q = None
    if m > 1:
        Q, R = np.linalg.qr(rng.standard_normal((m, m)))
        Q = Q * np.sign(np.diag(R))[None, :]
    return O.rht_matrix(n, log2_p, signs, Q)


def _sample_loss(X, G, dW):
    """(1/N^2) sum_{t,s} (g_t^T dW x_s)^2, the Kronecker loss written from the
    calibration samples with H_X = X^T X / N and H_G = G^T G / N."""
    N = X.shape[0]
    s = 0.0
    for t in range(N):
        gt = G[t] @ dW
        for u in range(N):
            s += float(gt @ X[u]) ** 2
    return s / N ** 2


def _sample_gptq_loss(X, dW):
    """(1/N) sum_s ||dW x_s||^2 (H_G = I)."""
    N = X.shape[0]
    return sum(float(np.sum((dW @ X[u]) ** 2)) for u in range(N)) / N


def _rotated_cov_loops(X, T):
    """H' [a, b] = (1/N) sum_t (T x_t)_a (T x_t)_b by explicit loops."""
    N, n = X.shape
    Z = [T @ X[t] for t in range(N)]
    H = np.zeros((n, n))
    for a in range(n):
        for b in range(n):
            H[a, b] = sum(z[a] * z[b] for z in Z) / N
    return H


CASES = [
    # d_out, d_in, N, log2_p_out, log2_p_in, bits, group
    (4, 8, 17, 2, 3, 2, 0),
    (12, 8, 23, 2, 3, 3, 0),     # d_out = 3 * 4: Q_3 mixes the output side
    (6, 12, 19, 1, 2, 4, 0),     # both sides with an odd factor
    (4, 64, 13, 2, 5, 3, 32),    # grouped grid, two groups
]


@pytest.mark.parametrize("d_out,d_in,N,kout,kin,bits,group", CASES)
def test_quantize_linear_against_sample_quantities(d_out, d_in, N, kout, kin, bits, group):
    rng = np.random.default_rng(1000 + 7 * d_out + d_in)
    W = rng.normal(0, 0.02, (d_out, d_in))
    X = rng.standard_normal((N, d_in)) * np.exp(rng.normal(0, 1.0, d_in))[None, :]
    G = rng.standard_normal((N, d_out)) * np.exp(rng.uniform(np.log(1e-3), 0, d_out))[None, :]
    U, V = _rht(rng, d_in, kin), _rht(rng, d_out, kout)
    r = O.quantize_linear(W, X, G, U, V, bits, group, block=128, damp_frac=0.01)

    # sensitivity: traces are mean squared norms of the samples
    tX = sum(float(X[t] @ X[t]) for t in range(N)) / N
    tG = sum(float(G[t] @ G[t]) for t in range(N)) / N
    assert np.allclose(r["sens"], (tX, tG, tX * tG), rtol=1e-12)

    # the rotated weights keep the layer's function: V^T W' U x = W x
    for _ in range(3):
        x = rng.standard_normal(d_in)
        assert np.max(np.abs(V.T @ (r["Wp"] @ (U @ x)) - W @ x)) < 1e-12

    # the factor is that of the damped ROTATED activation covariance, formed
    # here from the rotated samples by loops: Uc^T Uc (H_X' + lambda I) = I
    HXp = _rotated_cov_loops(X, U)
    lam = 0.01 * np.mean(np.diag(HXp))
    assert abs(r["lam"] - lam) <= 1e-12 * lam
    Uc = r["Uc"]
    assert np.allclose(Uc, np.triu(Uc)) and np.all(np.diag(Uc) > 0)
    res = Uc.T @ Uc @ (HXp + lam * np.eye(d_in)) - np.eye(d_in)
    assert np.max(np.abs(res)) < 1e-9

    # codes on the returned grid give the returned dequantized weights
    q = r["quant"]
    g = np.zeros(d_in, dtype=int) if not group else np.arange(d_in) // group
    deq = q.scales.astype(np.float64)[:, g] * (q.codes.astype(np.float64) - q.zeros.astype(np.float64)[:, g])
    assert np.array_equal(deq, q.W_hat)
    assert q.codes.max() <= 2 ** bits - 1

    # the loss, from the samples in ORIGINAL coordinates with the quantized
    # layer taken back through both rotations
    dW = W - V.T @ q.W_hat @ U
    assert np.isclose(r["loss"], _sample_loss(X, G, dW), rtol=1e-10)
    assert np.isclose(r["loss_gptq"], _sample_gptq_loss(X, dW), rtol=1e-10)
    assert r["loss"] > 0


def test_quantize_linear_dead_column():
    """An input channel that is zero in every token (after the rotation) is a
    dead column: the factor treats it as unit curvature before damping, its
    weights are zeroed before quantization (so its dequantized weight is 0),
    and the loss still equals the sample form.  The input rotation here is a
    signed permutation (log2_p = 0, Q_m a permutation), so the zero channel
    stays exactly zero in the rotated basis."""
    rng = np.random.default_rng(77)
    d_out, d_in, N = 4, 6, 15
    W = rng.normal(0, 0.02, (d_out, d_in))
    X = rng.standard_normal((N, d_in))
    X[:, 1] = 0.0
    G = rng.standard_normal((N, d_out))
    perm = np.eye(d_in)[[3, 0, 5, 1, 2, 4]]            # channel 1 goes to rotated index 3
    signs = np.where(rng.random(d_in) < 0.5, -1.0, 1.0)
    U = O.rht_matrix(d_in, 0, signs, perm)
    V = _rht(rng, d_out, 2)
    r = O.quantize_linear(W, X, G, U, V, 3, 0)
    dead = r["dead"]
    assert dead.tolist() == [False, False, False, True, False, False]
    q = r["quant"]
    assert np.all(q.W_hat[:, 3] == 0.0)

    # factor: the rotated covariance by loops with the dead diagonal set to
    # 1 before lambda is taken
    HXp = _rotated_cov_loops(X, U)
    assert np.all(HXp[3] == 0.0) and np.all(HXp[:, 3] == 0.0)
    HXp[3, 3] = 1.0
    lam = 0.01 * np.mean(np.diag(HXp))
    res = r["Uc"].T @ r["Uc"] @ (HXp + lam * np.eye(d_in)) - np.eye(d_in)
    assert np.max(np.abs(res)) < 1e-10

    dW = W - V.T @ q.W_hat @ U
    assert np.isclose(r["loss"], _sample_loss(X, G, dW), rtol=1e-10)


def test_quantize_linear_pins_catch_planted_mistakes():
    """The sample-form checks above fail for the composition mistakes a
    reviewer would look for: the factor of the unrotated H_X, the loss
    against the unrotated W, the rotations' roles swapped."""
    rng = np.random.default_rng(5)
    d_out, d_in, N = 4, 8, 17
    W = rng.normal(0, 0.02, (d_out, d_in))
    X = rng.standard_normal((N, d_in)) * np.exp(rng.normal(0, 1.0, d_in))[None, :]
    G = rng.standard_normal((N, d_out)) * np.exp(rng.uniform(np.log(1e-3), 0, d_out))[None, :]
    U, V = _rht(rng, d_in, 3), _rht(rng, d_out, 2)
    r = O.quantize_linear(W, X, G, U, V, 2, 0)
    HXp = _rotated_cov_loops(X, U)
    lam = 0.01 * np.mean(np.diag(HXp))
    # the factor of the UNROTATED covariance fails the residual check
    Uc_wrong, _, lam_w = O.chol_inv(O.covariance(X))
    res = Uc_wrong.T @ Uc_wrong @ (HXp + lam * np.eye(d_in)) - np.eye(d_in)
    assert np.max(np.abs(res)) > 1e-3
    # the loss against the unrotated W differs from the sample form
    q = r["quant"]
    wrong = O.kron_loss(W, q.W_hat, r["H_Xp"], r["H_Gp"])
    dW = W - V.T @ q.W_hat @ U
    assert not np.isclose(wrong, _sample_loss(X, G, dW), rtol=1e-3)
    # taking the quantized layer back with the rotations transposed differs too
    dW_swapped = W - V @ q.W_hat @ U.T
    assert not np.isclose(r["loss"], _sample_loss(X, G, dW_swapped), rtol=1e-3)
