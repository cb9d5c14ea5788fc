"""Pins of the oracle's output-side functions without the full H_G (CPU only).

KronQ review, Limitations (second limitation: BiIP holds H_G as a full
d_out x d_out matrix) and the research thread's "Sparks" list (how much of
the output-side flattening survives blockwise or low-rank H_G); KronQ paper
page, Abstract (1) (the output rotation uses the gradient covariance).  Each
function is checked against hand-derived values, brute force or an
independent library routine.
"""
import numpy as np
import pytest
import scipy.linalg as sla

import oracle as O


def test_balance_permutation_hand_values():
    # diag = [5, 1, 3, 2, 4, 0], k = 2 (3 blocks): ranks 0..5 are channels
    # 0, 4, 2, 3, 1, 5; rank q goes to block q % 3, slot q // 3
    perm = O.balance_permutation(np.array([5., 1., 3., 2., 4., 0.]), 2)
    assert perm.tolist() == [0, 3, 4, 1, 2, 5]
    # ties keep the lower index first: ranks 0, 1, 2, 3 = channels 0, 1, 2, 3
    assert O.balance_permutation(np.ones(4), 2).tolist() == [0, 2, 1, 3]
    with pytest.raises(ValueError):
        O.balance_permutation(np.ones(6), 4)


def test_balance_permutation_properties():
    rng = np.random.default_rng(3)
    d, k = 96, 8
    diag = np.exp(rng.uniform(np.log(1e-4), 0, d))
    perm = O.balance_permutation(diag, k)
    assert sorted(perm.tolist()) == list(range(d))
    sums = [diag[perm[b * k:(b + 1) * k]].sum() for b in range(d // k)]
    # dealt in descending order: block sums do not increase, and the first
    # and last differ by at most the largest entry
    assert all(a >= b - 1e-15 for a, b in zip(sums, sums[1:]))
    assert sums[0] - sums[-1] <= diag.max() + 1e-15
    P = O.permutation_matrix(perm)
    x = rng.standard_normal(d)
    assert np.array_equal(P @ x, x[perm])
    assert np.allclose(P @ P.T, np.eye(d))


def test_hg_blockwise_against_column_slices():
    rng = np.random.default_rng(4)
    N, d, k = 13, 6, 3
    G = rng.standard_normal((N, d))
    H = O.covariance(G)
    B = O.hg_blockwise(H, k)
    for b in range(0, d, k):
        for i in range(b, b + k):
            for j in range(b, b + k):
                s = sum(G[t, i] * G[t, j] for t in range(N)) / N
                assert abs(B[i, j] - s) < 1e-14
    assert not B[:3, 3:].any() and not B[3:, :3].any()
    assert np.array_equal(O.hg_blockwise(H, d), H)
    assert np.array_equal(O.hg_blockwise(H, 1), np.diag(np.diag(H)))


def test_hg_lowrank_eckart_young_and_order():
    rng = np.random.default_rng(5)
    d = 10
    A = rng.standard_normal((d, 3 * d)) * np.exp(rng.normal(0, 1, d))[:, None]
    H = A @ A.T / (3 * d)
    lam = np.sort(sla.eigvalsh(H))[::-1]
    assert np.allclose(O.hg_lowrank(H, d), H, atol=1e-12 * np.abs(H).max())
    D = rng.standard_normal((d, 7))
    HX = np.eye(7)
    prev = 0.0
    for r in (1, 3, 6, 10):
        Hr = O.hg_lowrank(H, r)
        # best rank-r error in the Frobenius norm is the tail of the spectrum
        assert np.isclose(np.linalg.norm(H - Hr) ** 2, np.sum(lam[r:] ** 2), rtol=1e-9, atol=1e-20)
        assert np.linalg.matrix_rank(Hr, tol=1e-10 * lam[0]) == r
        # H - H_r is positive semidefinite, so the loss grows with r up to the full one
        assert sla.eigvalsh(H - Hr).min() > -1e-12 * lam[0]
        L = O.kron_loss(D, 0 * D, HX, Hr)
        assert L >= prev - 1e-12
        prev = L
    assert np.isclose(prev, O.kron_loss(D, 0 * D, HX, H), rtol=1e-12)


def test_block_rht_matrix_orthogonal_and_blockwise():
    rng = np.random.default_rng(6)
    k, nb = 8, 3
    signs = np.where(rng.random(k) < 0.5, -1.0, 1.0)
    V = O.block_rht_matrix(k * nb, k, 3, signs)
    assert np.allclose(V @ V.T, np.eye(k * nb), atol=1e-14)
    Tk = O.rht_matrix(k, 3, signs)
    for b in range(nb):
        assert np.array_equal(V[b * k:(b + 1) * k, b * k:(b + 1) * k], Tk)
    assert not V[:k, k:].any()
    assert np.array_equal(O.block_rht_matrix(k, k, 3, signs), Tk)


def test_blockwise_loss_sample_form_and_special_cases():
    """sum_b tr(dW_b H_X dW_b^T H_G,b) with H_G,b the covariance of G's
    column block b equals (1/N^2) sum_b sum_{t,s} (g_{t,b}^T dW_b x_s)^2, is
    the full loss when H_G is block diagonal, and the full loss when k = d."""
    rng = np.random.default_rng(7)
    N, d_out, d_in, k = 9, 6, 5, 3
    X, G = rng.standard_normal((N, d_in)), rng.standard_normal((N, d_out))
    D = rng.standard_normal((d_out, d_in))
    HX, HG = O.covariance(X), O.covariance(G)
    blocks = np.stack([HG[b:b + k, b:b + k] for b in range(0, d_out, k)])
    s = 0.0
    for b in range(0, d_out, k):
        for t in range(N):
            for u in range(N):
                s += float(G[t, b:b + k] @ D[b:b + k] @ X[u]) ** 2
    got = O.blockwise_kron_loss(D, 0 * D, HX, blocks)
    assert np.isclose(got, s / N ** 2, rtol=1e-12)
    assert np.isclose(got, O.kron_loss(D, 0 * D, HX, O.hg_blockwise(HG, k)), rtol=1e-12)
    assert np.isclose(O.blockwise_kron_loss(D, 0 * D, HX, HG[None]), O.kron_loss(D, 0 * D, HX, HG), rtol=1e-12)


def test_weight_cv_hand_value_and_rotation():
    W = np.array([[3.0, 0.0], [0.0, 4.0]])
    assert np.isclose(O.weight_cv(W, "out"), 0.5 / 3.5)
    assert np.isclose(O.weight_cv(W, "in"), 0.5 / 3.5)
    assert O.weight_cv(np.ones((4, 4)), "out") == 0.0


def test_hg_informed_rotation_orthogonal_function_and_loss():
    """V = T P_G is orthogonal, keeps the layer's function, leaves the
    Kronecker loss unchanged, and with a block-diagonal T_k flattens the
    diagonal of the rotated H_G across blocks better than T_k alone (on this
    fixed draw: coefficient of variation 0.63 against 0.95)."""
    rng = np.random.default_rng(8)
    d_out, d_in, k = 32, 16, 8
    diagG = np.exp(rng.uniform(np.log(1e-4), 0, d_out))
    G = rng.standard_normal((400, d_out)) * np.sqrt(diagG)[None, :]
    HG = O.covariance(G)
    perm = O.balance_permutation(np.diag(HG), k)
    Pm = O.permutation_matrix(perm)
    sk = np.where(rng.random(k) < 0.5, -1.0, 1.0)
    Vk = O.block_rht_matrix(d_out, k, 3, sk)
    s_full = np.where(rng.random(d_out) < 0.5, -1.0, 1.0)
    T = O.rht_matrix(d_out, 5, s_full)
    U = O.rht_matrix(d_in, 4, np.where(rng.random(d_in) < 0.5, -1.0, 1.0))
    W = rng.normal(0, 0.02, (d_out, d_in))
    X = rng.standard_normal((50, d_in))
    HX = O.covariance(X)
    for V in (T @ Pm, Vk @ Pm):
        assert np.allclose(V @ V.T, np.eye(d_out), atol=1e-13)
        Wp, HXp, HGp = O.biip(W, HX, HG, U, V)
        x = rng.standard_normal(d_in)
        assert np.max(np.abs(V.T @ Wp @ U @ x - W @ x)) < 1e-12
        What = Wp + rng.normal(0, 1e-3, Wp.shape)
        back = V.T @ What @ U
        assert np.isclose(O.kron_loss(Wp, What, HXp, HGp), O.kron_loss(W, back, HX, HG), rtol=1e-10)
    spread = lambda M: np.std(np.diag(M)) / np.mean(np.diag(M))
    assert spread(Vk @ Pm @ HG @ Pm.T @ Vk.T) < 0.8 * spread(Vk @ HG @ Vk.T)


# --------------------------------------------------------------- act-order

def test_act_order_permutation_hand_values():
    H = np.diag([1.0, 5.0, 3.0, 5.0, 0.5])
    assert O.act_order_permutation(H).tolist() == [1, 3, 2, 0, 4]


def test_act_order_identity_when_already_sorted():
    """With the diagonal already descending the act-order solve is the
    natural-order solve."""
    rng = np.random.default_rng(21)
    d_out, d_in = 6, 10
    A = rng.standard_normal((d_in, 3 * d_in))
    H = A @ A.T / (3 * d_in)
    order = np.argsort(-np.diag(H), kind="stable")
    H = H[np.ix_(order, order)]
    W = rng.normal(0, 0.02, (d_out, d_in))
    q, perm, _ = O.quantize_layer_act_order(W, H, 3, 0, 4)
    assert perm.tolist() == list(range(d_in))
    Uc, dead, _ = O.chol_inv(H)
    ref = O.quantize_layer(W, Uc, 3, 0, 4, dead)
    assert np.array_equal(q.codes, ref.codes) and np.array_equal(q.W_hat, ref.W_hat)


def test_act_order_invariant_to_the_input_column_order():
    """Act-order depends on the diagonal, not on where a column sits: solving
    a layer whose columns were shuffled (W[:, s], H[s][:, s]) gives the same
    weights, shuffled the same way (distinct diagonal entries)."""
    rng = np.random.default_rng(22)
    d_out, d_in = 5, 12
    A = rng.standard_normal((d_in, 4 * d_in)) * np.exp(rng.normal(0, 1, d_in))[:, None]
    H = A @ A.T / (4 * d_in)
    W = rng.normal(0, 0.02, (d_out, d_in))
    s = rng.permutation(d_in)
    q1, p1, _ = O.quantize_layer_act_order(W, H, 2, 0, 4)
    q2, p2, _ = O.quantize_layer_act_order(W[:, s], H[np.ix_(s, s)], 2, 0, 4)
    assert np.array_equal(s[p2], p1)
    assert np.allclose(q2.W_hat, q1.W_hat[:, s], rtol=0, atol=1e-15)
    assert np.array_equal(q2.codes, q1.codes[:, s])


def test_act_order_least_squares_in_the_permuted_order():
    """The OBS property holds in the quantization order: after the solve, the
    last column's pre-rounding value equals W0 + (W0_p - W_hat_p) H_pr H_rr^-1
    for p = all earlier columns in act-order (damped H)."""
    rng = np.random.default_rng(23)
    d_out, d_in = 3, 7
    A = rng.standard_normal((d_in, 3 * d_in)) * np.exp(rng.normal(0, 1, d_in))[:, None]
    H = A @ A.T / (3 * d_in)
    W = rng.normal(0, 0.02, (d_out, d_in))
    q, perm, _ = O.quantize_layer_act_order(W, H, 3, 0, 128)
    Hd, _, _ = O.damp_and_dead(H[np.ix_(perm, perm)])
    Wp = W[:, perm]
    What_p = q.W_hat[:, perm]
    p, r = np.arange(d_in - 1), np.array([d_in - 1])
    cur = Wp[:, r] + (Wp[:, p] - What_p[:, p]) @ Hd[np.ix_(p, r)] @ np.linalg.inv(Hd[np.ix_(r, r)])
    scale, zero = q.scales[:, 0].astype(np.float64), q.zeros[:, 0].astype(np.float64)
    assert np.allclose(cur[:, 0] / scale + zero, q.V[:, perm[-1]], atol=1e-9)
