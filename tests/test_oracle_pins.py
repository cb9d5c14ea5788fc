"""Pins of the float64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: hand-worked
values (tests/golden), closed forms, brute force on tiny inputs, textbook
reductions and independent library routines.  CPU only.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg as sla

import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _spd(rng, n, cond_scale=1.0):
    A = rng.standard_normal((n, 2 * n))
    d = np.exp(rng.normal(0, cond_scale, n))
    A = A * d[:, None]
    return A @ A.T / (2 * n)


# --------------------------------------------------------------- covariance

def test_covariance_brute_force_loops():
    rng = np.random.default_rng(0)
    X = rng.standard_normal((7, 4))
    H = O.covariance(X)
    for i in range(4):
        for j in range(4):
            s = 0.0
            for t in range(7):
                s += X[t, i] * X[t, j]
            assert abs(H[i, j] - s / 7) < 1e-14


def test_covariance_symmetry_trace_and_chunks():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((1000, 33)).astype(np.float32)
    H = O.covariance(X, chunk=97)
    assert np.array_equal(H, H.T) or np.max(np.abs(H - H.T)) < 1e-15
    assert abs(np.trace(H) - np.sum(X.astype(np.float64) ** 2) / 1000) < 1e-10
    H2 = O.covariance_accumulate(O.covariance(X[:400], 1 / 1000), X[400:], 1 / 1000)
    assert np.max(np.abs(H - H2)) < 1e-13


def test_covariance_empty_tokens():
    H = O.covariance(np.zeros((0, 5)), alpha=1.0)
    assert H.shape == (5, 5) and not H.any()


# --------------------------------------------------------------- sensitivity

def test_sensitivity_golden():
    g = _gold("small_closed_forms.json")["sensitivity"]
    tX, tG, s = O.sensitivity(np.array(g["H_X"]), np.array(g["H_G"]))
    assert (tX, tG, s) == (g["tr_X"], g["tr_G"], g["s"])


def test_sensitivity_rotation_invariant():
    rng = np.random.default_rng(2)
    HX, HG = _spd(rng, 16), _spd(rng, 8)
    T_in = O.rht_matrix(16, 4, rng.choice([-1.0, 1.0], 16))
    T_out = O.rht_matrix(8, 3, rng.choice([-1.0, 1.0], 8))
    _, HXp, HGp = O.biip(np.zeros((8, 16)), HX, HG, T_in, T_out)
    a, b = O.sensitivity(HX, HG), O.sensitivity(HXp, HGp)
    assert np.allclose(a, b, rtol=1e-12)


# --------------------------------------------------------------- rotations

@pytest.mark.parametrize("p", [1, 2, 4, 8, 16, 64, 256])
def test_hadamard_matches_library(p):
    assert np.array_equal(O.sylvester_hadamard(p), sla.hadamard(p).astype(np.float64))


def test_rht_golden_n4():
    g = _gold("rht_n4.json")
    T = O.rht_matrix(4, 2, g["signs"])
    assert np.allclose(T, np.array(g["T"]), atol=0, rtol=0)


def _haar(rng, m):
    Q, R = np.linalg.qr(rng.standard_normal((m, m)))
    return Q * np.sign(np.diag(R))[None, :]


@pytest.mark.parametrize("n,k", [(64, 6), (24, 3), (56, 3), (43 * 4, 2)])
def test_rht_orthogonal(n, k):
    rng = np.random.default_rng(n)
    m = n >> k
    Q = None if m == 1 else _haar(rng, m)
    T = O.rht_matrix(n, k, rng.choice([-1.0, 1.0], n), Q)
    assert np.max(np.abs(T @ T.T - np.eye(n))) < 1e-12


def test_rht_kron_index_convention():
    # n = 3 * 2: element a*2 + b pairs row a of Q with row b of H_2.
    Q = np.array([[0.0, 1.0, 0.0], [0.0, 0.0, 1.0], [1.0, 0.0, 0.0]])  # a permutation
    T = O.rht_matrix(6, 1, np.ones(6), Q)
    x = np.arange(6, dtype=np.float64)  # pairs (0,1), (2,3), (4,5)
    r2 = math.sqrt(2.0)
    # Q moves pair 1 to slot 0, pair 2 to slot 1, pair 0 to slot 2; H_2/sqrt2 maps (u,v) -> (u+v, u-v)/sqrt2
    want = np.array([5, -1, 9, -1, 1, -1]) / r2
    assert np.allclose(T @ x, want, atol=1e-15)


def test_rotation_inverse_and_function_preserved():
    rng = np.random.default_rng(3)
    d_out, d_in = 24, 40
    W = rng.standard_normal((d_out, d_in))
    T_in = O.rht_matrix(d_in, 3, rng.choice([-1.0, 1.0], d_in), _haar(rng, 5))
    T_out = O.rht_matrix(d_out, 3, rng.choice([-1.0, 1.0], d_out), _haar(rng, 3))
    HX, HG = _spd(rng, d_in), _spd(rng, d_out)
    Wp, HXp, HGp = O.biip(W, HX, HG, T_in, T_out)
    x = rng.standard_normal(d_in)
    y = T_out.T @ (Wp @ (T_in @ x))
    assert np.max(np.abs(y - W @ x)) <= 1e-10
    back = O.rotate(O.rotate(Wp, "rows", T_out, inverse=True), "cols", T_in, inverse=True)
    assert np.max(np.abs(back - W)) < 1e-12
    assert abs(np.trace(HXp) - np.trace(HX)) < 1e-10 * np.trace(HX)
    assert abs(np.trace(HGp) - np.trace(HG)) < 1e-10 * np.trace(HG)
    # the loss is invariant: tr(dW' H_X' dW'^T H_G') = tr(dW H_X dW^T H_G)
    dW = rng.standard_normal((d_out, d_in)) * 1e-2
    dWp = T_out @ dW @ T_in.T
    assert np.isclose(O.kron_loss(dWp, 0 * dWp, HXp, HGp), O.kron_loss(dW, 0 * dW, HX, HG), rtol=1e-10)


# --------------------------------------------------------------- damping / cholesky

def test_damp_dead_golden():
    g = _gold("small_closed_forms.json")["damp"]
    H = np.diag(g["H_diag"])
    Uc, dead, lam = O.chol_inv(H, 0.01)
    assert list(dead) == g["dead"]
    assert abs(lam - g["lambda"]) < 1e-16
    assert np.allclose(np.diag(Uc), g["Uc_diag"], rtol=1e-14, atol=0)
    assert not np.any(np.triu(Uc, 1))


def test_chol_inv_identity_and_second_route():
    rng = np.random.default_rng(4)
    H = _spd(rng, 50, cond_scale=1.5)
    Uc, dead, lam = O.chol_inv(H, 0.01)
    Hd = H + lam * np.eye(50)
    assert not dead.any()
    assert np.allclose(np.tril(Uc, -1), 0)
    assert np.all(np.diag(Uc) > 0)
    assert np.max(np.abs(Uc.T @ Uc @ Hd - np.eye(50))) < 1e-9
    Uc2, _, _ = O.chol_inv_reversed(H, 0.01)
    assert np.max(np.abs(Uc - Uc2)) < 1e-9 * np.max(np.abs(Uc))
    # library cross-check: scipy's upper Cholesky of the inverse
    Ul = sla.cholesky(np.linalg.inv(Hd), lower=False)
    assert np.max(np.abs(Uc - Ul)) < 1e-9 * np.max(np.abs(Uc))


def test_chol_inv_not_pd_raises():
    H = np.diag([1.0, -5.0, 1.0])
    with pytest.raises(np.linalg.LinAlgError):
        O.chol_inv(H, 0.01)


# --------------------------------------------------------------- grid

def test_grid_golden():
    for c in _gold("grid_examples.json")["cases"]:
        w = np.array(c["w"], dtype=np.float32)
        sc, zr = O.fit_grid(w.min(), w.max(), c["bits"])
        assert float(sc) == c["scale"], c["name"]
        assert float(zr) == c["zero"], c["name"]
        v, q = O.quantize_codes(w, sc, zr, c["bits"])
        assert list(q.astype(int)) == c["codes"], c["name"]
        assert np.array_equal(O.dequantize(q, sc, zr), np.array(c["w_hat"])), c["name"]


def test_rtn_is_nearest_grid_point():
    """Brute force over all levels: the code is the nearest representable value."""
    rng = np.random.default_rng(5)
    for bits in (2, 3, 4):
        w = rng.standard_normal(2000).astype(np.float32)
        sc, zr = O.fit_grid(w.min(), w.max(), bits)
        _, q = O.quantize_codes(w, sc, zr, bits)
        levels = float(sc) * (np.arange(2 ** bits) - float(zr))
        best = np.argmin(np.abs(w.astype(np.float64)[:, None] - levels[None, :]), axis=1)
        assert np.array_equal(q.astype(int), best)


def test_rounding_noise_variance():
    """Uniform rounding noise: E[(w - w_hat)^2] / step^2 = 1/12 (within 5%)."""
    rng = np.random.default_rng(6)
    W = rng.standard_normal((256, 4096))
    res = O.quantize_layer(W, np.eye(4096), 4, group=0)
    r = (W - res.W_hat) / res.scales[:, :1]
    assert abs(np.mean(r ** 2) * 12 - 1) < 0.05


# --------------------------------------------------------------- solver

def test_solver_reduces_to_rtn_when_hx_identity():
    rng = np.random.default_rng(7)
    W = rng.normal(0, 0.02, (40, 300))
    Uc, dead, _ = O.chol_inv(np.eye(300), 0.01)
    for bits in (2, 3, 4):
        for group in (0, 64):
            res = O.quantize_layer(W, Uc, bits, group=group, block=128)
            for r in range(40):
                for g0 in range(0, 300, group or 300):
                    seg = W[r, g0:g0 + (group or 300)].astype(np.float32)
                    sc, zr = O.fit_grid(seg.min(), seg.max(), bits)
                    _, q = O.quantize_codes(seg, sc, zr, bits)
                    assert np.array_equal(res.codes[r, g0:g0 + len(seg)], q.astype(np.uint8))


def test_solver_golden_three_columns():
    g = _gold("obs_three_columns.json")
    Uc, _, _ = O.chol_inv(np.array(g["H"]), g["damp"])
    res = O.quantize_layer(np.array(g["W"]), Uc, g["bits"], snapshot_cols=(0, 1))
    assert float(res.scales[0, 0]) == g["scale"] and float(res.zeros[0, 0]) == g["zero"]
    assert np.allclose(res.snapshots[0][0], g["after_col0"], atol=1e-15)
    assert np.allclose(res.snapshots[1][0], g["after_col1"], atol=1e-15)
    assert list(res.codes[0]) == g["codes"]
    assert np.allclose(res.W_hat[0], g["w_hat"], atol=0)


def test_solver_equals_least_squares_resolve():
    """OBS optimality: after fixing the prefix p, the remaining weights solve the
    least-squares problem  w_r = w0_r + (w0_p - w_hat_p) H_pr H_rr^-1."""
    rng = np.random.default_rng(8)
    d_out, d_in = 6, 23
    W = rng.normal(0, 0.02, (d_out, d_in))
    H = _spd(rng, d_in, 1.0)
    Uc, _, lam = O.chol_inv(H, 0.01)
    Hd = H + lam * np.eye(d_in)
    cols = (0, 3, 4, 9, 15, 21)
    res = O.quantize_layer(W, Uc, 2, block=5, snapshot_cols=cols)
    for j in cols:
        p, r = slice(0, j + 1), slice(j + 1, d_in)
        want = W[:, r] + (W[:, p] - res.W_hat[:, p]) @ Hd[p, r] @ np.linalg.inv(Hd[r, r])
        assert np.max(np.abs(res.snapshots[j][:, r] - want)) < 1e-12


def test_solver_blocking_invariant():
    rng = np.random.default_rng(9)
    W = rng.normal(0, 0.02, (10, 70))
    H = _spd(rng, 70, 1.0)
    Uc, _, _ = O.chol_inv(H, 0.01)
    a = O.quantize_layer(W, Uc, 3, block=128)
    for b in (1, 3, 16):
        c = O.quantize_layer(W, Uc, 3, block=b)
        assert np.array_equal(a.codes, c.codes)
        assert np.max(np.abs(a.V - c.V)) < 1e-10
    g1 = O.quantize_layer(W, Uc, 3, group=8, block=8)
    g2 = O.quantize_layer(W, Uc, 3, group=8, block=32)
    assert np.array_equal(g1.codes, g2.codes) and np.array_equal(g1.zeros, g2.zeros)


def test_hg_cancels_full_kronecker_resolve():
    """Proposition 1: re-solving the remaining weights under the full Kronecker
    Hessian H_G kron H_X (row-major vec) gives the H_X-only OBS update."""
    rng = np.random.default_rng(10)
    d_out, d_in = 4, 9
    W = rng.normal(0, 0.02, (d_out, d_in))
    HX = _spd(rng, d_in, 1.0)
    HG = _spd(rng, d_out, 1.0)
    Uc, _, lam = O.chol_inv(HX, 0.01)
    HXd = HX + lam * np.eye(d_in)
    K = np.kron(HG, HXd)                      # index r * d_in + c
    cols = (0, 2, 5)
    res = O.quantize_layer(W, Uc, 2, block=4, snapshot_cols=cols)
    for j in cols:
        fixed = np.zeros((d_out, d_in), bool)
        fixed[:, :j + 1] = True
        f, u = fixed.reshape(-1), ~fixed.reshape(-1)
        dfix = (res.W_hat - W).reshape(-1)[f]
        du = -np.linalg.solve(K[np.ix_(u, u)], K[np.ix_(u, f)] @ dfix)
        want = W.reshape(-1)[u] + du
        got = res.snapshots[j].reshape(-1)[u]
        assert np.max(np.abs(got - want)) < 1e-12


def test_exhaustive_search_bounds_gptq():
    """Tiny layers: no code assignment on the same grid beats the exhaustive
    minimum; with H_X diagonal and H_G = I the problem separates and GPTQ
    (then plain RTN) attains it exactly."""
    rng = np.random.default_rng(11)
    bits = 2
    for trial in range(4):
        W = rng.normal(0, 1, (2, 4))
        HX = _spd(rng, 4, 0.5) if trial else np.diag(rng.uniform(0.5, 2, 4))
        HG = np.eye(2) if trial == 0 else _spd(rng, 2, 0.5)
        Uc, _, lam = O.chol_inv(HX, 0.0)
        res = O.quantize_layer(W, Uc, bits)
        sc, zr = res.scales[:, 0].astype(np.float64), res.zeros[:, 0].astype(np.float64)
        best = np.inf
        for combo in itertools.product(range(4), repeat=8):
            q = np.array(combo, dtype=np.float64).reshape(2, 4)
            Wh = sc[:, None] * (q - zr[:, None])
            best = min(best, O.kron_loss(W, Wh, HX, HG))
        got = O.kron_loss(W, res.W_hat, HX, HG)
        assert got >= best - 1e-12
        if trial == 0:
            assert abs(got - best) < 1e-12


def test_forced_code_excusal():
    """A disagreement is excused only within tol of a boundary and to an
    adjacent code; any other disagreement is reported."""
    rng = np.random.default_rng(12)
    W = rng.normal(0, 0.02, (3, 8))
    Uc = np.eye(8)
    base = O.quantize_layer(W, Uc, 2)
    sc, zr = float(base.scales[0, 0]), float(base.zeros[0, 0])
    W2 = W.copy()
    W2[0, 5] = sc * (1.5 + 2e-6 - zr)      # v = 1.5 + 2e-6: oracle rounds to 2
    ref = O.quantize_layer(W2, Uc, 2)
    assert ref.codes[0, 5] == 2
    forced = ref.codes.copy()
    forced[0, 5] = 1                        # the other adjacent code: excused
    forced[1, 2] = (forced[1, 2] + 2) % 4   # far from a boundary: reported
    out = O.quantize_layer(W2, Uc, 2, force_codes=forced)
    assert out.excused == 1 and out.codes[0, 5] == 1
    assert len(out.mismatches) == 1 and out.mismatches[0][:2] == (1, 2)
    tight = O.quantize_layer(W2, Uc, 2, force_codes=forced, excuse_tol=1e-6)
    assert tight.excused == 0 and len(tight.mismatches) == 2


# --------------------------------------------------------------- loss

def test_kron_loss_golden_and_identity_case():
    g = _gold("small_closed_forms.json")["kron_loss"]
    dW, HX, HG = np.array(g["dW"]), np.array(g["H_X"]), np.array(g["H_G"])
    assert O.kron_loss(dW, 0 * dW, HX, HG) == g["loss"]
    assert O.gptq_loss(dW, 0 * dW, HX) == g["loss_gptq"]


def test_kron_loss_single_entry_and_library_kron():
    rng = np.random.default_rng(13)
    HX, HG = _spd(rng, 7), _spd(rng, 5)
    D = np.zeros((5, 7))
    D[3, 2] = 0.7
    assert np.isclose(O.kron_loss(D, 0 * D, HX, HG), 0.49 * HX[2, 2] * HG[3, 3], rtol=1e-14)
    D = rng.standard_normal((5, 7))
    v = D.reshape(-1)
    assert np.isclose(O.kron_loss(D, 0 * D, HX, HG), v @ np.kron(HG, HX) @ v, rtol=1e-12)
    assert np.isclose(O.kron_loss(D, 0 * D, HX, None), v @ np.kron(np.eye(5), HX) @ v, rtol=1e-12)
    assert O.kron_loss(D, 0 * D, HX, HG) >= 0


def test_kron_loss_from_samples():
    """With H_X = X^T X / N and H_G = G^T G / N the loss equals
    (1/N^2) sum_{t,s} (g_t^T dW x_s)^2."""
    rng = np.random.default_rng(14)
    N = 11
    X, G = rng.standard_normal((N, 6)), rng.standard_normal((N, 4))
    D = rng.standard_normal((4, 6))
    s = 0.0
    for t in range(N):
        for u in range(N):
            s += float(G[t] @ D @ X[u]) ** 2
    L = O.kron_loss(D, 0 * D, O.covariance(X), O.covariance(G))
    assert np.isclose(L, s / N ** 2, rtol=1e-12)


# --------------------------------------------------------------- allocation

def test_allocation_golden():
    for c in _gold("small_closed_forms.json")["allocation"]:
        b = O.allocate_bits(c["sens"], c["n_params"], (2, 3, 4), c["avg"])
        assert list(b) == c["bits"]


def test_allocation_brute_force_lexicographic():
    """The greedy equals the lexicographically largest feasible assignment in
    descending-score order (brute force over all 3^5 assignments)."""
    rng = np.random.default_rng(15)
    for _ in range(30):
        k = 5
        s = rng.uniform(0, 1, k)
        n = rng.integers(1, 5, k)
        avg = float(rng.choice([2.4, 2.8, 3.0, 3.3]))
        order = sorted(range(k), key=lambda i: (-s[i], i))
        best = None
        for combo in itertools.product((2, 3, 4), repeat=k):
            if sum(n[i] * (combo[i] - 2) for i in range(k)) <= round(n.sum() * (avg - 2), 9) // 1:
                key = tuple(combo[i] for i in order)
                if best is None or key > best[0]:
                    best = (key, combo)
        got = O.allocate_bits(s, n, (2, 3, 4), avg)
        assert tuple(got) == best[1]
        assert (got * n).sum() <= avg * n.sum() + 1e-9


def test_allocation_monotone_equal_sizes():
    rng = np.random.default_rng(16)
    s = rng.uniform(0, 1, 20)
    b = O.allocate_bits(s, np.full(20, 7), (2, 3, 4), 3.0)
    order = np.argsort(-s)
    assert np.all(np.diff(b[order]) <= 0)
    assert b.mean() == 3.0
