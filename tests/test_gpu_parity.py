"""Parity of every C-ABI entry point with the float64 oracle, on the GPU.

Each stage is compared on the same inputs: the oracle receives the bits the
kernel received (bf16 X/G, fp32 W', H', Uc).  Sizes span several tiles and
ragged tails (d_out = 352 = 11*32, d_in = 704 = 11*64, N = 3000).

Tolerances (written out per test):
  covariances  Frobenius relative <= 1e-4 and |dH_ij| <= 1e-4 sqrt(H_ii H_jj);
  codes        identical except where the oracle's pre-rounding value lies
               within 1e-5 grid steps of a rounding boundary, and >= 99.9%
               identical;
  W_hat, loss  within 1e-3 relative;
  rotations    per vector ||dv|| <= 4e-6 ||v|| (fp32 butterflies: about
               (log2 p + m) unit roundoffs of the vector norm);
  Uc           |dUc_ij| <= 4e-7 |Uc_ij| + 1e-8 max_j |Uc_ij| (fp64 inside,
               one fp32 rounding at the end);
  traces       1e-12 relative (fp64 sums of the same fp32 diagonal).
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from gpu_util import cov_close, device_rht, need_gpu, np64, oracle_T

pytestmark = pytest.mark.gpu

SMALL = synth.scaled(synth.WORKLOADS["attn4096"], d_out=352, d_in=704, n_tokens=3000)


@pytest.fixture(scope="module")
def P():
    need_gpu()
    import post_weight_quantization_syrk_b200 as P
    P.load()
    return P


def _info():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _info_code(info):
    v = int(info.item())
    return (v >> 24) & 0xFF, v & 0xFFFFFF


# ------------------------------------------------------------------ covariance

@pytest.mark.parametrize("spec,seed", [(SMALL, 1), (synth.WORKLOADS["layer512"], 2),
                                       (synth.scaled(synth.WORKLOADS["mlp_down11008"], 64, 200, 777), 3),
                                       (synth.scaled(synth.WORKLOADS["down28672"], 64, 136, 1000), 4)])
def test_accum_cov_parity(P, spec, seed):
    X = synth.activations(spec, seed)
    G = synth.gradients(spec, seed)
    for A in (X, G):
        d = A.shape[1]
        C = torch.full((d, d), float("nan"), device="cuda")
        info = _info()
        P.kq_accum_cov(A.cuda(), C, 1.0 / A.shape[0], False, None, info)
        torch.cuda.synchronize()
        assert _info_code(info)[0] == 0
        ref = O.covariance(A.float().numpy())
        fro, ent = cov_close(np64(C), ref)
        assert fro <= 1e-4 and ent <= 1e-4, (fro, ent)
        assert torch.equal(C, C.T)


def test_accum_cov_streaming_and_empty(P):
    X = synth.activations(SMALL, 5).cuda()
    n = X.shape[0]
    C = torch.zeros((704, 704), device="cuda")
    info = _info()
    for t0 in range(0, n, 1100):
        P.kq_accum_cov(X[t0:t0 + 1100], C, 1.0 / n, t0 > 0, None, info)
    ref = O.covariance(X.cpu().float().numpy())
    fro, ent = cov_close(np64(C), ref)
    assert fro <= 1e-4 and ent <= 1e-4
    before = C.clone()
    P.kq_accum_cov(X[:0], C, 1.0, True, None, info)        # no tokens, accumulate: unchanged
    assert torch.equal(C, before)
    P.kq_accum_cov(X[:0], C, 1.0, False, None, info)       # no tokens, overwrite: zero
    assert not C.any()
    X8 = X[:, :8].contiguous()
    c1 = torch.zeros((1, 1), device="cuda")
    P.kq_accum_cov(X8[:, :1], c1, 1.0 / n, False, None, info)   # d = 1 (lda 8)
    torch.cuda.synchronize()
    assert _info_code(info)[0] == 0
    assert abs(c1.item() - float((X8[:, 0].double() ** 2).mean())) <= 1e-5 * c1.item()


def test_accum_cov_nonfinite_reported(P):
    X = synth.activations(SMALL, 6).cuda()
    X[17, 5] = float("inf")
    C = torch.zeros((704, 704), device="cuda")
    info = _info()
    P.kq_accum_cov(X, C, 1.0 / X.shape[0], False, None, info)
    code, _ = _info_code(info)
    assert code == 7


def test_accum_cov_wait_timeout_reported_then_recovers(P):
    """Failure detection without a fault: with the device-wait limit at 0 the
    SYRK's pipeline waits give up at their first incomplete poll, the call
    records KQ_ERR_TIMEOUT (index = the wait's site) in info, and the kernel
    drains its own copies and products with the normal bound before it frees
    its tensor memory and returns.  The context stays usable: the next call
    with the default limit matches the oracle."""
    X = synth.activations(SMALL, 7).cuda()
    n = X.shape[0]
    C = torch.zeros((704, 704), device="cuda")
    info = _info()
    old = P.kq_set_wait_limit_ns(0)
    try:
        P.kq_accum_cov(X, C, 1.0 / n, False, None, info)
        torch.cuda.synchronize()
    finally:
        P.kq_set_wait_limit_ns(old)
    assert old == P.KQ_WAIT_LIMIT_DEFAULT_NS
    code, where = _info_code(info)
    assert code == 8 and where in (1, 2, 3, 4), (code, where)
    info.zero_()
    C.fill_(float("nan"))
    P.kq_accum_cov(X, C, 1.0 / n, False, None, info)
    torch.cuda.synchronize()
    assert _info_code(info)[0] == 0
    fro, ent = cov_close(np64(C), O.covariance(X.cpu().float().numpy()))
    assert fro <= 1e-4 and ent <= 1e-4, (fro, ent)


# ------------------------------------------------------------------ sensitivity

def test_sensitivity_parity(P):
    rng = np.random.default_rng(0)
    HX = torch.from_numpy(rng.standard_normal((300, 300)).astype(np.float32)).cuda()
    HG = torch.from_numpy(rng.standard_normal((77, 77)).astype(np.float32)).cuda()
    out = torch.zeros(3, dtype=torch.float64, device="cuda")
    P.kq_sensitivity(HX, HG, out)
    ref = O.sensitivity(np64(HX), np64(HG))
    assert np.allclose(out.cpu().numpy(), ref, rtol=1e-12, atol=0)


# ------------------------------------------------------------------ rotations

@pytest.mark.parametrize("n", [512, 704, 352, 43 * 256, 7 * 4096 // 8, 96, 5, 4096, 2048, 16, 8, 7 * 1024, 8192])
@pytest.mark.parametrize("axis", ["rows", "cols"])
@pytest.mark.parametrize("inverse", [False, True])
def test_rotate_parity(P, n, axis, inverse):
    other = 80
    params = synth.rht_params(n, 1000 + n)
    T = oracle_T(params)
    rng = np.random.default_rng(n)
    shape = (n, other) if axis == "rows" else (other, n)
    M = rng.standard_normal(shape).astype(np.float32)
    pad = -shape[1] % 4                      # keep ld a multiple of 4
    buf = torch.zeros((shape[0], shape[1] + pad), device="cuda")
    Mg = buf[:, :shape[1]]
    Mg.copy_(torch.from_numpy(M))
    P.kq_rotate(Mg, P.KQ_AXIS_ROWS if axis == "rows" else P.KQ_AXIS_COLS, device_rht(params), inverse)
    ref = O.rotate(M.astype(np.float64), axis, T, inverse)
    got = np64(Mg)
    ax = 0 if axis == "rows" else 1
    err = np.linalg.norm(got - ref, axis=ax) / np.linalg.norm(ref, axis=ax)
    assert err.max() <= 4e-6, err.max()


def test_rotate_roundtrip_and_biip_function(P):
    spec = SMALL
    W = synth.weights(spec, 7)
    Ti, To = synth.rht_params(spec.d_in, 71), synth.rht_params(spec.d_out, 72)
    Wg = W.cuda().clone()
    P.kq_rotate(Wg, P.KQ_AXIS_COLS, device_rht(Ti))
    P.kq_rotate(Wg, P.KQ_AXIS_ROWS, device_rht(To))
    Wp_ref = oracle_T(To) @ W.double().numpy() @ oracle_T(Ti).T
    assert np.linalg.norm(np64(Wg) - Wp_ref) / np.linalg.norm(Wp_ref) < 2e-6
    P.kq_rotate(Wg, P.KQ_AXIS_ROWS, device_rht(To), True)
    P.kq_rotate(Wg, P.KQ_AXIS_COLS, device_rht(Ti), True)
    back = np64(Wg)
    # the fp32 Q_m is orthogonal to ~1e-7, so the round trip returns W to ~1e-6
    assert np.linalg.norm(back - W.double().numpy()) / np.linalg.norm(W.double().numpy()) < 4e-6


# ------------------------------------------------------------------ cholesky

def _spd(n, seed, cond_scale=1.5):
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((n, n + 16)) * np.exp(rng.normal(0, cond_scale, n))[:, None]
    return (A @ A.T / (n + 16)).astype(np.float32)


def _uc_ok(got, ref):
    rowmax = np.max(np.abs(ref), axis=1, keepdims=True)
    tol = 4e-7 * np.abs(ref) + 1e-8 * rowmax
    return np.max(np.abs(got - ref) - tol)


@pytest.mark.parametrize("n,seed", [(1, 0), (63, 1), (64, 2), (200, 3), (704, 4), (1000, 5), (1537, 6)])
def test_chol_inv_parity(P, n, seed):
    H = _spd(n, seed)
    Hg = torch.from_numpy(H).cuda()
    Uc = torch.full((n, n), float("nan"), device="cuda")
    dead = torch.full((n,), 7, dtype=torch.uint8, device="cuda")
    info = _info()
    P.kq_chol_inv(Hg, 0.01, Uc, dead, None, info)
    torch.cuda.synchronize()
    assert _info_code(info)[0] == 0
    ref, dref, _ = O.chol_inv(H.astype(np.float64), 0.01)
    assert _uc_ok(np64(Uc), ref) <= 0
    assert np.array_equal(dead.cpu().numpy().astype(bool), dref)


def test_chol_inv_grouped_bulk_update_residual(P):
    """From n = 8192 the bulk update runs once every four block steps; at
    n = 8200 (129 blocks of 64, the last one 8 wide) the last group of steps
    is incomplete.  A residual pin of the whole factor in fp64, for the first
    64, the last 64 and 64 random columns j: ||(Uc^T Uc (H + lambda I) - I) e_j||
    <= 2e-6 (H from 4n samples, so the exact factor rounded to fp32 leaves
    about 1e-7)."""
    n = 8200
    g = torch.Generator(device="cuda")
    g.manual_seed(41)
    A = torch.randn((n, 4 * n), device="cuda", generator=g)
    H = (A @ A.T) / (4 * n)
    del A
    Uc = torch.empty_like(H)
    info = _info()
    P.kq_chol_inv(H, 0.01, Uc, None, None, info)
    torch.cuda.synchronize()
    assert _info_code(info)[0] == 0
    lam = 0.01 * float(torch.diagonal(H).double().mean())
    rng = np.random.default_rng(43)
    S = np.unique(np.r_[np.arange(64), np.arange(n - 64, n), rng.choice(n, 64, replace=False)])
    St = torch.from_numpy(S).cuda()
    Hs = torch.triu(H.double())[:, St] + torch.triu(H.double(), 1).T[:, St]   # columns of the symmetric H
    Hs[St, torch.arange(len(S), device="cuda")] += lam
    U = Uc.double()
    R = U.T @ (U @ Hs)
    R[St, torch.arange(len(S), device="cuda")] -= 1.0
    r = torch.linalg.vector_norm(R, dim=0).cpu().numpy()
    assert float(torch.tril(Uc, -1).abs().max()) == 0.0
    assert r.max() <= 2e-6, (float(r.max()), int(S[int(np.argmax(r))]))


def test_chol_inv_dead_columns_and_errors(P):
    H = _spd(150, 9)
    H[[3, 77, 149], :] = 0
    H[:, [3, 77, 149]] = 0
    Uc = torch.zeros((150, 150), device="cuda")
    dead = torch.zeros(150, dtype=torch.uint8, device="cuda")
    info = _info()
    P.kq_chol_inv(torch.from_numpy(H).cuda(), 0.01, Uc, dead, None, info)
    torch.cuda.synchronize()
    assert _info_code(info)[0] == 0
    ref, dref, _ = O.chol_inv(H.astype(np.float64), 0.01)
    assert list(np.flatnonzero(dead.cpu().numpy())) == [3, 77, 149] == list(np.flatnonzero(dref))
    assert _uc_ok(np64(Uc), ref) <= 0
    # not positive definite
    Hn = -np.eye(100, dtype=np.float32)
    info = _info()
    P.kq_chol_inv(torch.from_numpy(Hn).cuda(), 0.01, torch.zeros((100, 100), device="cuda"), None, None, info)
    assert _info_code(info)[0] == 6
    # NaN input
    Hq = _spd(70, 10)
    Hq[5, 9] = np.nan
    info = _info()
    P.kq_chol_inv(torch.from_numpy(Hq).cuda(), 0.01, torch.zeros((70, 70), device="cuda"), None, None, info)
    assert _info_code(info)[0] == 7


# ------------------------------------------------------------------ quantize

def _quant_case(P, W, Uc, dead, bits, group, gemm_mode=None):
    d_out, d_in = W.shape
    ng = 1 if not group else -(-d_in // group)
    codes = torch.empty((d_out, d_in), dtype=torch.uint8, device="cuda")
    scales = torch.empty((d_out, ng), device="cuda")
    zeros = torch.empty((d_out, ng), device="cuda")
    W_hat = torch.empty((d_out, d_in), device="cuda")
    info = _info()
    mode = P.KQ_GEMM_FP32 if gemm_mode is None else gemm_mode
    P.kq_quantize_layer(W, Uc, dead, bits, group, codes, scales, zeros, W_hat, gemm_mode=mode, info=info)
    torch.cuda.synchronize()
    assert _info_code(info)[0] == 0
    return codes.cpu().numpy(), scales.cpu().numpy(), zeros.cpu().numpy(), np64(W_hat)


def excuse_tol(bits):
    """1e-5 grid steps for the pages' bit-widths (W2..W4).  The solver's fp32
    rounding error is absolute in w, so in grid steps it grows with
    2^b - 1; above 4 bits the tolerance is scaled by (2^b - 1) / 15."""
    return 1e-5 * max(1.0, (2 ** bits - 1) / 15.0)


def _check_quant(W, Uc, dead, bits, group, got):
    codes, scales, zeros, W_hat = got
    ref = O.quantize_layer(np64(W), np64(Uc), bits, group, 128,
                           dead=None if dead is None else dead.cpu().numpy().astype(bool),
                           force_codes=codes, force_zeros=zeros if group else None, excuse_tol=excuse_tol(bits))
    assert ref.mismatches == [], ref.mismatches[:5]
    assert ref.zero_mismatches == [], ref.zero_mismatches[:5]
    # in forced-code mode every non-excused code is identical; excused flips
    # are the only differences and must stay under 0.1%
    same = 1.0 - ref.excused / codes.size
    assert same >= 0.999, same
    if not group:
        assert np.array_equal(scales, ref.scales) and np.array_equal(zeros, ref.zeros)
    else:
        assert np.max(np.abs(scales / ref.scales - 1)) <= 1e-5
    rel = np.linalg.norm(W_hat - ref.W_hat) / np.linalg.norm(ref.W_hat)
    assert rel <= 1e-3, rel
    return ref


@pytest.fixture(scope="module")
def rotated_small(P):
    """The GPU's own rotated W' and factor Uc for the SMALL layer."""
    from post_weight_quantization_syrk_b200.pipeline import LayerQuantizer
    W, X, G, Ti, To = synth.layer(SMALL, 11)
    lq = LayerQuantizer(SMALL.d_out, SMALL.d_in)
    lq.statistics(X.cuda(), G.cuda())
    lq.rotate(W.cuda(), device_rht(Ti), device_rht(To))
    lq.factor(0.01)
    torch.cuda.synchronize()
    lq.check()
    return lq, (W, X, G, Ti, To)


@pytest.mark.parametrize("bits,group", [(2, 0), (3, 0), (4, 0), (3, 128), (2, 128), (8, 0), (4, 32)])
@pytest.mark.parametrize("mode", ["fp32", "3xtf32"])
def test_quantize_parity(P, rotated_small, bits, group, mode):
    lq, _ = rotated_small
    gm = P.KQ_GEMM_FP32 if mode == "fp32" else P.KQ_GEMM_3XTF32
    got = _quant_case(P, lq.Wp, lq.Uc, lq.dead, bits, group, gm)
    _check_quant(lq.Wp, lq.Uc, lq.dead, bits, group, got)


def test_quantize_identity_hessian_is_rtn(P):
    rng = np.random.default_rng(3)
    W = torch.from_numpy(rng.normal(0, 0.02, (100, 300)).astype(np.float32)).cuda()
    Uc = torch.zeros((300, 300), device="cuda")
    P.kq_chol_inv(torch.eye(300, device="cuda"), 0.01, Uc, None, None, _info())
    for bits in (2, 3, 4):
        codes, scales, zeros, W_hat = _quant_case(P, W, Uc, None, bits, 0)
        Wn = np64(W)
        sc, zr = O.fit_grid(W.cpu().numpy().min(1), W.cpu().numpy().max(1), bits)
        _, q = O.quantize_codes(Wn, sc[:, None], zr[:, None], bits)
        assert np.array_equal(codes, q.astype(np.uint8))


def test_quantize_dead_columns_degenerate_rows(P):
    """Dead columns, an all-zero row (zero-width range in every group: scale 1)
    and ragged d_out / d_in.  A constant non-zero row is not used with groups:
    after the OBS updates its later groups have a range at rounding-noise
    level, where the grid itself is decided by noise on either side."""
    rng = np.random.default_rng(4)
    d_out, d_in = 70, 260
    W = rng.normal(0, 0.02, (d_out, d_in)).astype(np.float32)
    W[5, :] = 0.0                        # degenerate row: zero-width range
    H = _spd(d_in, 12, 1.0)
    H[[0, 130], :] = 0
    H[:, [0, 130]] = 0
    Uc = torch.zeros((d_in, d_in), device="cuda")
    dead = torch.zeros(d_in, dtype=torch.uint8, device="cuda")
    P.kq_chol_inv(torch.from_numpy(H).cuda(), 0.01, Uc, dead, None, _info())
    Wg = torch.from_numpy(W).cuda()
    for group in (0, 128):
        for gm in (P.KQ_GEMM_FP32, P.KQ_GEMM_3XTF32):
            got = _quant_case(P, Wg, Uc, dead, 3, group, gm)
            _check_quant(Wg, Uc, dead, 3, group, got)


def test_quantize_constant_row_per_channel(P):
    """A constant non-zero row under the per-channel grid (fitted once on the
    initial row): scale 1, zero rint(-c)."""
    rng = np.random.default_rng(5)
    W = rng.normal(0, 0.02, (40, 256)).astype(np.float32)
    W[7, :] = 0.25
    Uc = torch.zeros((256, 256), device="cuda")
    P.kq_chol_inv(torch.from_numpy(_spd(256, 13, 1.0)).cuda(), 0.01, Uc, None, None, _info())
    Wg = torch.from_numpy(W).cuda()
    got = _quant_case(P, Wg, Uc, None, 2, 0)
    assert got[1][7, 0] == 1.0 and got[2][7, 0] == 0.0
    _check_quant(Wg, Uc, None, 2, 0, got)


def test_quantize_nonfinite_reported(P):
    W = torch.zeros((40, 200), device="cuda")
    W[3, 150] = float("nan")
    Uc = torch.zeros((200, 200), device="cuda")
    P.kq_chol_inv(torch.eye(200, device="cuda"), 0.01, Uc, None, None, _info())
    info = _info()
    P.kq_quantize_layer(W, Uc, None, 2, 0, torch.empty((40, 200), dtype=torch.uint8, device="cuda"),
                        torch.empty((40, 1), device="cuda"), torch.empty((40, 1), device="cuda"),
                        torch.empty((40, 200), device="cuda"), info=info)
    assert _info_code(info) == (7, 3)


# ------------------------------------------------------------------ loss

@pytest.mark.parametrize("d_out,d_in", [(352, 704), (200, 136), (40, 300), (513, 260)])
@pytest.mark.parametrize("with_hg", [True, False])
def test_kron_loss_shapes(P, d_out, d_in, with_hg):
    """Ragged tile edges and K tails of the tensor-core products."""
    rng = np.random.default_rng(d_out * 7 + d_in)
    W = rng.normal(0, 0.02, (d_out, d_in)).astype(np.float32)
    Wh = (W + rng.normal(0, 0.004, W.shape)).astype(np.float32)
    HX = _spd(d_in, 1, 1.0)
    HG = _spd(d_out, 2, 1.0)
    loss = torch.zeros(1, dtype=torch.float64, device="cuda")
    P.kq_kron_loss(torch.from_numpy(W).cuda(), torch.from_numpy(Wh).cuda(), torch.from_numpy(HX).cuda(),
                   torch.from_numpy(HG).cuda() if with_hg else None, loss)
    ref = O.kron_loss(W.astype(np.float64), Wh.astype(np.float64), HX.astype(np.float64),
                      HG.astype(np.float64) if with_hg else None)
    assert abs(loss.item() - ref) <= 1e-3 * abs(ref), (loss.item(), ref)


@pytest.mark.parametrize("with_hg", [True, False])
def test_kron_loss_parity(P, rotated_small, with_hg):
    lq, _ = rotated_small
    got = _quant_case(P, lq.Wp, lq.Uc, lq.dead, 2, 0)
    W_hat = torch.from_numpy(got[3].astype(np.float32)).cuda()
    loss = torch.zeros(1, dtype=torch.float64, device="cuda")
    P.kq_kron_loss(lq.Wp, W_hat, lq.H_X, lq.H_G if with_hg else None, loss)
    ref = O.kron_loss(np64(lq.Wp), np64(W_hat), np64(lq.H_X), np64(lq.H_G) if with_hg else None)
    assert abs(loss.item() - ref) <= 1e-3 * abs(ref), (loss.item(), ref)


# ------------------------------------------------------------------ whole layer

def test_layer512_whole_path_stagewise(P):
    """The 512x512 layer end to end; each stage against the oracle on the
    previous stage's GPU output, plus the oracle's own end-to-end loss."""
    from post_weight_quantization_syrk_b200.pipeline import LayerQuantizer
    spec = synth.WORKLOADS["layer512"]
    W, X, G, Ti, To = synth.layer(spec, synth.layer_seed(1))
    lq = LayerQuantizer(spec.d_out, spec.d_in)
    res = lq.run(W.cuda(), X.cuda(), G.cuda(), device_rht(Ti), device_rht(To), [(3, 0)])
    torch.cuda.synchronize()
    lq.check()
    Xn, Gn = X.float().numpy(), G.float().numpy()
    HX, HG = O.covariance(Xn), O.covariance(Gn)
    Tin, Tout = oracle_T(Ti), oracle_T(To)
    s = O.sensitivity(HX, HG)
    assert np.allclose(lq.sens.cpu().numpy(), s, rtol=1e-4)
    Wp, HXp, HGp = O.biip(W.double().numpy(), HX, HG, Tin, Tout)
    assert np.linalg.norm(np64(lq.Wp) - Wp) / np.linalg.norm(Wp) < 2e-6
    for got, ref in ((lq.H_X, HXp), (lq.H_G, HGp)):
        fro, ent = cov_close(np64(got), ref)
        assert fro <= 1e-4 and ent <= 1e-4
    Uc_ref, dead, _ = O.chol_inv(np64(lq.H_X), 0.01)
    assert _uc_ok(np64(lq.Uc), Uc_ref) <= 0
    r = res[0]
    got = (r.codes.cpu().numpy(), r.scales.cpu().numpy(), r.zeros.cpu().numpy(), np64(r.W_hat))
    _check_quant(lq.Wp, lq.Uc, lq.dead, 3, 0, got)
    L_ref = O.kron_loss(np64(lq.Wp), np64(r.W_hat), np64(lq.H_X), np64(lq.H_G))
    assert abs(r.loss.item() - L_ref) <= 1e-3 * L_ref
    # the oracle's own chain from the same X, G, W (float64 throughout): the
    # loss agrees to the statistical level the fp32 covariances allow
    full = O.quantize_linear(W.double().numpy(), Xn, Gn, Tin, Tout, 3)
    assert abs(r.loss.item() - full["loss"]) <= 0.05 * full["loss"]


# ------------------------------------------------------------------ multi-setting entry points

@pytest.mark.parametrize("gemm_mode", ["3xtf32", "fp32"])
def test_multi_entry_points_match_single_calls(P, rotated_small, gemm_mode):
    """kq_quantize_layer_multi / kq_kron_loss_multi share the operand splits
    across settings and must return exactly what the single calls return,
    whether the settings run side by side (four lanes, the fifth setting
    reusing lane 0) or one after the other (single-setting workspace)."""
    lq = rotated_small[0]
    mode = P.KQ_GEMM_3XTF32 if gemm_mode == "3xtf32" else P.KQ_GEMM_FP32
    settings = [(4, 0), (3, 128), (2, 0), (3, 0), (4, 64)]
    d_out, d_in = lq.Wp.shape

    def outputs():
        res = []
        for b, g in settings:
            ng = 1 if not g else -(-d_in // g)
            res.append((torch.empty((d_out, d_in), dtype=torch.uint8, device="cuda"),
                        torch.empty((d_out, ng), device="cuda"), torch.empty((d_out, ng), device="cuda"),
                        torch.empty((d_out, d_in), device="cuda"), torch.zeros(1, dtype=torch.float64, device="cuda")))
        return res

    one, many, seq = outputs(), outputs(), outputs()
    # the same settings with their W_hat stacked in one buffer: solved as one
    # problem (four settings, then the fifth), or one at a time when the
    # workspace holds one setting
    stk, stk1 = outputs(), outputs()
    for outs in (stk, stk1):
        buf = torch.empty((len(settings), d_out, d_in), device="cuda")
        for i, o in enumerate(outs):
            outs[i] = (o[0], o[1], o[2], buf[i], o[4])
    info = _info()
    for (b, g), (c, s, z, wh, l) in zip(settings, one):
        P.kq_quantize_layer(lq.Wp, lq.Uc, lq.dead, b, g, c, s, z, wh, gemm_mode=mode, info=info)
        P.kq_kron_loss(lq.Wp, wh, lq.H_X, lq.H_G, l)
    P.kq_quantize_layer_multi(lq.Wp, lq.Uc, lq.dead, settings, [o[0] for o in many], [o[1] for o in many],
                              [o[2] for o in many], [o[3] for o in many], gemm_mode=mode, info=info)
    P.kq_kron_loss_multi(lq.Wp, [o[3] for o in many], lq.H_X, lq.H_G, [o[4] for o in many])
    ws1 = P.workspace(P.kq_quantize_layer_workspace_size(d_out, d_in), lq.Wp.device)
    P.kq_quantize_layer_multi(lq.Wp, lq.Uc, lq.dead, settings, [o[0] for o in seq], [o[1] for o in seq],
                              [o[2] for o in seq], [o[3] for o in seq], gemm_mode=mode, ws=ws1, info=info)
    P.kq_kron_loss_multi(lq.Wp, [o[3] for o in seq], lq.H_X, lq.H_G, [o[4] for o in seq])
    P.kq_quantize_layer_multi(lq.Wp, lq.Uc, lq.dead, settings, [o[0] for o in stk], [o[1] for o in stk],
                              [o[2] for o in stk], [o[3] for o in stk], gemm_mode=mode, info=info)
    P.kq_kron_loss_multi(lq.Wp, [o[3] for o in stk], lq.H_X, lq.H_G, [o[4] for o in stk])
    P.kq_quantize_layer_multi(lq.Wp, lq.Uc, lq.dead, settings, [o[0] for o in stk1], [o[1] for o in stk1],
                              [o[2] for o in stk1], [o[3] for o in stk1], gemm_mode=mode, ws=ws1, info=info)
    P.kq_kron_loss_multi(lq.Wp, [o[3] for o in stk1], lq.H_X, lq.H_G, [o[4] for o in stk1])
    torch.cuda.synchronize()
    assert _info_code(info)[0] == 0
    for a, *rest in zip(one, many, seq, stk, stk1):
        for k, x in enumerate(a):
            for r in rest:
                assert torch.equal(x, r[k])


@pytest.mark.parametrize("d_out,d_in", [(200, 260), (33, 136), (3400, 260), (200, 1300)])
def test_stacked_solve_ragged_rows(P, d_out, d_in):
    """Settings stacked in one solve (M = count d_out rows in every trailing
    update, the first super-block reading W's row r mod d_out) against one
    call per setting, bit for bit, at row counts that leave partial CTAs and
    tiles, with dead columns (3 x 3400 rows: three CTAs per SM; 1300
    columns: the K = 1024 update after the first super-block reads W too);
    a non-finite weight is reported with its row in W."""
    rng = np.random.default_rng(d_out + d_in)
    W = torch.from_numpy(rng.normal(0, 0.02, (d_out, d_in)).astype(np.float32)).cuda()
    H = torch.from_numpy(_spd(d_in, 5, 1.0)).cuda()
    dead = torch.zeros(d_in, dtype=torch.uint8, device="cuda")
    dead[[3, d_in - 2]] = 1
    H[3, :] = 0
    H[:, 3] = 0
    H[d_in - 2, :] = 0
    H[:, d_in - 2] = 0
    Uc = torch.empty_like(H)
    info = _info()
    P.kq_chol_inv(H, 0.01, Uc, dead, None, info)
    settings = [(2, 0), (3, 32), (4, 0)]

    def outputs(stacked):
        buf = torch.empty((len(settings), d_out, d_in), device="cuda") if stacked else None
        res = []
        for i, (b, g) in enumerate(settings):
            ng = 1 if not g else -(-d_in // g)
            res.append((torch.empty((d_out, d_in), dtype=torch.uint8, device="cuda"),
                        torch.empty((d_out, ng), device="cuda"), torch.empty((d_out, ng), device="cuda"),
                        buf[i] if stacked else torch.empty((d_out, d_in), device="cuda")))
        return res

    one, stk = outputs(False), outputs(True)
    for (b, g), (c, s_, z, wh) in zip(settings, one):
        P.kq_quantize_layer(W, Uc, dead, b, g, c, s_, z, wh, gemm_mode=P.KQ_GEMM_3XTF32, info=info)
    P.kq_quantize_layer_multi(W, Uc, dead, settings, *[[o[k] for o in stk] for k in range(4)],
                              gemm_mode=P.KQ_GEMM_3XTF32, info=info)
    torch.cuda.synchronize()
    assert _info_code(info)[0] == 0
    for a, b in zip(one, stk):
        for x, y in zip(a, b):
            assert torch.equal(x, y)
    bad = W.clone()
    bad[d_out - 1, d_in // 2] = float("inf")
    info = _info()
    P.kq_quantize_layer_multi(bad, Uc, dead, settings, *[[o[k] for o in stk] for k in range(4)],
                              gemm_mode=P.KQ_GEMM_3XTF32, info=info)
    assert _info_code(info) == (7, d_out - 1)
