"""GPU parity of the output side without the full H_G, and of the H_G-informed
output rotation V = T P_G, against the float64 oracle.

KronQ review, Limitations (second limitation: BiIP holds H_G as a full
d_out x d_out matrix) and the research thread's "Sparks" (blockwise H_G);
KronQ paper page, Abstract (1) (the output rotation uses the gradient
covariance).  Integer and index work (the permutation, the gathers) is
compared bit for bit; covariances, rotations and losses with the tolerances
of test_gpu_parity.py.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from gpu_util import cov_close, device_rht, need_gpu, np64, oracle_T

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    need_gpu()
    import post_weight_quantization_syrk_b200 as P
    P.load()
    return P


def _info():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _code(info):
    return (int(info.item()) >> 24) & 0xFF


SPEC = synth.scaled(synth.WORKLOADS["attn4096"], d_out=1024, d_in=384, n_tokens=3000)


def test_channel_energy_and_balance_permutation(P):
    G = synth.gradients(SPEC, 5).cuda()
    e = torch.empty(SPEC.d_out, device="cuda")
    info = _info()
    P.kq_channel_energy(G, e, 1.0 / G.shape[0], None, info)
    torch.cuda.synchronize()
    assert _code(info) == 0
    ref = np.diag(O.covariance(G.cpu().float().numpy()))
    assert np.max(np.abs(np64(e) - ref) / ref) < 1e-6
    for k in (256, 512, 1024, 1):
        perm = torch.empty(SPEC.d_out, dtype=torch.int64, device="cuda")
        P.kq_balance_permutation(e, k, perm)
        want = O.balance_permutation(e.cpu().numpy(), k)      # the same fp32 energies decide
        assert np.array_equal(perm.cpu().numpy(), want), k
    # ties resolve to the lower index
    flat = torch.ones(512, device="cuda")
    perm = torch.empty(512, dtype=torch.int64, device="cuda")
    P.kq_balance_permutation(flat, 256, perm)
    assert np.array_equal(perm.cpu().numpy(), O.balance_permutation(np.ones(512), 256))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gather_bit_exact(P, dtype):
    rng = np.random.default_rng(9)
    rows, cols = 300, 520
    M = torch.from_numpy(rng.standard_normal((rows, cols)).astype(np.float32)).to(dtype).cuda()
    r = torch.from_numpy(rng.permutation(rows)).cuda()
    c = torch.from_numpy(rng.permutation(cols)).cuda()
    for ri, ci in ((r, None), (None, c), (r, c)):
        out = torch.empty_like(M)
        info = _info()
        P.kq_gather(M, out, ri, ci, info)
        torch.cuda.synchronize()
        assert _code(info) == 0
        ref = M.cpu()
        if ri is not None:
            ref = ref[ri.cpu()]
        if ci is not None:
            ref = ref[:, ci.cpu()]
        assert torch.equal(out.cpu(), ref)
    bad = c.clone()
    bad[7] = cols + 3
    out = torch.zeros_like(M)
    info = _info()
    P.kq_gather(M, out, None, bad, info)
    torch.cuda.synchronize()
    assert _code(info) == 1                              # reported, the index not read


@pytest.mark.parametrize("k", [256, 512])
def test_accum_cov_blocks_and_sensitivity(P, k):
    G = synth.gradients(SPEC, 6).cuda()
    X = synth.activations(SPEC, 6).cuda()
    Hb = torch.full((SPEC.d_out, k), float("nan"), device="cuda")
    info = _info()
    P.kq_accum_cov_blocks(G, k, Hb, 1.0 / G.shape[0], False, None, info)
    torch.cuda.synchronize()
    assert _code(info) == 0
    full = O.covariance(G.cpu().float().numpy())
    for b in range(SPEC.d_out // k):
        ref = full[b * k:(b + 1) * k, b * k:(b + 1) * k]
        fro, ent = cov_close(np64(Hb[b * k:(b + 1) * k]), ref)
        assert fro <= 1e-4 and ent <= 1e-4, (b, fro, ent)
    HX = torch.empty((SPEC.d_in, SPEC.d_in), device="cuda")
    P.kq_accum_cov(X, HX, 1.0 / X.shape[0], False, None, info)
    out = torch.zeros(3, dtype=torch.float64, device="cuda")
    P.kq_sensitivity_blocks(HX, Hb, out)
    tX = float(np.trace(np64(HX)))
    tG = sum(float(np.trace(np64(Hb[b * k:(b + 1) * k]))) for b in range(SPEC.d_out // k))
    assert np.allclose(out.cpu().numpy(), (tX, tG, tX * tG), rtol=1e-12)


def test_kron_loss_blocks(P):
    rng = np.random.default_rng(10)
    k = 256
    for d_out, d_in in ((1024, 384), (512, 200)):
        W = torch.from_numpy(rng.normal(0, 0.02, (d_out, d_in)).astype(np.float32)).cuda()
        Wh = W + torch.from_numpy(rng.normal(0, 0.004, (d_out, d_in)).astype(np.float32)).cuda()
        spec = synth.scaled(SPEC, d_out=d_out, d_in=d_in, n_tokens=1500)
        X = synth.activations(spec, 11).cuda().float()
        G = synth.gradients(spec, 11).cuda().float()
        HX = (X.T @ X / X.shape[0]).contiguous()
        HGfull = G.T @ G / G.shape[0]
        Hb = torch.cat([HGfull[b:b + k, b:b + k] for b in range(0, d_out, k)]).contiguous()
        loss = torch.zeros(1, dtype=torch.float64, device="cuda")
        P.kq_kron_loss_blocks(W, Wh, HX, Hb, loss)
        torch.cuda.synchronize()
        blocks = np64(Hb).reshape(d_out // k, k, k)
        ref = O.blockwise_kron_loss(np64(W), np64(Wh), np64(HX), blocks)
        assert abs(loss.item() - ref) <= 1e-3 * ref, (loss.item(), ref)


@pytest.mark.parametrize("balanced", [True, False])
def test_blockwise_layer_stagewise(P, balanced):
    """The blockwise layer path stage by stage against the oracle: W' =
    (I kron T_k) P_G W U^T, the rotated H_G blocks, codes (forced-code mode on
    the GPU's W' and U_c), the blockwise loss, and the layer's function after
    undoing both rotations."""
    from post_weight_quantization_syrk_b200.pipeline import BlockwiseLayerQuantizer
    k = 256
    W, X, G, Ti, _ = synth.layer(SPEC, 12)
    Tk = synth.rht_params(k, 77)
    lq = BlockwiseLayerQuantizer(SPEC.d_out, SPEC.d_in, k, balanced=balanced, gemm_mode=P.KQ_GEMM_3XTF32)
    res = lq.run(W.cuda(), X.cuda(), G.cuda(), device_rht(Ti), device_rht(Tk), [(3, 0)])
    torch.cuda.synchronize()
    lq.check("blockwise")
    Xn, Gn = X.float().numpy(), G.float().numpy()
    HG = O.covariance(Gn)
    perm = lq.perm.cpu().numpy()
    if balanced:
        # the same fp32 energies decide on both sides (their parity with the
        # oracle is test_channel_energy_and_balance_permutation's)
        assert np.array_equal(perm, O.balance_permutation(lq.energy.cpu().numpy(), k))
    else:
        assert np.array_equal(perm, np.arange(SPEC.d_out))
    Pm = O.permutation_matrix(perm)
    V = O.block_rht_matrix(SPEC.d_out, k, Tk.log2_p, Tk.signs.double().numpy()) @ Pm
    U = oracle_T(Ti)
    Wp_ref = V @ W.double().numpy() @ U.T
    assert np.linalg.norm(np64(lq.Wp) - Wp_ref) / np.linalg.norm(Wp_ref) < 4e-6
    HGp_ref = V @ HG @ V.T
    for b in range(SPEC.d_out // k):
        ref = HGp_ref[b * k:(b + 1) * k, b * k:(b + 1) * k]
        got = np64(lq.H_Gb[b * k:(b + 1) * k])
        assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-4
    r = res[0]
    q = O.quantize_layer(np64(lq.Wp), np64(lq.Uc), 3, 0, 128, lq.dead.cpu().numpy().astype(bool),
                         force_codes=r.codes.cpu().numpy())
    assert not q.mismatches, q.mismatches[:3]
    blocks = np64(lq.H_Gb).reshape(SPEC.d_out // k, k, k)
    Lref = O.blockwise_kron_loss(np64(lq.Wp), np64(r.W_hat), np64(lq.H_X), blocks)
    assert abs(r.loss.item() - Lref) <= 1e-3 * Lref
    # back to the original output order: V^T W' U = W
    back = torch.empty_like(lq.Wp)
    tmp = lq.Wp.clone()
    lq.unrotate_output(tmp, device_rht(Tk), back)
    P.kq_rotate(back, P.KQ_AXIS_COLS, device_rht(Ti), True)
    assert np.linalg.norm(np64(back) - W.double().numpy()) / np.linalg.norm(W.double().numpy()) < 4e-6


def test_full_rotation_with_hg_permutation(P):
    """LayerQuantizer with the H_G-informed factor: W' = T P_G W U^T and
    H_G' = T P_G H_G P_G^T T^T against the oracle."""
    from post_weight_quantization_syrk_b200.pipeline import LayerQuantizer
    W, X, G, Ti, To = synth.layer(SPEC, 13)
    lq = LayerQuantizer(SPEC.d_out, SPEC.d_in, gemm_mode=P.KQ_GEMM_3XTF32)
    Gc = G.cuda()
    lq.statistics(X.cuda(), Gc)
    lq.hg_permutation(Gc, 1 << To.log2_p)
    lq.rotate(W.cuda(), device_rht(Ti), device_rht(To))
    torch.cuda.synchronize()
    lq.check("hg permutation")
    HG = O.covariance(G.float().numpy())
    perm = lq.perm.cpu().numpy()
    assert sorted(perm.tolist()) == list(range(SPEC.d_out))
    e = torch.empty(SPEC.d_out, device="cuda")
    P.kq_channel_energy(Gc, e, 1.0 / Gc.shape[0], None, _info())
    assert np.array_equal(perm, O.balance_permutation(e.cpu().numpy(), 1 << To.log2_p))
    Pm = O.permutation_matrix(perm)
    V = oracle_T(To) @ Pm
    U = oracle_T(Ti)
    Wp_ref = V @ W.double().numpy() @ U.T
    assert np.linalg.norm(np64(lq.Wp) - Wp_ref) / np.linalg.norm(Wp_ref) < 4e-6
    HGp = V @ HG @ V.T
    assert np.linalg.norm(np64(lq.H_G) - HGp) / np.linalg.norm(HGp) < 1e-4
