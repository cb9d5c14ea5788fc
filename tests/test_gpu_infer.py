"""Inference side on the GPU against the oracle: packed codes bit for bit,
and the matvec with U and V reverted online (y = V^T W_hat' U x)."""
import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA GPU")
    import post_weight_quantization_syrk_b200 as P
    return P


def _info_code(info):
    v = int(info.item()) & 0xFFFFFFFF
    return v >> 24, v & 0xFFFFFF


def _rht_pair(P, n, seed):
    """Device RHT for the kernels and the same fp32 parameters as a dense
    float64 T for the oracle."""
    p = synth.rht_params(n, seed)
    dev = P.RHT(p.n, p.log2_p, p.m, p.signs.cuda(), None if p.Qm is None else p.Qm.cuda())
    T = O.rht_matrix(p.n, p.log2_p, p.signs.numpy().astype(np.float64),
                     None if p.Qm is None else p.Qm.numpy().astype(np.float64))
    return dev, T


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("rows,cols", [(37, 100), (64, 4096), (5, 31)])
def test_pack_codes_matches_oracle(P, bits, rows, cols):
    rng = np.random.default_rng(bits * 100 + cols)
    codes = rng.integers(0, 1 << bits, (rows, cols)).astype(np.uint8)
    packed = P.kq_pack_codes(torch.from_numpy(codes).cuda(), bits)
    torch.cuda.synchronize()
    got = packed.cpu().numpy().view(np.uint32)
    assert np.array_equal(got, O.pack_codes(codes, bits))


def test_pack_codes_reports_a_code_outside_the_width(P):
    codes = torch.zeros((4, 64), dtype=torch.uint8, device="cuda")
    codes[2, 40] = 8                      # does not fit in 3 bits
    info = P.new_info(codes.device)
    packed = P.kq_pack_codes(codes, 3, info=info)
    torch.cuda.synchronize()
    assert _info_code(info) == (1, 2)     # KQ_ERR_INVALID_ARG, row 2
    assert int(packed.abs().sum().item()) == 0   # masked to 0


@pytest.mark.parametrize("bits,group,d_out,d_in,batch", [
    (4, 0, 48, 96, 1),       # odd factor 3 on both sides (Q_m mixing)
    (3, 32, 48, 96, 5),
    (2, 64, 64, 128, 8),     # powers of two
    (4, 128, 200, 384, 3),   # ragged row count
    (3, 0, 40, 100, 2),      # d_in not a multiple of 32 (ragged last chunk)
    (3, 0, 96, 2496, 8),     # several 1024-column chunks of x, ragged last tile
    (8, 128, 72, 1312, 3),   # 8-bit codes, grouped, ragged last group
    (2, 32, 4864, 1056, 4),  # enough rows for four rows per warp
    (5, 0, 36, 70, 2),       # a width the row-tiled kernel does not take
])
def test_reverted_matvec_matches_oracle(P, bits, group, d_out, d_in, batch):
    rng = np.random.default_rng(bits * 1000 + d_in + batch)
    ng = 1 if not group else -(-d_in // group)
    codes = rng.integers(0, 1 << bits, (d_out, d_in)).astype(np.uint8)
    scales = rng.uniform(0.001, 0.02, (d_out, ng)).astype(np.float32)
    zeros = rng.integers(0, 1 << bits, (d_out, ng)).astype(np.float32)
    X = rng.standard_normal((batch, d_in)).astype(np.float32)
    Tin_d, Tin = _rht_pair(P, d_in, 31 + d_in)
    Tout_d, Tout = _rht_pair(P, d_out, 37 + d_out)
    packed = P.kq_pack_codes(torch.from_numpy(codes).cuda(), bits)
    Y = torch.empty((batch, d_out), device="cuda")
    P.kq_reverted_matvec(packed, bits, torch.from_numpy(scales).cuda(), torch.from_numpy(zeros).cuda(), group,
                         Tin_d, Tout_d, torch.from_numpy(X).cuda(), Y)
    Y0 = torch.empty((batch, d_out), device="cuda")
    P.kq_reverted_matvec(packed, bits, torch.from_numpy(scales).cuda(), torch.from_numpy(zeros).cuda(), group,
                         None, None, torch.from_numpy(X).cuda(), Y0)
    torch.cuda.synchronize()
    ref = O.reverted_apply(O.pack_codes(codes, bits), scales, zeros, bits, group, Tin, Tout,
                           X.astype(np.float64).T).T
    ref0 = O.reverted_apply(O.pack_codes(codes, bits), scales, zeros, bits, group, np.eye(d_in), np.eye(d_out),
                            X.astype(np.float64).T).T
    y, y0 = Y.cpu().numpy().astype(np.float64), Y0.cpu().numpy().astype(np.float64)
    assert np.linalg.norm(y - ref) <= 1e-5 * np.linalg.norm(ref)
    assert np.linalg.norm(y0 - ref0) <= 1e-5 * np.linalg.norm(ref0)


@pytest.mark.parametrize("d_out,d_in", [(4096, 4096), (11008, 4096)])
def test_reverted_matvec_full_size(P, d_out, d_in):
    """Layer sizes of the 7B model, 4-bit per-channel codes, one vector."""
    rng = np.random.default_rng(d_out)
    codes = rng.integers(0, 16, (d_out, d_in)).astype(np.uint8)
    scales = rng.uniform(0.001, 0.02, (d_out, 1)).astype(np.float32)
    zeros = rng.integers(0, 16, (d_out, 1)).astype(np.float32)
    X = rng.standard_normal((1, d_in)).astype(np.float32)
    Tin_d, Tin = _rht_pair(P, d_in, 7)
    Tout_d, Tout = _rht_pair(P, d_out, 8)
    packed = P.kq_pack_codes(torch.from_numpy(codes).cuda(), 4)
    Y = torch.empty((1, d_out), device="cuda")
    P.kq_reverted_matvec(packed, 4, torch.from_numpy(scales).cuda(), torch.from_numpy(zeros).cuda(), 0, Tin_d,
                         Tout_d, torch.from_numpy(X).cuda(), Y)
    torch.cuda.synchronize()
    ref = O.reverted_apply(O.pack_codes(codes, 4), scales, zeros, 4, 0, Tin, Tout, X[0].astype(np.float64))
    y = Y[0].cpu().numpy().astype(np.float64)
    assert np.linalg.norm(y - ref) <= 1e-5 * np.linalg.norm(ref)
