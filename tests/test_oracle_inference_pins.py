"""Pins of the oracle's inference side (packed codes, online reversion of U
and V) against hand-derived words, an independent big-integer statement of
the packed layout, and what the rotations must preserve."""
import math

import numpy as np
import pytest

import oracle as O


def _rht(n, log2_p, seed):
    """A randomised Hadamard T of order n = m 2^log2_p (random signs, a Haar
    Q_m from a sign-fixed QR when m > 1)."""
    rng = np.random.default_rng(seed)
    m = n >> log2_p
    signs = rng.choice([-1.0, 1.0], n)
    Qm = None
    if m > 1:
        Q, R = np.linalg.qr(rng.standard_normal((m, m)))
        Qm = Q * np.sign(np.diag(R))[None, :]
    return O.rht_matrix(n, log2_p, signs, Qm)


# ------------------------------------------------------------------ packing

def test_pack_hand_words():
    # 4 bits: nibbles fill each word from the least significant end
    assert O.pack_codes(np.array([[1, 2, 3, 4, 5, 6, 7, 8]]), 4)[0, 0] == 0x87654321
    # 2 bits: codes 1, 2, 3, 0 make the byte 0b00111001
    p = O.pack_codes(np.array([[1, 2, 3, 0] * 8]), 2)
    assert p.shape == (1, 2) and list(p[0]) == [0x39393939, 0x39393939]
    # 8 bits: one code per byte
    assert O.pack_codes(np.array([[0x11, 0x22, 0x33, 0x44]]), 8)[0, 0] == 0x44332211
    # 3 bits: code 10 sits at stream bits 30..32 and straddles words 0 and 1
    c = np.zeros((1, 32), dtype=np.int64)
    c[0, 10] = 7
    assert list(O.pack_codes(c, 3)[0]) == [0xC0000000, 0x00000001, 0]
    assert list(O.pack_codes(np.full((1, 32), 7), 3)[0]) == [0xFFFFFFFF] * 3
    # a 33rd column opens a second group of `bits` words, zero-padded
    c = np.zeros((1, 33), dtype=np.int64)
    c[0, 32] = 0xA
    assert list(O.pack_codes(c, 4)[0]) == [0, 0, 0, 0, 0xA, 0, 0, 0]


@pytest.mark.parametrize("bits", range(1, 9))
@pytest.mark.parametrize("cols", [1, 31, 32, 33, 100])
def test_pack_matches_big_integer_stream(bits, cols):
    """Each group of 32 codes is the integer sum_k code_k 2^(bits k), cut into
    32-bit words from the least significant end; unpacking restores the codes."""
    rng = np.random.default_rng(bits * 1000 + cols)
    codes = rng.integers(0, 1 << bits, (3, cols))
    packed = O.pack_codes(codes, bits)
    groups = -(-cols // 32)
    assert packed.shape == (3, groups * bits) and packed.dtype == np.uint32
    for r in range(3):
        for g in range(groups):
            s = sum(int(codes[r, c]) << (bits * (c - 32 * g)) for c in range(32 * g, min(32 * g + 32, cols)))
            want = [(s >> (32 * w)) & 0xFFFFFFFF for w in range(bits)]
            assert [int(v) for v in packed[r, g * bits:(g + 1) * bits]] == want
    assert np.array_equal(O.unpack_codes(packed, bits, cols), codes.astype(np.uint8))


def test_pack_rejects_codes_outside_the_width():
    with pytest.raises(ValueError):
        O.pack_codes(np.array([[4]]), 2)
    with pytest.raises(ValueError):
        O.pack_codes(np.array([[-1]]), 3)
    with pytest.raises(ValueError):
        O.unpack_codes(np.zeros((1, 3), dtype=np.uint32), 2, 64)


# ------------------------------------------------------------------ reversion

def _rtn(Wp, bits, group):
    """Round-to-nearest codes of Wp on per-row (or per-group) min/max grids."""
    rows, cols = Wp.shape
    gs = cols if not group else group
    ng = -(-cols // gs)
    codes = np.zeros((rows, cols), dtype=np.int64)
    scales = np.zeros((rows, ng), dtype=np.float32)
    zeros = np.zeros((rows, ng), dtype=np.float32)
    for g in range(ng):
        blk = Wp[:, g * gs:(g + 1) * gs]
        s, z = O.fit_grid(blk.min(axis=1), blk.max(axis=1), bits)
        scales[:, g], zeros[:, g] = s, z
        for r in range(rows):
            codes[r, g * gs:(g + 1) * gs] = O.quantize_codes(blk[r], s[r], z[r], bits)[1]
    return codes, scales, zeros


def test_dequantize_layer_elementwise():
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 16, (5, 96))
    scales = rng.uniform(0.5, 2.0, (5, 3))
    zeros = rng.integers(0, 16, (5, 3)).astype(np.float64)
    W = O.dequantize_layer(codes, scales, zeros, group=32)
    for r in range(5):
        for c in range(96):
            assert W[r, c] == scales[r, c // 32] * (codes[r, c] - zeros[r, c // 32])
    Wc = O.dequantize_layer(codes, scales[:, :1], zeros[:, :1], group=0)
    assert np.array_equal(Wc, scales[:, :1] * (codes - zeros[:, :1]))


def test_reverted_apply_with_identity_rotations_is_the_dequantized_matvec():
    rng = np.random.default_rng(4)
    d_out, d_in, bits = 7, 40, 3
    codes = rng.integers(0, 8, (d_out, d_in))
    scales = rng.uniform(0.01, 0.1, (d_out, 1))
    zeros = rng.integers(0, 8, (d_out, 1)).astype(np.float64)
    x = rng.standard_normal(d_in)
    y = O.reverted_apply(O.pack_codes(codes, bits), scales, zeros, bits, 0, np.eye(d_in), np.eye(d_out), x)
    for r in range(d_out):
        want = math.fsum(scales[r, 0] * (codes[r, c] - zeros[r, 0]) * x[c] for c in range(d_in))
        assert abs(y[r] - want) <= 1e-12 * (1 + abs(want))


def test_reverted_apply_recovers_the_layer_it_rotated():
    """For a layer exactly representable in the rotated basis (W' = W_hat'),
    V^T W_hat' U x is W x with W = V^T W' U: a transposed or swapped rotation
    fails this (T is not symmetric)."""
    rng = np.random.default_rng(5)
    d_out, d_in, bits = 48, 96, 4      # 48 = 3 * 16, 96 = 3 * 32: Q_m on both sides
    T_in, T_out = _rht(d_in, 5, 11), _rht(d_out, 4, 12)
    assert np.abs(T_in - T_in.T).max() > 0.1 and np.abs(T_out - T_out.T).max() > 0.1
    codes = rng.integers(0, 16, (d_out, d_in))
    scales = rng.uniform(0.001, 0.01, (d_out, 3)).astype(np.float32)
    zeros = rng.integers(0, 16, (d_out, 3)).astype(np.float32)
    Wp = O.dequantize_layer(codes, scales, zeros, group=32)
    W = T_out.T @ Wp @ T_in                      # the layer whose BiIP image is Wp
    assert np.allclose(O.biip(W, np.eye(d_in), np.eye(d_out), T_in, T_out)[0], Wp, atol=1e-14)
    x = rng.standard_normal((d_in, 5))
    y = O.reverted_apply(O.pack_codes(codes, bits), scales, zeros, bits, 32, T_in, T_out, x)
    assert np.allclose(y, W @ x, rtol=0, atol=1e-12)
    y0 = O.reverted_apply(O.pack_codes(codes, bits), scales, zeros, bits, 32, T_in, T_out, x[:, 0])
    assert np.allclose(y0, y[:, 0], rtol=0, atol=1e-13)


@pytest.mark.parametrize("bits,group", [(4, 0), (3, 32), (2, 0)])
def test_reverted_apply_error_is_the_rotated_quantization_error(bits, group):
    """y - W x = V^T (W_hat' - W') U x, so ||y - W x|| <= ||W_hat' - W'||_F ||x||,
    and each |W_hat' - W'| entry is at most half a grid step."""
    rng = np.random.default_rng(100 + bits)
    d_out, d_in = 32, 64
    T_in, T_out = _rht(d_in, 6, 21), _rht(d_out, 5, 22)
    W = rng.normal(0, 0.02, (d_out, d_in))
    Wp = O.biip(W, np.eye(d_in), np.eye(d_out), T_in, T_out)[0]
    codes, scales, zeros = _rtn(Wp, bits, group)
    W_hat_p = O.dequantize_layer(codes, scales, zeros, group)
    step = scales.astype(np.float64)[:, np.zeros(d_in, dtype=np.int64) if not group else np.arange(d_in) // group]
    assert np.all(np.abs(W_hat_p - Wp) <= 0.5 * step * (1 + 1e-6))
    x = rng.standard_normal(d_in)
    y = O.reverted_apply(O.pack_codes(codes, bits), scales, zeros, bits, group, T_in, T_out, x)
    err = np.linalg.norm(y - W @ x)
    assert err <= np.linalg.norm(W_hat_p - Wp) * np.linalg.norm(x) * (1 + 1e-9)
    assert np.isclose(err, np.linalg.norm((W_hat_p - Wp) @ (T_in @ x)), rtol=1e-9)
