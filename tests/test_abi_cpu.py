"""The C ABI without a GPU: the library loads, exports every declared symbol,
validates arguments on the host, and its host-only entry point (bit
allocation) matches the oracle bit for bit."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import oracle as O
import post_weight_quantization_syrk_b200 as P
from post_weight_quantization_syrk_b200 import _lib as K

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kronq.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_path():
    names = declared_functions()
    for fn in ("kq_accum_cov", "kq_rotate", "kq_chol_inv", "kq_quantize_layer", "kq_kron_loss",
               "kq_sensitivity", "kq_allocate_bits"):
        assert fn in names


def test_library_exports_every_declared_symbol():
    lib = K.load()
    names = declared_functions()
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", K.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (kq_\w+)", out))
    assert set(names) <= exported
    assert set(K.EXPORTS) == set(names)


def test_status_strings_and_version():
    assert P.kq_version() >= 100
    for code, name in K.STATUS_NAMES.items():
        assert P.kq_status_string(code) == name


def test_wait_limit_is_process_wide_and_returns_the_previous_value():
    assert P.kq_set_wait_limit_ns(123) == P.KQ_WAIT_LIMIT_DEFAULT_NS
    assert P.kq_set_wait_limit_ns(0) == 123
    assert P.kq_set_wait_limit_ns(P.KQ_WAIT_LIMIT_DEFAULT_NS) == 0


def test_allocation_matches_oracle_bit_exact():
    rng = np.random.default_rng(0)
    for _ in range(200):
        k = int(rng.integers(1, 40))
        s = rng.uniform(0, 10, k)
        if rng.random() < 0.3:
            s = np.round(s)          # ties
        n = rng.integers(1, 50, k) * int(rng.choice([1, 4096, 4096 * 11008]))
        avg = float(rng.choice([2.0, 2.5, 3.0, 3.25, 4.0]))
        ch = (2, 3, 4) if rng.random() < 0.7 else (2, 4, 8)
        assert P.kq_allocate_bits(s, n, ch, avg) == list(O.allocate_bits(s, n, ch, avg))


def test_allocation_llama7b_shapes():
    """The 7B-shaped model: 32 blocks x (q, k, v, o, gate, up, down)."""
    rng = np.random.default_rng(1)
    n = np.array([4096 * 4096] * 4 + [4096 * 11008] * 3, dtype=np.int64)
    n = np.tile(n, 32)
    s = rng.lognormal(0, 2, n.size)
    b = np.array(P.kq_allocate_bits(s, n, (2, 3, 4), 3.0))
    assert list(b) == list(O.allocate_bits(s, n, (2, 3, 4), 3.0))
    assert (b * n).sum() <= 3.0 * n.sum()
    assert (b * n).sum() > 2.99 * n.sum()


def test_allocation_validation():
    with pytest.raises(P.KronqError) as e:
        P.kq_allocate_bits([1.0], [0], (2, 3))
    assert e.value.status == 1
    with pytest.raises(P.KronqError):
        P.kq_allocate_bits([float("nan")], [5], (2, 3))
    with pytest.raises(P.KronqError):
        P.kq_allocate_bits([1.0], [5], (2, 2))
    assert P.kq_allocate_bits([], [], (2, 3)) == []


def _raw():
    return K.load()


def test_host_validation_without_gpu():
    """Argument checks return before any CUDA call: NULL pointers, bad sizes,
    misalignment and short workspaces are reported synchronously."""
    lib = _raw()
    NULL = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(0x10000)        # never dereferenced: validation fails first
    odd = ctypes.c_void_p(0x10002)
    s = lib.kq_accum_cov(NULL, 10, 8, 8, fake, 8, 1.0, 0, NULL, 0, fake, NULL)
    assert s == 1
    s = lib.kq_accum_cov(fake, 10, 0, 8, fake, 8, 1.0, 0, NULL, 0, fake, NULL)
    assert s == 2
    s = lib.kq_accum_cov(odd, 10, 8, 8, fake, 8, 1.0, 0, NULL, 0, fake, NULL)
    assert s == 3
    assert b"aligned" in lib.kq_last_error()
    s = lib.kq_accum_cov(fake, 10, 8, 9, fake, 8, 1.0, 0, NULL, 0, fake, NULL)
    assert s == 3
    s = lib.kq_chol_inv(fake, 16, 16, ctypes.c_float(0.01), fake, 16, NULL, fake, 8, fake, NULL)
    assert s == 4                           # workspace too small
    s = lib.kq_chol_inv(fake, 16, 8, ctypes.c_float(0.01), fake, 16, NULL, fake, 1 << 30, fake, NULL)
    assert s == 1                           # ldh < n
    s = lib.kq_chol_inv(fake, 0, 8, ctypes.c_float(0.01), fake, 16, NULL, fake, 1 << 30, fake, NULL)
    assert s == 2
    s = lib.kq_quantize_layer(fake, 8, 8, 8, fake, 8, NULL, 1, 0, 128, 0, fake, 8, fake, fake,
                              ctypes.c_void_p(0x20000), 8, fake, 1 << 20, fake, NULL)
    assert s == 1                           # bits outside 2..8
    s = lib.kq_quantize_layer(fake, 8, 8, 8, fake, 8, NULL, 3, 48, 128, 0, fake, 8, fake, fake,
                              ctypes.c_void_p(0x20000), 8, fake, 1 << 20, fake, NULL)
    assert s == 2                           # group not a multiple of 32 dividing 128
    s = lib.kq_quantize_layer(fake, 8, 8, 8, fake, 8, NULL, 3, 0, 64, 0, fake, 8, fake, fake,
                              ctypes.c_void_p(0x20000), 8, fake, 1 << 20, fake, NULL)
    assert s == 2                           # block != 128
    rht = K.kq_rht(12, 2, 3, 0x10000, 0)    # m = 3 needs Qm
    s = lib.kq_rotate(fake, 4, 12, 12, 1, ctypes.byref(rht), 0, NULL)
    assert s == 1
    rht = K.kq_rht(12, 2, 3, 0x10000, 0x10000)
    s = lib.kq_rotate(fake, 4, 16, 16, 1, ctypes.byref(rht), 0, NULL)
    assert s == 1                           # n does not match cols
    rht = K.kq_rht(13, 2, 3, 0x10000, 0x10000)
    s = lib.kq_rotate(fake, 4, 13, 16, 1, ctypes.byref(rht), 0, NULL)
    assert s == 2                           # n != m * 2^log2_p
    s = lib.kq_kron_loss(fake, 8, fake, 8, 8, 8, fake, 8, NULL, 0, fake, NULL, 0, NULL)
    assert s == 4
    s = lib.kq_sensitivity(fake, 0, 8, fake, 8, 8, fake, NULL)
    assert s == 1


def test_output_side_entry_points_validate_without_gpu():
    """The blockwise-H_G, permutation and act-order entry points reject bad
    arguments before any CUDA call."""
    lib = _raw()
    NULL = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(0x10000)
    # block size not a multiple of 256 dividing d
    s = lib.kq_accum_cov_blocks(fake, 10, 1024, 1024, 300, fake, 300, ctypes.c_float(1.0), 0, NULL, 0, fake, NULL)
    assert s == 2 and b"multiple of 256" in lib.kq_last_error()
    s = lib.kq_accum_cov_blocks(fake, 10, 768, 768, 512, fake, 512, ctypes.c_float(1.0), 0, NULL, 0, fake, NULL)
    assert s == 2
    s = lib.kq_accum_cov_blocks(fake, 10, 1024, 1024, 256, fake, 128, ctypes.c_float(1.0), 0, NULL, 0, fake, NULL)
    assert s == 1                           # ldc < k
    assert P.kq_accum_cov_blocks_workspace_size(1 << 18, 1000, 256) == 0
    assert P.kq_accum_cov_blocks_workspace_size(1 << 18, 4096, 512) > 0
    s = lib.kq_sensitivity_blocks(fake, 8, 8, fake, 1000, 256, 256, fake, NULL)
    assert s == 1                           # k does not divide d_out
    s = lib.kq_kron_loss_blocks(fake, 8, fake, 8, 512, 8, fake, 8, fake, 256, 256, fake, fake, 8, NULL)
    assert s == 4                           # workspace too small
    s = lib.kq_kron_loss_blocks(fake, 8, fake, 8, 500, 8, fake, 8, fake, 256, 256, fake, fake, 1 << 30, NULL)
    assert s == 1                           # k does not divide d_out
    s = lib.kq_channel_energy(fake, 10, 8, 8, ctypes.c_float(1.0), fake, fake, 8, fake, NULL)
    assert s == 4
    s = lib.kq_balance_permutation(fake, 12, 5, fake, NULL)
    assert s == 2
    s = lib.kq_balance_permutation(NULL, 12, 4, fake, NULL)
    assert s == 1
    s = lib.kq_act_order_permutation(fake, 0, 8, fake, NULL)
    assert s == 2
    s = lib.kq_act_order_permutation(fake, 16, 8, fake, NULL)
    assert s == 1                           # ldh < n
    s = lib.kq_gather(fake, 8, 3, NULL, NULL, 4, 8, ctypes.c_void_p(0x20000), 8, fake, NULL)
    assert s == 1 and b"elem_bytes" in lib.kq_last_error()
    s = lib.kq_gather(fake, 8, 4, NULL, NULL, 4, 8, fake, 8, fake, NULL)
    assert s == 1                           # out aliases M
    s = lib.kq_gather(fake, 4, 4, NULL, NULL, 4, 8, ctypes.c_void_p(0x20000), 8, fake, NULL)
    assert s == 1                           # ldm < cols


def test_workspace_sizes():
    assert P.kq_chol_inv_workspace_size(4096) >= 2 * 4096 * 4096 * 8
    assert P.kq_quantize_layer_workspace_size(4096, 4096) >= 4096 * 128 * 4
    assert P.kq_kron_loss_workspace_size(4096, 4096) >= 64 * 64 * 8
    assert P.kq_chol_inv_workspace_size(0) == 0


def test_chol_inv_workspace_holds_what_the_header_lists():
    """kq_chol_inv's workspace as its header documents it: the padded fp64
    matrix and its inverse (2 ld^2 doubles, ld = n rounded up to 128, + 128),
    eight panel buffers (8 * 64 * ld doubles) and the diagonal blocks'
    inverse factors (ceil(n/64) * 64^2 doubles), each rounded up to 256
    bytes, plus one double."""
    def up(x):
        return -(-x // 256) * 256
    for n in (1, 63, 64, 1000, 4096, 8200, 11008, 28672):
        ld = -(-n // 128) * 128 + 128
        want = up(ld * ld * 8) * 2 + up(8 * 64 * ld * 8) + up(-(-n // 64) * 64 * 64 * 8) + up(8)
        assert P.kq_chol_inv_workspace_size(n) == want, n


def test_multi_workspace_sizes():
    """One lane per setting up to four lanes; one lane is the single-setting size."""
    one = P.kq_quantize_layer_workspace_size(4096, 4096)
    sizes = [P.kq_quantize_layer_multi_workspace_size(4096, 4096, 128, c) for c in range(1, 7)]
    assert sizes[0] == one
    lane = sizes[1] - sizes[0]
    assert lane >= 2 * 4096 * 1024 * 4
    assert sizes[:4] == [one + k * lane for k in range(4)]
    assert sizes[4] == sizes[5] == sizes[3]
    assert P.kq_quantize_layer_multi_workspace_size(4096, 4096, 128, 0) == 0


def test_multi_entry_points_validate_before_enqueue():
    """Host-side rejections of the multi-setting calls (no device work)."""
    import ctypes
    lib = P.load()
    vp = ctypes.c_void_p
    dummy = vp(16)  # never dereferenced: validation fails first
    arr = (vp * 2)(vp(32), vp(48))
    bits = (ctypes.c_int * 2)(3, 9)          # second setting invalid
    groups = (ctypes.c_int * 2)(0, 0)
    st = lib.kq_quantize_layer_multi(dummy, 4, 128, 128, dummy, 128, None, 2, bits, groups, 128, 0, arr, 128, arr,
                                     arr, arr, 128, dummy, 1 << 30, dummy, None)
    assert st == 1 and b"bits" in lib.kq_last_error()   # KQ_ERR_INVALID_ARG
    st = lib.kq_kron_loss_multi(dummy, 128, 0, arr, 128, 4, 128, dummy, 128, dummy, 4, arr, dummy, 1 << 30, None)
    assert st == 1   # KQ_ERR_INVALID_ARG
    shared = (vp * 2)(vp(32), vp(32))        # both settings write the same W_hat
    bits = (ctypes.c_int * 2)(3, 4)
    st = lib.kq_quantize_layer_multi(dummy, 4, 128, 128, dummy, 128, None, 2, bits, groups, 128, 0, arr, 128, arr,
                                     arr, shared, 128, dummy, 1 << 30, dummy, None)
    assert st == 1 and b"share an output" in lib.kq_last_error()


def test_inference_entry_points_validate_before_enqueue():
    """Host-side rejections of kq_pack_codes / kq_reverted_matvec (nothing is
    launched: every check fails before a CUDA call)."""
    import ctypes
    lib = P.load()
    vp = ctypes.c_void_p
    d = vp(256)   # never dereferenced
    # kq_pack_codes: NULL codes, bits outside 1..8, packed row too short
    assert lib.kq_pack_codes(None, 4, 64, 64, 4, d, 8, d, None) == 1
    assert lib.kq_pack_codes(d, 4, 64, 64, 9, d, 18, d, None) == 1
    st = lib.kq_pack_codes(d, 4, 64, 64, 3, d, 5, d, None)      # needs 2 groups x 3 words
    assert st == 1 and b"leading dimension" in lib.kq_last_error()
    # kq_reverted_matvec
    T_ok = K.kq_rht(64, 6, 1, 256, None)
    T_bad = K.kq_rht(32, 5, 1, 256, None)
    def call(bits=4, group=0, batch=1, T_in=T_ok, ws_bytes=1 << 20, ldp=8):
        return lib.kq_reverted_matvec(d, 16, 64, ldp, bits, d, d, group, ctypes.byref(T_in), None, d, 64, batch, d,
                                      16, d, ws_bytes, None)
    assert call(bits=0) == 1
    assert call(batch=9) == 2 and b"batch" in lib.kq_last_error()
    assert call(group=48) == 2
    assert call(T_in=T_bad) == 1 and b"rotation order" in lib.kq_last_error()
    assert call(ldp=7) == 1
    assert call(ws_bytes=16) == 4
    assert P.kq_reverted_matvec_workspace_size(64, 3) >= 3 * 64 * 4
    assert P.kq_reverted_matvec_workspace_size(0, 1) == 0


def test_code_buffer_alignment_and_message_text():
    """The solver stores four codes at a time: a code buffer that is not
    4-byte aligned, or whose ldq is not a multiple of 4, is refused before
    anything is enqueued; error texts render their percent signs literally."""
    import ctypes
    lib = P.load()
    vp = ctypes.c_void_p
    d = vp(256)
    def quant(codes, ldq):
        return lib.kq_quantize_layer(d, 4, 128, 128, d, 128, None, 3, 0, 128, 0, codes, ldq, d, d, vp(512), 128, d,
                                     1 << 30, d, None)
    assert quant(vp(258), 128) == 3 and b"ldq % 4 == 0" in lib.kq_last_error()
    assert quant(vp(256), 129) == 3
    T = K.kq_rht(4, 2, 1, 256, None)
    st = lib.kq_rotate(vp(4), 4, 4, 4, P.KQ_AXIS_COLS, ctypes.byref(T), 0, None)
    assert st == 3 and b"ld % 4 == 0" in lib.kq_last_error()
