"""ctypes binding of libkronq.so (the C ABI declared in include/kronq.h).

Argument marshalling only: every computation runs in the library's CUDA
kernels.  Each wrapper takes torch CUDA tensors, checks dtype, device and
layout, passes raw pointers, leading dimensions and the current CUDA stream,
and raises KronqError on a non-OK status.  The library is loaded from the
package directory; if it is missing the import fails loudly (there is no
other implementation of these operations in the package).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkronq.so")

KQ_OK = 0
STATUS_NAMES = {
    0: "KQ_OK", 1: "KQ_ERR_INVALID_ARG", 2: "KQ_ERR_UNSUPPORTED_SHAPE", 3: "KQ_ERR_ALIGNMENT",
    4: "KQ_ERR_WORKSPACE", 5: "KQ_ERR_CUDA", 6: "KQ_ERR_NOT_PD", 7: "KQ_ERR_NONFINITE", 8: "KQ_ERR_TIMEOUT",
}
KQ_AXIS_ROWS, KQ_AXIS_COLS = 0, 1
KQ_GEMM_FP32, KQ_GEMM_3XTF32 = 0, 1

# Every symbol the header declares.
EXPORTS = (
    "kq_status_string", "kq_last_error", "kq_version", "kq_launch_count", "kq_set_wait_limit_ns",
    "kq_accum_cov_workspace_size", "kq_accum_cov", "kq_accum_cov_blocks_workspace_size", "kq_accum_cov_blocks",
    "kq_channel_energy_workspace_size", "kq_channel_energy", "kq_balance_permutation", "kq_gather",
    "kq_act_order_permutation",
    "kq_pack_codes", "kq_reverted_matvec_workspace_size", "kq_reverted_matvec",
    "kq_sensitivity", "kq_sensitivity_blocks",
    "kq_rotate",
    "kq_chol_inv_workspace_size", "kq_chol_inv",
    "kq_quantize_layer_workspace_size", "kq_quantize_layer", "kq_quantize_layer_multi_workspace_size",
    "kq_quantize_layer_multi", "kq_solver_timing",
    "kq_kron_loss_workspace_size", "kq_kron_loss", "kq_kron_loss_multi", "kq_kron_loss_noalloc",
    "kq_kron_loss_blocks_workspace_size", "kq_kron_loss_blocks",
    "kq_allocate_bits",
)


class KronqError(RuntimeError):
    def __init__(self, status, detail, where=""):
        self.status = int(status)
        self.name = STATUS_NAMES.get(int(status), f"status {status}")
        super().__init__(f"{where}: {self.name}: {detail}" if where else f"{self.name}: {detail}")


class kq_solver_times(ctypes.Structure):
    _fields_ = [("grid_ms", ctypes.c_double), ("inblock_ms", ctypes.c_double), ("update_ms", ctypes.c_double),
                ("grid_launches", ctypes.c_longlong), ("inblock_launches", ctypes.c_longlong),
                ("update_launches", ctypes.c_longlong), ("update_flops", ctypes.c_double),
                ("inblock_bytes", ctypes.c_double)]


class kq_rht(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int64), ("log2_p", ctypes.c_int32), ("m", ctypes.c_int32),
                ("signs", ctypes.c_void_p), ("Qm", ctypes.c_void_p)]


_i64, _i32, _f32, _f64, _vp, _sz = (ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_double,
                                    ctypes.c_void_p, ctypes.c_size_t)

_SIGS = {
    "kq_status_string": (ctypes.c_char_p, [_i32]),
    "kq_last_error": (ctypes.c_char_p, []),
    "kq_version": (_i32, []),
    "kq_launch_count": (ctypes.c_ulonglong, []),
    "kq_set_wait_limit_ns": (ctypes.c_ulonglong, [ctypes.c_ulonglong]),
    "kq_accum_cov_workspace_size": (_sz, [_i64, _i64]),
    "kq_accum_cov": (_i32, [_vp, _i64, _i64, _i64, _vp, _i64, _f32, _i32, _vp, _sz, _vp, _vp]),
    "kq_sensitivity": (_i32, [_vp, _i64, _i64, _vp, _i64, _i64, _vp, _vp]),
    "kq_sensitivity_blocks": (_i32, [_vp, _i64, _i64, _vp, _i64, _i64, _i64, _vp, _vp]),
    "kq_accum_cov_blocks_workspace_size": (_sz, [_i64, _i64, _i64]),
    "kq_accum_cov_blocks": (_i32, [_vp, _i64, _i64, _i64, _i64, _vp, _i64, _f32, _i32, _vp, _sz, _vp, _vp]),
    "kq_channel_energy_workspace_size": (_sz, [_i64]),
    "kq_channel_energy": (_i32, [_vp, _i64, _i64, _i64, _f32, _vp, _vp, _sz, _vp, _vp]),
    "kq_balance_permutation": (_i32, [_vp, _i64, _i64, _vp, _vp]),
    "kq_gather": (_i32, [_vp, _i64, _i32, _vp, _vp, _i64, _i64, _vp, _i64, _vp, _vp]),
    "kq_act_order_permutation": (_i32, [_vp, _i64, _i64, _vp, _vp]),
    "kq_rotate": (_i32, [_vp, _i64, _i64, _i64, _i32, ctypes.POINTER(kq_rht), _i32, _vp]),
    "kq_chol_inv_workspace_size": (_sz, [_i64]),
    "kq_chol_inv": (_i32, [_vp, _i64, _i64, _f32, _vp, _i64, _vp, _vp, _sz, _vp, _vp]),
    "kq_quantize_layer_workspace_size": (_sz, [_i64, _i64, _i32]),
    "kq_quantize_layer_multi_workspace_size": (_sz, [_i64, _i64, _i32, _i32]),
    "kq_quantize_layer": (_i32, [_vp, _i64, _i64, _i64, _vp, _i64, _vp, _i32, _i32, _i32, _i32,
                                 _vp, _i64, _vp, _vp, _vp, _i64, _vp, _sz, _vp, _vp]),
    "kq_quantize_layer_multi": (_i32, [_vp, _i64, _i64, _i64, _vp, _i64, _vp, _i32, ctypes.POINTER(ctypes.c_int),
                                       ctypes.POINTER(ctypes.c_int), _i32, _i32, ctypes.POINTER(_vp), _i64,
                                       ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.POINTER(_vp), _i64, _vp, _sz,
                                       _vp, _vp]),
    "kq_solver_timing": (_i32, [_i32, ctypes.POINTER(kq_solver_times)]),
    "kq_kron_loss_workspace_size": (_sz, [_i64, _i64]),
    "kq_kron_loss_blocks_workspace_size": (_sz, [_i64, _i64, _i64]),
    "kq_kron_loss_blocks": (_i32, [_vp, _i64, _vp, _i64, _i64, _i64, _vp, _i64, _vp, _i64, _i64, _vp, _vp, _sz, _vp]),
    "kq_kron_loss_multi": (_i32, [_vp, _i64, _i32, ctypes.POINTER(_vp), _i64, _i64, _i64, _vp, _i64, _vp, _i64,
                                  ctypes.POINTER(_vp), _vp, _sz, _vp]),
    "kq_kron_loss": (_i32, [_vp, _i64, _vp, _i64, _i64, _i64, _vp, _i64, _vp, _i64, _vp, _vp, _sz, _vp]),
    "kq_kron_loss_noalloc": (_i32, [_vp, _i64, _vp, _i64, _i64, _i64, _vp, _i64, _vp, _i64, _vp, _vp]),
    "kq_pack_codes": (_i32, [_vp, _i64, _i64, _i64, _i32, _vp, _i64, _vp, _vp]),
    "kq_reverted_matvec_workspace_size": (_sz, [_i64, _i32]),
    "kq_reverted_matvec": (_i32, [_vp, _i64, _i64, _i64, _i32, _vp, _vp, _i32, ctypes.POINTER(kq_rht),
                                  ctypes.POINTER(kq_rht), _vp, _i64, _i32, _vp, _i64, _vp, _sz, _vp]),
    "kq_allocate_bits": (_i32, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64), _i32,
                                ctypes.POINTER(ctypes.c_int), _i32, _f64, ctypes.POINTER(ctypes.c_int)]),
}

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libkronq.so (once) and declare every entry point's signature."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m post_weight_quantization_syrk_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status, where):
    if status != KQ_OK:
        detail = load().kq_last_error().decode(errors="replace")
        raise KronqError(status, detail, where)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _mat(t, dtype, name):
    """Row-major matrix check; returns the leading dimension."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D row-major tensor (unit column stride)")
    return t.stride(0) if t.shape[0] > 1 else max(t.shape[1], t.stride(0))


def _buf(ws):
    return (ctypes.c_void_p(0), 0) if ws is None else (ctypes.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size())


def workspace(nbytes: int, device) -> torch.Tensor:
    """A device byte buffer for a kq_* workspace (torch allocations are 256-byte aligned)."""
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def new_info(device) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def check_info(info: torch.Tensor, where: str = "device"):
    """Raise KronqError if a kernel recorded an error in `info` (synchronises)."""
    v = int(info.item())
    if v != 0:
        code, index = (v >> 24) & 0xFF, v & 0xFFFFFF
        raise KronqError(code, f"recorded by a kernel at index {index}", where)


# ----------------------------------------------------------------- wrappers

def kq_version() -> int:
    return int(load().kq_version())


def kq_launch_count() -> int:
    return int(load().kq_launch_count())


def kq_status_string(s: int) -> str:
    return load().kq_status_string(int(s)).decode()


def kq_accum_cov_workspace_size(n: int, d: int) -> int:
    return int(load().kq_accum_cov_workspace_size(int(n), int(d)))


def kq_accum_cov(A, C, alpha, accumulate=False, ws=None, info=None, stream=None):
    """C (+)= alpha * A^T A, A bf16 [n, d], C fp32 [d, d]."""
    lda = _mat(A, torch.bfloat16, "A")
    ldc = _mat(C, torch.float32, "C")
    n, d = A.shape
    if C.shape != (d, d):
        raise ValueError("C must be [d, d]")
    if ws is None:
        ws = workspace(kq_accum_cov_workspace_size(n, d), A.device)
    wp, wb = _buf(ws)
    _check(load().kq_accum_cov(_ptr(A), n, d, lda, _ptr(C), ldc, float(alpha), int(bool(accumulate)),
                               wp, wb, _ptr(info), _stream(stream)), "kq_accum_cov")


def kq_sensitivity_blocks(H_X, H_Gb, out3, stream=None):
    """out3 = tr H_X, tr H_G, product, with H_G in the block layout [d_out, k]."""
    ldx = _mat(H_X, torch.float32, "H_X")
    ldg = _mat(H_Gb, torch.float32, "H_Gb")
    if out3.dtype != torch.float64 or out3.numel() < 3 or not out3.is_cuda:
        raise TypeError("out3 must be a CUDA float64 tensor of 3 elements")
    _check(load().kq_sensitivity_blocks(_ptr(H_X), H_X.shape[0], ldx, _ptr(H_Gb), H_Gb.shape[0], H_Gb.shape[1], ldg,
                                        _ptr(out3), _stream(stream)), "kq_sensitivity_blocks")


def kq_accum_cov_blocks_workspace_size(n: int, d: int, k: int) -> int:
    return int(load().kq_accum_cov_blocks_workspace_size(int(n), int(d), int(k)))


def kq_accum_cov_blocks(A, k, C, alpha, accumulate=False, ws=None, info=None, stream=None):
    """The k x k diagonal blocks of alpha * A^T A into C fp32 [d, k] (block b in rows b k ..)."""
    lda = _mat(A, torch.bfloat16, "A")
    ldc = _mat(C, torch.float32, "C")
    n, d = A.shape
    if C.shape != (d, k):
        raise ValueError("C must be [d, k]")
    if ws is None:
        ws = workspace(kq_accum_cov_blocks_workspace_size(n, d, k), A.device)
    wp, wb = _buf(ws)
    _check(load().kq_accum_cov_blocks(_ptr(A), n, d, lda, int(k), _ptr(C), ldc, float(alpha), int(bool(accumulate)),
                                      wp, wb, _ptr(info), _stream(stream)), "kq_accum_cov_blocks")


def kq_channel_energy(A, out, alpha, ws=None, info=None, stream=None):
    """out fp32 [d] = alpha * sum_t A[t, j]^2 for bf16 A [n, d]."""
    lda = _mat(A, torch.bfloat16, "A")
    n, d = A.shape
    if out.dtype != torch.float32 or not out.is_cuda or out.numel() < d:
        raise TypeError("out must be a CUDA float32 tensor of d elements")
    if ws is None:
        ws = workspace(int(load().kq_channel_energy_workspace_size(d)), A.device)
    wp, wb = _buf(ws)
    _check(load().kq_channel_energy(_ptr(A), n, d, lda, float(alpha), _ptr(out), wp, wb, _ptr(info),
                                    _stream(stream)), "kq_channel_energy")


def kq_balance_permutation(energy, k, perm, stream=None):
    """perm int64 [d]: output channels dealt to d/k blocks by descending energy."""
    d = energy.numel()
    if energy.dtype != torch.float32 or perm.dtype != torch.int64 or perm.numel() < d:
        raise TypeError("energy float32 [d], perm int64 [d]")
    _check(load().kq_balance_permutation(_ptr(energy), d, int(k), _ptr(perm), _stream(stream)),
           "kq_balance_permutation")


def kq_act_order_permutation(H, perm, stream=None):
    """perm int64 [n]: columns by descending diagonal of H (ties: lower index)."""
    ldh = _mat(H, torch.float32, "H")
    n = H.shape[0]
    if perm.dtype != torch.int64 or perm.numel() < n or not perm.is_cuda:
        raise TypeError("perm must be a CUDA int64 tensor of n elements")
    _check(load().kq_act_order_permutation(_ptr(H), n, ldh, _ptr(perm), _stream(stream)), "kq_act_order_permutation")


def kq_gather(M, out, row_idx=None, col_idx=None, info=None, stream=None):
    """out[i, j] = M[row_idx[i], col_idx[j]] (either index may be None) for
    float32, bf16 or uint8 matrices of the same shape."""
    if M.dtype != out.dtype or M.dtype not in (torch.float32, torch.bfloat16, torch.uint8):
        raise TypeError("M and out must have the same dtype: float32, bf16 or uint8")
    ldm = _mat(M, M.dtype, "M")
    ldo = _mat(out, out.dtype, "out")
    if M.shape != out.shape:
        raise ValueError("M and out must have the same shape")
    for ix in (row_idx, col_idx):
        if ix is not None and (ix.dtype != torch.int64 or not ix.is_cuda):
            raise TypeError("indices must be CUDA int64 tensors")
    _check(load().kq_gather(_ptr(M), ldm, M.element_size(), _ptr(row_idx), _ptr(col_idx), M.shape[0], M.shape[1],
                            _ptr(out), ldo, _ptr(info), _stream(stream)), "kq_gather")


def kq_sensitivity(H_X, H_G, out3, stream=None):
    """out3 (fp64[3]) = tr H_X, tr H_G, their product."""
    ldx = _mat(H_X, torch.float32, "H_X")
    ldg = _mat(H_G, torch.float32, "H_G")
    if out3.dtype != torch.float64 or out3.numel() < 3 or not out3.is_cuda:
        raise TypeError("out3 must be a CUDA float64 tensor of 3 elements")
    _check(load().kq_sensitivity(_ptr(H_X), H_X.shape[0], ldx, _ptr(H_G), H_G.shape[0], ldg, _ptr(out3),
                                 _stream(stream)), "kq_sensitivity")


class RHT:
    """Device-side parameters of T = (Q_m kron H_p / sqrt(p)) diag(signs)."""

    def __init__(self, n, log2_p, m, signs, Qm=None):
        if signs.dtype != torch.float32 or not signs.is_cuda or signs.numel() != n:
            raise TypeError("signs must be a CUDA float32 tensor of n elements")
        if m > 1 and (Qm is None or Qm.dtype != torch.float32 or not Qm.is_cuda or Qm.numel() != m * m):
            raise TypeError("Qm must be a CUDA float32 [m, m] tensor when m > 1")
        self.signs = signs.contiguous()
        self.Qm = None if Qm is None else Qm.contiguous()
        self.c = kq_rht(int(n), int(log2_p), int(m), self.signs.data_ptr(),
                        0 if self.Qm is None else self.Qm.data_ptr())


def kq_rotate(M, axis, T: RHT, inverse=False, stream=None):
    """In place: axis ROWS: M <- T M; axis COLS: M <- M T^T (T^T when inverse)."""
    ld = _mat(M, torch.float32, "M")
    _check(load().kq_rotate(_ptr(M), M.shape[0], M.shape[1], ld, int(axis), ctypes.byref(T.c), int(bool(inverse)),
                            _stream(stream)), "kq_rotate")


def kq_chol_inv_workspace_size(n: int) -> int:
    return int(load().kq_chol_inv_workspace_size(int(n)))


def kq_chol_inv(H, damp_frac, Uc, dead_mask=None, ws=None, info=None, stream=None):
    ldh = _mat(H, torch.float32, "H")
    ldu = _mat(Uc, torch.float32, "Uc")
    n = H.shape[0]
    if dead_mask is not None and (dead_mask.dtype != torch.uint8 or dead_mask.numel() < n):
        raise TypeError("dead_mask must be uint8 [n]")
    if ws is None:
        ws = workspace(kq_chol_inv_workspace_size(n), H.device)
    wp, wb = _buf(ws)
    _check(load().kq_chol_inv(_ptr(H), n, ldh, float(damp_frac), _ptr(Uc), ldu, _ptr(dead_mask), wp, wb,
                              _ptr(info), _stream(stream)), "kq_chol_inv")


def kq_quantize_layer_workspace_size(d_out: int, d_in: int, block: int = 128) -> int:
    return int(load().kq_quantize_layer_workspace_size(int(d_out), int(d_in), int(block)))


def kq_quantize_layer_multi_workspace_size(d_out: int, d_in: int, block: int = 128, count: int = 1) -> int:
    """Workspace with which kq_quantize_layer_multi solves `count` settings side by side."""
    return int(load().kq_quantize_layer_multi_workspace_size(int(d_out), int(d_in), int(block), int(count)))


def kq_quantize_layer(W, Uc, dead_mask, bits, group, codes, scales, zeros, W_hat, block=128,
                      gemm_mode=KQ_GEMM_FP32, ws=None, info=None, stream=None):
    ldw = _mat(W, torch.float32, "W")
    ldu = _mat(Uc, torch.float32, "Uc")
    ldq = _mat(codes, torch.uint8, "codes")
    ldh = _mat(W_hat, torch.float32, "W_hat")
    d_out, d_in = W.shape
    ng = 1 if not group else -(-d_in // group)
    for t, nm in ((scales, "scales"), (zeros, "zeros")):
        if t.dtype != torch.float32 or not t.is_contiguous() or t.numel() < d_out * ng:
            raise TypeError(f"{nm} must be contiguous float32 [d_out, n_groups]")
    if ws is None:
        ws = workspace(kq_quantize_layer_workspace_size(d_out, d_in, block), W.device)
    wp, wb = _buf(ws)
    _check(load().kq_quantize_layer(_ptr(W), d_out, d_in, ldw, _ptr(Uc), ldu, _ptr(dead_mask), int(bits), int(group),
                                    int(block), int(gemm_mode), _ptr(codes), ldq, _ptr(scales), _ptr(zeros),
                                    _ptr(W_hat), ldh, wp, wb, _ptr(info), _stream(stream)), "kq_quantize_layer")


def _ptrs(ts):
    return (_vp * len(ts))(*[t.data_ptr() for t in ts])


def kq_quantize_layer_multi(W, Uc, dead_mask, settings, codes, scales, zeros, W_hat, block=128,
                            gemm_mode=KQ_GEMM_FP32, ws=None, info=None, stream=None):
    """kq_quantize_layer for several (bits, group) settings of one layer; the
    output lists hold one tensor per setting (same shapes as for one)."""
    k = len(settings)
    if not (k and len(codes) == len(scales) == len(zeros) == len(W_hat) == k):
        raise ValueError("one codes/scales/zeros/W_hat tensor per setting")
    ldw = _mat(W, torch.float32, "W")
    ldu = _mat(Uc, torch.float32, "Uc")
    ldq = _mat(codes[0], torch.uint8, "codes")
    ldh = _mat(W_hat[0], torch.float32, "W_hat")
    d_out, d_in = W.shape
    for (b, g), c, s_, z, wh in zip(settings, codes, scales, zeros, W_hat):
        ng = 1 if not g else -(-d_in // g)
        if _mat(c, torch.uint8, "codes") != ldq or _mat(wh, torch.float32, "W_hat") != ldh:
            raise ValueError("every codes / W_hat tensor needs the same leading dimension")
        for t, nm in ((s_, "scales"), (z, "zeros")):
            if t.dtype != torch.float32 or not t.is_contiguous() or t.numel() < d_out * ng:
                raise TypeError(f"{nm} must be contiguous float32 [d_out, n_groups]")
    if ws is None:
        ws = workspace(kq_quantize_layer_multi_workspace_size(d_out, d_in, block, k), W.device)
    wp, wb = _buf(ws)
    bits = (ctypes.c_int * k)(*[int(b) for b, _ in settings])
    groups = (ctypes.c_int * k)(*[int(g) for _, g in settings])
    _check(load().kq_quantize_layer_multi(_ptr(W), d_out, d_in, ldw, _ptr(Uc), ldu, _ptr(dead_mask), k, bits, groups,
                                          int(block), int(gemm_mode), _ptrs(codes), ldq, _ptrs(scales), _ptrs(zeros),
                                          _ptrs(W_hat), ldh, wp, wb, _ptr(info), _stream(stream)),
           "kq_quantize_layer_multi")


def kq_kron_loss_workspace_size(d_out: int, d_in: int) -> int:
    return int(load().kq_kron_loss_workspace_size(int(d_out), int(d_in)))


def kq_kron_loss(W, W_hat, H_X, H_G, loss, ws=None, stream=None):
    ldw = _mat(W, torch.float32, "W")
    ldh = _mat(W_hat, torch.float32, "W_hat")
    ldx = _mat(H_X, torch.float32, "H_X")
    ldg = 0 if H_G is None else _mat(H_G, torch.float32, "H_G")
    d_out, d_in = W.shape
    if loss.dtype != torch.float64 or not loss.is_cuda:
        raise TypeError("loss must be a CUDA float64 tensor")
    if ws is None:
        ws = workspace(kq_kron_loss_workspace_size(d_out, d_in), W.device)
    wp, wb = _buf(ws)
    _check(load().kq_kron_loss(_ptr(W), ldw, _ptr(W_hat), ldh, d_out, d_in, _ptr(H_X), ldx, _ptr(H_G), ldg,
                               _ptr(loss), wp, wb, _stream(stream)), "kq_kron_loss")


def kq_kron_loss_multi(W, W_hats, H_X, H_G, losses, ws=None, stream=None):
    """kq_kron_loss of several dequantized layers against one W, H_X, H_G."""
    k = len(W_hats)
    if not (k and len(losses) == k):
        raise ValueError("one loss tensor per W_hat")
    ldw = _mat(W, torch.float32, "W")
    ldh = _mat(W_hats[0], torch.float32, "W_hat")
    for wh, l in zip(W_hats, losses):
        if _mat(wh, torch.float32, "W_hat") != ldh:
            raise ValueError("every W_hat needs the same leading dimension")
        if l.dtype != torch.float64 or not l.is_cuda:
            raise TypeError("loss must be a CUDA float64 tensor")
    ldx = _mat(H_X, torch.float32, "H_X")
    ldg = 0 if H_G is None else _mat(H_G, torch.float32, "H_G")
    d_out, d_in = W.shape
    if ws is None:
        ws = workspace(kq_kron_loss_workspace_size(d_out, d_in), W.device)
    wp, wb = _buf(ws)
    _check(load().kq_kron_loss_multi(_ptr(W), ldw, k, _ptrs(W_hats), ldh, d_out, d_in, _ptr(H_X), ldx, _ptr(H_G), ldg,
                                     _ptrs(losses), wp, wb, _stream(stream)), "kq_kron_loss_multi")


def kq_kron_loss_blocks_workspace_size(d_out: int, d_in: int, k: int) -> int:
    return int(load().kq_kron_loss_blocks_workspace_size(int(d_out), int(d_in), int(k)))


def kq_kron_loss_blocks(W, W_hat, H_X, H_Gb, loss, ws=None, stream=None):
    """Kronecker loss with the block-diagonal H_G given as H_Gb [d_out, k]."""
    ldw = _mat(W, torch.float32, "W")
    ldh = _mat(W_hat, torch.float32, "W_hat")
    ldx = _mat(H_X, torch.float32, "H_X")
    ldg = _mat(H_Gb, torch.float32, "H_Gb")
    d_out, d_in = W.shape
    k = H_Gb.shape[1]
    if H_Gb.shape[0] != d_out:
        raise ValueError("H_Gb must be [d_out, k]")
    if loss.dtype != torch.float64 or not loss.is_cuda:
        raise TypeError("loss must be a CUDA float64 tensor")
    if ws is None:
        ws = workspace(kq_kron_loss_blocks_workspace_size(d_out, d_in, k), W.device)
    wp, wb = _buf(ws)
    _check(load().kq_kron_loss_blocks(_ptr(W), ldw, _ptr(W_hat), ldh, d_out, d_in, _ptr(H_X), ldx, _ptr(H_Gb), k, ldg,
                                      _ptr(loss), wp, wb, _stream(stream)), "kq_kron_loss_blocks")


def kq_kron_loss_noalloc(W, W_hat, H_X, H_G, loss, stream=None):
    """kq_kron_loss with the library's own fixed scratch (no workspace argument)."""
    ldw = _mat(W, torch.float32, "W")
    ldh = _mat(W_hat, torch.float32, "W_hat")
    ldx = _mat(H_X, torch.float32, "H_X")
    ldg = 0 if H_G is None else _mat(H_G, torch.float32, "H_G")
    d_out, d_in = W.shape
    if loss.dtype != torch.float64 or not loss.is_cuda:
        raise TypeError("loss must be a CUDA float64 tensor")
    _check(load().kq_kron_loss_noalloc(_ptr(W), ldw, _ptr(W_hat), ldh, d_out, d_in, _ptr(H_X), ldx, _ptr(H_G), ldg,
                                       _ptr(loss), _stream(stream)), "kq_kron_loss_noalloc")


def kq_allocate_bits(sens, n_params, choices=(2, 3, 4), avg_bits=3.0):
    """Host call: greedy bit allocation; returns a list of ints."""
    k = len(sens)
    s = (ctypes.c_double * k)(*[float(x) for x in sens])
    n = (ctypes.c_int64 * k)(*[int(x) for x in n_params])
    c = (ctypes.c_int * len(choices))(*[int(x) for x in choices])
    out = (ctypes.c_int * max(k, 1))()
    _check(load().kq_allocate_bits(s, n, k, c, len(choices), float(avg_bits), out), "kq_allocate_bits")
    return [int(out[i]) for i in range(k)]


def kq_pack_codes(codes, bits, packed=None, info=None, stream=None):
    """uint8 codes [rows, cols] -> packed words [rows, ceil(cols / 32) * bits]
    (int32 storage of the uint32 words; layout in kronq.h)."""
    ldq = _mat(codes, torch.uint8, "codes")
    rows, cols = codes.shape
    words = -(-cols // 32) * int(bits)
    if packed is None:
        packed = torch.empty((rows, words), dtype=torch.int32, device=codes.device)
    ldp = _mat(packed, torch.int32, "packed")
    if packed.shape[0] != rows or packed.shape[1] < words:
        raise ValueError("packed must be [rows, >= ceil(cols / 32) * bits]")
    if info is None:
        info = new_info(codes.device)
    _check(load().kq_pack_codes(_ptr(codes), rows, cols, ldq, int(bits), _ptr(packed), ldp, _ptr(info),
                                _stream(stream)), "kq_pack_codes")
    return packed


def kq_reverted_matvec_workspace_size(d_in: int, batch: int) -> int:
    return int(load().kq_reverted_matvec_workspace_size(int(d_in), int(batch)))


def kq_reverted_matvec(packed, bits, scales, zeros, group, T_in, T_out, X, Y, ws=None, stream=None):
    """Y = V^T (W_hat' (U X^T))^T for X [batch, d_in]: the packed layer with its
    rotations reverted (T_in / T_out None: the identity)."""
    ldp = _mat(packed, torch.int32, "packed")
    ldx = _mat(X, torch.float32, "X")
    ldy = _mat(Y, torch.float32, "Y")
    batch, d_in = X.shape
    d_out = Y.shape[1]
    if Y.shape[0] != batch or packed.shape[0] != d_out:
        raise ValueError("X [batch, d_in], Y [batch, d_out], packed [d_out, words]")
    for t, nm in ((scales, "scales"), (zeros, "zeros")):
        if t.dtype != torch.float32 or not t.is_contiguous() or not t.is_cuda:
            raise TypeError(f"{nm} must be a contiguous CUDA float32 tensor")
    if ws is None:
        ws = workspace(kq_reverted_matvec_workspace_size(d_in, batch), X.device)
    wp, wb = _buf(ws)
    _check(load().kq_reverted_matvec(_ptr(packed), d_out, d_in, ldp, int(bits), _ptr(scales), _ptr(zeros), int(group),
                                     None if T_in is None else ctypes.byref(T_in.c),
                                     None if T_out is None else ctypes.byref(T_out.c),
                                     _ptr(X), ldx, batch, _ptr(Y), ldy, wp, wb, _stream(stream)),
           "kq_reverted_matvec")
    return Y


KQ_WAIT_LIMIT_DEFAULT_NS = 4_000_000_000


def kq_set_wait_limit_ns(ns):
    """Set the time limit of the tensor-core kernels' device waits (process
    wide); 0 makes a wait give up at its first incomplete poll.  Returns the
    previous limit."""
    return int(load().kq_set_wait_limit_ns(int(ns)))


def kq_solver_timing(enable):
    """Diagnostic: kq_solver_timing(True) starts recording CUDA events around
    this thread's solver launches; kq_solver_timing(False) synchronises and
    returns the per-class sums as a dict."""
    t = kq_solver_times()
    _check(load().kq_solver_timing(1 if enable else 0, None if enable else ctypes.byref(t)), "kq_solver_timing")
    if enable:
        return None
    return {f: getattr(t, f) for f, _ in kq_solver_times._fields_}
