"""KronQ per-linear-layer weight quantization on B200 (sm_100a).

The computation lives in libkronq.so (C ABI, include/kronq.h); this package
is its thin Python binding (``_lib``) plus a layer driver (``pipeline``) that
sequences the ABI calls on torch-provided device memory and streams.
"""
from . import _lib  # noqa: F401
from ._lib import (  # noqa: F401
    KQ_AXIS_COLS, KQ_AXIS_ROWS, KQ_GEMM_3XTF32, KQ_GEMM_FP32, RHT, KronqError, check_info, kq_accum_cov,
    kq_accum_cov_workspace_size, kq_allocate_bits, kq_chol_inv, kq_chol_inv_workspace_size, kq_kron_loss,
    kq_kron_loss_multi, kq_kron_loss_workspace_size, kq_launch_count, kq_pack_codes, kq_quantize_layer,
    kq_quantize_layer_multi, kq_reverted_matvec, kq_reverted_matvec_workspace_size, kq_set_wait_limit_ns, KQ_WAIT_LIMIT_DEFAULT_NS,
    kq_solver_timing, kq_accum_cov_blocks, kq_accum_cov_blocks_workspace_size, kq_channel_energy,
    kq_balance_permutation, kq_gather, kq_sensitivity_blocks, kq_kron_loss_blocks,
    kq_kron_loss_blocks_workspace_size, kq_act_order_permutation,
    kq_quantize_layer_multi_workspace_size, kq_quantize_layer_workspace_size, kq_rotate, kq_sensitivity,
    kq_status_string, kq_version, load, new_info, workspace,
)
