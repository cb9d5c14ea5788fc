"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
import numpy as np
import pytest
import torch

import synth


def need_gpu():
    if not torch.cuda.is_available():
        pytest.fail("these tests need a CUDA GPU; run them with -m 'not gpu' on a CPU-only machine")


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def device_rht(params: synth.RHTParams, device="cuda"):
    from post_weight_quantization_syrk_b200 import RHT
    Qm = None if params.Qm is None else params.Qm.to(device)
    return RHT(params.n, params.log2_p, params.m, params.signs.to(device), Qm)


def oracle_T(params: synth.RHTParams):
    """Dense T from the same float32 parameters the GPU gets."""
    import oracle as O
    Q = None if params.Qm is None else params.Qm.double().numpy()
    return O.rht_matrix(params.n, params.log2_p, params.signs.double().numpy(), Q)


def cov_close(H_gpu, H_ref, tol=1e-4):
    """Covariance tolerance: Frobenius relative and per entry relative to
    sqrt(H_ii H_jj) (near-zero off-diagonals carry no relative meaning)."""
    H_gpu = np.asarray(H_gpu, dtype=np.float64)
    fro = np.linalg.norm(H_gpu - H_ref) / max(np.linalg.norm(H_ref), 1e-300)
    d = np.sqrt(np.abs(np.diag(H_ref)))
    scale = np.outer(d, d)
    ent = np.max(np.abs(H_gpu - H_ref) / np.maximum(scale, 1e-300)) if H_ref.size else 0.0
    return fro, ent
