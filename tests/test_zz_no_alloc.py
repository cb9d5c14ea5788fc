"""kq_kron_loss_noalloc: the Kronecker loss for callers that cannot allocate
device memory (an embedding application that owns all device allocations, or
a loop that cannot afford cudaMalloc's implicit synchronisation).  It keeps its
per-tile partial sums in a fixed array inside the library instead of a caller
workspace; its results must agree with kq_kron_loss on the same inputs.

The file name sorts last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _layer(seed, d_out, d_in):
    rng = np.random.default_rng(seed)
    W = torch.from_numpy(rng.normal(0, 0.02, (d_out, d_in)).astype(np.float32)).cuda()
    W_hat = W + torch.from_numpy(rng.normal(0, 0.005, (d_out, d_in)).astype(np.float32)).cuda()
    spec = synth.scaled(synth.WORKLOADS["attn4096"], d_out=d_out, d_in=d_in, n_tokens=1024)
    X = synth.activations(spec, seed).cuda().float()
    G = synth.gradients(spec, seed).cuda().float()
    H_X = (X.T @ X) / X.shape[0]
    H_G = (G.T @ G) / G.shape[0]
    return W, W_hat, H_X.contiguous(), H_G.contiguous()


def test_noalloc_loss_matches_workspace_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA GPU")
    import post_weight_quantization_syrk_b200 as P
    P.load()
    # two calls in a row, different shapes, so the second call runs over
    # whatever the first one left in the shared scratch array
    for seed, (d_out, d_in), with_hg in ((1, (352, 704), True), (2, (200, 136), False)):
        W, W_hat, H_X, H_G = _layer(seed, d_out, d_in)
        hg = H_G if with_hg else None
        ref = torch.zeros(1, dtype=torch.float64, device="cuda")
        got = torch.full((1,), float("nan"), dtype=torch.float64, device="cuda")
        P.kq_kron_loss(W, W_hat, H_X, hg, ref)
        P._lib.kq_kron_loss_noalloc(W, W_hat, H_X, hg, got)
        torch.cuda.synchronize()
        r, g = ref.item(), got.item()
        assert np.isfinite(g) and r > 0
        assert abs(g - r) <= 1e-3 * abs(r), (g, r)


def test_noalloc_rejects_sizes_above_the_fixed_scratch():
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA GPU")
    import post_weight_quantization_syrk_b200 as P
    P.load()
    d_out, d_in = 64 * 257, 64 * 256                 # 65792 tiles > 65536
    W = torch.zeros((1, 1), device="cuda")
    big = torch.zeros((1, 1), device="cuda").expand(d_out, d_in)   # never read: rejected first
    loss = torch.zeros(1, dtype=torch.float64, device="cuda")
    lib = P._lib.load()
    import ctypes
    s = lib.kq_kron_loss_noalloc(ctypes.c_void_p(W.data_ptr()), d_in, ctypes.c_void_p(W.data_ptr()), d_in, d_out,
                                 d_in, ctypes.c_void_p(W.data_ptr()), d_in, None, 0,
                                 ctypes.c_void_p(loss.data_ptr()), None)
    assert s == 2
    assert b"fixed scratch" in lib.kq_last_error()
    del big
