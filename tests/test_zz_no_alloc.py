"""kq_kron_loss_noalloc: the Kronecker loss for callers that cannot allocate
device memory (an embedding application that owns all device allocations, or
a loop that cannot afford cudaMalloc's implicit synchronisation).  It keeps its
per-tile partial sums in a fixed array inside the library instead of a caller
workspace.  Its results must agree with the float64 oracle and, where both
apply (symmetric Hessians), with kq_kron_loss, within the loss tolerance of
the parity tests (1e-3 relative).

The file name sorts last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu
TOL = 1e-3


def _need():
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA GPU")
    import post_weight_quantization_syrk_b200 as P
    P.load()
    return P


def _np(t):
    return t.detach().to("cpu", torch.float64).numpy()


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


def _padded(t, extra):
    """The same matrix as a view with a leading dimension `extra` columns wider."""
    big = torch.full((t.shape[0], t.shape[1] + extra), float("nan"), dtype=t.dtype, device=t.device)
    big[:, :t.shape[1]] = t
    return big[:, :t.shape[1]]


def _noalloc(P, W, W_hat, H_X, H_G):
    got = torch.full((1,), float("nan"), dtype=torch.float64, device="cuda")
    P._lib.kq_kron_loss_noalloc(W, W_hat, H_X, H_G, got)
    torch.cuda.synchronize()
    return got.item()


def test_noalloc_loss_matches_oracle_and_workspace_entry_point():
    P = _need()
    # calls in a row with different shapes, so each runs over whatever the
    # previous one left in the shared scratch array
    for seed, (d_out, d_in), with_hg in ((1, (352, 704), True), (2, (200, 136), False), (3, (256, 4096), True)):
        W, W_hat, H_X, H_G = _layer(seed, d_out, d_in)
        hg = H_G if with_hg else None
        g = _noalloc(P, W, W_hat, H_X, hg)
        ref = O.kron_loss(_np(W), _np(W_hat), _np(H_X), None if hg is None else _np(hg))
        assert np.isfinite(g) and ref > 0
        assert abs(g - ref) <= TOL * ref, (d_out, d_in, g, ref)
        ws_loss = torch.zeros(1, dtype=torch.float64, device="cuda")
        P.kq_kron_loss(W, W_hat, H_X, hg, ws_loss)
        torch.cuda.synchronize()
        assert abs(g - ws_loss.item()) <= TOL * abs(ws_loss.item()), (g, ws_loss.item())


def test_noalloc_loss_nonsymmetric_hessians_and_wide_leading_dimensions():
    """With both H_X and H_G non-symmetric, reading H_G by rows instead of by
    columns would give tr(dW H_X dW^T H_G^T), a different number: the case is
    built so that the two differ by far more than the tolerance.  Every matrix
    is passed as a view with a leading dimension wider than its width."""
    P = _need()
    d_out, d_in = 160, 96
    W, W_hat, H_X, H_G = _layer(11, d_out, d_in)
    rng = np.random.default_rng(12)

    def one_sided(H, upper):
        # entries above (or below) the diagonal perturbed by half of
        # sqrt(H_ii H_jj) times a standard normal: far from symmetric
        d = np.sqrt(np.diag(_np(H)))
        S = np.outer(d, d) * rng.standard_normal(H.shape) * 0.5
        S = np.triu(S, 1) if upper else np.tril(S, -1)
        return torch.from_numpy(S.astype(np.float32)).cuda()

    HXn, HGn = (H_X + one_sided(H_X, True)).contiguous(), (H_G + one_sided(H_G, False)).contiguous()
    ref = O.kron_loss(_np(W), _np(W_hat), _np(HXn), _np(HGn))
    transposed = O.kron_loss(_np(W), _np(W_hat), _np(HXn), _np(HGn).T)
    assert abs(transposed - ref) > 10 * TOL * abs(ref), "case does not separate the two readings"
    for extra in (0, 8):
        g = _noalloc(P, _padded(W, extra), _padded(W_hat, extra + 4), _padded(HXn, extra), _padded(HGn, extra + 12))
        assert abs(g - ref) <= TOL * abs(ref), (extra, g, ref)


def test_noalloc_rejects_sizes_above_the_fixed_scratch():
    P = _need()
    lib = P._lib.load()
    W = torch.zeros((1, 1), device="cuda")
    loss = torch.zeros(1, dtype=torch.float64, device="cuda")

    def call(d_out, d_in):
        # the pointers are never read: the shape is rejected before any launch
        return lib.kq_kron_loss_noalloc(ctypes.c_void_p(W.data_ptr()), d_in, ctypes.c_void_p(W.data_ptr()), d_in,
                                        d_out, d_in, ctypes.c_void_p(W.data_ptr()), d_in, None, 0,
                                        ctypes.c_void_p(loss.data_ptr()), None)

    assert call(64 * 257, 64 * 256) == 2                 # 65792 tiles > 65536
    assert b"fixed scratch" in lib.kq_last_error()
    assert call(64 * 65536, 64) == 2                     # 65536 tiles, but 65536 tile rows > 65535
    assert b"65535" in lib.kq_last_error()
