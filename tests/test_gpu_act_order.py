"""GPU parity of the act-order solve (columns quantized by descending diagonal
of H_X') against the float64 oracle.

"A Unified Hessian-Guided Framework for Post-Training Quantization",
block-LDL rounding: like GPTQ, the blocks with the larger traces are
quantized first.  Stage by stage on the same inputs, as in
test_gpu_parity.py: the permutation bit for bit (both sides decide on the
same fp32 diagonal), the permuted H and W bit for bit, the factor of the
permuted H within the factor tolerance, codes in forced-code mode on the
GPU's permuted W' and factor, and the results in the original column order.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from gpu_util import device_rht, need_gpu, np64

pytestmark = pytest.mark.gpu

SMALL = synth.scaled(synth.WORKLOADS["attn4096"], d_out=352, d_in=704, n_tokens=3000)


@pytest.fixture(scope="module")
def P():
    need_gpu()
    import post_weight_quantization_syrk_b200 as P
    P.load()
    return P


@pytest.mark.parametrize("bits,group", [(3, 0), (2, 0), (4, 128)])
def test_act_order_layer_stagewise(P, bits, group):
    from post_weight_quantization_syrk_b200.pipeline import LayerQuantizer
    W, X, G, Ti, To = synth.layer(SMALL, 31)
    lq = LayerQuantizer(SMALL.d_out, SMALL.d_in, gemm_mode=P.KQ_GEMM_3XTF32, act_order=True)
    res = lq.run(W.cuda(), X.cuda(), G.cuda(), device_rht(Ti), device_rht(To), [(bits, group)])
    torch.cuda.synchronize()
    lq.check("act-order")
    r = res[0]
    HXp = np64(lq.H_X)
    perm = lq.perm_in.cpu().numpy()
    assert np.array_equal(perm, O.act_order_permutation(lq.H_X.cpu().numpy()))
    assert perm.tolist() != list(range(SMALL.d_in))        # the order really changes
    inv = np.empty_like(perm)
    inv[perm] = np.arange(len(perm))
    assert np.array_equal(lq.inv_in.cpu().numpy(), inv)
    Hq = HXp[np.ix_(perm, perm)]
    assert np.array_equal(np64(lq.Hq), Hq)
    assert np.array_equal(np64(lq.Wq), np64(lq.Wp)[:, perm])
    # the factor of the permuted, damped H_X' (fp64 inside, fp32 out)
    ref_uc, dead, _ = O.chol_inv(Hq, 0.01)
    got_uc = np64(lq.Uc)
    rowmax = np.max(np.abs(ref_uc), axis=1, keepdims=True)
    assert np.max(np.abs(got_uc - ref_uc) - (4e-7 * np.abs(ref_uc) + 1e-8 * rowmax)) <= 0
    # codes in the quantization order, forced-code mode on the GPU's inputs
    q = O.quantize_layer(np64(lq.Wq), got_uc, bits, group, 128, lq.dead.cpu().numpy().astype(bool),
                         force_codes=r.codes_q.cpu().numpy(), force_zeros=r.zeros.cpu().numpy() if group else None)
    assert not q.mismatches, q.mismatches[:3]
    assert not q.zero_mismatches
    total = q.codes.size
    assert (total - q.excused) / total >= 0.999
    if not group:
        assert np.array_equal(r.scales.cpu().numpy()[:, 0], q.scales[:, 0])
    rel = np.linalg.norm(np64(r.W_hat_q) - q.W_hat) / np.linalg.norm(q.W_hat)
    assert rel <= 1e-3
    # results back in the original column order, bit for bit
    assert torch.equal(r.codes, r.codes_q[:, lq.inv_in])
    assert torch.equal(r.W_hat, r.W_hat_q[:, lq.inv_in])
    # the loss of the un-permuted result against the unpermuted Hessians
    L = O.kron_loss(np64(lq.Wp), np64(r.W_hat), HXp, np64(lq.H_G))
    assert abs(r.loss.item() - L) <= 1e-3 * L


def test_act_order_permutation_ties_and_ld(P):
    H = torch.zeros((9, 12), device="cuda")
    d = torch.tensor([1.0, 5.0, 3.0, 5.0, 0.5, 3.0, 3.0, 7.0, 0.0])
    H[torch.arange(9), torch.arange(9)] = d.cuda()
    perm = torch.empty(9, dtype=torch.int64, device="cuda")
    P.kq_act_order_permutation(H[:, :9], perm)
    assert perm.cpu().tolist() == [7, 1, 3, 2, 5, 6, 0, 4, 8]
