"""pipeline.quantize_from_host (inputs in pinned host memory, the next
layer's copies overlapped with the current layer's compute) returns exactly
what the same calls return on device-resident inputs, layer by layer."""
import pytest
import torch

import synth
from gpu_util import device_rht, need_gpu

pytestmark = pytest.mark.gpu


def test_quantize_from_host_matches_device_run():
    need_gpu()
    import post_weight_quantization_syrk_b200 as P
    from post_weight_quantization_syrk_b200.pipeline import LayerQuantizer, quantize_from_host
    P.load()
    spec = synth.WORKLOADS["layer512"]
    settings = [(3, 0), (2, 128)]
    layers, expect = [], []
    Ti, To = synth.rht_params(spec.d_in, 71), synth.rht_params(spec.d_out, 72)
    T_in, T_out = device_rht(Ti), device_rht(To)
    lq = LayerQuantizer(spec.d_out, spec.d_in, gemm_mode=P.KQ_GEMM_3XTF32)
    for k in range(3):   # three layers of one shape, different data
        seed = synth.layer_seed(0, k)
        W, X, G = synth.weights(spec, seed), synth.activations(spec, seed), synth.gradients(spec, seed)
        layers.append((W.pin_memory(), X.pin_memory(), G.pin_memory()))
        res = lq.run(W.cuda(), X.cuda(), G.cuda(), T_in, T_out, settings)
        torch.cuda.synchronize()
        expect.append([(r.codes.cpu(), r.scales.cpu(), r.zeros.cpu(), r.loss.cpu()) for r in res])
    results = [lq.alloc_result(b, g) for b, g in settings]
    outs = [[(torch.empty(r.codes.shape, dtype=torch.uint8, pin_memory=True),
              torch.empty(r.scales.shape, pin_memory=True), torch.empty(r.zeros.shape, pin_memory=True),
              torch.empty(1, dtype=torch.float64, pin_memory=True)) for r in results] for _ in layers]
    quantize_from_host(lq, layers, T_in, T_out, settings, results, outs)
    torch.cuda.synchronize()
    lq.check("quantize_from_host")
    for got_layer, exp_layer in zip(outs, expect):
        for got, exp in zip(got_layer, exp_layer):
            for g, e in zip(got, exp):
                assert torch.equal(g, e)
