"""Latency of the inference-side matvec with U and V reverted online against
the same packed matvec without rotations.

    python -m post_weight_quantization_syrk_b200.infer_bench    (from the repository root:
                                                                it draws the rotations with synth/)

For each layer shape of the 7B model (4-bit, per-channel grid) and batch 1
and 8, it cycles through 24 distinct packed layers (more bytes than L2, so
the weights stream from HBM as in decode) and reports the CUDA-event time per
kq_reverted_matvec call, issued back to back from Python (at batch 1 the
plain call is bound by the host's launch rate, so its time is an upper bound
of the device time), and the device time per call with the 24 calls captured
in one CUDA graph and replayed.  The rotation parameters are seeded synthetic
draws.
"""
import torch

import post_weight_quantization_syrk_b200 as P


def _rht(n, seed, dev):
    import synth
    p = synth.rht_params(n, seed)
    return P.RHT(p.n, p.log2_p, p.m, p.signs.to(dev), None if p.Qm is None else p.Qm.to(dev))


def main(shapes=((4096, 4096), (11008, 4096), (4096, 11008)), batches=(1, 8), n_layers=24, bits=4):
    dev = torch.device("cuda")
    for d_out, d_in in shapes:
        g = torch.Generator(device=dev)
        g.manual_seed(1)
        layers = []
        for _ in range(n_layers):
            codes = torch.randint(0, 1 << bits, (d_out, d_in), dtype=torch.uint8, device=dev, generator=g)
            layers.append(P.kq_pack_codes(codes, bits))
        del codes
        scales = torch.rand((d_out, 1), device=dev) * 0.01 + 0.001
        zeros = torch.full((d_out, 1), float(1 << (bits - 1)), device=dev)
        T_in, T_out = _rht(d_in, 3, dev), _rht(d_out, 4, dev)
        for batch in batches:
            X = torch.randn((batch, d_in), device=dev)
            Y = torch.empty((batch, d_out), device=dev)
            ws = P.workspace(P.kq_reverted_matvec_workspace_size(d_in, batch), dev)
            us = {}
            for name, a, b in (("reverted", T_in, T_out), ("plain", None, None)):
                for i in range(3 * n_layers):
                    P.kq_reverted_matvec(layers[i % n_layers], bits, scales, zeros, 0, a, b, X, Y, ws)
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                n = 10 * n_layers
                e0.record()
                for i in range(n):
                    P.kq_reverted_matvec(layers[i % n_layers], bits, scales, zeros, 0, a, b, X, Y, ws)
                e1.record()
                torch.cuda.synchronize()
                us[name] = e0.elapsed_time(e1) / n * 1e3
                # device time: the calls of one pass over the layers as a CUDA graph
                side = torch.cuda.Stream()
                side.wait_stream(torch.cuda.current_stream())
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.stream(side):
                    with torch.cuda.graph(graph, stream=side):
                        for i in range(n_layers):
                            P.kq_reverted_matvec(layers[i], bits, scales, zeros, 0, a, b, X, Y, ws)
                torch.cuda.current_stream().wait_stream(side)
                graph.replay()
                torch.cuda.synchronize()
                e0.record()
                for _ in range(10):
                    graph.replay()
                e1.record()
                torch.cuda.synchronize()
                us[name + "_dev"] = e0.elapsed_time(e1) / (10 * n_layers) * 1e3
                del graph
            gb = d_out * d_in * bits / 8 / 1e9
            print(f"{d_out}x{d_in} {bits}-bit batch {batch}: reverted {us['reverted']:.2f} us "
                  f"(device {us['reverted_dev']:.2f}), plain {us['plain']:.2f} us (device {us['plain_dev']:.2f}, "
                  f"{gb / (us['plain_dev'] * 1e-6):.0f} GB/s of packed weights), weights {gb * 1e3:.1f} MB, "
                  f"rotation overhead on the device {us['reverted_dev'] - us['plain_dev']:.2f} us", flush=True)
        del layers
        torch.cuda.empty_cache()


if __name__ == "__main__":
    main()
