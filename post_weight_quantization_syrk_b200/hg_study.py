"""How much of the output-side flattening survives without the full H_G.

    python -m post_weight_quantization_syrk_b200.hg_study [--layers attn4096,mlp_up11008,mlp_down11008]
                                                         [--tokens 262144] [--out FILE]

KronQ review, Limitations (second limitation): BiIP holds H_G as a full
d_out x d_out matrix, a transient peak of memory; the research thread's
"Sparks" list asks how much of the outlier flattening of bidirectional
incoherence processing survives under blockwise (or low-rank) H_G.  KronQ
paper page, Abstract (1): the output rotation uses the gradient covariance.

For each synthetic layer (the bench's attention and MLP recipes) and each
output side:
  full         V = T (randomised Hadamard on all d_out channels; the default)
  full+P_G     V = T P_G (the H_G-informed permutation, blocks of T's Hadamard size)
  block k      V = (I kron T_k) with only the k x k diagonal blocks of H_G formed
  block k+P_G  the same with P_G dealing channels to the blocks by energy
(with --recipe stress the weights carry outliers on both axes and the
gradient channels are correlated) it reports the exact Kronecker loss tr(dW H_X dW^T H_G) of the quantized
layer in original coordinates (full H_X and H_G, formed here for the
measurement only), the loss the path itself estimates (the blockwise one for
the block variants), the coefficient of variation of W's output-row and
input-column norms before and after the rotations, and the bytes held for
H_G.  The solver does not read H_G (its update is the H_X-only one), so the
quantized weights differ between variants only through V.  Every step runs
in libkronq.so; torch is used for buffers and for the norms of the CV
diagnostic.
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

SETTINGS = {"attn4096": [(4, 0), (3, 0), (2, 0)], "mlp_up11008": [(3, 128), (2, 0)],
            "mlp_down11008": [(3, 128), (2, 0)]}


def cv(W, dim):
    """Coefficient of variation of the L2 norms of W's rows (dim=1) or columns (dim=0)."""
    n = W.double().norm(dim=dim)
    return float(n.std(unbiased=False) / n.mean())


def stress_inputs(spec, seed, dev):
    """A harder variant than the pages' recipes, for this study only: W with
    log-normal(0, 1) output-row and input-column scales (outliers on both
    axes, CV near 1.3) and G with a rank-32 component shared by all output
    channels (off-diagonal H_G) on top of the independent per-channel part."""
    import torch

    import synth
    g = torch.Generator(device=dev)
    g.manual_seed(seed * 7 + 3)
    W = synth.weights(spec, seed, dev)
    W *= torch.exp(torch.randn(spec.d_out, 1, generator=g, device=dev))
    W *= torch.exp(torch.randn(1, spec.d_in, generator=g, device=dev))
    X = synth.activations(spec, seed, dev)
    G = synth.gradients(spec, seed, dev).float()
    r = G.std(dim=0, keepdim=True)
    C = torch.randn(32, spec.d_out, generator=g, device=dev) * r
    G += 0.3 * (torch.randn(spec.n_tokens, 32, generator=g, device=dev) @ C)
    return W, X, G.to(torch.bfloat16)


def run_layer(name, n_tokens, ks, dev, recipe="pages"):
    import torch

    import synth
    import post_weight_quantization_syrk_b200 as P
    from post_weight_quantization_syrk_b200.pipeline import BlockwiseLayerQuantizer, LayerQuantizer

    spec = synth.scaled(synth.WORKLOADS[name], n_tokens=n_tokens)
    seed = synth.layer_seed(3 if name.startswith("mlp") else 2, 0)
    settings = SETTINGS[name]
    with torch.no_grad():
        if recipe == "stress":
            W, X, G = stress_inputs(spec, seed, dev)
        else:
            W = synth.weights(spec, seed, dev)
            X = synth.activations(spec, seed, dev)
            G = synth.gradients(spec, seed, dev)
    Ti, To = synth.rht_params(spec.d_in, seed * 2 + 11), synth.rht_params(spec.d_out, seed * 2 + 12)

    def drht(p):
        return P.RHT(p.n, p.log2_p, p.m, p.signs.to(dev), None if p.Qm is None else p.Qm.to(dev))

    T_in, T_out = drht(Ti), drht(To)
    info = P.new_info(dev)
    # the unrotated covariances, for the exact loss in original coordinates
    HX0 = torch.empty((spec.d_in, spec.d_in), device=dev)
    HG0 = torch.empty((spec.d_out, spec.d_out), device=dev)
    P.kq_accum_cov(X, HX0, 1.0 / n_tokens, False, None, info)
    P.kq_accum_cov(G, HG0, 1.0 / n_tokens, False, None, info)
    out = {"layer": name, "recipe": recipe, "d_out": spec.d_out, "d_in": spec.d_in, "tokens": n_tokens,
           "settings": ["W%d%s" % (b, " g%d" % g if g else "") for b, g in settings],
           "cv_before": {"out": cv(W, 1), "in": cv(W, 0)}, "variants": {}}

    def exact_loss(W_hat_orig):
        loss = torch.zeros(1, dtype=torch.float64, device=dev)
        P.kq_kron_loss(W, W_hat_orig, HX0, HG0, loss)
        return float(loss.item())

    def finish(label, lq, results, to_orig, hg_bytes, ms):
        torch.cuda.synchronize()
        lq.check(label)
        rows = []
        for (b, g), r in zip(settings, results):
            Wh = r.W_hat.clone()
            orig = to_orig(Wh)
            P.kq_rotate(orig, P.KQ_AXIS_COLS, T_in, True)
            rows.append({"setting": "W%d%s" % (b, " g%d" % g if g else ""), "loss_exact": exact_loss(orig),
                         "loss_path": float(r.loss.item())})
        out["variants"][label] = {"cv_after": {"out": cv(lq.Wp, 1), "in": cv(lq.Wp, 0)}, "hg_bytes": hg_bytes,
                                  "path_ms": ms, "results": rows}

    def timed_run(lq, T_o, before_rotate=None):
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        lq.statistics(X, G)
        lq.sensitivity()
        if before_rotate:
            before_rotate(lq)
        lq.rotate(W, T_in, T_o)
        lq.factor(0.01)
        res = lq.alloc_results(settings)
        lq.quantize_all(res)
        lq.loss_all(res)
        e.record()
        torch.cuda.synchronize()
        return res, s.elapsed_time(e)

    # full V = T, and V = T P_G (P_G over blocks of T's Hadamard size)
    for label, perm_k in (("full", None), ("full+P_G", 1 << To.log2_p)):
        lq = LayerQuantizer(spec.d_out, spec.d_in, dev, gemm_mode=P.KQ_GEMM_3XTF32)
        res, ms = timed_run(lq, T_out, (lambda q: q.hg_permutation(G, perm_k)) if perm_k else None)

        def back(Wh, lq=lq):
            P.kq_rotate(Wh, P.KQ_AXIS_ROWS, T_out, True)
            if lq.perm is None:
                return Wh
            inv = torch.empty_like(lq.perm)
            inv.scatter_(0, lq.perm, torch.arange(spec.d_out, dtype=torch.int64, device=dev))
            o = torch.empty_like(Wh)
            P.kq_gather(Wh, o, inv, None, info)
            return o
        finish(label, lq, res, back, spec.d_out * spec.d_out * 4, ms)
        del lq, res
        torch.cuda.empty_cache()
    # blockwise H_G with a block-diagonal V
    for k in ks:
        if spec.d_out % k:
            continue
        Tk = drht(synth.rht_params(k, seed * 2 + 13))
        for balanced in (False, True):
            label = f"block{k}" + ("+P_G" if balanced else "")
            lq = BlockwiseLayerQuantizer(spec.d_out, spec.d_in, k, balanced=balanced, device=dev,
                                         gemm_mode=P.KQ_GEMM_3XTF32)
            res, ms = timed_run(lq, Tk)

            def back(Wh, lq=lq, Tk=Tk):
                o = torch.empty_like(Wh)
                lq.unrotate_output(Wh, Tk, o)
                return o
            finish(label, lq, res, back, spec.d_out * k * 4, ms)
            del lq, res
            torch.cuda.empty_cache()
    return out


def main(argv=None):
    import torch
    import post_weight_quantization_syrk_b200 as P
    ap = argparse.ArgumentParser()
    ap.add_argument("--layers", default="attn4096,mlp_up11008,mlp_down11008")
    ap.add_argument("--tokens", type=int, default=262144)
    ap.add_argument("--blocks", default="256,1024")
    ap.add_argument("--recipe", default="pages", choices=["pages", "stress"],
                    help="pages: the bench's input recipes; stress: weight outliers on both axes and "
                         "correlated gradient channels (see stress_inputs)")
    ap.add_argument("--out", default=None)
    a = ap.parse_args(argv)
    P.load()
    dev = torch.device("cuda", 0)
    t0 = time.time()
    res = [run_layer(n, a.tokens, [int(k) for k in a.blocks.split(",")], dev, a.recipe) for n in a.layers.split(",")]
    doc = {"study": "output side without the full H_G", "wall_s": time.time() - t0, "layers": res}
    text = json.dumps(doc, indent=1)
    if a.out:
        with open(a.out, "w") as f:
            f.write(text)
    print(text)


if __name__ == "__main__":
    main()
