"""A whole Llama-2-7B-shaped model through the KronQ path (32 decoder blocks x
7 linears), driven through the C ABI.

Order (KronQ paper page, Abstract; KronQ review, Method and Comparison):
  pass 1, per block: covariances of the four distinct linear inputs
    (attention input shared by q/k/v, o-projection input, MLP input shared by
    gate/up, down-projection input) and of the seven output gradients, kept
    resident; the trace sensitivity tr(H_G) tr(H_X) of each linear;
  allocation of {2,3,4} bits to an average of 3.0 over all 224 linears from
    the scores (kq_allocate_bits);
  pass 2, per block: BiIP of each input covariance once (q/k/v and gate/up
    share U and H_X, hence one damped Cholesky factor), then per linear the
    rotation of W and H_G, the blocked OBS solve at its allocated bit-width
    and its Kronecker loss.
In pass 2 the weights of all blocks are generated first; then the rotation
of H_X and the Cholesky factorisation of every input group run block after
block on two factor streams (the widest group, the down projection's input
and the longest factorisation, on the caller's stream, the three 4096-wide
groups on a second stream beside it), and every linear's rotations, solve
and loss run on a third stream as soon as its group's factor is ready, so
the factorisations overlap one another and the linears of earlier blocks
(the factorisations are latency-bound chains).  GPU time is the elapsed
time of pass 1's blocks and of pass 2 as a whole, taken with CUDA events;
generating the synthetic inputs is reported separately and is not part of
it.  Phase seconds are each phase's own event time, summed over its calls
(with the overlap they add up to more than the GPU time).  On several ranks
each takes the blocks of dist.shard and the score table is merged across
ranks before the (identical) allocation.
"""
from __future__ import annotations

import dataclasses
import time

import torch

from . import _lib as K
from . import dist as D

D_MODEL = 4096
D_FF = 11008
N_BLOCKS = 32
LINEARS = ("q", "k", "v", "o", "gate", "up", "down")
# input group of each linear, its (d_out, d_in)
INPUT_OF = {"q": "attn", "k": "attn", "v": "attn", "o": "oin", "gate": "mlp", "up": "mlp", "down": "dn"}
SHAPE = {"q": (D_MODEL, D_MODEL), "k": (D_MODEL, D_MODEL), "v": (D_MODEL, D_MODEL), "o": (D_MODEL, D_MODEL),
         "gate": (D_FF, D_MODEL), "up": (D_FF, D_MODEL), "down": (D_MODEL, D_FF)}
INPUT_WIDTH = {"attn": D_MODEL, "oin": D_MODEL, "mlp": D_MODEL, "dn": D_FF}


def synthetic_model(n_tokens, n_blocks=N_BLOCKS, device="cuda", **kw):
    """A ModelQuantizer over the seeded synthetic 7B-shaped model."""
    import synth

    def make_inputs(b, stats_only):
        return synth.model_block(b, n_tokens, stats_only, device)

    def make_rht(b, name, n):
        p = synth.model_rht(b, name, n)
        return K.RHT(p.n, p.log2_p, p.m, p.signs.to(device), None if p.Qm is None else p.Qm.to(device))

    return ModelQuantizer(make_inputs, make_rht, n_tokens, n_blocks, device, **kw)


@dataclasses.dataclass
class Phase:
    ms: float = 0.0

    def add(self, e0, e1):
        self.ms += e0.elapsed_time(e1)


class ModelQuantizer:
    """Drives the 7B-shaped model; `make_inputs(block)` supplies the synthetic
    tensors of one block (X per input group, G and W per linear)."""

    def __init__(self, make_inputs, make_rht, n_tokens, n_blocks=N_BLOCKS, device="cuda",
                 choices=(2, 3, 4), avg_bits=3.0, gemm_mode=K.KQ_GEMM_3XTF32, damp=0.01, rank=0, world=1,
                 overlap=True):
        self.make_inputs, self.make_rht = make_inputs, make_rht
        self.n_tokens, self.n_blocks, self.dev = n_tokens, n_blocks, torch.device(device)
        self.choices, self.avg_bits, self.gemm_mode, self.damp = choices, avg_bits, gemm_mode, damp
        self.info = K.new_info(self.dev)
        self.overlap = overlap
        self.ws = K.workspace(256, self.dev)        # calls on the caller's stream
        self.ws_lin = None                          # calls of the linears (their stream)
        self.ws_fac = None                          # factorisations on the second factor stream
        self.fac_stream = None
        self.phases = {k: Phase() for k in ("statistics", "sensitivity", "rotate", "chol_inv", "quantize", "loss")}
        self.gen_s = 0.0
        self.rank, self.world = rank, world
        self.blocks = D.shard(n_blocks, rank, world)

    def _ws(self, nbytes):
        if nbytes > self.ws.numel():
            self.ws = K.workspace(nbytes, self.dev)
        return self.ws

    def _ws_fac(self, nbytes):
        # the second factor stream's workspace (its factorisations overlap the first's)
        if self.ws_fac is None or nbytes > self.ws_fac.numel():
            self.ws_fac = K.workspace(nbytes, self.dev)
        return self.ws_fac

    def _ws_lin(self, nbytes):
        # allocated while the linears' stream is current, so that the caching
        # allocator ties it to that stream
        if self.ws_lin is None or nbytes > self.ws_lin.numel():
            self.ws_lin = K.workspace(nbytes, self.dev)
        return self.ws_lin

    def _timed(self, name, fn):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        self._events.append((name, e0, e1))

    def allocate(self, sens):
        """Bits for every linear of the model from this rank's scores: sens
        maps (block, linear) -> (tr_X, tr_G, score) for the blocks of this
        rank; the table is merged across ranks, then every rank runs the
        same allocation.  Returns (alloc, full table)."""
        table = torch.zeros((self.n_blocks, len(LINEARS), 3), dtype=torch.float64,
                            device=self.dev if self.world > 1 and self.dev.type == "cuda" else "cpu")
        for (b, lin), v in sens.items():
            table[b, LINEARS.index(lin)] = torch.tensor(v, dtype=torch.float64)
        table = D.merge_table(table).cpu()
        keys = [(b, lin) for b in range(self.n_blocks) for lin in LINEARS]
        full = {k: table[k[0], LINEARS.index(k[1])].tolist() for k in keys}
        n_params = [SHAPE[lin][0] * SHAPE[lin][1] for _, lin in keys]
        bits = K.kq_allocate_bits([full[k][2] for k in keys], n_params, self.choices, self.avg_bits)
        return dict(zip(keys, bits)), full

    def _span_start(self):
        e = torch.cuda.Event(enable_timing=True)
        e.record()
        return e

    def _span_end(self, e0):
        e1 = torch.cuda.Event(enable_timing=True)
        e1.record()
        self._spans.append((e0, e1))

    def _linears(self, b, weights, U, Uc, dead, ready, HX, HG, alloc, results, lin_stream, dev):
        """Rotations of W and H_G, solve and loss of block b's linears on the
        linears' stream, each after its input group's factor."""
        with torch.cuda.stream(lin_stream):
            for lin in LINEARS:
                g = INPUT_OF[lin]
                lin_stream.wait_event(ready[(b, g)])
                d_out, d_in = SHAPE[lin]
                V = self.make_rht(b, "out:" + lin, d_out)
                W = weights[b][lin]
                Hg = HG.pop((b, lin))
                self._timed("rotate", lambda: (K.kq_rotate(W, K.KQ_AXIS_COLS, U[b][g]),
                                               K.kq_rotate(W, K.KQ_AXIS_ROWS, V),
                                               K.kq_rotate(Hg, K.KQ_AXIS_COLS, V),
                                               K.kq_rotate(Hg, K.KQ_AXIS_ROWS, V)))
                nb = alloc[(b, lin)]
                codes = torch.empty((d_out, d_in), dtype=torch.uint8, device=dev)
                scales = torch.empty((d_out, 1), dtype=torch.float32, device=dev)
                zeros = torch.empty((d_out, 1), dtype=torch.float32, device=dev)
                W_hat = torch.empty((d_out, d_in), dtype=torch.float32, device=dev)
                loss = torch.zeros(1, dtype=torch.float64, device=dev)
                ws = self._ws_lin(max(K.kq_quantize_layer_workspace_size(d_out, d_in),
                                      K.kq_kron_loss_workspace_size(d_out, d_in)))
                self._timed("quantize", lambda: K.kq_quantize_layer(W, Uc[(b, g)], dead[(b, g)], nb, 0, codes,
                                                                     scales, zeros, W_hat, gemm_mode=self.gemm_mode,
                                                                     ws=ws, info=self.info))
                self._timed("loss", lambda: K.kq_kron_loss(W, W_hat, HX[(b, g)], Hg, loss, ws))
                results[(b, lin)] = {"bits": nb, "loss": loss, "codes_bytes": codes.numel()}
                del Hg, codes, W_hat

    def run(self):
        self._events, self._spans = [], []
        dev = self.dev
        HX, HG, sens = {}, {}, {}
        sens_dev = {}
        # ---------------- pass 1: statistics and sensitivities (this rank's blocks)
        for b in self.blocks:
            t0 = time.perf_counter()
            inp = self.make_inputs(b, stats_only=True)
            torch.cuda.synchronize()
            self.gen_s += time.perf_counter() - t0
            span = self._span_start()
            for g, X in inp["X"].items():
                d = X.shape[1]
                H = torch.empty((d, d), dtype=torch.float32, device=dev)
                ws = self._ws(K.kq_accum_cov_workspace_size(X.shape[0], d))
                self._timed("statistics", lambda: K.kq_accum_cov(X, H, 1.0 / X.shape[0], False, ws, self.info))
                HX[(b, g)] = H
            for lin, G in inp["G"].items():
                d = G.shape[1]
                H = torch.empty((d, d), dtype=torch.float32, device=dev)
                ws = self._ws(K.kq_accum_cov_workspace_size(G.shape[0], d))
                self._timed("statistics", lambda: K.kq_accum_cov(G, H, 1.0 / G.shape[0], False, ws, self.info))
                HG[(b, lin)] = H
            for lin in LINEARS:
                out = torch.zeros(3, dtype=torch.float64, device=dev)
                self._timed("sensitivity",
                            lambda: K.kq_sensitivity(HX[(b, INPUT_OF[lin])], HG[(b, lin)], out))
                sens_dev[(b, lin)] = out
            self._span_end(span)
            del inp
        torch.cuda.synchronize()
        K.check_info(self.info, "model statistics")
        for k, v in sens_dev.items():
            sens[k] = v.cpu().tolist()
        alloc, sens = self.allocate(sens)
        keys = [(b, lin) for b in range(self.n_blocks) for lin in LINEARS]
        mine = [(b, lin) for b in self.blocks for lin in LINEARS]

        # ---------------- pass 2: BiIP, Cholesky, solver, loss (this rank's blocks)
        # The weights of every block are generated first (untimed).  Then, in
        # one timed span: the factor streams rotate every input group's H_X
        # and factor it, block after block (the widest group on the caller's
        # stream, the three 4096-wide ones on a second factor stream), while
        # the linears' stream quantizes each block's linears as soon as their
        # group's factor is ready; so the factorisations of later blocks
        # overlap the linears of earlier ones.
        main = torch.cuda.current_stream(dev)
        lin_stream = torch.cuda.Stream(device=dev) if self.overlap else main
        if self.overlap and self.fac_stream is None:
            self.fac_stream = torch.cuda.Stream(device=dev)
        fac = self.fac_stream if self.overlap else main
        weights = {}
        for b in self.blocks:
            t0 = time.perf_counter()
            weights[b] = self.make_inputs(b, stats_only=False)["W"]
            torch.cuda.synchronize()
            self.gen_s += time.perf_counter() - t0
        results = {}
        U = {b: {g: self.make_rht(b, "in:" + g, INPUT_WIDTH[g]) for g in INPUT_WIDTH} for b in self.blocks}
        Uc, dead, ready = {}, {}, {}
        span = self._span_start()
        fork = torch.cuda.Event()
        fork.record(main)
        fac.wait_event(fork)
        order = sorted(INPUT_WIDTH, key=lambda g: -INPUT_WIDTH[g])
        for b in self.blocks:
            for i, g in enumerate(order):
                st = main if i == 0 else fac
                H = HX[(b, g)]
                with torch.cuda.stream(st):
                    self._timed("rotate", lambda: (K.kq_rotate(H, K.KQ_AXIS_COLS, U[b][g]),
                                                   K.kq_rotate(H, K.KQ_AXIS_ROWS, U[b][g])))
                    n = H.shape[0]
                    Uc[(b, g)] = torch.empty_like(H)
                    dead[(b, g)] = torch.zeros(n, dtype=torch.uint8, device=dev)
                    ws = self._ws(K.kq_chol_inv_workspace_size(n)) if i == 0 else \
                        self._ws_fac(K.kq_chol_inv_workspace_size(n))
                    self._timed("chol_inv", lambda: K.kq_chol_inv(H, self.damp, Uc[(b, g)], dead[(b, g)], ws,
                                                                  self.info))
                ready[(b, g)] = torch.cuda.Event()
                ready[(b, g)].record(st)
            if not self.overlap:
                self._linears(b, weights, U, Uc, dead, ready, HX, HG, alloc, results, lin_stream, dev)
        if self.overlap:
            for b in self.blocks:
                self._linears(b, weights, U, Uc, dead, ready, HX, HG, alloc, results, lin_stream, dev)
        for st in (lin_stream, fac):
            if st is not main:
                done = torch.cuda.Event()
                done.record(st)
                main.wait_event(done)
        self._span_end(span)
        torch.cuda.synchronize()
        K.check_info(self.info, "model quantization")
        for name, e0, e1 in self._events:
            self.phases[name].add(e0, e1)
        total_ms = sum(e0.elapsed_time(e1) for e0, e1 in self._spans)
        # the job's GPU time is the slowest rank's
        total_s = D.all_max(total_ms / 1e3, self.dev)
        n_weights = sum(SHAPE[lin][0] * SHAPE[lin][1] for _, lin in keys)
        avg = sum(alloc[k] * SHAPE[k[1]][0] * SHAPE[k[1]][1] for k in keys) / n_weights
        return {
            "blocks": self.n_blocks, "linears": len(keys), "weights": n_weights, "ranks": self.world,
            "gpu_seconds": total_s,
            "weights_per_s": n_weights / total_s,
            "phase_seconds": {k: v.ms / 1e3 for k, v in self.phases.items()},
            "input_generation_seconds": self.gen_s,
            "average_bits": avg,
            "bits_histogram": {str(c): sum(1 for k in keys if alloc[k] == c) for c in self.choices},
            "loss_sum_this_rank": float(sum(r["loss"].item() for r in results.values())),
            "per_linear": [{"block": b, "linear": lin, "score": sens[(b, lin)][2], "tr_X": sens[(b, lin)][0],
                            "tr_G": sens[(b, lin)][1], "bits": alloc[(b, lin)],
                            "loss": results[(b, lin)]["loss"].item()} for b, lin in mine],
        }
