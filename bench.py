"""Throughput of the KronQ per-layer quantization path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kronq|reference]
                    [--workload attn4096] [--bits 4,3,2]

One step is the whole path for one Llama-2-7B attention-projection-shaped
layer (W 4096x4096, 128 x 2048 = 262144 calibration tokens of bf16 X and G):
both covariance SYRKs, the trace sensitivity, the BiIP rotations of W, H_X and
H_G, the damped Cholesky factor of the inverse, and for each bit-width (W4, W3,
W2 per-channel) the blocked OBS quantization and the Kronecker loss.  The
metric counts the weights quantized: d_out * d_in per bit-width per step.
Inputs are synthetic (seeded), resident in HBM before timing, and larger than
L2 (X and G are 2 GiB each), so no L2 flush is needed between steps.

With N > 1 (torchrun) every rank quantizes its own layer (weak scaling, no
data-path collective); timing is the max over ranks.  Rank 0 prints one JSON
line.  --impl reference times the float64 CPU oracle on a bounded sample of
the same workload on the host cores and prints the same line for it.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "weights quantized/sec per layer"
UNIT = "weights/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="kronq", choices=["kronq", "reference"])
    ap.add_argument("--workload", default="attn4096")
    ap.add_argument("--bits", default="4,3,2")
    ap.add_argument("--group", type=int, default=0)
    ap.add_argument("--gemm", default="3xtf32", choices=["3xtf32", "fp32"],
                    help="precision mode of the solver's trailing update")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-model", action="store_true", help="skip the whole 7B-shaped model run")
    ap.add_argument("--model-blocks", type=int, default=32)
    a = ap.parse_args()
    a.warmup = max(a.warmup, 3)
    return a


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during timing."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.idx)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------- GPU arm

def run_kronq(a):
    import torch
    import torch.distributed as dist

    import synth
    import post_weight_quantization_syrk_b200 as P
    from post_weight_quantization_syrk_b200.pipeline import LayerQuantizer

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    P.load()
    spec = synth.WORKLOADS[a.workload]
    bits = [int(b) for b in a.bits.split(",")]
    settings = [(b, a.group) for b in bits]
    seed = synth.layer_seed(2, rank)
    with torch.no_grad():
        W = synth.weights(spec, seed, dev)
        X = synth.activations(spec, seed, dev)
        G = synth.gradients(spec, seed, dev)
    Ti, To = synth.rht_params(spec.d_in, seed * 2 + 11), synth.rht_params(spec.d_out, seed * 2 + 12)

    def dev_rht(p):
        return P.RHT(p.n, p.log2_p, p.m, p.signs.to(dev), None if p.Qm is None else p.Qm.to(dev))

    T_in, T_out = dev_rht(Ti), dev_rht(To)
    gemm_mode = P.KQ_GEMM_3XTF32 if a.gemm == "3xtf32" else P.KQ_GEMM_FP32
    lq = LayerQuantizer(spec.d_out, spec.d_in, dev, gemm_mode=gemm_mode)
    results = [lq.alloc_result(b, g) for b, g in settings]
    stream = torch.cuda.current_stream()

    stage_events = []   # per timed step: [(name, start_event, end_event), ...]

    def step(timed):
        marks = []

        def mark(name):
            if timed:
                e = torch.cuda.Event(enable_timing=True)
                e.record(stream)
                marks.append((name, e))

        mark("start")
        lq.statistics(X, G)   # the two covariance SYRKs (H_X, then H_G)
        mark("syrk_x2")
        lq.sensitivity()
        mark("sensitivity")
        lq.rotate(W, T_in, T_out)
        mark("rotate")
        lq.factor(0.01)
        mark("chol_inv")
        tag = "".join(f"w{r.bits}" for r in results)
        lq.quantize_all(results)   # every bit-width, one operand split of Uc
        mark(f"quantize_{tag}")
        lq.loss_all(results)       # every bit-width, one split of the smaller Hessian
        mark(f"loss_{tag}")
        if timed:
            stage_events.append(marks)

    for _ in range(a.warmup):
        step(False)
    torch.cuda.synchronize()
    lq.check("warmup")
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    launches0 = P.kq_launch_count()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(a.steps):
        step(True)
    end.record(stream)
    torch.cuda.synchronize()
    launches = P.kq_launch_count() - launches0
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    lq.check("timed steps")
    ms = start.elapsed_time(end)
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_max = float(t.item())
    stages = {}
    for marks in stage_events:
        for (_, e0), (name, e1) in zip(marks[:-1], marks[1:]):
            stages.setdefault(name, []).append(e0.elapsed_time(e1))
    stages_ms = {k: statistics.mean(v) for k, v in stages.items()}
    syrk_ms = [v / 2.0 for v in stages["syrk_x2"]]   # two SYRK launches per step
    weights_per_step = spec.d_out * spec.d_in * len(settings)
    value = weights_per_step * a.steps * world / (ms_max / 1e3)

    # ---- end to end through the public API with host buffers
    e2e = None
    if not a.no_e2e:
        e2e = run_e2e(a, lq, results, W, X, G, T_in, T_out, spec, settings, world, dev)

    # ---- the whole 7B-shaped model (32 blocks x 7 linears); on N ranks each
    # takes every N-th block and the sensitivity table is merged for the
    # allocation (the model's total work is fixed: strong scaling)
    model = None
    if not a.no_model:
        from post_weight_quantization_syrk_b200.model import synthetic_model
        del X, G
        torch.cuda.empty_cache()
        r = synthetic_model(n_tokens=spec.n_tokens, n_blocks=a.model_blocks, device=dev, gemm_mode=gemm_mode,
                            rank=rank, world=world).run()
        model = {k: r[k] for k in ("blocks", "linears", "weights", "ranks", "gpu_seconds", "weights_per_s",
                                   "phase_seconds", "input_generation_seconds", "average_bits", "bits_histogram")}
        model["tokens"] = spec.n_tokens
        model["note"] = ("end-to-end GPU time of the whole path for all linears (statistics, sensitivity, bit "
                         "allocation, BiIP, Cholesky, solver, loss), the slowest rank's when sharded; phase "
                         "seconds are rank 0's; synthetic inputs generated per block, untimed")

    pk, src = peaks()
    flops = spec.n_tokens * spec.d_in * (spec.d_in + 1)    # one SYRK launch on X (d_out == d_in here)
    traffic = syrk_traffic(a.workload)
    syrk_avg = statistics.mean(syrk_ms)
    achieved = flops / (syrk_avg / 1e3) / 1e12
    peak = pk.get("bf16_tflops_sustained", pk.get("bf16_tflops"))
    burst = pk.get("bf16_tflops") or peak
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": ms_max / a.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16->fp32 (SYRK), fp64 (Cholesky), fp32 (solver, loss)", "data": "synthetic",
        "config": {"workload": f"{a.workload}: W {spec.d_out}x{spec.d_in}, N={spec.n_tokens} tokens, "
                               f"{'+'.join('W%d' % b for b in bits)} {'per-channel' if not a.group else 'g%d' % a.group}",
                   "layers_per_rank_per_step": 1, "bit_widths": bits, "group": a.group,
                   "trailing_update": a.gemm,
                   "l2": "inputs larger than L2 (X, G 2 GiB each); no flush"},
        "roofline": {"kernel": "kq_accum_cov (SYRK)", "bound": "tensor", "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{src} bf16 sustained",
                     # the burst figure too: the sustained one was taken at power-capped clocks
                     "burst_peak": burst, "frac_of_burst": achieved / burst,
                     "algorithmic_flops_per_launch": flops,
                     "avg_launch_ms": syrk_avg},
        "stages_ms": stages_ms,
        "gpu_launches": launches,
        "clocks": clk,
        "e2e": e2e,
        "model_7b": model,
    }
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        out["cpu_baseline"] = oracle_sample(spec, settings)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


# DRAM bytes (read + write) of one kq_accum_cov call at 262144 x 4096, from the
# ncu capture summarised in profiles/syrk_tc_kernel_attn4096_traffic.md; valid
# only for the kernel sources it was taken on.
SYRK_TRAFFIC = {"attn4096": 5.00e9}
SYRK_SOURCE_SHA = {"kq_syrk.cu": "219987dcfe1d0668", "kq_tc.cuh": "f59b54090d782541"}


def syrk_traffic(workload):
    import hashlib
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "post_weight_quantization_syrk_b200", "csrc")
    for name, want in SYRK_SOURCE_SHA.items():
        with open(os.path.join(csrc, name), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest()[:16] != want:
                return None
    return SYRK_TRAFFIC.get(workload)


def run_e2e(a, lq, results, W, X, G, T_in, T_out, spec, settings, world, dev):
    """Same step through the public API from pinned host buffers: every step
    copies its inputs host->device and its results (codes, grids, losses)
    device->host inside the timed region.  pipeline.quantize_from_host
    overlaps step i+1's input copies with step i's compute."""
    import torch
    from post_weight_quantization_syrk_b200.pipeline import quantize_from_host
    Wh, Xh, Gh = W.cpu().pin_memory(), X.cpu().pin_memory(), G.cpu().pin_memory()
    n = max(3, min(a.steps, 5))

    def outputs():
        return [(torch.empty(r.codes.shape, dtype=torch.uint8, pin_memory=True),
                 torch.empty(r.scales.shape, pin_memory=True), torch.empty(r.zeros.shape, pin_memory=True),
                 torch.empty(1, dtype=torch.float64, pin_memory=True)) for r in results]

    outs = [outputs() for _ in range(n)]
    h2d = Wh.numel() * 4 + Xh.numel() * 2 + Gh.numel() * 2
    d2h = sum(o[0].numel() + o[1].numel() * 4 + o[2].numel() * 4 + 8 for o in outs[0])
    stream = torch.cuda.current_stream()
    quantize_from_host(lq, [(Wh, Xh, Gh)], T_in, T_out, settings, results, outs[:1])   # warm
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    quantize_from_host(lq, [(Wh, Xh, Gh)] * n, T_in, T_out, settings, results, outs)
    e.record(stream)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e)
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item())
    return {"value": spec.d_out * spec.d_in * len(settings) * n * world / (ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms / n, "steps": n,
            "overlap": "step i+1's host->device copies run on a second stream during step i's compute"}


# ----------------------------------------------------------------- CPU oracle

def oracle_sample(spec, settings, seed=1234):
    """Time the float64 oracle on a bounded sample of the workload and scale
    each stage to the full layer by its work:
      covariances: n_s of the N tokens (cost linear in tokens),
      BiIP rotations, damped Cholesky factor: full size,
      solver: r_s of the d_out rows (rows are independent given Uc),
      Kronecker loss: full size, once, counted for every bit-width."""
    import numpy as np
    import torch

    import oracle as O
    import synth
    n_s, r_s = 1024, 32
    sp = synth.scaled(spec, n_tokens=n_s)
    W = synth.weights(sp, seed).double().numpy()
    X = synth.activations(sp, seed).float().numpy()
    G = synth.gradients(sp, seed).float().numpy()
    Ti, To = synth.rht_params(spec.d_in, 7), synth.rht_params(spec.d_out, 8)
    Tin = O.rht_matrix(Ti.n, Ti.log2_p, Ti.signs.double().numpy(), None if Ti.Qm is None else Ti.Qm.double().numpy())
    Tout = O.rht_matrix(To.n, To.log2_p, To.signs.double().numpy(), None if To.Qm is None else To.Qm.double().numpy())
    t = {}
    c0 = time.perf_counter()
    HX = O.covariance(X)
    HG = O.covariance(G)
    t["cov"] = (time.perf_counter() - c0) * spec.n_tokens / n_s
    c0 = time.perf_counter()
    O.sensitivity(HX, HG)
    Wp, HXp, HGp = O.biip(W, HX, HG, Tin, Tout)
    t["rot"] = time.perf_counter() - c0
    c0 = time.perf_counter()
    Uc, dead, _ = O.chol_inv(HXp, 0.01)
    t["chol"] = time.perf_counter() - c0
    t["quant"] = 0.0
    for b, g in settings:
        c0 = time.perf_counter()
        q = O.quantize_layer(Wp[:r_s], Uc, b, g, 128, dead)
        t["quant"] += (time.perf_counter() - c0) * spec.d_out / r_s
    Wh = np.array(Wp, copy=True)
    Wh[:r_s] = q.W_hat
    c0 = time.perf_counter()
    O.kron_loss(Wp, Wh, HXp, HGp)
    t["loss"] = (time.perf_counter() - c0) * len(settings)
    total = sum(t.values())
    threads = torch.get_num_threads()
    return {"value": spec.d_out * spec.d_in * len(settings) / total, "unit": UNIT,
            "cores": os.cpu_count(), "threads": threads, "kind": "oracle",
            "seconds_per_step_extrapolated": total, "stage_seconds": t,
            "sample": f"covariances on {n_s} of {spec.n_tokens} tokens (x{spec.n_tokens // n_s}); solver on "
                      f"{r_s} of {spec.d_out} rows (x{spec.d_out // r_s}); rotations, Cholesky and one "
                      f"Kronecker loss at full size (loss x{len(settings)}); NumPy float64 on the host cores"}


def run_reference(a):
    rank = int(os.environ.get("RANK", 0))
    if rank != 0:
        return
    import synth
    spec = synth.WORKLOADS[a.workload]
    bits = [int(b) for b in a.bits.split(",")]
    settings = [(b, a.group) for b in bits]
    for _ in range(a.warmup if a.warmup <= 1 else 1):
        oracle_sample(spec, settings)
    vals, secs = [], []
    for k in range(a.steps):
        r = oracle_sample(spec, settings, seed=1234 + k)
        vals.append(r["value"])
        secs.append(r["seconds_per_step_extrapolated"])
    value = len(vals) / sum(1.0 / v for v in vals)
    last = r
    out = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup,
           "ms_per_step": 1e3 * statistics.mean(secs), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
           "config": {"workload": f"{a.workload}: W {spec.d_out}x{spec.d_in}, N={spec.n_tokens} tokens, "
                                  f"{'+'.join('W%d' % b for b in bits)} "
                                  f"{'per-channel' if not a.group else 'g%d' % a.group}",
                      "bit_widths": bits, "group": a.group},
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": last["cores"], "kind": "oracle",
                            "sample": last["sample"]},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_kronq(a)


if __name__ == "__main__":
    main()
