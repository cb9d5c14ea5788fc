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

Besides the headline the line carries, all measured outside the timed
region: `roofline` for the dominant kernel (the covariance SYRK, against the
measured burst bf16 peak: the runs hold the maximum SM clock);
`stage_roofline`, every stage of the step against its own bound (SYRK and
trailing-update GEMMs on the tensor pipe, rotations and the quantize pass
against HBM, the Cholesky against an fp64 DGEMM measured in the same run);
`configs`, the per-layer numbers of the other workloads (the 512 x 512
layer, the MLP gate/up and down layers, the 70B-shaped down projection);
`model_7b`, the whole 7B-shaped model.
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
    ap.add_argument("--configs", default="layer512,mlp_up11008,mlp_down11008,down28672",
                    help="other workloads reported per layer (comma list; empty for none)")
    ap.add_argument("--no-diag", action="store_true", help="skip the untimed per-kernel-class diagnostics")
    ap.add_argument("--act-order", action="store_true",
                    help="solve the columns in descending order of the H_X' diagonal (results returned in the "
                         "original order)")
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


def tf32x3_peak(pk, src):
    """Effective peak of a 3xTF32 product: dense tf32 runs at half the bf16
    rate (1.1 against 2.25 PFLOP/s nominal), and every product issues three
    tf32 MMAs (big*big + big*small + small*big)."""
    return {"value": pk["bf16_tflops"] / 2.0 / 3.0, "unit": "TFLOP/s",
            "source": f"{src} burst bf16 {pk['bf16_tflops']} / 2 (tf32 : bf16 nominal) / 3 (MMAs per product)"}


def fp64_peak(dev):
    """fp64 denominator for the Cholesky: a cuBLAS DGEMM (torch.matmul, 8192^3)
    timed here with CUDA events, best of 5; MEASURED_PEAKS.json has no fp64
    figure.  A library GEMM is used only as this yardstick."""
    import torch
    n = 8192
    a = torch.randn((n, n), dtype=torch.float64, device=dev)
    b = torch.randn((n, n), dtype=torch.float64, device=dev)
    torch.matmul(a, b)
    best = None
    for _ in range(5):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        torch.matmul(a, b)
        e.record()
        torch.cuda.synchronize()
        ms = s.elapsed_time(e)
        best = ms if best is None else min(best, ms)
    del a, b
    return {"value": 2.0 * n ** 3 / (best / 1e3) / 1e12, "unit": "TFLOP/s",
            "source": "cuBLAS DGEMM 8192^3 (torch.matmul fp64) measured in this run, best of 5"}


def stage_roofline(spec, settings, stages_ms, pk, src, fp64):
    """Every stage of one step against its own bound.  Algorithmic work per
    unit (one layer): SYRK N d (d + 1) flops per covariance (lower triangle);
    rotations 8 bytes per element per pass, 2 passes each for W, H_X, H_G;
    Cholesky n^3/3 + n^3/3 fp64 flops; quantize pass 13 bytes per weight per
    setting (W slab read; W_hat, codes, errors written); Kronecker loss
    2 d_out d_in (min + max/2) flops per setting as formed (2 d_out d_in
    (d_in + d_out) if both products of the trace were formed in full, also
    reported)."""
    d_out, d_in, N, k = spec.d_out, spec.d_in, spec.n_tokens, len(settings)
    hbm = pk["hbm_gbs"]
    x3 = tf32x3_peak(pk, src)
    q_ms = next(v for n, v in stages_ms.items() if n.startswith("quantize"))
    l_ms = next(v for n, v in stages_ms.items() if n.startswith("loss"))
    out = {}

    def put(name, work, unit, ms, peak, peak_unit, peak_src, note):
        ach = work / (ms / 1e3) / (1e12 if peak_unit == "TFLOP/s" else 1e9)
        out[name] = {"ms": ms, "work": work, "work_unit": unit, "achieved": ach, "unit": peak_unit, "peak": peak,
                     "frac": ach / peak, "peak_source": peak_src, "note": note}

    put("syrk", float(N) * (d_in * (d_in + 1) + d_out * (d_out + 1)), "flop", stages_ms["syrk_x2"],
        pk["bf16_tflops"], "TFLOP/s", f"{src} burst bf16", "both covariances incl. the fixed-order split sum")
    put("rotate", 8.0 * 2 * (d_out * d_in + d_in * d_in + d_out * d_out), "byte", stages_ms["rotate"], hbm, "GB/s",
        f"{src} HBM copy", "6 algorithmic passes (W, H_X, H_G 2 each); the column transform takes 2 passes, so "
                           "9 passes move 1.5x these bytes")
    put("chol_inv", 2.0 * d_in ** 3 / 3.0, "flop", stages_ms["chol_inv"], fp64["value"], "TFLOP/s",
        fp64["source"], "fp64 throughout (DMMA trailing updates, serial 64-column diagonal chain)")
    put("quantize", 13.0 * d_out * d_in * k, "byte", q_ms, hbm, "GB/s", f"{src} HBM copy",
        f"{k} settings solved as one stacked problem (grid fit, in-block recursion, trailing updates)")
    lo, hi = min(d_in, d_out), max(d_in, d_out)
    put("loss", 2.0 * d_out * d_in * (lo + hi / 2.0) * k, "flop", l_ms, x3["value"], "TFLOP/s", x3["source"],
        "3xTF32; work = the products as formed, one Hessian in the first product and the upper block triangle "
        "of the second: 2 d_out d_in (min + max/2) flops per setting")
    full = 2.0 * d_out * d_in * (d_in + d_out) * k
    out["loss"]["work_both_products_full"] = full
    out["loss"]["achieved_vs_full_products"] = full / (l_ms / 1e3) / 1e12
    return out


def run_layer_steps(P, LayerQuantizer, spec, settings, seed, dev, steps, warmup, gemm_mode):
    """Generate one layer, run `warmup` + `steps` whole-path steps with CUDA
    events per stage; returns (ms per step, stage ms, the quantizer)."""
    import torch
    import synth
    with torch.no_grad():
        W = synth.weights(spec, seed, dev)
        X = synth.activations(spec, seed, dev)
        G = synth.gradients(spec, seed, dev)
    Ti, To = synth.rht_params(spec.d_in, seed * 2 + 11), synth.rht_params(spec.d_out, seed * 2 + 12)
    T_in = P.RHT(Ti.n, Ti.log2_p, Ti.m, Ti.signs.to(dev), None if Ti.Qm is None else Ti.Qm.to(dev))
    T_out = P.RHT(To.n, To.log2_p, To.m, To.signs.to(dev), None if To.Qm is None else To.Qm.to(dev))
    lq = LayerQuantizer(spec.d_out, spec.d_in, dev, gemm_mode=gemm_mode)
    results = lq.alloc_results(settings)
    stream = torch.cuda.current_stream()
    names = ["syrk_x2", "sensitivity", "rotate", "chol_inv", "quantize", "loss"]
    per = {n: [] for n in names}
    total = 0.0
    for it in range(warmup + steps):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
        ev[0].record(stream)
        lq.statistics(X, G)
        ev[1].record(stream)
        lq.sensitivity()
        ev[2].record(stream)
        lq.rotate(W, T_in, T_out)
        ev[3].record(stream)
        lq.factor(0.01)
        ev[4].record(stream)
        lq.quantize_all(results)
        ev[5].record(stream)
        lq.loss_all(results)
        ev[6].record(stream)
        torch.cuda.synchronize()
        if it >= warmup:
            for i, n in enumerate(names):
                per[n].append(ev[i].elapsed_time(ev[i + 1]))
            total += ev[0].elapsed_time(ev[-1])
    lq.check(spec.name)
    del X, G
    return total / steps, {n: statistics.mean(v) for n, v in per.items()}, lq, results, W, T_in, T_out


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
    lq = LayerQuantizer(spec.d_out, spec.d_in, dev, gemm_mode=gemm_mode, act_order=a.act_order)
    results = lq.alloc_results(settings)
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

    # ---- untimed diagnostics: fp64 yardstick, solver split by kernel class,
    # host enqueue time per stage
    pk, src = peaks()
    fp64 = fp64_peak(dev)
    solver = None
    host_ms = None
    if not a.no_diag:
        solver = {k: 0.0 for k in ("grid_ms", "inblock_ms", "update_ms", "grid_launches", "inblock_launches",
                                   "update_launches", "update_flops", "inblock_bytes")}
        # the step's own form: every setting in one stacked solve
        P.kq_solver_timing(True)
        lq.quantize_all(results)
        t = P.kq_solver_timing(False)
        for k_ in solver:
            solver[k_] += t[k_]
        torch.cuda.synchronize()
        host_ms = {}
        c0 = time.perf_counter()
        for name, fn in (("statistics", lambda: lq.statistics(X, G)), ("sensitivity", lq.sensitivity),
                         ("rotate", lambda: lq.rotate(W, T_in, T_out)), ("chol_inv", lambda: lq.factor(0.01)),
                         ("quantize", lambda: lq.quantize_all(results)), ("loss", lambda: lq.loss_all(results))):
            t0 = time.perf_counter()
            fn()
            host_ms[name] = (time.perf_counter() - t0) * 1e3
        host_ms["total"] = (time.perf_counter() - c0) * 1e3
        torch.cuda.synchronize()
        lq.check("diagnostics")
    sr = stage_roofline(spec, settings, stages_ms, pk, src, fp64)
    if solver:
        x3 = tf32x3_peak(pk, src)
        ib_ach = solver["inblock_bytes"] / (solver["inblock_ms"] / 1e3) / 1e9
        up_ach = solver["update_flops"] / (solver["update_ms"] / 1e3) / 1e12
        sr["solver_inblock"] = {
            "ms": solver["inblock_ms"], "launches": int(solver["inblock_launches"]),
            "us_per_launch": 1e3 * solver["inblock_ms"] / max(1, solver["inblock_launches"]),
            "work": solver["inblock_bytes"], "work_unit": "byte", "achieved": ib_ach, "unit": "GB/s",
            "peak": pk["hbm_gbs"], "frac": ib_ach / pk["hbm_gbs"], "peak_source": f"{src} HBM copy",
            "note": "per-launch CUDA events over the stacked solve of all settings (untimed diagnostic pass; "
                    "each launch covers every setting's rows)"}
        sr["solver_trailing_gemm"] = {
            "ms": solver["update_ms"], "launches": int(solver["update_launches"]), "work": solver["update_flops"],
            "work_unit": "flop", "achieved": up_ach, "unit": "TFLOP/s", "peak": x3["value"],
            "frac": up_ach / x3["value"], "peak_source": x3["source"],
            "note": "3xTF32 trailing updates of the stacked solve (M = settings x d_out), per-launch CUDA events"}
        sr["solver_grid"] = {"ms": solver["grid_ms"], "launches": int(solver["grid_launches"])}

    # ---- the other workloads, per layer (untimed by the headline; each its
    # own short run with per-stage CUDA events)
    configs = {}
    cfg_settings = {"layer512": [(3, 0)], "mlp_up11008": [(3, 128), (2, 0)], "mlp_down11008": [(3, 128), (2, 0)],
                    "down28672": [(2, 0)]}
    cfg_index = {"layer512": 1, "mlp_up11008": 3, "mlp_down11008": 3, "down28672": 4}
    for name in [c for c in a.configs.split(",") if c]:
        cspec = synth.WORKLOADS[name]
        cset = cfg_settings.get(name, settings)
        small = cspec.d_out * cspec.d_in <= 1 << 20
        ms_c, st_c, lq_c, res_c, W_c, Ti_c, To_c = run_layer_steps(
            P, LayerQuantizer, cspec, cset, synth.layer_seed(cfg_index.get(name, 9), rank), dev,
            steps=10 if small else 2, warmup=3 if small else 1, gemm_mode=gemm_mode)
        configs[name] = {
            "workload": f"{name}: W {cspec.d_out}x{cspec.d_in}, N={cspec.n_tokens} tokens, "
                        + "+".join(f"W{b}" + (f" g{g}" if g else "") for b, g in cset),
            "ms_per_step": ms_c, "weights_per_s": cspec.d_out * cspec.d_in * len(cset) / (ms_c / 1e3),
            "stages_ms": st_c, "stage_roofline": stage_roofline(cspec, cset, st_c, pk, src, fp64),
            "losses": [float(r.loss.item()) for r in res_c], "steps": 10 if small else 2}
        del lq_c, res_c, W_c
        torch.cuda.empty_cache()

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

    flops = spec.n_tokens * spec.d_in * (spec.d_in + 1)    # one SYRK launch on X (d_out == d_in here)
    traffic = syrk_traffic(a.workload)
    syrk_avg = statistics.mean(syrk_ms)
    achieved = flops / (syrk_avg / 1e3) / 1e12
    peak = pk.get("bf16_tflops")
    sustained = pk.get("bf16_tflops_sustained") or peak
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": ms_max / a.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16->fp32 (SYRK), fp64 (Cholesky), fp32 (solver, loss)", "data": "synthetic",
        "config": {"workload": f"{a.workload}: W {spec.d_out}x{spec.d_in}, N={spec.n_tokens} tokens, "
                               f"{'+'.join('W%d' % b for b in bits)} {'per-channel' if not a.group else 'g%d' % a.group}",
                   "layers_per_rank_per_step": 1, "bit_widths": bits, "group": a.group,
                   "trailing_update": a.gemm, "column_order": "act-order" if a.act_order else "natural",
                   "l2": "inputs larger than L2 (X, G 2 GiB each); no flush"},
        "roofline": {"kernel": "kq_accum_cov (SYRK)", "bound": "tensor", "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{src} bf16 burst (the step runs at the maximum SM clock, see clocks)",
                     # the sustained figure too: it was taken at power-capped clocks
                     "sustained_peak": sustained, "frac_of_sustained": achieved / sustained,
                     "algorithmic_flops_per_launch": flops,
                     "avg_launch_ms": syrk_avg},
        "stages_ms": stages_ms,
        "stage_roofline": sr,
        "host_enqueue_ms": host_ms,
        "configs": configs,
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


# DRAM bytes (read + write, both launches) of one kq_accum_cov call at
# 262144 x 4096, from one ncu capture of dram__bytes_read.sum and
# dram__bytes_write.sum; valid only for the kernel sources it was taken on
# (their hashes), else the bench reports null.
SYRK_TRAFFIC = {"attn4096": 5.09e9}
SYRK_SOURCE_SHA = {"kq_syrk.cu": "3634edf2f04853fc", "kq_tc.cuh": "91f487fc41a449d7"}


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
