"""Single calls of the hot path on seeded inputs, to profile one kernel in isolation.

    python -m post_weight_quantization_syrk_b200.prof_cases chol N [--reps R]
    python -m post_weight_quantization_syrk_b200.prof_cases solve D_OUT D_IN [--settings 4,3,2] [--reps R]

`chol` factors H = A A^T / (N + 64) (A a seeded Gaussian N x (N + 64) on the
device) with kq_chol_inv, R times.  `solve` factors a D_IN-wide H of the same
kind and then quantizes a seeded W (D_OUT x D_IN, entries N(0, 0.02^2)) with
kq_quantize_layer_multi, R times, the settings' W_hat stacked in one buffer
(one stacked solve per call), 3xTF32 trailing updates.  Every step runs in
libkronq.so; torch provides the buffers and the seeded inputs.  It prints one
line with the device error word, so that a profiler's plain run can be checked.
"""
from __future__ import annotations

import argparse

import torch

from . import _lib as K


def _spd(n: int, seed: int, dev) -> torch.Tensor:
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    A = torch.randn((n, n + 64), device=dev, generator=g)
    H = (A @ A.T) / (n + 64)
    del A
    return H


def chol(n: int, reps: int, dev) -> int:
    H = _spd(n, 5, dev)
    Uc = torch.empty_like(H)
    dead = torch.zeros(n, dtype=torch.uint8, device=dev)
    ws = K.workspace(K.kq_chol_inv_workspace_size(n), dev)
    info = K.new_info(dev)
    for _ in range(reps):
        K.kq_chol_inv(H, 0.01, Uc, dead, ws, info)
    torch.cuda.synchronize()
    return int(info.item())


def solve(d_out: int, d_in: int, settings, reps: int, dev) -> int:
    H = _spd(d_in, 1, dev)
    Uc = torch.empty_like(H)
    info = K.new_info(dev)
    K.kq_chol_inv(H, 0.01, Uc, None, None, info)
    g = torch.Generator(device=dev)
    g.manual_seed(2)
    W = torch.randn((d_out, d_in), device=dev, generator=g) * 0.02
    k = len(settings)
    codes = [torch.empty((d_out, d_in), dtype=torch.uint8, device=dev) for _ in range(k)]
    ng = [1 if not grp else -(-d_in // grp) for _, grp in settings]
    scales = [torch.empty((d_out, n), device=dev) for n in ng]
    zeros = [torch.empty_like(s) for s in scales]
    stack = torch.empty((k, d_out, d_in), device=dev)
    W_hat = [stack[i] for i in range(k)]
    ws = K.workspace(K.kq_quantize_layer_multi_workspace_size(d_out, d_in, 128, k), dev)
    for _ in range(reps):
        K.kq_quantize_layer_multi(W, Uc, None, settings, codes, scales, zeros, W_hat, gemm_mode=K.KQ_GEMM_3XTF32,
                                  ws=ws, info=info)
    torch.cuda.synchronize()
    return int(info.item())


def main(argv=None):
    ap = argparse.ArgumentParser()
    sub = ap.add_subparsers(dest="case", required=True)
    c = sub.add_parser("chol")
    c.add_argument("n", type=int)
    c.add_argument("--reps", type=int, default=1)
    s = sub.add_parser("solve")
    s.add_argument("d_out", type=int)
    s.add_argument("d_in", type=int)
    s.add_argument("--settings", default="4,3,2", help="bit-widths, per-channel grids")
    s.add_argument("--reps", type=int, default=1)
    a = ap.parse_args(argv)
    K.load()
    dev = torch.device("cuda", 0)
    if a.case == "chol":
        info = chol(a.n, a.reps, dev)
        print(f"chol n={a.n} reps={a.reps} info={info}")
    else:
        settings = [(int(b), 0) for b in a.settings.split(",")]
        info = solve(a.d_out, a.d_in, settings, a.reps, dev)
        print(f"solve {a.d_out}x{a.d_in} settings={settings} reps={a.reps} info={info}")


if __name__ == "__main__":
    main()
