"""Seeded synthetic inputs for the KronQ layer-quantization path.

This module only draws random numbers.  It holds none of the method's
arithmetic, and it serves both the float64 oracle and the CUDA library, which
therefore see bit-identical inputs.  The pages quantize Llama-family layers
with WikiText-2 / web-text calibration data; neither trained weights nor the
datasets are available here, so these recipes stand in for them with the
shapes and value distributions the workloads name:

* weights ~ N(0, std^2), optionally with a fraction of entries scaled up;
* activations X [tokens, d_in]: N(0,1) times a per-channel scale
  (log-normal), optionally with "massive" channels, SiLU-gated Gaussian
  products (MLP down-projection inputs) or Student-t(3) heavy tails;
* output gradients G [tokens, d_out]: N(0,1) times a per-output-channel
  scale drawn log-uniformly over [lo, 1];
* the random rotation parameters the method draws (+-1 signs, and a Haar
  random orthogonal m x m factor when the dimension is m * 2^k with odd m > 1).

Everything is produced with torch generators seeded from the layer seed, on
the CPU for small parity cases and on the GPU for full-size runs.  X and G are
rounded to bf16, the calibration storage format of the path.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

SEED_BASE = 20260000


def layer_seed(cfg_index: int, layer: int = 0) -> int:
    """Seed of layer `layer` of workload number `cfg_index` (1-based)."""
    return SEED_BASE + 100 * int(cfg_index) + int(layer)


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    """Shape and distribution recipe of one synthetic linear layer y = W x."""
    name: str
    d_out: int
    d_in: int
    n_tokens: int
    w_std: float = 0.02
    w_outlier_frac: float = 0.0      # fraction of W entries multiplied by w_outlier_mult
    w_outlier_mult: float = 10.0
    w_bf16: bool = True              # weights stored as bf16 values (else fp32)
    x_kind: str = "lognormal"        # "lognormal" | "silu_gated" | "student_t3"
    x_sigma: float = 1.0             # log-normal sigma of the per-channel scales
    x_massive: int = 0               # channels multiplied by x_massive_mult
    x_massive_mult: float = 100.0
    g_lo: float = 1e-3               # per-output-channel gradient scales ~ LogUniform[g_lo, 1]


# The named workloads.  Sizes: (d_out x d_in, calibration tokens).
WORKLOADS = {
    # 512x512 layer, 2048 tokens; fp32 weights with 1% outliers x10.
    "layer512": LayerSpec("layer512", 512, 512, 2048, w_std=0.02, w_outlier_frac=0.01,
                          w_outlier_mult=10.0, w_bf16=False, x_sigma=1.0, g_lo=1e-3),
    # Llama-2-7B attention projection: 4096x4096, 128 x 2048 tokens.
    "attn4096": LayerSpec("attn4096", 4096, 4096, 262144, w_std=0.02, x_sigma=1.5,
                          x_massive=8, g_lo=1e-4),
    # Llama-2-7B MLP gate/up (4096 -> 11008) and down (11008 -> 4096).
    "mlp_up11008": LayerSpec("mlp_up11008", 11008, 4096, 262144, x_sigma=1.0, g_lo=1e-3),
    "mlp_down11008": LayerSpec("mlp_down11008", 4096, 11008, 262144, x_kind="silu_gated",
                               x_sigma=1.0, g_lo=1e-3),
    # The attention-projection layer with a quarter of the tokens (profiling
    # captures: inputs still larger than L2, a few GB on the device).
    "attn4096_n65536": LayerSpec("attn4096_n65536", 4096, 4096, 65536, w_std=0.02, x_sigma=1.5,
                                 x_massive=8, g_lo=1e-4),
    # The MLP gate/up layer with 16384 tokens (profiling captures of the
    # 11008-wide rotations: H_G is 485 MB, larger than L2; about 2.5 GB on
    # the device in all).
    "mlp_up11008_n16384": LayerSpec("mlp_up11008_n16384", 11008, 4096, 16384, x_sigma=1.0, g_lo=1e-3),
    # Llama-70B-shaped down projection: 28672 -> 8192, 65536 tokens, Student-t(3).
    "down28672": LayerSpec("down28672", 8192, 28672, 65536, w_std=0.01,
                           x_kind="student_t3", g_lo=1e-4),
}


def scaled(spec: LayerSpec, d_out=None, d_in=None, n_tokens=None) -> LayerSpec:
    """The same recipe at other sizes (small parity cases)."""
    return dataclasses.replace(spec, d_out=d_out or spec.d_out, d_in=d_in or spec.d_in,
                               n_tokens=n_tokens or spec.n_tokens)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(shape, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def weights(spec: LayerSpec, seed: int, device="cpu") -> torch.Tensor:
    """W [d_out, d_in] float32 (values bf16-representable when spec.w_bf16)."""
    g = _gen(seed * 4 + 0, device)
    W = _randn((spec.d_out, spec.d_in), g, device) * spec.w_std
    if spec.w_outlier_frac > 0:
        k = int(round(spec.w_outlier_frac * W.numel()))
        idx = torch.randperm(W.numel(), generator=g, device=device)[:k]
        W.view(-1)[idx] *= spec.w_outlier_mult
    if spec.w_bf16:
        W = W.to(torch.bfloat16).to(torch.float32)
    return W


def channel_scales(spec: LayerSpec, seed: int, device="cpu") -> torch.Tensor:
    """Per-input-channel scales of X: LogNormal(0, sigma), massive channels x mult."""
    g = _gen(seed * 4 + 1, device)
    c = torch.exp(_randn((spec.d_in,), g, device) * spec.x_sigma)
    if spec.x_massive:
        idx = torch.randperm(spec.d_in, generator=g, device=device)[:spec.x_massive]
        c[idx] *= spec.x_massive_mult
    return c


def activations(spec: LayerSpec, seed: int, device="cpu", n_tokens=None,
                token_offset_chunks=0) -> torch.Tensor:
    """X [n, d_in] bf16 drawn per spec.x_kind."""
    n = spec.n_tokens if n_tokens is None else n_tokens
    g = _gen(seed * 4 + 2 + 1000003 * token_offset_chunks, device)
    if spec.x_kind == "lognormal":
        Z = _randn((n, spec.d_in), g, device)
        Z *= channel_scales(spec, seed, device)[None, :]
    elif spec.x_kind == "silu_gated":
        a = _randn((n, spec.d_in), g, device)
        Z = torch.nn.functional.silu(a)
        del a
        Z *= _randn((n, spec.d_in), g, device)
        Z *= channel_scales(spec, seed, device)[None, :]
    elif spec.x_kind == "student_t3":
        # t_3 = z0 / sqrt((z1^2 + z2^2 + z3^2) / 3)
        chi = torch.zeros((n, spec.d_in), device=device)
        for _ in range(3):
            z = _randn((n, spec.d_in), g, device)
            chi.addcmul_(z, z)
            del z
        Z = _randn((n, spec.d_in), g, device)
        Z /= torch.sqrt(chi / 3.0)
        del chi
    else:
        raise ValueError(spec.x_kind)
    return Z.to(torch.bfloat16)


def gradients(spec: LayerSpec, seed: int, device="cpu", n_tokens=None,
              token_offset_chunks=0) -> torch.Tensor:
    """G [n, d_out] bf16: N(0,1) times per-output-channel LogUniform[g_lo, 1]."""
    n = spec.n_tokens if n_tokens is None else n_tokens
    g = _gen(seed * 4 + 3, device)
    r = torch.exp(torch.rand((spec.d_out,), generator=g, device=device) * math.log(spec.g_lo))
    g2 = _gen(seed * 4 + 3 + 7919 * (1 + token_offset_chunks), device)
    Z = _randn((n, spec.d_out), g2, device)
    Z *= r[None, :]
    return Z.to(torch.bfloat16)


@dataclasses.dataclass
class RHTParams:
    """Parameters of T = (Q_m kron H_p / sqrt(p)) diag(signs), n = m * 2^log2_p."""
    n: int
    log2_p: int
    m: int
    signs: torch.Tensor              # float32 [n], +-1
    Qm: torch.Tensor | None          # float32 [m, m] (None when m == 1)
    Qm64: np.ndarray | None          # the float64 draw Qm was rounded from


def split_pow2(n: int):
    """n = m * 2^k with m odd."""
    k = (n & -n).bit_length() - 1
    return n >> k, k


def rht_params(n: int, seed: int) -> RHTParams:
    """Random signs and (for odd m > 1) a Haar-random orthogonal m x m matrix.

    The orthogonal draw is the Q factor of a Gaussian matrix with the signs of
    R's diagonal folded in, which makes it Haar distributed.
    """
    m, k = split_pow2(n)
    g = _gen(seed * 4 + 5, "cpu")
    signs = torch.where(torch.rand((n,), generator=g) < 0.5, -1.0, 1.0).to(torch.float32)
    Qm = Qm64 = None
    if m > 1:
        rs = np.random.default_rng(seed * 4 + 6)
        A = rs.standard_normal((m, m))
        Q, R = np.linalg.qr(A)
        Qm64 = Q * np.sign(np.diag(R))[None, :]
        Qm = torch.from_numpy(Qm64.astype(np.float32))
    return RHTParams(n, k, m, signs, Qm, Qm64)


def layer(spec: LayerSpec, seed: int, device="cpu"):
    """(W, X, G, T_in, T_out) for one layer."""
    W = weights(spec, seed, device)
    X = activations(spec, seed, device)
    G = gradients(spec, seed, device)
    T_in = rht_params(spec.d_in, seed * 2 + 11)
    T_out = rht_params(spec.d_out, seed * 2 + 12)
    return W, X, G, T_in, T_out


# ---------------------------------------------------------------------------
# Whole 7B-shaped model (32 blocks x 7 linears): per-block synthetic inputs.
# 4096-wide inputs follow the attention-projection recipe (log-normal(0, 1.5)
# channel scales, 8 massive channels), the 11008-wide down-projection input is
# the SiLU-gated product; gradients get LogUniform[1e-4, 1] output scales.
# ---------------------------------------------------------------------------
MODEL_LINEARS = ("q", "k", "v", "o", "gate", "up", "down")
MODEL_INPUT_OF = {"q": "attn", "k": "attn", "v": "attn", "o": "oin", "gate": "mlp", "up": "mlp", "down": "dn"}
MODEL_SHAPE = {"q": (4096, 4096), "k": (4096, 4096), "v": (4096, 4096), "o": (4096, 4096),
               "gate": (11008, 4096), "up": (11008, 4096), "down": (4096, 11008)}


def model_block(block: int, n_tokens: int, stats_only: bool, device="cuda"):
    """{"X": {group: X}, "G": {linear: G}} (stats_only) or {"W": {linear: W}}."""
    base = WORKLOADS["attn4096"]
    out = {}
    if stats_only:
        X = {}
        for gi, g in enumerate(("attn", "oin", "mlp", "dn")):
            seed = layer_seed(5, 100 * block + gi)
            spec = (scaled(WORKLOADS["mlp_down11008"], d_in=11008, n_tokens=n_tokens) if g == "dn"
                    else scaled(base, d_in=4096, n_tokens=n_tokens))
            X[g] = activations(spec, seed, device)
        G = {}
        for li, lin in enumerate(MODEL_LINEARS):
            d_out, d_in = MODEL_SHAPE[lin]
            spec = scaled(base, d_out=d_out, d_in=d_in, n_tokens=n_tokens)
            G[lin] = gradients(spec, layer_seed(5, 100 * block + 10 + li), device)
        out["X"], out["G"] = X, G
    else:
        W = {}
        for li, lin in enumerate(MODEL_LINEARS):
            d_out, d_in = MODEL_SHAPE[lin]
            spec = scaled(base, d_out=d_out, d_in=d_in)
            W[lin] = weights(spec, layer_seed(5, 100 * block + 20 + li), device)
        out["W"] = W
    return out


def model_rht(block: int, name: str, n: int) -> RHTParams:
    """Rotation parameters of input group / output of one linear of a block."""
    tag = sum((i + 1) * ord(c) for i, c in enumerate(name))
    return rht_params(n, layer_seed(5, 100 * block + 50) * 7 + tag)
