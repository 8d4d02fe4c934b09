"""Seeded synthetic inputs for the bidirectional Mamba mixer layer.

This module only draws random numbers; it holds none of the layer's
arithmetic, so both the CUDA path and the fp64 oracle can be fed from it.

Distributions (the layer's already-projected inputs and S4D-real-initialised
parameters, as the throughput workloads use them):

  x, z, dt_raw             ~ N(0, 1)                       [b, L, D]  (dt per direction)
  B, C                     ~ N(0, 1) per direction          [b, L, N]
  dt_bias[r, d]            = log(expm1(s)), s log-uniform in [1e-3, 1e-1]
                             (so that softplus(dt_bias) = s)
  A[r, d, n]               = -(n + 1)                        (S4D-real)
  D[r, d]                  = 1
  conv_w[r, d, k], conv_b  ~ U(-0.5, 0.5)
  separate parameters for the forward (r = 0) and reverse (r = 1) layers.

Draw order from one ``torch.Generator`` seeded with ``seed`` (fixed, so a
seed names one input set):
  bias_f, bias_b, w_f, b_f, w_b, b_b, x, z, dt_f, dt_b, B_f, C_f, B_b, C_b

The Mamba-2 mixer at the pages' shape (H heads of P channels, one group of B
and C with N states, conv over the C_conv = H*P + 2N channels of xBC):

  xbc_r (x | B | C per direction), z, dt_raw ~ N(0, 1)   [b, L, C_conv], [b, L, H*P], [b, L, H]
  dt_bias[r, h]            = log(expm1(s)), s log-uniform in [1e-3, 1e-1]
  A[r, h]                  = -a, a ~ U(1, 16)               (Mamba-2 initialisation range)
  D[r, h]                  = 1
  conv_w[r, c, k], conv_b  ~ U(-0.5, 0.5)
  draw order: bias_f, bias_b, A_f, A_b, w_f, b_f, w_b, b_b, xbc_f, xbc_b, z, dt_f, dt_b
Floating tensors are drawn in fp32 and then rounded (RNE) to the I/O dtype;
the oracle receives exactly the rounded values widened to fp64.  A CPU
generator and a CUDA generator give different streams for the same seed, so
``device`` is part of an input set's name.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

D_CONV = 4


@dataclass(frozen=True)
class Workload:
    """One named synthetic workload (sizes, dtype and seed)."""
    name: str
    batch: int
    L: int
    d_inner: int
    d_state: int = 16
    dtype: str = "bf16"          # I/O dtype of x, z, dt, B, C and out
    seed: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def tokens(self) -> int:
        return self.batch * self.L

    @property
    def elements(self) -> int:
        return self.batch * self.L * self.d_inner


# The workloads the layer is specified on.
TINY = Workload("tiny_b1_L256_D64_fp32", 1, 256, 64, 16, "fp32", 0)
LAYER_1P3B = Workload("layer_1p3b_b8_L2048_D4096_bf16", 8, 2048, 4096, 16, "bf16", 1)
LONG_SEQ = {L: Workload(f"long_b1_L{L}_D4096_bf16", 1, L, 4096, 16, "bf16", 2)
            for L in (4096, 16384, 65536, 131072)}
BLOCK_CACHED = Workload("block_cached_b16_P65536_G32_D4096_bf16", 16, 32, 4096, 16, "bf16", 4,
                        extra={"prefix": 65536, "block": 32, "blocks": 16, "steps_per_block": 128})
# Block-cached decoding through a stack of layers (the pages' 1.3B denoiser
# has 24 blocks), one cache per layer; the per-step shape of BLOCK_CACHED.
BLOCK_DECODE = Workload("decode_24layers_b16_P65536_G32_K128_D4096_bf16", 16, 32, 4096, 16, "bf16", 7,
                        extra={"layers": 24, "prefix": 65536, "block": 32, "steps_per_block": 128})
def make_proj_case(batch: int, L: int, d_model: int, d_inner: int, N: int = 16, seed: int = 0, device="cpu") -> dict:
    """Inputs of the layer's neighbours (bf16 activations and weights, fp32
    modulation).  Draws h, gamma, beta, w_in, y, w_out: h, y ~ N(0, 1);
    gamma ~ 1 + 0.1 N(0, 1), beta ~ 0.1 N(0, 1) per (batch row, feature);
    weights ~ N(0, 1 / fan_in), so projected values are O(1)."""
    g = _gen(seed, device)

    def randn(*shape, scale=1.0):
        return torch.randn(*shape, generator=g, device=device, dtype=torch.float32) * scale

    bf = torch.bfloat16
    return {
        "h": randn(batch, L, d_model).to(bf),
        "gamma": (1.0 + randn(batch, d_model, scale=0.1)).contiguous(),
        "beta": randn(batch, d_model, scale=0.1).contiguous(),
        "w_in": randn(4 * d_inner + 4 * N, d_model, scale=d_model ** -0.5).to(bf),
        "y": randn(batch, L, d_inner).to(bf),
        "w_out": randn(d_model, d_inner, scale=d_inner ** -0.5).to(bf),
    }


# The projections around the 1.3B-shape layer: d_model 2048 -> d_inner 4096, b 8, L 2048.
PROJ_1P3B = Workload("proj_1p3b_b8_L2048_dmodel2048_D4096_bf16", 8, 2048, 4096, 16, "bf16", 9,
                     extra={"d_model": 2048})

# One sequence of 262,144 tokens cut into contiguous segments, one per GPU
# (the sequence-sharded scan; total work fixed as the GPU count grows).
SHARDED_SEQ = Workload("sharded_b1_L262144_D4096_bf16", 1, 262144, 4096, 16, "bf16", 8)

# The same decoding through 24 Mamba-2 mixers at the pages' shape (a shorter
# prompt: the prefix scan's fp32 workspace grows with its length).
BLOCK_DECODE_M2 = Workload("decode_mamba2_24layers_b16_P8192_G32_K128_H120x32_N128_bf16", 16, 32, 3840, 128, "bf16",
                           8, extra={"layers": 24, "prefix": 8192, "block": 32, "steps_per_block": 128,
                                     "nheads": 120, "headdim": 32, "mixer": "mamba2"})
DENOISER_SWEEP = {L: Workload(f"denoiser_48x128_b1_L{L}_D4096_bf16", 1, L, 4096, 16, "bf16", 3,
                              extra={"layers": 48, "steps": 128})
                  for L in (2048, 8192, 32768, 131072)}


def torch_dtype(name: str) -> torch.dtype:
    return {"fp32": torch.float32, "bf16": torch.bfloat16}[name]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_params(D: int, N: int, g: torch.Generator, device="cpu") -> dict:
    """Parameters of both directions (fp32).  Draws bias_f, bias_b, w_f, b_f, w_b, b_b."""
    lo, hi = math.log(1e-3), math.log(1e-1)
    bias = []
    for _ in range(2):
        s = torch.exp(torch.rand(D, generator=g, device=device, dtype=torch.float64) * (hi - lo) + lo)
        bias.append(torch.log(torch.expm1(s)).float())
    w, cb = [], []
    for _ in range(2):
        w.append(torch.rand(D, D_CONV, generator=g, device=device) - 0.5)
        cb.append(torch.rand(D, generator=g, device=device) - 0.5)
    A = -torch.arange(1, N + 1, device=device, dtype=torch.float32).repeat(2, D, 1).contiguous()
    return {
        "A": A,                                             # [2, D, N]
        "D": torch.ones(2, D, device=device),               # [2, D]
        "dt_bias": torch.stack(bias).contiguous(),          # [2, D]
        "conv_w": torch.stack(w).contiguous(),              # [2, D, 4]
        "conv_b": torch.stack(cb).contiguous(),             # [2, D]
    }


def make_inputs(batch: int, L: int, D: int, N: int, dtype: str, g: torch.Generator,
                device="cpu") -> dict:
    """Layer inputs.  Draws x, z, dt_f, dt_b, B_f, C_f, B_b, C_b."""
    td = torch_dtype(dtype)

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=device, dtype=torch.float32).to(td)

    x = randn(batch, L, D)
    z = randn(batch, L, D)
    dt = torch.empty(2, batch, L, D, device=device, dtype=td)
    dt[0] = randn(batch, L, D)
    dt[1] = randn(batch, L, D)
    B = torch.empty(2, batch, L, N, device=device, dtype=td)
    C = torch.empty(2, batch, L, N, device=device, dtype=td)
    B[0] = randn(batch, L, N)
    C[0] = randn(batch, L, N)
    B[1] = randn(batch, L, N)
    C[1] = randn(batch, L, N)
    return {"x": x, "z": z, "dt": dt, "B": B, "C": C}


def make_case(batch: int, L: int, D: int, N: int = 16, dtype: str = "bf16", seed: int = 0,
              device="cpu"):
    """(inputs, params) for one layer call, drawn in the documented order."""
    g = _gen(seed, device)
    params = make_params(D, N, g, device)
    inputs = make_inputs(batch, L, D, N, dtype, g, device)
    return inputs, params


def make_workload(w: Workload, device="cpu"):
    return make_case(w.batch, w.L, w.d_inner, w.d_state, w.dtype, w.seed, device)


# ---------------------------------------------------------------- Mamba-2 mixer

def make_mamba2_params(H: int, P: int, N: int, g: torch.Generator, device="cpu") -> dict:
    """Parameters of both directions (fp32).  Draws bias_f, bias_b, A_f, A_b, w_f, b_f, w_b, b_b."""
    CH = H * P + 2 * N
    lo, hi = math.log(1e-3), math.log(1e-1)
    bias = []
    for _ in range(2):
        s = torch.exp(torch.rand(H, generator=g, device=device, dtype=torch.float64) * (hi - lo) + lo)
        bias.append(torch.log(torch.expm1(s)).float())
    A = [-(1.0 + 15.0 * torch.rand(H, generator=g, device=device)) for _ in range(2)]
    w, cb = [], []
    for _ in range(2):
        w.append(torch.rand(CH, D_CONV, generator=g, device=device) - 0.5)
        cb.append(torch.rand(CH, generator=g, device=device) - 0.5)
    return {
        "A": torch.stack(A).contiguous(),                   # [2, H]
        "D": torch.ones(2, H, device=device),               # [2, H]
        "dt_bias": torch.stack(bias).contiguous(),          # [2, H]
        "conv_w": torch.stack(w).contiguous(),              # [2, CH, 4]
        "conv_b": torch.stack(cb).contiguous(),             # [2, CH]
    }


def make_mamba2_inputs(batch: int, L: int, H: int, P: int, N: int, dtype: str, g: torch.Generator,
                       device="cpu") -> dict:
    """Mixer inputs.  Draws xbc_f, xbc_b, z, dt_f, dt_b."""
    td = torch_dtype(dtype)
    CH = H * P + 2 * N

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=device, dtype=torch.float32).to(td)

    xbc = torch.empty(2, batch, L, CH, device=device, dtype=td)
    xbc[0] = randn(batch, L, CH)
    xbc[1] = randn(batch, L, CH)
    z = randn(batch, L, H * P)
    dt = torch.empty(2, batch, L, H, device=device, dtype=td)
    dt[0] = randn(batch, L, H)
    dt[1] = randn(batch, L, H)
    return {"xbc": xbc, "z": z, "dt": dt}


def make_mamba2_case(batch: int, L: int, H: int, P: int, N: int, dtype: str = "bf16", seed: int = 0,
                     device="cpu"):
    """(inputs, params) for one Mamba-2 mixer call, drawn in the documented order."""
    g = _gen(seed, device)
    params = make_mamba2_params(H, P, N, g, device)
    inputs = make_mamba2_inputs(batch, L, H, P, N, dtype, g, device)
    return inputs, params


# The pages' 1.3B denoiser layer: d_inner 3840 = 120 heads x 32, d_state 128.
MAMBA2_1P3B = Workload("mamba2_1p3b_b8_L2048_H120x32_N128_bf16", 8, 2048, 3840, 128, "bf16", 5,
                       extra={"nheads": 120, "headdim": 32})
MAMBA2_LONG = {L: Workload(f"mamba2_b1_L{L}_H120x32_N128_bf16", 1, L, 3840, 128, "bf16", 6,
                           extra={"nheads": 120, "headdim": 32})
               for L in (4096, 16384, 65536)}
