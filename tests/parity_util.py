"""Shared helpers of the GPU parity tests: channel subsets and the error bounds.

Error measures against the fp64 oracle (y = oracle, g = CUDA result):
  normwise  = max_i |g_i - y_i| / max_i |y_i|
  bf16-out  : |g_i - y_i| <= 2^-8 |y_i| + TOL_BF16 * max|y|   per element
              (2^-8 |y| bounds the round-to-nearest error of a bf16 store)
Bounds:
  TOL_FP32  = 1e-5   fp32 inputs, fp32 output
  TOL_BF16  = 2e-3   bf16 inputs, fp32 state; measured on the fp32-output mode
  GUARD     = 5e-5   fp32-arithmetic guard for any input dtype: the inputs the
                     oracle sees are exactly the kernel's, so only fp32
                     rounding and the approximate exp2/log2/rcp separate the
                     two; an emulation of the scan with 2^-22 systematic error
                     in every transcendental stays below 3e-6, so 5e-5 leaves
                     >15x margin while catching errors that 2e-3 would not.
"""
from __future__ import annotations

import numpy as np
import torch

TOL_FP32 = 1e-5
TOL_BF16 = 2e-3
GUARD = 5e-5


def normwise(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    return float(np.max(np.abs(got - want)) / max(np.max(np.abs(want)), 1e-300))


def bf16_out_ok(got, want, tol=TOL_BF16) -> bool:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    bound = 2.0 ** -8 * np.abs(want) + tol * np.max(np.abs(want))
    return bool(np.all(np.abs(got - want) <= bound))


def to_cpu64(t) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def to_device(d: dict, device="cuda") -> dict:
    return {k: (v.to(device) if v is not None else None) for k, v in d.items()}


def channel_subset(inp: dict, par: dict, chans) -> tuple[dict, dict]:
    """The exact sub-problem on channels `chans` (channels are independent:
    conv, step size, A, D and the gate are all per channel; B and C are
    shared by every channel)."""
    idx = torch.as_tensor(chans, device=inp["x"].device, dtype=torch.long)
    si = {
        "x": inp["x"].index_select(-1, idx).cpu(),
        "z": inp["z"].index_select(-1, idx).cpu() if inp.get("z") is not None else None,
        "dt": inp["dt"].index_select(-1, idx).cpu(),
        "B": inp["B"].cpu(),
        "C": inp["C"].cpu() if inp.get("C") is not None else None,
    }
    pidx = idx.to(par["A"].device)
    sp = {
        "A": par["A"].index_select(1, pidx).cpu(),
        "D": par["D"].index_select(1, pidx).cpu(),
        "dt_bias": par["dt_bias"].index_select(1, pidx).cpu(),
        "conv_w": par["conv_w"].index_select(1, pidx).cpu(),
        "conv_b": par["conv_b"].index_select(1, pidx).cpu() if par.get("conv_b") is not None else None,
    }
    return si, sp


def sample_channels(D: int, k: int, seed: int) -> list[int]:
    """k channels spread over [0, D): both ends plus random ones."""
    rng = np.random.default_rng(seed)
    picks = {0, D - 1}
    while len(picks) < min(k, D):
        picks.add(int(rng.integers(0, D)))
    return sorted(picks)


def head_subset(inp: dict, par: dict, heads, P: int = 32, N: int = 128):
    """The exact Mamba-2 sub-problem on `heads` (heads are independent once B
    and C, shared by all heads after their own conv, are kept whole).
    Returns (inputs, params, the output channels of those heads)."""
    H = inp["dt"].shape[-1]
    HP = H * P
    dev = inp["z"].device
    hidx = torch.as_tensor(list(heads), device=dev, dtype=torch.long)
    xch = torch.cat([torch.arange(h * P, (h + 1) * P, device=dev) for h in heads])
    cch = torch.cat([xch, torch.arange(HP, HP + 2 * N, device=dev)])
    si = {"xbc": inp["xbc"].index_select(-1, cch).cpu(),
          "z": inp["z"].index_select(-1, xch).cpu(),
          "dt": inp["dt"].index_select(-1, hidx).cpu()}
    pd = par["A"].device
    sp = {"A": par["A"].index_select(1, hidx.to(pd)).cpu(),
          "D": par["D"].index_select(1, hidx.to(pd)).cpu(),
          "dt_bias": par["dt_bias"].index_select(1, hidx.to(pd)).cpu(),
          "conv_w": par["conv_w"].index_select(1, cch.to(pd)).cpu(),
          "conv_b": par["conv_b"].index_select(1, cch.to(pd)).cpu() if par.get("conv_b") is not None else None}
    return si, sp, xch.cpu().numpy()
