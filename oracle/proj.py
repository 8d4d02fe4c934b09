"""fp64 oracle of the mixer layer's neighbours (test infrastructure; only the
test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
use it).  Plain numpy in double precision, written from "DiffuMamba:
High-Throughput Diffusion LMs with Mamba Backbone", App. A.1 Eq. (10)-(11)
and Table 12; shares no code with the CUDA library.

  adaln     Eq. (10): gamma_t * (x - mu(x)) / sigma(x) + beta_t over each
            token's hidden vector, sigma = sqrt(biased variance + eps)
            (the pages give no eps; the reading takes LayerNorm's 1e-5)
  in_proj   the linear input projection, split into the layer's inputs in
            the column order [x | z | dt_f | dt_b | B_f | C_f | B_b | C_b]
  out_proj  the linear output projection of the layer's gated output
"""
from __future__ import annotations

import numpy as np


def _f64(t) -> np.ndarray:
    if hasattr(t, "detach"):
        t = t.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(t, dtype=np.float64))


def adaln(x, gamma, beta, eps: float = 1e-5) -> np.ndarray:
    """x [b, L, d]; gamma, beta [b, d].  Returns [b, L, d]."""
    x, g, be = _f64(x), _f64(gamma), _f64(beta)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return g[:, None, :] * (x - mu) / np.sqrt(var + eps) + be[:, None, :]


def in_proj(a, w_in, d_inner: int, d_state: int = 16) -> dict:
    """a [b, L, d_model]; w_in [4 d_inner + 4 d_state, d_model].  Returns the
    layer inputs {"x", "z" [b, L, D]; "dt" [2, b, L, D]; "B", "C" [2, b, L, N]}."""
    y = _f64(a) @ _f64(w_in).T
    D, N = d_inner, d_state
    o = 4 * D
    return {"x": y[..., :D], "z": y[..., D:2 * D],
            "dt": np.stack([y[..., 2 * D:3 * D], y[..., 3 * D:4 * D]]),
            "B": np.stack([y[..., o:o + N], y[..., o + 2 * N:o + 3 * N]]),
            "C": np.stack([y[..., o + N:o + 2 * N], y[..., o + 3 * N:o + 4 * N]])}


def out_proj(y, w_out) -> np.ndarray:
    """y [b, L, d_inner]; w_out [d_model, d_inner].  Returns [b, L, d_model]."""
    return _f64(y) @ _f64(w_out).T
