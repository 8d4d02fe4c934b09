"""fp64 CPU oracle for the bidirectional Mamba mixer layer (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps ``bimamba_oracle.c`` (plain C,
double precision, OpenMP over (batch, channel)) through ctypes and shares no
code with the CUDA library.

Every function takes numpy arrays; they are converted to contiguous float64
before the call, so bf16/fp32 inputs are widened exactly.  See the C file's
header for the definitions and the passages of "DiffuMamba: High-Throughput
Diffusion LMs with Mamba Backbone" (§3.2 Eq. (4)-(6), App. A.1 Eq. (7)-(9),
§4.3) that each part follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bimamba_oracle.c")
_SRC2 = os.path.join(_HERE, "mamba2_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

FWD_ONLY = 1
REV_ONLY = 2

MUTATIONS = {
    1: "D skip dropped",
    2: "sign of A flipped",
    3: "forward conv taps reversed",
    4: "reverse direction walks forwards",
    5: "reverse conv made causal",
    6: "dt bias dropped",
    7: "B and C swapped",
    8: "C reads the state before the update",
    9: "delta missing on the B term",
    10: "gate is silu of the sum instead of silu(z)",
    11: "block step ignores the cached conv tail",
    12: "block step ignores the cached state",
    13: "last state dropped",
    14: "conv bias dropped",
    15: "reverse output added after the gate",
}


MUTATIONS2 = {
    1: "B and C skip the conv",
    2: "A taken from the next head",
    3: "delta taken from the next head",
    4: "reverse conv made causal",
    5: "C reads the state before the update",
    6: "D skip dropped",
    7: "B read from the C slice",
    8: "dt bias dropped",
    9: "reverse direction walks forwards",
    10: "delta missing on the drive",
    11: "gate is silu of the sum times z",
    12: "x channels laid out p-major instead of head-major",
}


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (-O2, OpenMP, no fast-math)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_SRC2))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-fno-fast-math", "-o", _LIB, _SRC, _SRC2, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I, Lg, U = ctypes.c_int, ctypes.c_long, ctypes.c_uint
        lib.oracle_layer_fwd.argtypes = [I, Lg, I, I] + [P] * 13 + [U, P, P, P]
        lib.oracle_layer_fwd.restype = I
        lib.oracle_features.argtypes = [I, Lg, I, I] + [P] * 10 + [P, P]
        lib.oracle_features.restype = I
        lib.oracle_prefix_state.argtypes = [I, Lg, I, I] + [P] * 8 + [P, P]
        lib.oracle_prefix_state.restype = I
        lib.oracle_block_step.argtypes = [I, Lg, I, I, P, P] + [P] * 13 + [U, P, P, P, P, P]
        lib.oracle_block_step.restype = I
        lib.oracle2_layer_fwd.argtypes = [I, Lg, I, I, I] + [P] * 10 + [U, P, P, P]
        lib.oracle2_layer_fwd.restype = I
        lib.oracle2_set_mutation.argtypes = [I]
        lib.oracle_set_mutation.argtypes = [I]
        lib.oracle_get_mutation.restype = I
        lib.oracle_set_threads.argtypes = [I]
        lib.oracle_max_threads.restype = I
        _lib = lib
    return _lib


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu")
        a = a.double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def set_mutation(m: int) -> None:
    """Plant mistake ``m`` (see MUTATIONS) in the oracle; 0 restores it."""
    _load().oracle_set_mutation(int(m))


def set_mutation2(m: int) -> None:
    """Plant mistake ``m`` (see MUTATIONS2) in the Mamba-2 oracle; 0 restores it."""
    _load().oracle2_set_mutation(int(m))


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _params(p):
    keys = ("A", "D", "dt_bias", "conv_w", "conv_b")
    return [_f64(p.get(k)) for k in keys]


def layer_fwd(inp: dict, params: dict, flags: int = 0, return_dirs: bool = False):
    """Full-sequence bidirectional layer.

    inp: x, z [b, L, D]; dt [2, b, L, D]; B, C [2, b, L, N]
    params: A [2, D, N]; D, dt_bias [2, D]; conv_w [2, D, 4]; conv_b [2, D] or None
    Returns out [b, L, D] (and y_fwd, y_rev when return_dirs).
    """
    x, z = _f64(inp["x"]), _f64(inp["z"])
    dt, B, C = _f64(inp["dt"]), _f64(inp["B"]), _f64(inp["C"])
    b, L, D = x.shape
    N = B.shape[-1]
    A, Dk, bias, w, cb = _params(params)
    dt0, dt1 = np.ascontiguousarray(dt[0]), np.ascontiguousarray(dt[1])
    B0, B1 = np.ascontiguousarray(B[0]), np.ascontiguousarray(B[1])
    C0, C1 = np.ascontiguousarray(C[0]), np.ascontiguousarray(C[1])
    out = np.empty((b, L, D), np.float64)
    yf = np.empty_like(out) if return_dirs else None
    yr = np.empty_like(out) if return_dirs else None
    rc = _load().oracle_layer_fwd(b, L, D, N, *map(_ptr, (x, z, dt0, dt1, B0, C0, B1, C1, A, Dk, bias, w, cb)),
                                  flags, _ptr(out), _ptr(yf), _ptr(yr))
    if rc != 0:
        raise RuntimeError("oracle_layer_fwd failed")
    return (out, yf, yr) if return_dirs else out


def features(inp: dict, params: dict):
    """u (conv+SiLU output) and delta (softplus step) of both directions, [2, b, L, D]."""
    x = _f64(inp["x"])
    dt, B = _f64(inp["dt"]), _f64(inp["B"])
    b, L, D = x.shape
    N = B.shape[-1]
    A, Dk, bias, w, cb = _params(params)
    dt0, dt1 = np.ascontiguousarray(dt[0]), np.ascontiguousarray(dt[1])
    B0, B1 = np.ascontiguousarray(B[0]), np.ascontiguousarray(B[1])
    u = np.empty((2, b, L, D), np.float64)
    dl = np.empty_like(u)
    rc = _load().oracle_features(b, L, D, N, *map(_ptr, (x, dt0, dt1, B0, B1, A, Dk, bias, w, cb)),
                                 _ptr(u), _ptr(dl))
    if rc != 0:
        raise RuntimeError("oracle_features failed")
    return u, dl


def prefix_state(inp: dict, params: dict):
    """Forward scan over the whole input from zero state: (h [b, D, N], tail [b, 3, D])."""
    x = _f64(inp["x"])
    dt, B = _f64(inp["dt"]), _f64(inp["B"])
    b, P, D = x.shape
    N = B.shape[-1]
    A, Dk, bias, w, cb = _params(params)
    dt0 = np.ascontiguousarray(dt[0])
    B0 = np.ascontiguousarray(B[0])
    h = np.empty((b, D, N), np.float64)
    tail = np.empty((b, 3, D), np.float64)
    rc = _load().oracle_prefix_state(b, P, D, N, *map(_ptr, (x, dt0, B0, A, Dk, bias, w, cb)),
                                     _ptr(h), _ptr(tail))
    if rc != 0:
        raise RuntimeError("oracle_prefix_state failed")
    return h, tail


def block_step(h, tail, inp: dict, params: dict, flags: int = 0, commit: bool = False,
               return_dirs: bool = False):
    """Block step from the cached (h, tail).  Returns out [b, G, D], plus
    (h_new, tail_new) when commit, plus (y_fwd, y_rev) when return_dirs."""
    h, tail = _f64(h), _f64(tail)
    x, z = _f64(inp["x"]), _f64(inp["z"])
    dt, B, C = _f64(inp["dt"]), _f64(inp["B"]), _f64(inp["C"])
    b, G, D = x.shape
    N = B.shape[-1]
    A, Dk, bias, w, cb = _params(params)
    dt0, dt1 = np.ascontiguousarray(dt[0]), np.ascontiguousarray(dt[1])
    B0, B1 = np.ascontiguousarray(B[0]), np.ascontiguousarray(B[1])
    C0, C1 = np.ascontiguousarray(C[0]), np.ascontiguousarray(C[1])
    out = np.empty((b, G, D), np.float64)
    h_new = np.empty_like(h) if commit else None
    t_new = np.empty_like(tail) if commit else None
    yf = np.empty_like(out) if return_dirs else None
    yr = np.empty_like(out) if return_dirs else None
    rc = _load().oracle_block_step(b, G, D, N, _ptr(h), _ptr(tail),
                                   *map(_ptr, (x, z, dt0, dt1, B0, C0, B1, C1, A, Dk, bias, w, cb)),
                                   flags, _ptr(out), _ptr(h_new), _ptr(t_new), _ptr(yf), _ptr(yr))
    if rc != 0:
        raise RuntimeError("oracle_block_step failed")
    res = [out]
    if commit:
        res += [h_new, t_new]
    if return_dirs:
        res += [yf, yr]
    return res[0] if len(res) == 1 else tuple(res)


# ---------------------------------------------------------------- Mamba-2 mixer

def mamba2_dims(inp: dict):
    """(batch, L, H, P, N) of a Mamba-2 input dict."""
    dt, z, xbc = inp["dt"], inp["z"], inp["xbc"]
    b, L, H = dt.shape[1], dt.shape[2], dt.shape[3]
    HP = z.shape[-1]
    P = HP // H
    N = (xbc.shape[-1] - HP) // 2
    return b, L, H, P, N


def mamba2_layer_fwd(inp: dict, params: dict, flags: int = 0, return_dirs: bool = False):
    """Full-sequence bidirectional Mamba-2 mixer (mamba2_oracle.c).

    inp: xbc [2, b, L, H*P + 2N] (per direction: x | B | C before the conv);
         z [b, L, H*P]; dt [2, b, L, H]
    params: A, D, dt_bias [2, H]; conv_w [2, H*P + 2N, 4]; conv_b [2, H*P + 2N] or None
    Returns out [b, L, H*P] (and y_fwd, y_rev when return_dirs).
    """
    b, L, H, P, N = mamba2_dims(inp)
    xbc, z, dt = _f64(inp["xbc"]), _f64(inp["z"]), _f64(inp["dt"])
    x0, x1 = np.ascontiguousarray(xbc[0]), np.ascontiguousarray(xbc[1])
    dt0, dt1 = np.ascontiguousarray(dt[0]), np.ascontiguousarray(dt[1])
    A, Dk, bias, w, cb = _params(params)
    out = np.empty((b, L, H * P), np.float64)
    yf = np.empty_like(out) if return_dirs else None
    yr = np.empty_like(out) if return_dirs else None
    rc = _load().oracle2_layer_fwd(b, L, H, P, N, *map(_ptr, (x0, x1, z, dt0, dt1, A, Dk, bias, w, cb)),
                                   flags, _ptr(out), _ptr(yf), _ptr(yr))
    if rc != 0:
        raise RuntimeError("oracle2_layer_fwd failed")
    return (out, yf, yr) if return_dirs else out


from .proj import adaln, in_proj, out_proj  # noqa: E402  (the layer's neighbours, plain numpy)
