"""Python binding of the C ABI in include/bimamba.h (ctypes, marshalling only).

Each function has the name of the C entry point it calls.  Tensors are torch
tensors on the CUDA device; torch allocates outputs and workspaces and
supplies the current stream.  Every step of the layer runs in the CUDA
library: if ``libbimamba.so`` is missing this module raises on import, and
there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

_LIB_PATH = _build.LIB

BIMAMBA_OK = 0
BIMAMBA_ERR_INVALID_ARG = -1
BIMAMBA_ERR_UNSUPPORTED = -2
BIMAMBA_ERR_MISALIGNED = -3
BIMAMBA_ERR_WORKSPACE = -4
BIMAMBA_ERR_CUDA = -5

BIMAMBA_F32 = 0
BIMAMBA_BF16 = 1

BIMAMBA_FWD_ONLY = 0x1
BIMAMBA_REV_ONLY = 0x2
BIMAMBA_LANES_SHIFT = 8
BIMAMBA_NO_TMA = 0x4000
BIMAMBA_CHUNK_SHIFT = 16
BIMAMBA_FAMILY_SHIFT = 18
BIMAMBA_CHUNKED_WIDE = 0x2000
BIMAMBA_M2_NO_CLUSTER = 0x8000
BIMAMBA_TEST_STARVE = 0x100000

D_STATE = 16


class BimambaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {status_string(status)} (status {status})")
        self.status = status


class Params(ctypes.Structure):
    _fields_ = [("A", ctypes.c_void_p), ("D", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p),
                ("conv_w", ctypes.c_void_p), ("conv_b", ctypes.c_void_p)]


class Inputs(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("z", ctypes.c_void_p), ("dt", ctypes.c_void_p * 2),
                ("B", ctypes.c_void_p * 2), ("C", ctypes.c_void_p * 2), ("dtype", ctypes.c_int)]


class FwdState(ctypes.Structure):
    _fields_ = [("h", ctypes.c_void_p), ("conv_x", ctypes.c_void_p)]


class Carry(ctypes.Structure):
    _fields_ = [("h_in", ctypes.c_void_p * 2), ("h_out", ctypes.c_void_p * 2), ("delta_sum", ctypes.c_void_p * 2),
                ("conv_halo", ctypes.c_void_p * 2)]


class Params2(ctypes.Structure):
    _fields_ = [("A", ctypes.c_void_p), ("D", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p),
                ("conv_w", ctypes.c_void_p), ("conv_b", ctypes.c_void_p)]


class FwdState2(ctypes.Structure):
    _fields_ = [("S", ctypes.c_void_p), ("conv_xbc", ctypes.c_void_p)]


class Inputs2(ctypes.Structure):
    _fields_ = [("xbc", ctypes.c_void_p * 2), ("z", ctypes.c_void_p), ("dt", ctypes.c_void_p * 2),
                ("dtype", ctypes.c_int)]


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is not built; run `python -c \"import __graft_entry__ as g; g.build()\"` "
                          "or `python bidirectional_mamba_denoiser_b200/build.py`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, I64, U, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint, ctypes.c_size_t
    lib.bimamba_workspace_bytes.argtypes = [I, I64, I, I, U]
    lib.bimamba_workspace_bytes.restype = SZ
    lib.bimamba_layer_fwd.argtypes = [ctypes.POINTER(Inputs), ctypes.POINTER(Params), P, I,
                                      I, I64, I, I, U, P, SZ, P]
    lib.bimamba_layer_fwd.restype = I
    lib.bimamba_layer_fwd_carry.argtypes = [ctypes.POINTER(Inputs), ctypes.POINTER(Params), ctypes.POINTER(Carry), P,
                                            I, I, I64, I, I, U, P, SZ, P]
    lib.bimamba_layer_fwd_carry.restype = I
    lib.bimamba_compose_carries.argtypes = [P, P, ctypes.POINTER(Params), I, I, I, I, I, P, P]
    lib.bimamba_compose_carries.restype = I
    lib.bimamba_adaln.argtypes = [P, P, P, P, I, I64, I, ctypes.c_float, P]
    lib.bimamba_adaln.restype = I
    lib.bimamba_in_proj.argtypes = [P, P, I, I64, I, I, I, P, P, P, P, P, P]
    lib.bimamba_in_proj.restype = I
    lib.bimamba_out_proj.argtypes = [P, P, I, I64, I, I, P, P]
    lib.bimamba_out_proj.restype = I
    lib.bimamba_layer_fwd_noalloc.argtypes = [ctypes.POINTER(Inputs), ctypes.POINTER(Params), P, I,
                                              I, I64, I, I, U, P]
    lib.bimamba_layer_fwd_noalloc.restype = I
    lib.bimamba_prefix_state.argtypes = [ctypes.POINTER(Inputs), ctypes.POINTER(Params), I, I64, I, I,
                                         ctypes.POINTER(FwdState), P]
    lib.bimamba_prefix_state.restype = I
    lib.bimamba_block_step.argtypes = [ctypes.POINTER(FwdState), ctypes.POINTER(Inputs), I, ctypes.POINTER(Params),
                                       P, I, I, I, I, ctypes.POINTER(FwdState), U, P]
    lib.bimamba_block_step.restype = I
    lib.bimamba2_workspace_bytes.argtypes = [I, I64, I, I, I]
    lib.bimamba2_workspace_bytes.restype = SZ
    lib.bimamba2_layer_fwd.argtypes = [ctypes.POINTER(Inputs2), ctypes.POINTER(Params2), P, I,
                                       I, I64, I, I, I, U, P, SZ, P]
    lib.bimamba2_layer_fwd.restype = I
    lib.bimamba2_prefix_state.argtypes = [ctypes.POINTER(Inputs2), ctypes.POINTER(Params2), I, I64, I, I, I,
                                          ctypes.POINTER(FwdState2), P, SZ, P]
    lib.bimamba2_prefix_state.restype = I
    lib.bimamba2_block_step.argtypes = [ctypes.POINTER(FwdState2), ctypes.POINTER(Inputs2), I64, ctypes.POINTER(Params2),
                                        P, I, I, I, I, I, ctypes.POINTER(FwdState2), U, P, SZ, P]
    lib.bimamba2_block_step.restype = I
    lib.bimamba_features.argtypes = [ctypes.POINTER(Inputs), ctypes.POINTER(Params), I, I64, I, P, P, P]
    lib.bimamba_features.restype = I
    lib.bimamba_status_string.argtypes = [I]
    lib.bimamba_status_string.restype = ctypes.c_char_p
    lib.bimamba_abi_version.restype = I
    lib.bimamba_device_error.argtypes = [I]
    lib.bimamba_device_error.restype = I
    return lib


lib = _load()


def bimamba_device_error(reset: bool = True) -> int:
    """The device error word (0 = no kernel gave up waiting); synchronises."""
    return int(lib.bimamba_device_error(1 if reset else 0))


def status_string(status: int) -> str:
    return lib.bimamba_status_string(int(status)).decode()


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return BIMAMBA_F32
    if t == torch.bfloat16:
        return BIMAMBA_BF16
    raise TypeError(f"unsupported dtype {t}")


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensors passed to the CUDA library must be contiguous CUDA tensors")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _pair(t):
    """A per-direction input: a [2, ...] tensor or a (fwd, rev) pair."""
    if isinstance(t, (tuple, list)):
        return t[0], t[1]
    return t[0], t[1]


def make_params(params: dict) -> Params:
    return Params(_ptr(params["A"]), _ptr(params["D"]), _ptr(params["dt_bias"]),
                  _ptr(params["conv_w"]), _ptr(params.get("conv_b")))


def make_inputs(x, z, dt, B, C) -> Inputs:
    dt0, dt1 = _pair(dt)
    B0, B1 = _pair(B)
    C0, C1 = _pair(C)
    inp = Inputs()
    inp.x = _ptr(x)
    inp.z = _ptr(z)
    inp.dt[0], inp.dt[1] = _ptr(dt0), _ptr(dt1)
    inp.B[0], inp.B[1] = _ptr(B0), _ptr(B1)
    inp.C[0], inp.C[1] = _ptr(C0), _ptr(C1)
    inp.dtype = _dtype_code(x.dtype)
    return inp


def bimamba_workspace_bytes(batch: int, L: int, d_inner: int, d_state: int = D_STATE, flags: int = 0) -> int:
    return int(lib.bimamba_workspace_bytes(batch, L, d_inner, d_state, flags))


def bimamba_layer_fwd(x, z, dt, B, C, params: dict, out=None, out_dtype=None, flags: int = 0,
                      workspace=None, stream=None):
    """Full-sequence bidirectional layer.  x, z [b, L, D]; dt [2, b, L, D];
    B, C [2, b, L, 16]; params as produced by workloads.make_params (on the
    device).  Returns out [b, L, D]."""
    b, L, D = x.shape
    N = (B[0] if isinstance(B, (tuple, list)) else B).shape[-1]
    if out is None:
        out = torch.empty(b, L, D, device=x.device, dtype=out_dtype or x.dtype)
    need = bimamba_workspace_bytes(b, L, D, N, flags)
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=x.device, dtype=torch.uint8)
    inp = make_inputs(x, z, dt, B, C)
    par = make_params(params)
    rc = lib.bimamba_layer_fwd(ctypes.byref(inp), ctypes.byref(par), _ptr(out), _dtype_code(out.dtype),
                               b, L, D, N, flags, _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _stream(stream))
    if rc != BIMAMBA_OK:
        raise BimambaError("bimamba_layer_fwd", rc)
    return out


def bimamba_features(x, dt, params: dict, stream=None):
    """The layer's per-token features (diagnostic): x [b, L, D], dt [2, b, L, D]
    (or a (fwd, rev) pair).  Returns (u, delta), each [2, b, L, D] fp32."""
    b, L, D = x.shape
    u = torch.empty(2, b, L, D, device=x.device, dtype=torch.float32)
    delta = torch.empty_like(u)
    dt0, dt1 = _pair(dt)
    inp = Inputs()
    inp.x = _ptr(x)
    inp.dt[0], inp.dt[1] = _ptr(dt0), _ptr(dt1)
    inp.dtype = _dtype_code(x.dtype)
    par = make_params(params)
    rc = lib.bimamba_features(ctypes.byref(inp), ctypes.byref(par), b, L, D, _ptr(u), _ptr(delta), _stream(stream))
    if rc != BIMAMBA_OK:
        raise BimambaError("bimamba_features", rc)
    return u, delta


def _dir_pair(t):
    """None, a [2, ...] tensor or a (fwd, rev) pair (entries may be None) ->
    two device pointers (or None)."""
    if t is None:
        return None, None
    if isinstance(t, (tuple, list)):
        return _ptr(t[0]), _ptr(t[1])
    return _ptr(t[0]), _ptr(t[1])


def bimamba_layer_fwd_carry(x, z, dt, B, C, params: dict, h_in=None, h_out=None, delta_sum=None, out=None,
                            out_dtype=None, flags: int = 0, workspace=None, stream=None, conv_halo=None):
    """bimamba_layer_fwd with scan carries.  h_in, h_out: [2, b, D, 16] fp32
    (or (fwd, rev) pairs, entries may be None): the states entering / leaving
    each direction; delta_sum: [2, b, D] fp32, each direction's sum of step
    sizes; conv_halo: [2, b, 3, D] of x's dtype (or a (before, after) pair):
    the x rows of the three tokens before token 0 and after token L-1 that the
    convs read instead of zeros.  Returns out [b, L, D]."""
    b, L, D = x.shape
    N = (B[0] if isinstance(B, (tuple, list)) else B).shape[-1]
    if out is None:
        out = torch.empty(b, L, D, device=x.device, dtype=out_dtype or x.dtype)
    need = bimamba_workspace_bytes(b, L, D, N, flags)
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=x.device, dtype=torch.uint8)
    inp = make_inputs(x, z, dt, B, C)
    par = make_params(params)
    car = Carry()
    car.h_in[0], car.h_in[1] = _dir_pair(h_in)
    car.h_out[0], car.h_out[1] = _dir_pair(h_out)
    car.delta_sum[0], car.delta_sum[1] = _dir_pair(delta_sum)
    car.conv_halo[0], car.conv_halo[1] = _dir_pair(conv_halo)
    rc = lib.bimamba_layer_fwd_carry(ctypes.byref(inp), ctypes.byref(par), ctypes.byref(car), _ptr(out),
                                     _dtype_code(out.dtype), b, L, D, N, flags, _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != BIMAMBA_OK:
        raise BimambaError("bimamba_layer_fwd_carry", rc)
    return out


def bimamba_compose_carries(h_out_all, delta_sum_all, params: dict, seg: int, out=None, stream=None):
    """The carries entering segment ``seg``: h_out_all [nseg, 2, b, D, 16] and
    delta_sum_all [nseg, 2, b, D] (every segment's run from zero).  Returns
    h_in [2, b, D, 16] fp32."""
    nseg, _, b, D, N = h_out_all.shape
    if out is None:
        out = torch.empty(2, b, D, N, device=h_out_all.device, dtype=torch.float32)
    par = make_params(params)
    rc = lib.bimamba_compose_carries(_ptr(h_out_all), _ptr(delta_sum_all), ctypes.byref(par), nseg, seg, b, D, N,
                                     _ptr(out), _stream(stream))
    if rc != BIMAMBA_OK:
        raise BimambaError("bimamba_compose_carries", rc)
    return out


def bimamba_adaln(x, gamma, beta, eps: float = 1e-5, out=None, stream=None):
    """AdaLN: gamma[b] * (x - mean) / sqrt(var + eps) + beta[b] per token row.
    x [b, L, d] bf16; gamma, beta [b, d] fp32.  Returns [b, L, d] bf16."""
    b, L, d = x.shape
    if out is None:
        out = torch.empty_like(x)
    rc = lib.bimamba_adaln(_ptr(x), _ptr(gamma), _ptr(beta), _ptr(out), b, L, d, eps, _stream(stream))
    if rc != BIMAMBA_OK:
        raise BimambaError("bimamba_adaln", rc)
    return out


def bimamba_in_proj(a, w_in, d_inner: int, d_state: int = D_STATE, out: dict | None = None, stream=None) -> dict:
    """Input projection into the layer's input arrays: a [b, L, d_model] bf16,
    w_in [4 d_inner + 4 d_state, d_model] bf16.  Returns {"x", "z" [b, L, D];
    "dt" [2, b, L, D]; "B", "C" [2, b, L, d_state]} (bf16)."""
    b, L, dm = a.shape
    if out is None:
        kw = dict(device=a.device, dtype=a.dtype)
        out = {"x": torch.empty(b, L, d_inner, **kw), "z": torch.empty(b, L, d_inner, **kw),
               "dt": torch.empty(2, b, L, d_inner, **kw), "B": torch.empty(2, b, L, d_state, **kw),
               "C": torch.empty(2, b, L, d_state, **kw)}
    rc = lib.bimamba_in_proj(_ptr(a), _ptr(w_in), b, L, dm, d_inner, d_state, _ptr(out["x"]), _ptr(out["z"]),
                             _ptr(out["dt"]), _ptr(out["B"]), _ptr(out["C"]), _stream(stream))
    if rc != BIMAMBA_OK:
        raise BimambaError("bimamba_in_proj", rc)
    return out


def bimamba_out_proj(y, w_out, out=None, stream=None):
    """Output projection: y [b, L, d_inner] bf16, w_out [d_model, d_inner]
    bf16.  Returns [b, L, d_model] bf16."""
    b, L, D = y.shape
    dm = w_out.shape[0]
    if out is None:
        out = torch.empty(b, L, dm, device=y.device, dtype=y.dtype)
    rc = lib.bimamba_out_proj(_ptr(y), _ptr(w_out), b, L, D, dm, _ptr(out), _stream(stream))
    if rc != BIMAMBA_OK:
        raise BimambaError("bimamba_out_proj", rc)
    return out


def bimamba_layer_fwd_noalloc(x, z, dt, B, C, params: dict, out=None, out_dtype=None, flags: int = 0,
                              stream=None):
    """bimamba_layer_fwd for callers that cannot allocate device memory: the
    library's built-in 64 MiB scratch replaces the workspace (sizes whose
    bimamba_workspace_bytes fits in it).  Calls that overlap on the GPU race on that
    scratch.  ``out`` is still the caller's; pass it in to allocate nothing
    here either."""
    b, L, D = x.shape
    N = (B[0] if isinstance(B, (tuple, list)) else B).shape[-1]
    if out is None:
        out = torch.empty(b, L, D, device=x.device, dtype=out_dtype or x.dtype)
    inp = make_inputs(x, z, dt, B, C)
    par = make_params(params)
    rc = lib.bimamba_layer_fwd_noalloc(ctypes.byref(inp), ctypes.byref(par), _ptr(out), _dtype_code(out.dtype),
                                       b, L, D, N, flags, _stream(stream))
    if rc != BIMAMBA_OK:
        raise BimambaError("bimamba_layer_fwd_noalloc", rc)
    return out


def bimamba_prefix_state(x, dt, B, params: dict, h_out=None, conv_x_out=None, stream=None):
    """Forward scan over the prefix x [b, P, D] (dt, B: the forward direction's,
    [b, P, D] / [b, P, 16], or [2, ...] stacks whose first entry is used).
    Returns (h [b, D, 16] fp32, conv_x [b, 3, D])."""
    b, P, D = x.shape
    dt0 = dt[0] if (isinstance(dt, (tuple, list)) or dt.dim() == 4) else dt
    B0 = B[0] if (isinstance(B, (tuple, list)) or B.dim() == 4) else B
    N = B0.shape[-1]
    if h_out is None:
        h_out = torch.empty(b, D, N, device=x.device, dtype=torch.float32)
    if conv_x_out is None:
        conv_x_out = torch.empty(b, 3, D, device=x.device, dtype=x.dtype)
    inp = Inputs()
    inp.x = _ptr(x)
    inp.dt[0] = _ptr(dt0)
    inp.B[0] = _ptr(B0)
    inp.dtype = _dtype_code(x.dtype)
    par = make_params(params)
    st = FwdState(_ptr(h_out), _ptr(conv_x_out))
    rc = lib.bimamba_prefix_state(ctypes.byref(inp), ctypes.byref(par), b, P, D, N, ctypes.byref(st),
                                  _stream(stream))
    if rc != BIMAMBA_OK:
        raise BimambaError("bimamba_prefix_state", rc)
    return h_out, conv_x_out


def bimamba_block_step(state, x, z, dt, B, C, params: dict, out=None, out_dtype=None, new_state=None,
                       flags: int = 0, stream=None):
    """One step on the active block x [b, G, D] from state = (h, conv_x).
    new_state = (h, conv_x) tensors to commit into (may be `state` itself)."""
    b, G, D = x.shape
    N = state[0].shape[-1]
    if out is None:
        out = torch.empty(b, G, D, device=x.device, dtype=out_dtype or x.dtype)
    inp = make_inputs(x, z, dt, B, C)
    par = make_params(params)
    st = FwdState(_ptr(state[0]), _ptr(state[1]))
    ns = FwdState(_ptr(new_state[0]), _ptr(new_state[1])) if new_state is not None else None
    rc = lib.bimamba_block_step(ctypes.byref(st), ctypes.byref(inp), G, ctypes.byref(par), _ptr(out),
                                _dtype_code(out.dtype), b, D, N, ctypes.byref(ns) if ns is not None else None,
                                flags, _stream(stream))
    if rc != BIMAMBA_OK:
        raise BimambaError("bimamba_block_step", rc)
    return out


# ---------------------------------------------------------------- Mamba-2 mixer

M2_HEADDIM = 32
M2_D_STATE = 128


def bimamba2_workspace_bytes(batch: int, L: int, nheads: int, headdim: int = M2_HEADDIM,
                             d_state: int = M2_D_STATE) -> int:
    return int(lib.bimamba2_workspace_bytes(batch, L, nheads, headdim, d_state))


def bimamba2_layer_fwd(xbc, z, dt, params: dict, out=None, out_dtype=None, flags: int = 0,
                       workspace=None, stream=None):
    """Full-sequence bidirectional Mamba-2 mixer.  xbc [2, b, L, H*P + 2N]
    (or a (fwd, rev) pair); z [b, L, H*P]; dt [2, b, L, H] (or a pair);
    params as produced by workloads.make_mamba2_params (on the device).
    Returns out [b, L, H*P]."""
    x0, x1 = _pair(xbc)
    d0, d1 = _pair(dt)
    b, L, H = d0.shape
    HP = z.shape[-1]
    P = HP // H
    N = (x0.shape[-1] - HP) // 2
    if out is None:
        out = torch.empty(b, L, HP, device=z.device, dtype=out_dtype or z.dtype)
    need = bimamba2_workspace_bytes(b, L, H, P, N)
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=z.device, dtype=torch.uint8)
    inp = Inputs2()
    inp.xbc[0], inp.xbc[1] = _ptr(x0), _ptr(x1)
    inp.z = _ptr(z)
    inp.dt[0], inp.dt[1] = _ptr(d0), _ptr(d1)
    inp.dtype = _dtype_code(z.dtype)
    par = Params2(_ptr(params["A"]), _ptr(params["D"]), _ptr(params["dt_bias"]),
                  _ptr(params["conv_w"]), _ptr(params.get("conv_b")))
    rc = lib.bimamba2_layer_fwd(ctypes.byref(inp), ctypes.byref(par), _ptr(out), _dtype_code(out.dtype),
                                b, L, H, P, N, flags, _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _stream(stream))
    if rc != BIMAMBA_OK:
        raise BimambaError("bimamba2_layer_fwd", rc)
    return out


def _params2(params: dict) -> Params2:
    return Params2(_ptr(params["A"]), _ptr(params["D"]), _ptr(params["dt_bias"]), _ptr(params["conv_w"]),
                   _ptr(params.get("conv_b")))


def _workspace2(workspace, batch, L, H, P, N, device):
    need = bimamba2_workspace_bytes(batch, L, H, P, N)
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=device, dtype=torch.uint8)
    return workspace


def bimamba2_prefix_state(xbc, dt, params: dict, S_out=None, conv_out=None, workspace=None, stream=None):
    """Forward scan of the Mamba-2 mixer over a prefix: xbc, dt of the forward
    direction ([b, P, CH], [b, P, H], or [2, ...] stacks whose first entry is
    used).  Returns (S [b, H, 32, N] fp32, conv_xbc [b, 3, CH])."""
    x0 = xbc[0] if (isinstance(xbc, (tuple, list)) or xbc.dim() == 4) else xbc
    d0 = dt[0] if (isinstance(dt, (tuple, list)) or dt.dim() == 4) else dt
    b, L, CH = x0.shape
    H = d0.shape[-1]
    P = M2_HEADDIM
    N = (CH - H * P) // 2
    if S_out is None:
        S_out = torch.empty(b, H, P, N, device=x0.device, dtype=torch.float32)
    if conv_out is None:
        conv_out = torch.empty(b, 3, CH, device=x0.device, dtype=x0.dtype)
    workspace = _workspace2(workspace, b, L, H, P, N, x0.device)
    inp = Inputs2()
    inp.xbc[0] = _ptr(x0)
    inp.dt[0] = _ptr(d0)
    inp.dtype = _dtype_code(x0.dtype)
    par = _params2(params)
    st = FwdState2(_ptr(S_out), _ptr(conv_out))
    rc = lib.bimamba2_prefix_state(ctypes.byref(inp), ctypes.byref(par), b, L, H, P, N, ctypes.byref(st),
                                   _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != BIMAMBA_OK:
        raise BimambaError("bimamba2_prefix_state", rc)
    return S_out, conv_out


def bimamba2_block_step(state, xbc, z, dt, params: dict, out=None, out_dtype=None, new_state=None, flags: int = 0,
                        workspace=None, stream=None):
    """One denoising step of the Mamba-2 mixer on the active block from
    state = (S, conv_xbc): xbc [2, b, G, CH] (or a pair), z [b, G, H*P],
    dt [2, b, G, H].  new_state = (S, conv_xbc) to commit into (may be
    `state` itself).  Returns out [b, G, H*P]."""
    x0, x1 = _pair(xbc)
    d0, d1 = _pair(dt)
    b, G, H = d0.shape
    HP = z.shape[-1]
    P = HP // H
    N = (x0.shape[-1] - HP) // 2
    if out is None:
        out = torch.empty(b, G, HP, device=z.device, dtype=out_dtype or z.dtype)
    workspace = _workspace2(workspace, b, G, H, P, N, z.device)
    inp = Inputs2()
    inp.xbc[0], inp.xbc[1] = _ptr(x0), _ptr(x1)
    inp.z = _ptr(z)
    inp.dt[0], inp.dt[1] = _ptr(d0), _ptr(d1)
    inp.dtype = _dtype_code(z.dtype)
    par = _params2(params)
    st = FwdState2(_ptr(state[0]), _ptr(state[1]))
    ns = FwdState2(_ptr(new_state[0]), _ptr(new_state[1])) if new_state is not None else None
    rc = lib.bimamba2_block_step(ctypes.byref(st), ctypes.byref(inp), G, ctypes.byref(par), _ptr(out),
                                 _dtype_code(out.dtype), b, H, P, N, ctypes.byref(ns) if ns is not None else None,
                                 flags, _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != BIMAMBA_OK:
        raise BimambaError("bimamba2_block_step", rc)
    return out
