"""The C ABI on the host: symbols, sizes and argument checks (no kernel runs).

Every call here fails a check before anything is launched: the pointers are
fake addresses that no code ever dereferences.  Each case breaks exactly one
rule, and the rule checked before it is satisfied, so the expected status
names the check that must fire.
"""
import ctypes
import os
import re

import pytest

from bidirectional_mamba_denoiser_b200 import bimamba as bm

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "bimamba.h")

FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced
NULL = object()        # "pass a NULL struct pointer"


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bimamba2?_[a-z_]+)\s*\(", text)))


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("bimamba_layer_fwd", "bimamba_prefix_state", "bimamba_block_step",
              "bimamba_workspace_bytes", "bimamba_status_string", "bimamba_abi_version",
              "bimamba2_layer_fwd", "bimamba2_workspace_bytes"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(bm._LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_abi_version_and_status_strings():
    assert bm.lib.bimamba_abi_version() == 2
    for s in (0, -1, -2, -3, -4, -5):
        assert bm.status_string(s) and bm.status_string(s) != "unknown status"
    assert bm.status_string(-99) == "unknown status"


def test_workspace_bytes():
    # fp32 partial outputs [b][L][D] rounded up to 256 bytes, then fp32 B/C quads [2][b][L][32]
    assert bm.bimamba_workspace_bytes(8, 2048, 4096) == 8 * 2048 * 4096 * 4 + 2 * 8 * 2048 * 32 * 4
    assert bm.bimamba_workspace_bytes(1, 1, 1) == 256 + 2 * 32 * 4
    assert bm.bimamba_workspace_bytes(0, 10, 10) == 0
    assert bm.bimamba_workspace_bytes(1, 0, 10) == 0
    assert bm.bimamba_workspace_bytes(1, 10, 10, d_state=8) == 0


def _inputs(dtype=bm.BIMAMBA_BF16, base=FAKE):
    inp = bm.Inputs()
    inp.x, inp.z = base, base + 0x1000
    inp.dt[0], inp.dt[1] = base + 0x2000, base + 0x3000
    inp.B[0], inp.B[1] = base + 0x4000, base + 0x5000
    inp.C[0], inp.C[1] = base + 0x6000, base + 0x7000
    inp.dtype = dtype
    return inp


def _params():
    return bm.Params(FAKE + 0x10000, FAKE + 0x11000, FAKE + 0x12000, FAKE + 0x13000, FAKE + 0x14000)


def _byref(s):
    return None if s is NULL else ctypes.byref(s)


def _layer(inp=None, par=None, out=FAKE + 0x20000, out_dtype=bm.BIMAMBA_BF16, batch=2, L=64, D=32, N=16,
           flags=0, ws=FAKE + 0x30000, ws_bytes=None, broken=True):
    # Refuse to issue a call in which nothing was broken: with every argument
    # valid the library would launch a kernel on the fake addresses.
    assert broken, "a validation case must break some argument"
    inp = _inputs() if inp is None else inp
    par = _params() if par is None else par
    if ws_bytes is None:
        ws_bytes = bm.bimamba_workspace_bytes(max(batch, 1), max(L, 1), max(D, 1)) or 16
    return bm.lib.bimamba_layer_fwd(_byref(inp), _byref(par), out, out_dtype, batch, L, D, N, flags, ws,
                                    ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(batch=0), bm.BIMAMBA_ERR_INVALID_ARG),
    (dict(batch=70000), bm.BIMAMBA_ERR_INVALID_ARG),
    (dict(L=0), bm.BIMAMBA_ERR_INVALID_ARG),
    (dict(L=-5), bm.BIMAMBA_ERR_INVALID_ARG),
    (dict(D=0), bm.BIMAMBA_ERR_INVALID_ARG),
    (dict(out=None), bm.BIMAMBA_ERR_INVALID_ARG),
    (dict(N=8), bm.BIMAMBA_ERR_UNSUPPORTED),
    (dict(N=32), bm.BIMAMBA_ERR_UNSUPPORTED),
    (dict(flags=0x4), bm.BIMAMBA_ERR_UNSUPPORTED),
    (dict(flags=3 << bm.BIMAMBA_LANES_SHIFT), bm.BIMAMBA_ERR_UNSUPPORTED),
    (dict(flags=3 << bm.BIMAMBA_CHUNK_SHIFT), bm.BIMAMBA_ERR_UNSUPPORTED),
    (dict(flags=bm.BIMAMBA_FWD_ONLY | bm.BIMAMBA_REV_ONLY), bm.BIMAMBA_ERR_INVALID_ARG),
    (dict(out_dtype=7), bm.BIMAMBA_ERR_UNSUPPORTED),
    (dict(inp=NULL), bm.BIMAMBA_ERR_INVALID_ARG),
    (dict(par=NULL), bm.BIMAMBA_ERR_INVALID_ARG),
    (dict(out=FAKE + 0x20001), bm.BIMAMBA_ERR_MISALIGNED),
    (dict(ws=None), bm.BIMAMBA_ERR_WORKSPACE),
    (dict(ws=FAKE + 0x30008), bm.BIMAMBA_ERR_WORKSPACE),
    (dict(ws_bytes=100), bm.BIMAMBA_ERR_WORKSPACE),
])
def test_layer_rejects(kw, status):
    assert kw
    assert _layer(**kw) == status


def test_layer_rejects_bad_inputs_and_params():
    inp = _inputs()
    inp.z = None
    assert _layer(inp=inp) == bm.BIMAMBA_ERR_INVALID_ARG
    inp = _inputs()
    inp.C[1] = None
    assert _layer(inp=inp) == bm.BIMAMBA_ERR_INVALID_ARG
    inp = _inputs()
    inp.dtype = 5
    assert _layer(inp=inp) == bm.BIMAMBA_ERR_UNSUPPORTED
    inp = _inputs()
    inp.dt[1] = FAKE + 0x3001  # odd address for a 2-byte element
    assert _layer(inp=inp) == bm.BIMAMBA_ERR_MISALIGNED
    inp = _inputs(dtype=bm.BIMAMBA_F32)
    inp.B[0] = FAKE + 0x4002  # 2-byte aligned, 4-byte element
    assert _layer(inp=inp) == bm.BIMAMBA_ERR_MISALIGNED
    par = _params()
    par.A = None
    assert _layer(par=par) == bm.BIMAMBA_ERR_INVALID_ARG
    par = _params()
    par.conv_w = FAKE + 0x13002
    assert _layer(par=par) == bm.BIMAMBA_ERR_MISALIGNED


def _state(h=FAKE + 0x40000, cx=FAKE + 0x41000):
    return bm.FwdState(h, cx)


def _prefix(inp=None, par=None, batch=2, P=64, D=32, N=16, st=None):
    inp = _inputs() if inp is None else inp
    par = _params() if par is None else par
    st = _state() if st is None else st
    return bm.lib.bimamba_prefix_state(_byref(inp), _byref(par), batch, P, D, N, _byref(st), None)


def test_prefix_rejects():
    assert _prefix(batch=0) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _prefix(P=0) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _prefix(N=4) == bm.BIMAMBA_ERR_UNSUPPORTED
    assert _prefix(st=NULL) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _prefix(st=_state(h=None)) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _prefix(st=_state(h=FAKE + 0x40002)) == bm.BIMAMBA_ERR_MISALIGNED
    inp = _inputs()
    inp.x = None
    assert _prefix(inp=inp) == bm.BIMAMBA_ERR_INVALID_ARG


def _block(st=None, inp=None, G=32, par=None, out=FAKE + 0x20000, out_dtype=bm.BIMAMBA_BF16, batch=2, D=32,
           N=16, new=NULL, flags=0):
    st = _state() if st is None else st
    inp = _inputs() if inp is None else inp
    par = _params() if par is None else par
    return bm.lib.bimamba_block_step(_byref(st), _byref(inp), G, _byref(par), out, out_dtype, batch, D, N,
                                     _byref(new), flags, None)


def test_block_rejects():
    assert _block(G=0) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _block(G=65) == bm.BIMAMBA_ERR_UNSUPPORTED
    assert _block(batch=0) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _block(N=15) == bm.BIMAMBA_ERR_UNSUPPORTED
    assert _block(out=None) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _block(st=NULL) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _block(new=_state(cx=None)) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _block(new=_state(cx=FAKE + 0x41001)) == bm.BIMAMBA_ERR_MISALIGNED
    assert _block(flags=bm.BIMAMBA_FWD_ONLY | bm.BIMAMBA_REV_ONLY) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _block(flags=0x100000) == bm.BIMAMBA_ERR_UNSUPPORTED


# ---------------------------------------------------------------- Mamba-2 mixer

def _inputs2(dtype=bm.BIMAMBA_BF16, base=FAKE):
    inp = bm.Inputs2()
    inp.xbc[0], inp.xbc[1] = base, base + 0x10000
    inp.z = base + 0x20000
    inp.dt[0], inp.dt[1] = base + 0x30000, base + 0x31000
    inp.dtype = dtype
    return inp


def _params2(base=FAKE + 0x40000):
    return bm.Params2(base, base + 0x1000, base + 0x2000, base + 0x3000, base + 0x4000)


def _m2(**broken):
    # Refuse to issue a call in which nothing was broken: with every argument
    # valid the library would launch kernels on the fake addresses.
    assert broken, "a validation case must break some argument"
    return _m2_call(**broken)


def _m2_call(inp=None, par=None, out=FAKE + 0x50000, out_dtype=bm.BIMAMBA_BF16, batch=2, L=64, H=4, P=32, N=128,
             flags=0, ws=FAKE + 0x100000, ws_bytes=None):
    inp = _inputs2() if inp is None else inp
    par = _params2() if par is None else par
    if ws_bytes is None:
        ws_bytes = bm.bimamba2_workspace_bytes(batch, L, H, P, N)
    return bm.lib.bimamba2_layer_fwd(_byref(inp), _byref(par), out, out_dtype, batch, L, H, P, N, flags,
                                     ws, ws_bytes, None)


def test_mamba2_workspace_bytes():
    # conv features 2*b*L*CH + step sizes 2*b*H*L + forward and reverse outputs 2*b*L*H*P,
    # fp32, then fp16 C and B tiles of 128 x 128 per chunk of 128 steps and direction, then
    # the ticket counter and one flag per (batch row, head), int32 (every part a multiple of
    # 256 bytes at this size)
    b, L, H = 8, 2048, 120
    CH = H * 32 + 256
    want = (2 * b * L * CH * 4 + 2 * b * H * L * 4 + 2 * b * L * H * 32 * 4 + 2 * b * (L // 128) * 2 * 128 * 128 * 2
            + (1 + b * H) * 4)
    assert bm.bimamba2_workspace_bytes(b, L, H) == want
    assert bm.bimamba2_workspace_bytes(0, 10, 4) == 0
    assert bm.bimamba2_workspace_bytes(1, 0, 4) == 0
    assert bm.bimamba2_workspace_bytes(1, 10, 0) == 0


def test_mamba2_rejects():
    assert _m2(inp=NULL) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _m2(par=NULL) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _m2(out=None) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _m2(batch=0) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _m2(L=0) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _m2(H=0) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _m2(P=64) == bm.BIMAMBA_ERR_UNSUPPORTED
    assert _m2(N=64) == bm.BIMAMBA_ERR_UNSUPPORTED
    assert _m2(flags=0x4) == bm.BIMAMBA_ERR_UNSUPPORTED  # no such flag
    assert _m2(flags=1 << 8) == bm.BIMAMBA_ERR_UNSUPPORTED  # lane field: not a Mamba-2 option
    assert _m2(flags=bm.BIMAMBA_FWD_ONLY | bm.BIMAMBA_REV_ONLY) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _m2(inp=_inputs2(dtype=7)) == bm.BIMAMBA_ERR_UNSUPPORTED
    assert _m2(out_dtype=7) == bm.BIMAMBA_ERR_UNSUPPORTED
    bad = _inputs2()
    bad.z = None
    assert _m2(inp=bad) == bm.BIMAMBA_ERR_INVALID_ARG
    bad = _inputs2()
    bad.dt[1] = FAKE + 0x31001
    assert _m2(inp=bad) == bm.BIMAMBA_ERR_MISALIGNED
    bad = _inputs2()
    bad.z = FAKE + 0x20008  # element-aligned but not 16-byte aligned
    assert _m2(inp=bad) == bm.BIMAMBA_ERR_MISALIGNED
    bad = _inputs2()
    bad.xbc[1] = FAKE + 0x10008
    assert _m2(inp=bad) == bm.BIMAMBA_ERR_MISALIGNED
    par = _params2()
    par.conv_w = FAKE + 0x43008
    assert _m2(par=par) == bm.BIMAMBA_ERR_MISALIGNED
    par = _params2()
    par.conv_w = None
    assert _m2(par=par) == bm.BIMAMBA_ERR_INVALID_ARG
    par = _params2()
    par.A = FAKE + 0x40002
    assert _m2(par=par) == bm.BIMAMBA_ERR_MISALIGNED
    assert _m2(out=FAKE + 0x50008) == bm.BIMAMBA_ERR_MISALIGNED
    assert _m2(ws=None) == bm.BIMAMBA_ERR_WORKSPACE
    assert _m2(ws_bytes=bm.bimamba2_workspace_bytes(2, 64, 4) - 1) == bm.BIMAMBA_ERR_WORKSPACE
    assert _m2(ws=FAKE + 0x100080) == bm.BIMAMBA_ERR_MISALIGNED


def _state2(base=FAKE + 0x200000):
    return bm.FwdState2(base, base + 0x100000)


def _m2_prefix(**broken):
    assert broken, "a validation case must break some argument"
    kw = dict(inp=None, par=None, batch=2, P=64, H=4, Pd=32, N=128, state=None, ws=FAKE + 0x400000, ws_bytes=None)
    kw.update(broken)
    inp = _inputs2() if kw["inp"] is None else kw["inp"]
    par = _params2() if kw["par"] is None else kw["par"]
    st = _state2() if kw["state"] is None else kw["state"]
    wsb = kw["ws_bytes"] if kw["ws_bytes"] is not None else bm.bimamba2_workspace_bytes(2, 64, 4)
    return bm.lib.bimamba2_prefix_state(_byref(inp), _byref(par), kw["batch"], kw["P"], kw["H"], kw["Pd"], kw["N"],
                                        _byref(st), kw["ws"], wsb, None)


def _m2_block(**broken):
    assert broken, "a validation case must break some argument"
    kw = dict(state=None, inp=None, G=32, par=None, out=FAKE + 0x50000, out_dtype=bm.BIMAMBA_BF16, batch=2, H=4,
              Pd=32, N=128, new=None, flags=0, ws=FAKE + 0x400000, ws_bytes=None)
    kw.update(broken)
    st = _state2() if kw["state"] is None else kw["state"]
    inp = _inputs2() if kw["inp"] is None else kw["inp"]
    par = _params2() if kw["par"] is None else kw["par"]
    wsb = kw["ws_bytes"] if kw["ws_bytes"] is not None else bm.bimamba2_workspace_bytes(2, 32, 4)
    new = kw["new"]
    return bm.lib.bimamba2_block_step(_byref(st), _byref(inp), kw["G"], _byref(par), kw["out"], kw["out_dtype"],
                                      kw["batch"], kw["H"], kw["Pd"], kw["N"], None if new is None else _byref(new),
                                      kw["flags"], kw["ws"], wsb, None)


def test_mamba2_prefix_and_block_rejects():
    assert _m2_prefix(inp=NULL) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _m2_prefix(P=0) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _m2_prefix(N=64) == bm.BIMAMBA_ERR_UNSUPPORTED
    assert _m2_prefix(state=NULL) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _m2_prefix(state=bm.FwdState2(FAKE + 0x200008, FAKE + 0x300000)) == bm.BIMAMBA_ERR_MISALIGNED
    assert _m2_prefix(ws_bytes=16) == bm.BIMAMBA_ERR_WORKSPACE
    bad = _inputs2()
    bad.xbc[0] = FAKE + 0x8
    assert _m2_prefix(inp=bad) == bm.BIMAMBA_ERR_MISALIGNED
    assert _m2_block(state=NULL) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _m2_block(G=0) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _m2_block(out=None) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _m2_block(flags=bm.BIMAMBA_NO_TMA) == bm.BIMAMBA_ERR_UNSUPPORTED
    assert _m2_block(flags=3) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _m2_block(new=bm.FwdState2(FAKE + 0x200000, None)) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _m2_block(new=bm.FwdState2(FAKE + 0x200000, FAKE + 0x300008)) == bm.BIMAMBA_ERR_MISALIGNED
    assert _m2_block(ws=None) == bm.BIMAMBA_ERR_WORKSPACE
    assert _m2_block(out=FAKE + 0x50008) == bm.BIMAMBA_ERR_MISALIGNED


def _carry(**ptrs):
    c = bm.Carry()
    for name, (a, b) in ptrs.items():
        getattr(c, name)[0], getattr(c, name)[1] = a, b
    return c


def _layer_carry(carry, flags=0, **kw):
    inp, par = _inputs(), _params()
    ws_bytes = bm.bimamba_workspace_bytes(2, 64, 32)
    return bm.lib.bimamba_layer_fwd_carry(ctypes.byref(inp), ctypes.byref(par), _byref(carry), FAKE + 0x20000,
                                          bm.BIMAMBA_BF16, kw.get("batch", 2), 64, 32, 16, flags, FAKE + 0x30000,
                                          ws_bytes, None)


def test_layer_carry_rejects():
    # no carry struct; NO_TMA (carries live in the TMA-fed kernels); a misaligned carry pointer;
    # the layer's own checks still apply (batch 0)
    assert _layer_carry(NULL) == bm.BIMAMBA_ERR_INVALID_ARG
    assert _layer_carry(_carry(h_out=(FAKE + 0x40000, None)), flags=bm.BIMAMBA_NO_TMA) == bm.BIMAMBA_ERR_UNSUPPORTED
    for name in ("h_in", "h_out", "delta_sum"):
        assert _layer_carry(_carry(**{name: (None, FAKE + 0x40002)})) == bm.BIMAMBA_ERR_MISALIGNED
    # conv halos: aligned to the input element (bf16 here); a halo alone runs with carries
    assert _layer_carry(_carry(conv_halo=(FAKE + 0x40001, None))) == bm.BIMAMBA_ERR_MISALIGNED
    assert _layer_carry(_carry(conv_halo=(None, FAKE + 0x40000)), flags=bm.BIMAMBA_NO_TMA) == \
        bm.BIMAMBA_ERR_UNSUPPORTED
    assert _layer_carry(_carry(h_out=(FAKE + 0x40000, None)), batch=0) == bm.BIMAMBA_ERR_INVALID_ARG


@pytest.mark.parametrize("kw,status", [
    (dict(h_all=None), bm.BIMAMBA_ERR_INVALID_ARG),
    (dict(ds_all=None), bm.BIMAMBA_ERR_INVALID_ARG),
    (dict(h_in=None), bm.BIMAMBA_ERR_INVALID_ARG),
    (dict(nseg=0), bm.BIMAMBA_ERR_INVALID_ARG),
    (dict(seg=-1), bm.BIMAMBA_ERR_INVALID_ARG),
    (dict(seg=4), bm.BIMAMBA_ERR_INVALID_ARG),
    (dict(batch=0), bm.BIMAMBA_ERR_INVALID_ARG),
    (dict(D=0), bm.BIMAMBA_ERR_INVALID_ARG),
    (dict(N=8), bm.BIMAMBA_ERR_UNSUPPORTED),
    (dict(par=NULL), bm.BIMAMBA_ERR_INVALID_ARG),
    (dict(h_in=FAKE + 0x50002), bm.BIMAMBA_ERR_MISALIGNED),
])
def test_compose_carries_rejects(kw, status):
    a = dict(h_all=FAKE, ds_all=FAKE + 0x1000, par=_params(), nseg=4, seg=1, batch=2, D=32, N=16,
             h_in=FAKE + 0x50000)
    a.update(kw)
    assert bm.lib.bimamba_compose_carries(a["h_all"], a["ds_all"], _byref(a["par"]), a["nseg"], a["seg"],
                                          a["batch"], a["D"], a["N"], a["h_in"], None) == status


def test_neighbours_reject():
    L = bm.lib
    # AdaLN: null, sizes, d % 8, eps, misalignment
    assert L.bimamba_adaln(None, FAKE, FAKE, FAKE, 2, 8, 64, 1e-5, None) == bm.BIMAMBA_ERR_INVALID_ARG
    assert L.bimamba_adaln(FAKE, FAKE, FAKE, FAKE, 0, 8, 64, 1e-5, None) == bm.BIMAMBA_ERR_INVALID_ARG
    assert L.bimamba_adaln(FAKE, FAKE, FAKE, FAKE, 2, 8, 64, 0.0, None) == bm.BIMAMBA_ERR_INVALID_ARG
    assert L.bimamba_adaln(FAKE, FAKE, FAKE, FAKE, 2, 8, 60, 1e-5, None) == bm.BIMAMBA_ERR_UNSUPPORTED
    assert L.bimamba_adaln(FAKE + 8, FAKE, FAKE, FAKE, 2, 8, 64, 1e-5, None) == bm.BIMAMBA_ERR_MISALIGNED
    assert L.bimamba_adaln(FAKE, FAKE + 4, FAKE, FAKE, 2, 8, 64, 1e-5, None) == bm.BIMAMBA_ERR_MISALIGNED
    assert L.bimamba_adaln(FAKE, FAKE, FAKE, FAKE, 2, 8, 8200, 1e-5, None) == bm.BIMAMBA_ERR_UNSUPPORTED
    # input projection
    ok = [FAKE, FAKE + 0x1000, 2, 8, 64, 32, 16] + [FAKE + 0x2000 * i for i in range(1, 6)] + [None]
    def inp(**kw):
        a = list(ok)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return L.bimamba_in_proj(*a)
    assert inp(_0=None) == bm.BIMAMBA_ERR_INVALID_ARG
    assert inp(_2=0) == bm.BIMAMBA_ERR_INVALID_ARG
    assert inp(_3=0) == bm.BIMAMBA_ERR_INVALID_ARG
    assert inp(_3=65535 * 128) == bm.BIMAMBA_ERR_INVALID_ARG  # 2 x that many rows: past the grid
    assert inp(_4=96) == bm.BIMAMBA_ERR_UNSUPPORTED           # d_model % 64
    assert inp(_5=36) == bm.BIMAMBA_ERR_UNSUPPORTED           # d_inner % 8
    assert inp(_6=8) == bm.BIMAMBA_ERR_UNSUPPORTED            # d_state
    assert inp(_9=FAKE + 0x6008) == bm.BIMAMBA_ERR_MISALIGNED
    # output projection
    assert L.bimamba_out_proj(FAKE, FAKE, 2, 8, 64, 32, None, None) == bm.BIMAMBA_ERR_INVALID_ARG
    assert L.bimamba_out_proj(FAKE, FAKE, 2, 8, 72, 32, FAKE, None) == bm.BIMAMBA_ERR_UNSUPPORTED
    assert L.bimamba_out_proj(FAKE, FAKE, 2, 8, 64, 36, FAKE, None) == bm.BIMAMBA_ERR_UNSUPPORTED
    assert L.bimamba_out_proj(FAKE, FAKE + 4, 2, 8, 64, 32, FAKE, None) == bm.BIMAMBA_ERR_MISALIGNED


def test_header_serves_a_plain_c_program(tmp_path):
    """A C99 program includes the header, links the library and calls it with
    no torch and no C++: status strings, the ABI version, workspace queries
    and a rejected call (nothing runs on a GPU)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_abi.c"
    src.write_text(r"""
#include <stdio.h>
#include <string.h>
#include "bimamba.h"
int main(void) {
    if (bimamba_abi_version() != 2) return 1;
    if (strlen(bimamba_status_string(BIMAMBA_ERR_INVALID_ARG)) == 0) return 2;
    if (bimamba_workspace_bytes(8, 2048, 4096, 16, 0) != (size_t)8 * 2048 * 4096 * 4 + (size_t)2 * 8 * 2048 * 32 * 4)
        return 3;
    if (bimamba2_workspace_bytes(0, 10, 4, 32, 128) != 0) return 4;
    /* a call with no inputs is rejected before anything is launched */
    if (bimamba_layer_fwd(NULL, NULL, NULL, BIMAMBA_BF16, 1, 16, 32, 16, 0, NULL, 0, NULL) !=
        BIMAMBA_ERR_INVALID_ARG) return 5;
    printf("ok\n");
    return 0;
}
""")
    lib_dir = os.path.dirname(bm._LIB_PATH)
    exe = tmp_path / "use_abi"
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), str(src), "-L", lib_dir,
                    "-lbimamba", f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)


def test_scratch_address_cache_is_keyed_by_context(tmp_path):
    """The no-allocation entry point caches its scratch array's device address
    per CUDA context.  A context destroyed and created anew (same device, new
    context id) must miss the cache, so the address is looked up again; the
    cache's own header is compiled here into a small C++ program."""
    import shutil
    import subprocess
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no C++ compiler")
    csrc = os.path.join(os.path.dirname(bm._LIB_PATH), "csrc")
    src = tmp_path / "cache.cc"
    src.write_text(r"""
#include <stdio.h>
#include "context_cache.h"
using bimamba::ContextAddressCache;
int main() {
    ContextAddressCache<4> c;
    int a, b, d;
    if (c.find({0, 7})) return 1;
    c.put({0, 7}, &a);
    if (c.find({0, 7}) != &a) return 2;
    if (c.find({0, 8})) return 3;            /* same device, new context: miss */
    if (c.find({1, 7})) return 4;            /* other device: miss */
    c.put({0, 8}, &b);                       /* the new context's address */
    if (c.find({0, 8}) != &b || c.find({0, 7}) != &a) return 5;
    c.put({0, 8}, &d);                       /* an entry is replaced, not duplicated */
    if (c.find({0, 8}) != &d) return 6;
    for (unsigned long long id = 100; id < 110; ++id) c.put({2, id}, &a);  /* overflow: oldest evicted */
    if (c.find({2, 109}) != &a) return 7;
    if (c.find({2, 100})) return 8;
    printf("ok\n");
    return 0;
}
""")
    exe = tmp_path / "cache"
    subprocess.run([cxx, "-std=c++17", "-Wall", "-Werror", "-I", csrc, str(src), "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)


def test_features_rejects():
    L = bm.lib
    inp, par = _inputs(), _params()
    assert L.bimamba_features(None, ctypes.byref(par), 2, 8, 32, FAKE, FAKE + 0x100, None) == \
        bm.BIMAMBA_ERR_INVALID_ARG
    assert L.bimamba_features(ctypes.byref(inp), None, 2, 8, 32, FAKE, FAKE + 0x100, None) == \
        bm.BIMAMBA_ERR_INVALID_ARG
    assert L.bimamba_features(ctypes.byref(inp), ctypes.byref(par), 0, 8, 32, FAKE, FAKE + 0x100, None) == \
        bm.BIMAMBA_ERR_INVALID_ARG
    assert L.bimamba_features(ctypes.byref(inp), ctypes.byref(par), 2, 8, 32, None, FAKE + 0x100, None) == \
        bm.BIMAMBA_ERR_INVALID_ARG
    assert L.bimamba_features(ctypes.byref(inp), ctypes.byref(par), 2, 8, 32, FAKE + 2, FAKE + 0x100, None) == \
        bm.BIMAMBA_ERR_MISALIGNED
    bad = _inputs()
    bad.dtype = 9
    assert L.bimamba_features(ctypes.byref(bad), ctypes.byref(par), 2, 8, 32, FAKE, FAKE + 0x100, None) == \
        bm.BIMAMBA_ERR_UNSUPPORTED
