"""bimamba_layer_fwd_noalloc: the full layer for callers that cannot allocate.

Such callers (a plugin inside a host that owns all GPU memory, or code that
only has the C ABI and no CUDA allocator) cannot pass a workspace, so this
entry point uses the library's built-in 64 MiB scratch instead.  It launches
the same kernel with the same arguments as bimamba_layer_fwd, only the
workspace address differs, so the two outputs must agree bit for bit.

The tests call it through the C ABI twice in a row on different inputs.
Before the second call a call on NaN inputs fills the scratch with NaN, so a
kernel that read a scratch value before writing it would show.  They also
check sampled channels against the fp64 oracle, the bf16 and fp32 outputs,
a single-direction flag, and that a problem too large for the scratch is
rejected in the full entry point's order of checks.  This file is collected
last.
"""
import ctypes

import pytest
import torch

import oracle
from bidirectional_mamba_denoiser_b200 import workloads as W
from tests import parity_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bm():
    from bidirectional_mamba_denoiser_b200 import bimamba
    return bimamba


def _call_noalloc(bm, d, p, out, flags=0):
    """Straight through the C ABI: no workspace argument exists."""
    b, L, D = d["x"].shape
    inp = bm.make_inputs(d["x"], d["z"], d["dt"], d["B"], d["C"])
    par = bm.make_params(p)
    return bm.lib.bimamba_layer_fwd_noalloc(ctypes.byref(inp), ctypes.byref(par), out.data_ptr(),
                                            bm.BIMAMBA_F32 if out.dtype == torch.float32 else bm.BIMAMBA_BF16,
                                            b, L, D, 16, flags, torch.cuda.current_stream().cuda_stream)


def _poison_scratch(bm, shape):
    """A call on NaN inputs: its half-sequence partial outputs, all NaN, are
    left in the shared scratch."""
    b, L, D = shape
    inp, par = W.make_case(b, L, D, 16, "bf16", seed=1, device="cuda")
    inp["x"].fill_(float("nan"))
    out = torch.empty(b, L, D, device="cuda", dtype=torch.float32)
    assert _call_noalloc(bm, inp, par, out) == bm.BIMAMBA_OK
    torch.cuda.synchronize()
    assert torch.isnan(out).any()


@pytest.mark.parametrize("flags", [0, 1])  # 1 = BIMAMBA_FWD_ONLY
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(2, 1000, 512), (1, 3000, 256)])
def test_noalloc_matches_layer_fwd_twice(bm, shape, out_dtype, flags):
    b, L, D = shape
    for k, seed in enumerate((41, 42)):  # two calls in a row, different inputs
        if k == 1:
            _poison_scratch(bm, shape)
        inp, par = W.make_case(b, L, D, 16, "bf16", seed=seed, device="cuda")
        want = bm.bimamba_layer_fwd(inp["x"], inp["z"], inp["dt"], inp["B"], inp["C"], par,
                                    out_dtype=out_dtype, flags=flags)
        got = torch.full_like(want, float("nan"))
        assert _call_noalloc(bm, inp, par, got, flags) == bm.BIMAMBA_OK
        torch.cuda.synchronize()
        assert torch.equal(got, want), (k, seed)
        # and against the fp64 oracle on sampled channels
        chans = U.sample_channels(D, 6, seed=seed)
        si, sp = U.channel_subset(inp, par, chans)
        ref = oracle.layer_fwd(si, sp, flags=oracle.FWD_ONLY if flags else 0)
        g = U.to_cpu64(got.index_select(-1, torch.as_tensor(chans, device="cuda")))
        if out_dtype == torch.float32:
            assert U.normwise(g, ref) <= U.GUARD
        else:
            assert U.bf16_out_ok(g, ref)


def _oversize_inputs():
    L = 4096 + 8  # workspace 4104 * (4096 * 4 + 256) bytes > 64 MiB
    x = torch.empty(1, L, 4096, device="cuda", dtype=torch.bfloat16)
    bc = torch.empty(2, 1, L, 16, device="cuda", dtype=torch.bfloat16)
    return {"x": x, "z": x, "dt": torch.stack([x, x]), "B": bc, "C": bc}


def test_noalloc_rejects_sizes_beyond_its_scratch(bm):
    """A workspace above 64 MiB does not fit the scratch:
    the call returns BIMAMBA_ERR_WORKSPACE and launches nothing."""
    inp = _oversize_inputs()
    _, par = W.make_case(1, 4, 4096, 16, "bf16", seed=1, device="cuda")
    out = torch.empty_like(inp["x"])
    assert _call_noalloc(bm, inp, par, out) == bm.BIMAMBA_ERR_WORKSPACE


def test_noalloc_checks_in_the_full_entry_points_order(bm):
    """An oversize call with another fault reports that fault first, as
    bimamba_layer_fwd does: its workspace check comes last."""
    inp = _oversize_inputs()
    _, par = W.make_case(1, 4, 4096, 16, "bf16", seed=1, device="cuda")
    out = torch.empty_like(inp["x"])
    assert _call_noalloc(bm, inp, par, out, flags=0x80000000) == bm.BIMAMBA_ERR_UNSUPPORTED
    assert _call_noalloc(bm, inp, par, out, flags=bm.BIMAMBA_FWD_ONLY | bm.BIMAMBA_REV_ONLY) == \
        bm.BIMAMBA_ERR_INVALID_ARG
    x = inp["x"]
    ci = bm.make_inputs(x, x, inp["dt"], inp["B"], inp["C"])
    ci.z = None
    b, L, D = x.shape
    rc = bm.lib.bimamba_layer_fwd_noalloc(ctypes.byref(ci), ctypes.byref(bm.make_params(par)), out.data_ptr(),
                                          bm.BIMAMBA_BF16, b, L, D, 16, 0, torch.cuda.current_stream().cuda_stream)
    assert rc == bm.BIMAMBA_ERR_INVALID_ARG
