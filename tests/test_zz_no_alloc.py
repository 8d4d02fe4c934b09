"""bimamba_layer_fwd_noalloc: the full layer for callers that cannot allocate.

Such callers (a plugin inside a host that owns all GPU memory, or code that
only has the C ABI and no CUDA allocator) cannot pass a workspace, so this
entry point uses the library's built-in 64 MiB scratch instead.  The test
calls it through the C ABI twice in a row, on two different inputs, and
checks each result against bimamba_layer_fwd with a caller workspace, with
the same fp32-arithmetic bound the other parity tests use.  Running two
calls back to back also shows that a call does not depend on what the
previous call left in the shared scratch.  This file is collected last.
"""
import ctypes

import pytest
import torch

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


@pytest.mark.parametrize("shape", [(2, 1000, 512), (1, 3000, 256)])
def test_noalloc_matches_layer_fwd_twice(bm, shape):
    b, L, D = shape
    for seed in (41, 42):  # two calls in a row, different inputs
        inp, par = W.make_case(b, L, D, 16, "bf16", seed=seed, device="cuda")
        want = bm.bimamba_layer_fwd(inp["x"], inp["z"], inp["dt"], inp["B"], inp["C"], par,
                                    out_dtype=torch.float32)
        got = torch.empty_like(want)
        assert _call_noalloc(bm, inp, par, got) == bm.BIMAMBA_OK
        torch.cuda.synchronize()
        assert U.normwise(U.to_cpu64(got), U.to_cpu64(want)) <= U.GUARD


def test_noalloc_rejects_sizes_beyond_its_scratch(bm):
    """batch * L * d_inner above 16,777,216 does not fit the 64 MiB scratch:
    the call returns BIMAMBA_ERR_WORKSPACE and launches nothing."""
    x = torch.empty(1, 4096 + 8, 4096, device="cuda", dtype=torch.bfloat16)
    inp = {"x": x, "z": x, "dt": torch.stack([x, x]),
           "B": torch.empty(2, 1, 4104, 16, device="cuda", dtype=torch.bfloat16),
           "C": torch.empty(2, 1, 4104, 16, device="cuda", dtype=torch.bfloat16)}
    _, par = W.make_case(1, 4, 4096, 16, "bf16", seed=1, device="cuda")
    out = torch.empty_like(x)
    assert _call_noalloc(bm, inp, par, out) == bm.BIMAMBA_ERR_WORKSPACE
