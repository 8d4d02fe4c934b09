"""Failure detection on the GPU without a fault: a wait that runs out.

The TMA-fed kernels wait for each tile on an mbarrier with a bound.  With the
test flag BIMAMBA_TEST_STARVE no tile load is ever issued, so every such
wait must give up (after ~0.1 ms each), set bit 0 of the device error word
and let the kernel finish -- no hang, no trap.  Afterwards the context must
still work: a normal call gives the right answer and leaves the word clear.
"""
import time

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


@pytest.mark.parametrize("family", [1, 2])
def test_starved_waits_give_up_and_report(bm, family):
    inp, par = W.make_case(1, 64, 64, 16, "bf16", seed=5)
    d = U.to_device(inp)
    p = U.to_device(par)
    assert bm.bimamba_device_error(reset=True) >= 0  # clear whatever came before
    flags = bm.BIMAMBA_TEST_STARVE | (family << bm.BIMAMBA_FAMILY_SHIFT)
    t0 = time.perf_counter()
    bm.bimamba_layer_fwd(d["x"], d["z"], d["dt"], d["B"], d["C"], p, out_dtype=torch.float32, flags=flags)
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 10.0
    assert bm.bimamba_device_error(reset=True) & 1
    # the context is still usable and the word was cleared
    ref = oracle.layer_fwd(inp, par)
    got = bm.bimamba_layer_fwd(d["x"], d["z"], d["dt"], d["B"], d["C"], p, out_dtype=torch.float32,
                               flags=family << bm.BIMAMBA_FAMILY_SHIFT)
    torch.cuda.synchronize()
    assert U.normwise(U.to_cpu64(got), ref) <= U.GUARD
    assert bm.bimamba_device_error(reset=False) == 0
