"""The fp64 Mamba-2 oracle against routes other than itself (CPU only)."""
import numpy as np
import pytest

import oracle
from tests import mamba2_pins as M


@pytest.fixture(autouse=True)
def _no_mutation():
    oracle.set_mutation2(0)
    yield
    oracle.set_mutation2(0)


@pytest.mark.parametrize("name", sorted(M.PINS))
def test_pin(name):
    fn, tol = M.PINS[name]
    err = fn()
    assert np.isfinite(err) and err <= tol, f"{name}: discrepancy {err:.3e} > {tol:.1e}"


def test_mutations_are_caught():
    """Plant each plausible mistake in the Mamba-2 oracle; some pin must fail."""
    missed = []
    for m, what in oracle.MUTATIONS2.items():
        oracle.set_mutation2(m)
        caught = []
        for name, (fn, tol) in M.PINS.items():
            try:
                err = fn()
            except Exception:
                err = np.inf
            if not (np.isfinite(err) and err <= max(tol, 1e-9)):
                caught.append(name)
        oracle.set_mutation2(0)
        if not caught:
            missed.append(f"{m}: {what}")
    assert not missed, "mutations no pin catches: " + "; ".join(missed)


def test_bad_sizes_raise():
    inp, par = M.np_case2(1, 4, 2, 2, 2, seed=1)
    inp["dt"] = inp["dt"][:, :, :0]
    inp["xbc"] = inp["xbc"][:, :, :0]
    inp["z"] = inp["z"][:, :0]
    with pytest.raises(RuntimeError):
        oracle.mamba2_layer_fwd(inp, par)


def test_conv_bias_absent_reads_as_zero():
    inp, par = M.np_case2(1, 12, 2, 2, 3, seed=2)
    par0 = dict(par)
    par0["conv_b"] = np.zeros_like(par["conv_b"])
    parn = dict(par)
    parn["conv_b"] = None
    assert np.array_equal(oracle.mamba2_layer_fwd(inp, par0), oracle.mamba2_layer_fwd(inp, parn))
