"""The fp64 oracle against routes other than itself (CPU only)."""
import numpy as np
import pytest

import oracle
from tests import oracle_pins as P


@pytest.fixture(autouse=True)
def _no_mutation():
    oracle.set_mutation(0)
    yield
    oracle.set_mutation(0)


@pytest.mark.parametrize("name", sorted(P.PINS))
def test_pin(name):
    fn, tol = P.PINS[name]
    err = fn()
    assert np.isfinite(err) and err <= tol, f"{name}: discrepancy {err:.3e} > {tol:.1e}"


def test_softplus_and_silu_special_values():
    """softplus(0) = ln 2 and softplus(v) -> v for large v; silu(0) = 0 and
    silu(v) -> v for large v -- read through the oracle's delta and u."""
    inp, par = P.np_case(1, 4, 2, seed=1)
    par["dt_bias"][:] = 0.0
    inp["dt"][:] = 0.0
    inp["dt"][:, :, 1, :] = 50.0
    inp["x"][:] = 0.0
    par["conv_b"][:] = 0.0
    u, dl = oracle.features(inp, par)
    assert np.allclose(dl[:, :, 0], np.log(2.0), rtol=0, atol=1e-15)
    assert np.allclose(dl[:, :, 1], 50.0, rtol=1e-15, atol=0)
    assert np.all(u == 0.0)
    par["conv_b"][:] = 40.0
    u, _ = oracle.features(inp, par)
    assert np.allclose(u, 40.0, rtol=1e-15)


def test_mutations_are_caught():
    """Plant each plausible mistake in the oracle; some pin must fail."""
    missed = []
    for m, what in oracle.MUTATIONS.items():
        oracle.set_mutation(m)
        caught = []
        for name, (fn, tol) in P.PINS.items():
            try:
                err = fn()
            except Exception:
                err = np.inf
            if not (np.isfinite(err) and err <= max(tol, 1e-9)):
                caught.append(name)
        oracle.set_mutation(0)
        if not caught:
            missed.append(f"{m}: {what}")
    assert not missed, "mutations no pin catches: " + "; ".join(missed)


def test_bad_sizes_raise():
    inp, par = P.np_case(1, 4, 2, seed=1)
    inp["x"] = inp["x"][:, :0]
    with pytest.raises(RuntimeError):
        oracle.layer_fwd(inp, par)


def test_conv_bias_absent_reads_as_zero():
    inp, par = P.np_case(1, 20, 3, seed=2)
    par0 = dict(par)
    par0["conv_b"] = np.zeros_like(par["conv_b"])
    parn = dict(par)
    parn["conv_b"] = None
    a = oracle.layer_fwd(inp, par0)
    b = oracle.layer_fwd(inp, parn)
    assert np.array_equal(a, b)
