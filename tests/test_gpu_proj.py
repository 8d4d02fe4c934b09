"""The layer's neighbours on a B200 (AdaLN, input and output projections on
the tcgen05 tensor cores) against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from bidirectional_mamba_denoiser_b200 import workloads as W
from tests import parity_util as U

pytestmark = pytest.mark.gpu

# bf16 results of fp32-accumulated sums of exact bf16 products: the store's
# rounding (2^-8 relative) plus fp32 accumulation over K terms, far below
# 1e-4 of the largest value at these sizes
TOL = 1e-4


@pytest.fixture(scope="module")
def bm():
    from bidirectional_mamba_denoiser_b200 import bimamba
    return bimamba


def _dev(c):
    return {k: v.cuda() for k, v in c.items()}


@pytest.mark.parametrize("shape", [(2, 37, 256), (1, 5, 2048), (3, 4, 72)])
def test_adaln(bm, shape):
    b, L, d = shape
    c = W.make_proj_case(b, L, d, 8, seed=31)
    g = _dev(c)
    got = bm.bimamba_adaln(g["h"], g["gamma"], g["beta"], eps=1e-5)
    torch.cuda.synchronize()
    want = oracle.adaln(c["h"], c["gamma"], c["beta"], 1e-5)
    assert U.bf16_out_ok(U.to_cpu64(got), want, TOL)


def _check_in_proj(got, want, tol=TOL):
    for k in ("x", "z", "dt", "B", "C"):
        assert U.bf16_out_ok(U.to_cpu64(got[k]), want[k], tol), k


@pytest.mark.parametrize("shape", [(2, 200, 256, 256), (1, 128, 64, 8), (3, 77, 192, 520)])
def test_in_proj_ragged_tiles(bm, shape):
    """M = batch * L and N = 4 D + 64 not multiples of the 128 x 256 tile."""
    b, L, dm, D = shape
    c = W.make_proj_case(b, L, dm, D, seed=32)
    g = _dev(c)
    got = bm.bimamba_in_proj(g["h"], g["w_in"], D)
    torch.cuda.synchronize()
    assert bm.bimamba_device_error() == 0
    _check_in_proj(got, oracle.in_proj(c["h"], c["w_in"], D))


@pytest.mark.parametrize("shape", [(2, 200, 256, 256), (1, 100, 1024, 72)])
def test_out_proj(bm, shape):
    b, L, dm, D = shape
    D = (D + 63) // 64 * 64
    c = W.make_proj_case(b, L, dm, D, seed=33)
    g = _dev(c)
    got = bm.bimamba_out_proj(g["y"], g["w_out"])
    torch.cuda.synchronize()
    assert U.bf16_out_ok(U.to_cpu64(got), oracle.out_proj(c["y"], c["w_out"]), TOL)


def test_full_size_sampled_rows(bm):
    """b 8, L 2048, d_model 2048, d_inner 4096 (the bench's launch): 64 sampled
    token rows of every output against the oracle."""
    w = W.PROJ_1P3B
    c = W.make_proj_case(w.batch, w.L, w.extra["d_model"], w.d_inner, seed=w.seed, device="cuda")
    a = bm.bimamba_adaln(c["h"], c["gamma"], c["beta"])
    got = bm.bimamba_in_proj(a, c["w_in"], w.d_inner)
    o = bm.bimamba_out_proj(c["y"], c["w_out"])
    torch.cuda.synchronize()
    rows = np.random.default_rng(0).choice(w.batch * w.L, 64, replace=False)
    bi, ti = rows // w.L, rows % w.L
    a_cpu = a.cpu()
    want_a = oracle.adaln(c["h"].cpu()[bi, ti][:, None], c["gamma"].cpu()[bi], c["beta"].cpu()[bi])[:, 0]
    assert U.bf16_out_ok(U.to_cpu64(a_cpu[bi, ti]), want_a, TOL)
    want = oracle.in_proj(a_cpu[bi, ti][None], c["w_in"].cpu(), w.d_inner)
    for k in ("x", "z"):
        assert U.bf16_out_ok(U.to_cpu64(got[k][bi, ti]), want[k][0], TOL), k
    for k in ("dt", "B", "C"):
        assert U.bf16_out_ok(U.to_cpu64(got[k][:, bi, ti]), want[k][:, 0], TOL), k
    want_o = oracle.out_proj(c["y"].cpu()[bi, ti][None], c["w_out"].cpu())[0]
    assert U.bf16_out_ok(U.to_cpu64(o[bi, ti]), want_o, TOL)


def test_mixer_sublayer_chain(bm):
    """AdaLN -> in_proj -> layer -> out_proj (Eq. (11) without the residual)
    against the same chain in the oracle, fed the kernels' own bf16
    intermediates so that each stage is checked on identical inputs."""
    b, L, dm, D = 2, 96, 128, 64
    c = W.make_proj_case(b, L, dm, D, seed=34)
    _, par = W.make_case(1, 4, D, 16, "bf16", 35)
    g, p = _dev(c), U.to_device(par)
    a = bm.bimamba_adaln(g["h"], g["gamma"], g["beta"])
    inp = bm.bimamba_in_proj(a, g["w_in"], D)
    y = bm.bimamba_layer_fwd(inp["x"], inp["z"], inp["dt"], inp["B"], inp["C"], p)
    o = bm.bimamba_out_proj(y, g["w_out"])
    torch.cuda.synchronize()
    assert U.bf16_out_ok(U.to_cpu64(a), oracle.adaln(c["h"], c["gamma"], c["beta"]), TOL)
    _check_in_proj(inp, oracle.in_proj(a.cpu(), c["w_in"], D))
    want_y = oracle.layer_fwd({k: v.cpu() for k, v in inp.items()}, par)
    assert U.bf16_out_ok(U.to_cpu64(y), want_y)
    assert U.bf16_out_ok(U.to_cpu64(o), oracle.out_proj(y.cpu(), c["w_out"]), TOL)
