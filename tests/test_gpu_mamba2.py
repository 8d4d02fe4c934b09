"""The Mamba-2 mixer's CUDA path (through the C ABI) against the fp64 oracle, on a B200."""
import numpy as np
import pytest
import torch

import oracle
from bidirectional_mamba_denoiser_b200 import workloads as W
from tests import parity_util as U

pytestmark = pytest.mark.gpu

P, N = 32, 128


@pytest.fixture(scope="module")
def bm():
    from bidirectional_mamba_denoiser_b200 import bimamba
    return bimamba


def run(bm, inp, par, out_dtype, flags=0):
    d = U.to_device(inp)
    p = U.to_device(par)
    out = bm.bimamba2_layer_fwd(d["xbc"], d["z"], d["dt"], p, out_dtype=out_dtype, flags=flags)
    torch.cuda.synchronize()
    return U.to_cpu64(out)


@pytest.mark.parametrize("shape", [(1, 37, 2), (2, 100, 3), (1, 8, 1), (1, 1, 2), (2, 257, 4), (1, 9, 2)])
def test_small_fp32(bm, shape):
    """fp32 in and out, ragged lengths around the 8-token chunk: normwise <= 1e-5."""
    b, L, H = shape
    inp, par = W.make_mamba2_case(b, L, H, P, N, "fp32", seed=50 + L)
    got = run(bm, inp, par, torch.float32)
    want = oracle.mamba2_layer_fwd(inp, par)
    assert U.normwise(got, want) <= U.TOL_FP32


# bf16 inputs run the chunked dual form on the tensor cores (fp16 operands,
# bound 2e-3); BIMAMBA_NO_TMA selects the step-by-step CUDA-core scan, which
# also meets the fp32-arithmetic guard.
PATHS = {"tensor": (0, U.TOL_BF16), "cuda_core": (0x4000, U.GUARD)}


@pytest.mark.parametrize("path", sorted(PATHS))
def test_bf16_inputs(bm, path):
    """bf16 in, fp32 state: fp32-output mode within the path's bound;
    bf16-output mode within one bf16 rounding + 2e-3."""
    flags, tol = PATHS[path]
    inp, par = W.make_mamba2_case(2, 300, 4, P, N, "bf16", seed=61)
    want = oracle.mamba2_layer_fwd(inp, par)
    got32 = run(bm, inp, par, torch.float32, flags=flags)
    err = U.normwise(got32, want)
    assert err <= tol, err
    got16 = run(bm, inp, par, torch.bfloat16, flags=flags)
    assert U.bf16_out_ok(got16, want)


# the two launch forms of the tensor path: clusters whose CTAs meet halfway
# (chosen while batch * nheads <= 2 x the SM count), and ticket-ordered CTAs
# (forwards first, each reverse after its forward; forced by the flag)
FORMS = {"cluster": 0, "tickets": 0x8000}


@pytest.mark.parametrize("shape", [(3, 300, 120), (1, 383, 300), (3, 129, 100)])
def test_tensor_path_both_launch_forms(bm, shape):
    """batch * nheads above 2 x the SM count (360, 300 and 300 (head, batch
    row) pairs against 296) takes the ticket-ordered form without the flag;
    here with ragged L (the chunks of the two directions aligned in token
    space) and, in the 3-row cases, reverse CTAs of one batch row waiting on
    forwards of another.  Each form once more below the threshold, forced."""
    b, L, H = shape
    inp, par = W.make_mamba2_case(b, L, H, P, N, "bf16", seed=66 + L)
    want = oracle.mamba2_layer_fwd(inp, par)
    got = run(bm, inp, par, torch.float32)
    assert bm.bimamba_device_error() == 0
    assert U.normwise(got, want) <= U.TOL_BF16
    small, spar = W.make_mamba2_case(2, 300, 40, P, N, "bf16", seed=67)
    swant = oracle.mamba2_layer_fwd(small, spar)
    for flags in FORMS.values():
        assert U.normwise(run(bm, small, spar, torch.float32, flags=flags), swant) <= U.TOL_BF16


@pytest.mark.parametrize("form", sorted(FORMS))
@pytest.mark.parametrize("L", [1, 2, 127, 128, 129, 256, 383])
def test_tensor_path_ragged_lengths(bm, L, form):
    """Chunks of 128 steps: lengths around the chunk edge, both directions,
    both launch forms."""
    inp, par = W.make_mamba2_case(2, L, 3, P, N, "bf16", seed=70 + L)
    got = run(bm, inp, par, torch.float32, flags=FORMS[form])
    assert bm.bimamba_device_error() == 0
    assert U.normwise(got, oracle.mamba2_layer_fwd(inp, par)) <= U.TOL_BF16


@pytest.mark.parametrize("form", sorted(FORMS))
@pytest.mark.parametrize("which", ["fwd", "rev"])
def test_tensor_path_direction_flags(bm, which, form):
    inp, par = W.make_mamba2_case(1, 200, 2, P, N, "bf16", seed=71)
    f_or = oracle.FWD_ONLY if which == "fwd" else oracle.REV_ONLY
    f_bm = bm.BIMAMBA_FWD_ONLY if which == "fwd" else bm.BIMAMBA_REV_ONLY
    got = run(bm, inp, par, torch.float32, flags=f_bm | FORMS[form])
    assert U.normwise(got, oracle.mamba2_layer_fwd(inp, par, flags=f_or)) <= U.TOL_BF16


def test_tensor_path_tickets_bf16_output(bm):
    """The ticket-ordered form with bf16 output: within one bf16 rounding + 2e-3."""
    inp, par = W.make_mamba2_case(3, 260, 5, P, N, "bf16", seed=74)
    want = oracle.mamba2_layer_fwd(inp, par)
    got16 = run(bm, inp, par, torch.bfloat16, flags=FORMS["tickets"])
    assert U.bf16_out_ok(got16, want)


@pytest.mark.parametrize("dt_value", [4.0, -9.0])
def test_tensor_path_extreme_step_sizes(bm, dt_value):
    inp, par = W.make_mamba2_case(1, 300, 2, P, N, "bf16", seed=72)
    inp["dt"][:] = dt_value
    got = run(bm, inp, par, torch.float32)
    assert U.normwise(got, oracle.mamba2_layer_fwd(inp, par)) <= U.TOL_BF16


@pytest.mark.parametrize("form", sorted(FORMS))
def test_tensor_path_starved_waits_give_up(bm, form):
    """With BIMAMBA_TEST_STARVE no tile copy is issued: every wait for a tile
    gives up after ~0.1 ms and bit 0 of the device error word is set; in the
    ticket-ordered form no forward sets its flag either, so every reverse
    CTA's wait for it gives up too and sets bit 1.  The kernel finishes, and
    the context still works afterwards."""
    inp, par = W.make_mamba2_case(1, 130, 2, P, N, "bf16", seed=73)
    assert bm.bimamba_device_error(reset=True) >= 0
    run(bm, inp, par, torch.float32, flags=bm.BIMAMBA_TEST_STARVE | FORMS[form])
    word = bm.bimamba_device_error(reset=True)
    assert word & 1
    assert bool(word & 2) == (form == "tickets")
    got = run(bm, inp, par, torch.float32, flags=FORMS[form])
    assert U.normwise(got, oracle.mamba2_layer_fwd(inp, par)) <= U.TOL_BF16
    assert bm.bimamba_device_error(reset=True) == 0


@pytest.mark.parametrize("which", ["fwd", "rev"])
def test_direction_flags(bm, which):
    inp, par = W.make_mamba2_case(1, 70, 2, P, N, "fp32", seed=62)
    f_or = oracle.FWD_ONLY if which == "fwd" else oracle.REV_ONLY
    f_bm = bm.BIMAMBA_FWD_ONLY if which == "fwd" else bm.BIMAMBA_REV_ONLY
    got = run(bm, inp, par, torch.float32, flags=f_bm)
    assert U.normwise(got, oracle.mamba2_layer_fwd(inp, par, flags=f_or)) <= U.TOL_FP32


def test_shared_xbc_pointer(bm):
    """The same xBC buffer for both directions (one in_proj)."""
    inp, par = W.make_mamba2_case(1, 45, 2, P, N, "fp32", seed=63)
    inp["xbc"][1] = inp["xbc"][0]
    d, p = U.to_device(inp), U.to_device(par)
    x = d["xbc"][0].contiguous()
    out = bm.bimamba2_layer_fwd((x, x), d["z"], d["dt"], p, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert U.normwise(U.to_cpu64(out), oracle.mamba2_layer_fwd(inp, par)) <= U.TOL_FP32


@pytest.mark.parametrize("dt_value", [4.0, -9.0])
def test_extreme_step_sizes(bm, dt_value):
    """Large steps (decay products fall below 2^-60 within a few tokens, so the
    kernel folds them into the state again and again) and tiny steps (memory
    over the whole sequence)."""
    inp, par = W.make_mamba2_case(1, 150, 3, P, N, "fp32", seed=64)
    inp["dt"][:] = dt_value
    got = run(bm, inp, par, torch.float32)
    assert U.normwise(got, oracle.mamba2_layer_fwd(inp, par)) <= U.TOL_FP32


def test_conv_bias_absent(bm):
    inp, par = W.make_mamba2_case(1, 33, 2, P, N, "fp32", seed=65)
    par = dict(par)
    par["conv_b"] = None
    d, p = U.to_device(inp), U.to_device(par)
    out = bm.bimamba2_layer_fwd(d["xbc"], d["z"], d["dt"], p, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert U.normwise(U.to_cpu64(out), oracle.mamba2_layer_fwd(inp, par)) <= U.TOL_FP32


def test_repeatable(bm):
    inp, par = W.make_mamba2_case(2, 64, 3, P, N, "bf16", seed=66)
    a = run(bm, inp, par, torch.float32)
    b = run(bm, inp, par, torch.float32)
    assert np.array_equal(a, b)


def test_full_size_sampled_heads(bm):
    """The pages' layer: b 8, L 2048, 120 heads x 32, N 128, bf16, in the
    launch configuration the bench times; three heads against the oracle."""
    w = W.MAMBA2_1P3B
    H = w.extra["nheads"]
    inp, par = W.make_mamba2_case(w.batch, w.L, H, P, N, "bf16", w.seed, device="cuda")
    heads = [0, 77, H - 1]
    si, sp, xch = U.head_subset(inp, par, heads)
    want = oracle.mamba2_layer_fwd(si, sp)
    idx = torch.as_tensor(xch, device="cuda")
    for flags, tol in PATHS.values():
        out32 = bm.bimamba2_layer_fwd(inp["xbc"], inp["z"], inp["dt"], par, out_dtype=torch.float32, flags=flags)
        out16 = bm.bimamba2_layer_fwd(inp["xbc"], inp["z"], inp["dt"], par, out_dtype=torch.bfloat16, flags=flags)
        torch.cuda.synchronize()
        err = U.normwise(U.to_cpu64(out32.index_select(-1, idx)), want)
        assert err <= tol, (flags, err)
        assert U.bf16_out_ok(U.to_cpu64(out16.index_select(-1, idx)), want)


def test_long_batch1_sampled_heads(bm):
    """b 1, L 16,384, 120 heads (the clustered launch form of the tensor path:
    both directions at once, meeting halfway), the bench's mamba2_long
    configuration: three heads against the oracle on both paths."""
    w = W.MAMBA2_LONG[16384]
    H = w.extra["nheads"]
    inp, par = W.make_mamba2_case(w.batch, w.L, H, P, N, "bf16", w.seed, device="cuda")
    heads = [0, 60, H - 1]
    si, sp, xch = U.head_subset(inp, par, heads)
    want = oracle.mamba2_layer_fwd(si, sp)
    idx = torch.as_tensor(xch, device="cuda")
    for flags, tol in PATHS.values():
        out32 = bm.bimamba2_layer_fwd(inp["xbc"], inp["z"], inp["dt"], par, out_dtype=torch.float32, flags=flags)
        torch.cuda.synchronize()
        assert bm.bimamba_device_error() == 0
        err = U.normwise(U.to_cpu64(out32.index_select(-1, idx)), want)
        assert err <= tol, (flags, err)


def test_workspace_too_small_is_rejected(bm):
    inp, par = W.make_mamba2_case(1, 16, 2, P, N, "bf16", seed=1, device="cuda")
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(bm.BimambaError) as e:
        bm.bimamba2_layer_fwd(inp["xbc"], inp["z"], inp["dt"], par, workspace=ws)
    assert e.value.status == bm.BIMAMBA_ERR_WORKSPACE


def _tok(inp, lo, hi):
    """Tokens [lo, hi) of a Mamba-2 input dict (xbc, dt: [2, b, L, .]; z: [b, L, .])."""
    return {"xbc": inp["xbc"][:, :, lo:hi].contiguous(), "z": inp["z"][:, lo:hi].contiguous(),
            "dt": inp["dt"][:, :, lo:hi].contiguous()}


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_block_chain_from_prefix_state(bm, dtype):
    """Prefix of 100 tokens, then two committed blocks of 37.  Expected values
    from the layer oracle by the definition of the block step: the forward
    part is the full-sequence forward over prefix + blocks restricted to the
    block, the reverse part is the layer on the block alone.  The second
    block's output checks the first commit's state; the tail is compared
    bit for bit."""
    b, H, Pn, G = 2, 3, 100, 37
    inp, par = W.make_mamba2_case(b, Pn + 2 * G, H, P, N, dtype, seed=80)
    d, p = U.to_device(inp), U.to_device(par)
    pre = _tok(d, 0, Pn)
    S, tail = bm.bimamba2_prefix_state(pre["xbc"], pre["dt"], p)
    # bf16 inputs: the prefix state comes from the dual form's state updates on the tensor cores
    # (fp16 operands), held to the 2e-3 bound of bf16 I/O; the blocks (G 37) run the fp32 scan
    tol = U.TOL_FP32 if dtype == "fp32" else U.TOL_BF16
    for k in range(2):
        lo, hi = Pn + k * G, Pn + (k + 1) * G
        blk = _tok(d, lo, hi)
        out = bm.bimamba2_block_step((S, tail), blk["xbc"], blk["z"], blk["dt"], p, out_dtype=torch.float32,
                                     new_state=(S, tail))
        torch.cuda.synchronize()
        _, yf, _ = oracle.mamba2_layer_fwd(_tok(inp, 0, hi), par, return_dirs=True)
        bi = _tok(inp, lo, hi)
        _, _, yr = oracle.mamba2_layer_fwd(bi, par, return_dirs=True)
        z = bi["z"].double().numpy()
        want = (yf[:, lo:hi] + yr) * (z / (1.0 + np.exp(-z)))
        assert U.normwise(U.to_cpu64(out), want) <= tol, k
        want_tail = inp["xbc"][0, :, hi - 3:hi].double().numpy()
        assert np.array_equal(U.to_cpu64(tail), want_tail), k


def test_block_step_without_commit_leaves_state(bm):
    inp, par = W.make_mamba2_case(1, 60, 2, P, N, "fp32", seed=81)
    d, p = U.to_device(inp), U.to_device(par)
    pre = _tok(d, 0, 40)
    S, tail = bm.bimamba2_prefix_state(pre["xbc"], pre["dt"], p)
    S0, t0 = S.clone(), tail.clone()
    blk = _tok(d, 40, 60)
    bm.bimamba2_block_step((S, tail), blk["xbc"], blk["z"], blk["dt"], p, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(S, S0) and torch.equal(tail, t0)


# bf16 inputs, a block of at most 32 steps and a multiple of 4 heads: the block
# step's closed form on the tensor cores (fp16 operands, fp32 state), within the
# dual form's 2e-3 bound.
@pytest.mark.parametrize("G,H", [(32, 4), (31, 8), (17, 4), (1, 4)])
def test_block_chain_tensor_path(bm, G, H):
    """Prefix of 100 tokens, then two committed blocks of G; expected values
    from the layer oracle by the definition of the block step (forward: the
    full-sequence forward restricted to the block; reverse: the layer on the
    block alone).  The second block checks the first commit's state; the
    tail is compared bit for bit."""
    b, Pn = 2, 100
    inp, par = W.make_mamba2_case(b, Pn + 2 * G, H, P, N, "bf16", seed=90 + G)
    d, p = U.to_device(inp), U.to_device(par)
    pre = _tok(d, 0, Pn)
    S, tail = bm.bimamba2_prefix_state(pre["xbc"], pre["dt"], p)
    for k in range(2):
        lo, hi = Pn + k * G, Pn + (k + 1) * G
        blk = _tok(d, lo, hi)
        out = bm.bimamba2_block_step((S, tail), blk["xbc"], blk["z"], blk["dt"], p, out_dtype=torch.float32,
                                     new_state=(S, tail))
        torch.cuda.synchronize()
        assert bm.bimamba_device_error() == 0
        _, yf, _ = oracle.mamba2_layer_fwd(_tok(inp, 0, hi), par, return_dirs=True)
        bi = _tok(inp, lo, hi)
        _, _, yr = oracle.mamba2_layer_fwd(bi, par, return_dirs=True)
        z = bi["z"].double().numpy()
        want = (yf[:, lo:hi] + yr) * (z / (1.0 + np.exp(-z)))
        assert U.normwise(U.to_cpu64(out), want) <= U.TOL_BF16, k
        want_tail = inp["xbc"][0, :, hi - 3:hi].double().numpy()
        assert np.array_equal(U.to_cpu64(tail), want_tail), k


@pytest.mark.parametrize("which", ["fwd", "rev", "bf16_out"])
def test_block_step_tensor_path_flags_and_output(bm, which):
    """One block of 32 after a 64-token prefix, without commit: a single
    direction by flag, or bf16 output (within one bf16 rounding + 2e-3); the
    cached state is left unchanged."""
    b, H, Pn, G = 2, 4, 64, 32
    inp, par = W.make_mamba2_case(b, Pn + G, H, P, N, "bf16", seed=97)
    d, p = U.to_device(inp), U.to_device(par)
    pre = _tok(d, 0, Pn)
    S, tail = bm.bimamba2_prefix_state(pre["xbc"], pre["dt"], p)
    S0, t0 = S.clone(), tail.clone()
    blk = _tok(d, Pn, Pn + G)
    flags = {"fwd": bm.BIMAMBA_FWD_ONLY, "rev": bm.BIMAMBA_REV_ONLY, "bf16_out": 0}[which]
    out_dtype = torch.bfloat16 if which == "bf16_out" else torch.float32
    out = bm.bimamba2_block_step((S, tail), blk["xbc"], blk["z"], blk["dt"], p, out_dtype=out_dtype, flags=flags)
    torch.cuda.synchronize()
    assert bm.bimamba_device_error() == 0
    _, yf, _ = oracle.mamba2_layer_fwd(_tok(inp, 0, Pn + G), par, return_dirs=True)
    bi = _tok(inp, Pn, Pn + G)
    _, _, yr = oracle.mamba2_layer_fwd(bi, par, return_dirs=True)
    yf, yr = yf[:, Pn:], yr
    if which == "fwd":
        yr = np.zeros_like(yr)
    elif which == "rev":
        yf = np.zeros_like(yf)
    z = bi["z"].double().numpy()
    want = (yf + yr) * (z / (1.0 + np.exp(-z)))
    if which == "bf16_out":
        assert U.bf16_out_ok(U.to_cpu64(out), want)
    else:
        assert U.normwise(U.to_cpu64(out), want) <= U.TOL_BF16
    assert torch.equal(S, S0) and torch.equal(tail, t0)


@pytest.mark.parametrize("Pn", [128, 300, 1])
def test_prefix_state_tensor_path_lengths(bm, Pn):
    """bf16 prefixes of one whole chunk, several chunks with a ragged last one,
    and a single token (the prefix state's state updates on the tensor cores),
    each followed by one committed block of 32: the block's output against the
    layer oracle by the block step's definition, and the tail bit for bit."""
    b, H, G = 2, 4, 32
    inp, par = W.make_mamba2_case(b, Pn + G, H, P, N, "bf16", seed=110 + Pn)
    d, p = U.to_device(inp), U.to_device(par)
    pre = _tok(d, 0, Pn)
    S, tail = bm.bimamba2_prefix_state(pre["xbc"], pre["dt"], p)
    blk = _tok(d, Pn, Pn + G)
    out = bm.bimamba2_block_step((S, tail), blk["xbc"], blk["z"], blk["dt"], p, out_dtype=torch.float32,
                                 new_state=(S, tail))
    torch.cuda.synchronize()
    assert bm.bimamba_device_error() == 0
    _, yf, _ = oracle.mamba2_layer_fwd(_tok(inp, 0, Pn + G), par, return_dirs=True)
    bi = _tok(inp, Pn, Pn + G)
    _, _, yr = oracle.mamba2_layer_fwd(bi, par, return_dirs=True)
    z = bi["z"].double().numpy()
    want = (yf[:, Pn:] + yr) * (z / (1.0 + np.exp(-z)))
    assert U.normwise(U.to_cpu64(out), want) <= U.TOL_BF16
    assert np.array_equal(U.to_cpu64(tail), inp["xbc"][0, :, Pn + G - 3:Pn + G].double().numpy())
