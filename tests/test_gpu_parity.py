"""The CUDA path (through the C ABI) against the fp64 oracle, on a B200."""
import numpy as np
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


def run_layer(bm, inp, par, out_dtype, flags=0):
    d = U.to_device(inp)
    p = U.to_device(par)
    out = bm.bimamba_layer_fwd(d["x"], d["z"], d["dt"], d["B"], d["C"], p, out_dtype=out_dtype, flags=flags)
    torch.cuda.synchronize()
    return U.to_cpu64(out)


@pytest.mark.parametrize("flags", [0, 0x4000, 1 << 18, 2 << 18])
def test_tiny_fp32_case(bm, flags):
    """b=1, L=256, D=64, fp32 in and out, seed 0: normwise <= 1e-5 (both kernels)."""
    inp, par = W.make_workload(W.TINY)
    ref = oracle.layer_fwd(inp, par)
    got = run_layer(bm, inp, par, torch.float32, flags)
    assert U.normwise(got, ref) <= U.TOL_FP32


@pytest.mark.parametrize("lanes", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("shape", [(1, 257, 72), (3, 100, 40), (2, 33, 8), (1, 17, 24)])
def test_bf16_ragged_staged_kernel(bm, shape, lanes):
    """The kernel without TMA staging: ragged L (not a multiple of its
    16-token chunk) and ragged D (not a multiple of a CTA's channels), each
    lane split."""
    b, L, D = shape
    inp, par = W.make_case(b, L, D, 16, "bf16", seed=100 + L + D)
    ref = oracle.layer_fwd(inp, par)
    flags = (lanes << 8) | bm.BIMAMBA_NO_TMA
    got32 = run_layer(bm, inp, par, torch.float32, flags)
    assert U.normwise(got32, ref) <= U.GUARD
    got16 = run_layer(bm, inp, par, torch.bfloat16, flags)
    assert U.bf16_out_ok(got16, ref)


@pytest.mark.parametrize("chunk", [1, 2])
@pytest.mark.parametrize("lanes", [4, 8, 16])
@pytest.mark.parametrize("shape", [(1, 257, 72), (3, 100, 40), (2, 33, 8), (1, 95, 24), (2, 1, 16),
                                   (1, 32, 32), (1, 64, 48), (1, 65, 8)])
def test_bf16_ragged_tma_kernel(bm, shape, lanes, chunk):
    """The TMA-fed kernel with 16- and 32-token chunks: one, two and three
    chunks, a ragged last chunk, and channel counts that leave the last
    CTA's tile partly empty."""
    b, L, D = shape
    inp, par = W.make_case(b, L, D, 16, "bf16", seed=200 + L + D)
    ref = oracle.layer_fwd(inp, par)
    flags = (lanes << 8) | (chunk << bm.BIMAMBA_CHUNK_SHIFT) | (1 << bm.BIMAMBA_FAMILY_SHIFT)
    got32 = run_layer(bm, inp, par, torch.float32, flags)
    assert U.normwise(got32, ref) <= U.GUARD
    got16 = run_layer(bm, inp, par, torch.bfloat16, flags)
    assert U.bf16_out_ok(got16, ref)
    assert bm.bimamba_device_error() == 0


@pytest.mark.parametrize("group", [1, 2, 4, 8, "2u", "4f"])
@pytest.mark.parametrize("shape", [(1, 257, 72), (3, 100, 40), (2, 33, 8), (1, 95, 24), (2, 1, 16),
                                   (1, 16, 32), (1, 32, 64), (2, 17, 96)])
def test_bf16_ragged_fused_kernel(bm, shape, group):
    """The per-token fused kernel (16-token chunks, one lane per channel,
    B/C shared by groups of lanes; 2 lanes widen B/C to fp32 once per chunk
    unless the chunk field is 1 ("u": per use), 4 lanes per use unless it
    is 2 ("f")): one, two and many chunks, ragged last chunks and a last CTA
    whose 32 channels are partly past d_inner."""
    b, L, D = shape
    inp, par = W.make_case(b, L, D, 16, "bf16", seed=300 + L + D)
    ref = oracle.layer_fwd(inp, par)
    g = int(group[0]) if isinstance(group, str) else group
    chunk = {"u": 1, "f": 2}[group[1]] if isinstance(group, str) else 0
    flags = (g << 8) | (2 << bm.BIMAMBA_FAMILY_SHIFT) | (chunk << bm.BIMAMBA_CHUNK_SHIFT)
    got32 = run_layer(bm, inp, par, torch.float32, flags)
    assert U.normwise(got32, ref) <= U.GUARD
    got16 = run_layer(bm, inp, par, torch.bfloat16, flags)
    assert U.bf16_out_ok(got16, ref)
    assert bm.bimamba_device_error() == 0


WIDE = 0x2000  # BIMAMBA_CHUNKED_WIDE


@pytest.mark.parametrize("shape", [(1, 257, 72), (3, 100, 40), (2, 33, 8), (1, 95, 24), (2, 1, 16),
                                   (1, 32, 32), (1, 64, 48), (1, 65, 8), (1, 200, 20)])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_ragged_chunked_direct_kernel(bm, shape, dtype):
    """The chunked kernel at 8 lanes per channel in both forms: one warp per
    direction (4-channel CTAs whose bf16 tiles are the aligned 8 channels
    around them) reading B/C straight from the tiles (the default), and the
    4-warp CTAs with B/C widened once per chunk (BIMAMBA_CHUNKED_WIDE)."""
    b, L, D = shape
    if D * (4 if dtype == "fp32" else 2) % 16:
        pytest.skip("rows must be 16-byte units for the TMA-fed kernels")
    inp, par = W.make_case(b, L, D, 16, dtype, seed=800 + L + D)
    ref = oracle.layer_fwd(inp, par)
    for flags in ((8 << 8) | (1 << bm.BIMAMBA_FAMILY_SHIFT), (8 << 8) | (1 << bm.BIMAMBA_FAMILY_SHIFT) | WIDE):
        got32 = run_layer(bm, inp, par, torch.float32, flags)
        assert U.normwise(got32, ref) <= (U.GUARD if dtype == "bf16" else U.TOL_FP32), hex(flags)
        if dtype == "bf16":
            got16 = run_layer(bm, inp, par, torch.bfloat16, flags)
            assert U.bf16_out_ok(got16, ref)
        assert bm.bimamba_device_error() == 0


PSCAN = 3 << 18  # the chunked parallel scan (8 pieces of 8 steps per channel and chunk)


@pytest.mark.parametrize("shape", [(1, 257, 72), (3, 100, 40), (2, 33, 8), (1, 95, 24), (2, 1, 16),
                                   (1, 64, 32), (1, 128, 48), (1, 65, 8), (1, 200, 20), (2, 129, 16), (1, 63, 8)])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_ragged_pscan_kernel(bm, shape, dtype):
    """The chunked parallel scan: chunks of 64 steps cut into 8 pieces whose
    affine carries are combined by warp shuffles; one, two and many chunks,
    ragged last chunks (where the reverse walk starts with identity steps),
    and channel counts that leave the last CTA's 8 channels partly empty."""
    b, L, D = shape
    if D * (4 if dtype == "fp32" else 2) % 16:
        pytest.skip("rows must be 16-byte units for the TMA-fed kernels")
    inp, par = W.make_case(b, L, D, 16, dtype, seed=900 + L + D)
    ref = oracle.layer_fwd(inp, par)
    got32 = run_layer(bm, inp, par, torch.float32, PSCAN)
    assert U.normwise(got32, ref) <= (U.GUARD if dtype == "bf16" else U.TOL_FP32)
    if dtype == "bf16":
        got16 = run_layer(bm, inp, par, torch.bfloat16, PSCAN)
        assert U.bf16_out_ok(got16, ref)
    assert bm.bimamba_device_error() == 0


@pytest.mark.parametrize("flag", ["fwd", "rev"])
def test_pscan_single_direction_and_general_A(bm, flag):
    inp, par = W.make_case(1, 300, 24, 16, "fp32", seed=23)
    g = torch.Generator().manual_seed(29)
    par = dict(par)
    par["A"] = -torch.exp(torch.rand(par["A"].shape, generator=g) * 5.0 - 3.0)
    par["D"] = torch.rand(par["D"].shape, generator=g) * 2.0 - 1.0
    f = oracle.FWD_ONLY if flag == "fwd" else oracle.REV_ONLY
    ref = oracle.layer_fwd(inp, par, flags=f)
    fl = bm.BIMAMBA_FWD_ONLY if flag == "fwd" else bm.BIMAMBA_REV_ONLY
    got = run_layer(bm, inp, par, torch.float32, PSCAN | fl)
    assert U.normwise(got, ref) <= U.TOL_FP32


def test_pscan_rejects_staging(bm):
    inp, par = W.make_case(1, 64, 16, 16, "bf16", seed=1, device="cuda")
    with pytest.raises(bm.BimambaError) as e:
        bm.bimamba_layer_fwd(inp["x"], inp["z"], inp["dt"], inp["B"], inp["C"], par, flags=PSCAN | bm.BIMAMBA_NO_TMA)
    assert e.value.status == bm.BIMAMBA_ERR_UNSUPPORTED


@pytest.mark.parametrize("flags", [(8 << 8) | (1 << 18) | WIDE, PSCAN])
@pytest.mark.parametrize("L", [4096, 65536])
def test_long_sequence_other_kernels_sampled(bm, L, flags):
    """b=1, D=4096, bf16, seed 2: the 4-warp chunked kernel and the parallel
    scan at long L (the default kernel is checked by test_long_sequence_sampled)."""
    err, ok16 = _sampled_layer_check(bm, W.LONG_SEQ[L], 12, flags)
    assert err <= U.GUARD and ok16


def test_unaligned_channel_count_uses_staged_kernel(bm):
    """d_inner = 20: a bf16 row is not a whole number of 16-byte units, so
    the library must take the kernel without TMA -- and still be right."""
    inp, par = W.make_case(2, 70, 20, 16, "bf16", seed=11)
    ref = oracle.layer_fwd(inp, par)
    got = run_layer(bm, inp, par, torch.float32)
    assert U.normwise(got, ref) <= U.GUARD


@pytest.mark.parametrize("L", [1, 2, 3, 4, 5, 15, 16, 31, 32, 33, 63, 64, 65, 96, 97])
def test_short_sequences(bm, L):
    inp, par = W.make_case(2, L, 16, 16, "fp32", seed=7 + L)
    ref = oracle.layer_fwd(inp, par)
    for flags in (1 << 8 | bm.BIMAMBA_NO_TMA, 4 << 8 | bm.BIMAMBA_NO_TMA, 16 << 8 | bm.BIMAMBA_NO_TMA,
                  4 << 8 | 1 << 18, 8 << 8 | 1 << 18, 16 << 8 | 1 << 18, 4 << 8 | 1 << 16 | 1 << 18,
                  16 << 8 | 1 << 16 | 1 << 18, 1 << 8 | 2 << 18, 2 << 8 | 2 << 18, 4 << 8 | 2 << 18,
                  8 << 8 | 2 << 18):
        got = run_layer(bm, inp, par, torch.float32, flags)
        assert U.normwise(got, ref) <= U.TOL_FP32, (L, hex(flags))


@pytest.mark.parametrize("flag", ["fwd", "rev"])
def test_single_direction_flags(bm, flag):
    """FWD_ONLY / REV_ONLY give y_0 * silu(z) / y_1 * silu(z) (Eq. (6) additivity)."""
    inp, par = W.make_case(2, 130, 24, 16, "fp32", seed=3)
    f = oracle.FWD_ONLY if flag == "fwd" else oracle.REV_ONLY
    ref = oracle.layer_fwd(inp, par, flags=f)
    got = run_layer(bm, inp, par, torch.float32, bm.BIMAMBA_FWD_ONLY if flag == "fwd" else bm.BIMAMBA_REV_ONLY)
    assert U.normwise(got, ref) <= U.TOL_FP32


def test_conv_bias_absent(bm):
    inp, par = W.make_case(1, 90, 16, 16, "fp32", seed=4)
    par = dict(par)
    par["conv_b"] = None
    ref = oracle.layer_fwd(inp, par)
    got = run_layer(bm, inp, par, torch.float32)
    assert U.normwise(got, ref) <= U.TOL_FP32


def test_general_A_and_D(bm):
    """A not of the S4D-real form and D != 1: nothing may rely on either."""
    inp, par = W.make_case(2, 200, 40, 16, "fp32", seed=5)
    g = torch.Generator().manual_seed(9)
    par = dict(par)
    par["A"] = -torch.exp(torch.rand(par["A"].shape, generator=g) * 5.0 - 3.0)
    par["D"] = torch.rand(par["D"].shape, generator=g) * 2.0 - 1.0
    ref = oracle.layer_fwd(inp, par)
    got = run_layer(bm, inp, par, torch.float32)
    assert U.normwise(got, ref) <= U.TOL_FP32


def test_repeatable(bm):
    """Same inputs, same bits: no reduction order depends on timing."""
    inp, par = W.make_case(2, 300, 64, 16, "bf16", seed=6)
    a = run_layer(bm, inp, par, torch.bfloat16)
    b = run_layer(bm, inp, par, torch.bfloat16)
    assert np.array_equal(a, b)


def _sampled_layer_check(bm, w: W.Workload, nchan: int, flags=0):
    inp, par = W.make_case(w.batch, w.L, w.d_inner, w.d_state, w.dtype, w.seed, device="cuda")
    out32 = bm.bimamba_layer_fwd(inp["x"], inp["z"], inp["dt"], inp["B"], inp["C"], par,
                                 out_dtype=torch.float32, flags=flags)
    out16 = bm.bimamba_layer_fwd(inp["x"], inp["z"], inp["dt"], inp["B"], inp["C"], par,
                                 out_dtype=torch.bfloat16, flags=flags)
    torch.cuda.synchronize()
    chans = U.sample_channels(w.d_inner, nchan, seed=w.seed)
    si, sp = U.channel_subset(inp, par, chans)
    ref = oracle.layer_fwd(si, sp)
    idx = torch.as_tensor(chans, device="cuda")
    g32 = U.to_cpu64(out32.index_select(-1, idx))
    g16 = U.to_cpu64(out16.index_select(-1, idx))
    return U.normwise(g32, ref), U.bf16_out_ok(g16, ref)


@pytest.mark.parametrize("flags", [0, 1 << 18, (2 << 18) | (2 << 8) | (1 << 16)])
def test_layer_1p3b_shape_sampled(bm, flags):
    """b=8, L=2048, D=4096, bf16, seed 1 -- the launch configuration the
    bench times (flags 0) and the chunked kernel; 48 channels of every batch
    row against the oracle."""
    err, ok16 = _sampled_layer_check(bm, W.LAYER_1P3B, 48, flags)
    assert err <= U.GUARD and ok16


@pytest.mark.parametrize("L", [4096, 65536, 131072])
def test_long_sequence_sampled(bm, L):
    """b=1, D=4096, bf16, seed 2 at long L; 12 channels against the oracle."""
    err, ok16 = _sampled_layer_check(bm, W.LONG_SEQ[L], 12)
    assert err <= U.TOL_BF16 and ok16
    assert err <= U.GUARD


# ------------------------------------------------------------------ block step

def _slice_tokens(inp, lo, hi):
    return {k: (v[:, :, lo:hi] if k in ("dt", "B", "C") else v[:, lo:hi]).contiguous()
            for k, v in inp.items() if v is not None}


# block-step kernels: 0 = rows staged by cp.async, NO_TMA = ordinary loads,
# a lane count = the kernel that splits a channel's states over lanes
BLOCK_KERNELS = {"async": 0, "plain": 0x4000, "split4": 4 << 8, "split8": 8 << 8}


@pytest.mark.parametrize("kernel", ["async", "plain", "split4"])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_block_chain_matches_oracle(bm, dtype, kernel):
    """Prefix of 512 tokens, then 16 blocks of 32 committed one after another
    (L = 1024 in all): every block's output and the committed state against
    the oracle's own block chain."""
    b, D, P, G = 2, 40, 512, 32
    inp, par = W.make_case(b, P + 16 * G, D, 16, dtype, seed=21)
    pre = _slice_tokens(inp, 0, P)
    h_ref, t_ref = oracle.prefix_state(pre, par)
    dpar = U.to_device(par)
    dpre = U.to_device(pre)
    h, tail = bm.bimamba_prefix_state(dpre["x"], dpre["dt"], dpre["B"], dpar)
    torch.cuda.synchronize()
    assert U.normwise(U.to_cpu64(h), h_ref) <= U.GUARD
    assert np.array_equal(U.to_cpu64(tail), t_ref)
    tol = U.TOL_FP32 if dtype == "fp32" else U.GUARD
    for k in range(16):
        blk = _slice_tokens(inp, P + k * G, P + (k + 1) * G)
        ref, h_ref, t_ref = oracle.block_step(h_ref, t_ref, blk, par, commit=True)
        dblk = U.to_device(blk)
        out = bm.bimamba_block_step((h, tail), dblk["x"], dblk["z"], dblk["dt"], dblk["B"], dblk["C"], dpar,
                                    out_dtype=torch.float32, new_state=(h, tail), flags=BLOCK_KERNELS[kernel])
        torch.cuda.synchronize()
        assert U.normwise(U.to_cpu64(out), ref) <= tol, k
        assert U.normwise(U.to_cpu64(h), h_ref) <= U.GUARD, k
        assert np.array_equal(U.to_cpu64(tail), t_ref), k


@pytest.mark.parametrize("kernel", ["async", "plain", "split8"])
@pytest.mark.parametrize("G", [1, 2, 3, 5, 31, 33, 64])
@pytest.mark.parametrize("D", [24, 18])
def test_block_step_ragged_lengths(bm, G, kernel, D):
    """d_inner 18 (72-byte rows) cannot take 16-byte copies: the default then
    falls back to ordinary loads."""
    b, P = 2, 70
    inp, par = W.make_case(b, P + G, D, 16, "fp32", seed=30 + G)
    pre, blk = _slice_tokens(inp, 0, P), _slice_tokens(inp, P, P + G)
    h_ref, t_ref = oracle.prefix_state(pre, par)
    ref, h2_ref, t2_ref = oracle.block_step(h_ref, t_ref, blk, par, commit=True)
    dpar, dpre, dblk = U.to_device(par), U.to_device(pre), U.to_device(blk)
    h, tail = bm.bimamba_prefix_state(dpre["x"], dpre["dt"], dpre["B"], dpar)
    h2, t2 = torch.empty_like(h), torch.empty_like(tail)
    out = bm.bimamba_block_step((h, tail), dblk["x"], dblk["z"], dblk["dt"], dblk["B"], dblk["C"], dpar,
                                out_dtype=torch.float32, new_state=(h2, t2), flags=BLOCK_KERNELS[kernel])
    torch.cuda.synchronize()
    assert U.normwise(U.to_cpu64(out), ref) <= U.TOL_FP32
    assert U.normwise(U.to_cpu64(h2), h2_ref) <= U.TOL_FP32
    assert np.array_equal(U.to_cpu64(t2), t2_ref)
    # without commit the cached state is left alone
    h_before = h.clone()
    bm.bimamba_block_step((h, tail), dblk["x"], dblk["z"], dblk["dt"], dblk["B"], dblk["C"], dpar,
                          out_dtype=torch.float32, flags=BLOCK_KERNELS[kernel])
    torch.cuda.synchronize()
    assert torch.equal(h, h_before)


@pytest.mark.parametrize("kernel", ["async", "plain"])
def test_block_step_flags(bm, kernel):
    b, D, P, G = 1, 16, 40, 32
    inp, par = W.make_case(b, P + G, D, 16, "fp32", seed=41)
    pre, blk = _slice_tokens(inp, 0, P), _slice_tokens(inp, P, P + G)
    h_ref, t_ref = oracle.prefix_state(pre, par)
    dpar, dpre, dblk = U.to_device(par), U.to_device(pre), U.to_device(blk)
    h, tail = bm.bimamba_prefix_state(dpre["x"], dpre["dt"], dpre["B"], dpar)
    for f_or, f_bm in ((oracle.FWD_ONLY, bm.BIMAMBA_FWD_ONLY), (oracle.REV_ONLY, bm.BIMAMBA_REV_ONLY)):
        ref = oracle.block_step(h_ref, t_ref, blk, par, flags=f_or)
        out = bm.bimamba_block_step((h, tail), dblk["x"], dblk["z"], dblk["dt"], dblk["B"], dblk["C"], dpar,
                                    out_dtype=torch.float32, flags=f_bm | BLOCK_KERNELS[kernel])
        torch.cuda.synchronize()
        assert U.normwise(U.to_cpu64(out), ref) <= U.TOL_FP32


def test_block_cached_full_prefix_sampled(bm):
    """b=16, P=65536, D=4096, bf16: the prefix state over the full prefix and
    two committed block steps of 32 tokens, on 8 sampled channels."""
    w = W.BLOCK_CACHED
    P, G = w.extra["prefix"], w.extra["block"]
    inp, par = W.make_case(w.batch, P + 2 * G, w.d_inner, 16, "bf16", w.seed, device="cuda")
    pre = {"x": inp["x"][:, :P], "dt": inp["dt"][0, :, :P].contiguous(), "B": inp["B"][0, :, :P].contiguous()}
    h, tail = bm.bimamba_prefix_state(pre["x"].contiguous(), pre["dt"], pre["B"], par)
    chans = U.sample_channels(w.d_inner, 8, seed=5)
    idx = torch.as_tensor(chans, device="cuda")
    si, sp = U.channel_subset(inp, par, chans)
    spre = _slice_tokens(si, 0, P)
    h_ref, t_ref = oracle.prefix_state(spre, sp)
    torch.cuda.synchronize()
    assert U.normwise(U.to_cpu64(h.index_select(1, idx)), h_ref) <= U.GUARD
    assert np.array_equal(U.to_cpu64(tail.index_select(-1, idx)), t_ref)
    for k in range(2):
        blk = _slice_tokens(inp, P + k * G, P + (k + 1) * G)
        out = bm.bimamba_block_step((h, tail), blk["x"], blk["z"], blk["dt"], blk["B"], blk["C"], par,
                                    out_dtype=torch.float32, new_state=(h, tail))
        sblk = _slice_tokens(si, P + k * G, P + (k + 1) * G)
        ref, h_ref, t_ref = oracle.block_step(h_ref, t_ref, sblk, sp, commit=True)
        torch.cuda.synchronize()
        assert U.normwise(U.to_cpu64(out.index_select(-1, idx)), ref) <= U.GUARD
        assert U.normwise(U.to_cpu64(h.index_select(1, idx)), h_ref) <= U.GUARD


def test_workspace_too_small_is_rejected(bm):
    inp, par = W.make_case(1, 64, 16, 16, "bf16", seed=1, device="cuda")
    ws = torch.empty(100, dtype=torch.uint8, device="cuda")
    with pytest.raises(bm.BimambaError) as e:
        bm.bimamba_layer_fwd(inp["x"], inp["z"], inp["dt"], inp["B"], inp["C"], par, workspace=ws)
    assert e.value.status == bm.BIMAMBA_ERR_WORKSPACE
