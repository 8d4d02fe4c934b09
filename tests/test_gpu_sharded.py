"""The sequence-sharded layer on one B200: every segment's two passes and the
carry composition run through the C ABI (bimamba_layer_fwd_carry,
bimamba_compose_carries), the collectives replaced by stacking
(sharded.emulate_sharded, the same phase functions as the distributed path);
the joined output against the fp64 oracle's full-sequence layer."""
import pytest
import torch

import oracle
from bidirectional_mamba_denoiser_b200 import sharded as SH
from bidirectional_mamba_denoiser_b200 import workloads as W
from tests import parity_util as U

pytestmark = pytest.mark.gpu

FAMILIES = {"fused": 2 << 18, "chunked": 1 << 18, "pscan": 3 << 18}


@pytest.fixture(scope="module")
def bm():
    from bidirectional_mamba_denoiser_b200 import bimamba
    return bimamba


@pytest.mark.parametrize("family", list(FAMILIES))
@pytest.mark.parametrize("lengths", [[300, 212], [100, 57, 3, 200, 40], [512]])
def test_fp32_segments_match_the_full_layer(bm, family, lengths):
    """fp32 in and out, b=2, D=64: normwise <= 1e-5 for 1, 2 and 5 segments (one of 3 tokens)."""
    inp, par = W.make_case(2, sum(lengths), 64, 16, "fp32", 21)
    want = oracle.layer_fwd(inp, par)
    got = SH.emulate_sharded(U.to_device(inp), U.to_device(par), lengths, ops=SH.CudaOps(FAMILIES[family]))
    torch.cuda.synchronize()
    assert bm.bimamba_device_error() == 0
    assert U.normwise(U.to_cpu64(got), want) <= U.TOL_FP32


@pytest.mark.parametrize("family", list(FAMILIES))
def test_bf16_segments_match_the_full_layer(bm, family):
    """bf16 in and out, b=1, L=4096 in 4 segments, D=256: the bf16-output bound."""
    lengths = [1024, 1000, 1100, 972]
    inp, par = W.make_case(1, sum(lengths), 256, 16, "bf16", 22)
    want = oracle.layer_fwd(inp, par)
    got = SH.emulate_sharded(U.to_device(inp), U.to_device(par), lengths, ops=SH.CudaOps(FAMILIES[family]))
    torch.cuda.synchronize()
    assert U.bf16_out_ok(U.to_cpu64(got), want)


@pytest.mark.parametrize("family", list(FAMILIES))
def test_aggregates_are_the_segment_scans(bm, family):
    """Pass 1 of a segment: the forward h_out is the oracle's prefix state of
    the segment (with its left halo), delta_sum the sum of its step sizes,
    and the composed carry into the next segment that same state."""
    inp, par = W.make_case(2, 160, 64, 16, "fp32", 23)
    lengths = [96, 64]
    d, p = U.to_device(inp), U.to_device(par)
    ops = SH.CudaOps(FAMILIES[family])
    segs = [{k: v.contiguous() for k, v in s.items()} for s in SH.split_sequence(d, lengths)]
    edges = torch.stack([SH.halo_edges(s) for s in segs])
    aggs = [SH.pass_from_zero(s, SH.neighbour_halos(edges, r), p, ops) for r, s in enumerate(segs)]
    torch.cuda.synchronize()
    head = {k: (v[:, :96] if k in ("x", "z") else v[:, :, :96]) for k, v in inp.items()}
    h_prefix, _ = oracle.prefix_state(head, par)
    assert U.normwise(U.to_cpu64(aggs[0][0][0]), h_prefix) <= U.TOL_FP32
    _, dl = oracle.features(head, par)
    assert U.normwise(U.to_cpu64(aggs[0][1]), dl.sum(axis=2)) <= U.TOL_FP32
    h_in = ops.compose(torch.stack([a[0] for a in aggs]), torch.stack([a[1] for a in aggs]), p, 1)
    torch.cuda.synchronize()
    assert U.normwise(U.to_cpu64(h_in[0]), h_prefix) <= U.TOL_FP32
    assert not h_in[1].any()


@pytest.mark.parametrize("family", list(FAMILIES))
def test_zero_carries_change_nothing(bm, family):
    """Carries of zero in, states out: the output is bit for bit the plain layer's."""
    inp, par = W.make_case(2, 200, 64, 16, "bf16", 24)
    d, p = U.to_device(inp), U.to_device(par)
    flags = FAMILIES[family]
    plain = bm.bimamba_layer_fwd(d["x"], d["z"], d["dt"], d["B"], d["C"], p, flags=flags)
    zeros = torch.zeros(2, 2, 64, 16, device="cuda")
    h_out = torch.empty(2, 2, 64, 16, device="cuda")
    ds = torch.empty(2, 2, 64, device="cuda")
    got = bm.bimamba_layer_fwd_carry(d["x"], d["z"], d["dt"], d["B"], d["C"], p, h_in=zeros, h_out=h_out,
                                     delta_sum=ds, flags=flags)
    torch.cuda.synchronize()
    assert torch.equal(got, plain)
    assert torch.isfinite(h_out).all() and (ds > 0).all()


def test_full_size_sampled_channels(bm):
    """The bench's sharded workload (b 1, L 262,144, D 4096, bf16) cut into 4
    segments of 65,536 (one rank's share at 4 GPUs), all channels on the GPU;
    16 sampled channels against the oracle's full-sequence layer."""
    w = W.SHARDED_SEQ
    inp, par = W.make_case(w.batch, w.L, w.d_inner, w.d_state, w.dtype, w.seed, device="cuda")
    got = SH.emulate_sharded(inp, par, [w.L // 4] * 4)
    torch.cuda.synchronize()
    assert bm.bimamba_device_error() == 0
    chans = U.sample_channels(w.d_inner, 16, seed=3)
    si, sp = U.channel_subset(inp, par, chans)
    want = oracle.layer_fwd(si, sp)
    idx = torch.as_tensor(chans, device="cuda")
    assert U.bf16_out_ok(U.to_cpu64(got.index_select(-1, idx)), want)


@pytest.mark.parametrize("nseg", [2, 8])
def test_chunked_layer_matches_single_pass(nseg):
    """The batch-1 layer scanned as segments side by side with carries
    (two passes) against the single-pass layer and the oracle."""
    from bidirectional_mamba_denoiser_b200 import bimamba as bm
    from bidirectional_mamba_denoiser_b200 import sharded as SH
    inp, par = W.make_case(1, 1024, 64, 16, "fp32", seed=71)
    ref = oracle.layer_fwd(inp, par)
    d, p = U.to_device(inp), U.to_device(par)
    plan = SH.ChunkedLayer(d, p, nseg)
    got = plan.output(plan.run())
    torch.cuda.synchronize()
    assert U.normwise(U.to_cpu64(got), ref) <= U.TOL_FP32
    one = bm.bimamba_layer_fwd(d["x"], d["z"], d["dt"], d["B"], d["C"], p, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert U.normwise(U.to_cpu64(got), U.to_cpu64(one)) <= U.TOL_FP32
