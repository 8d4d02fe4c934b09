"""Host logic of the sequence-sharded layer (bidirectional_mamba_denoiser_b200/
sharded.py), on CPU: halo selection and the whole exchange (all-gathers over
real gloo groups of 2 and 3 ranks) with a plain fp64 numpy stand-in for the
CUDA compute steps, against the oracle's full-sequence layer."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from bidirectional_mamba_denoiser_b200 import sharded as SH
from bidirectional_mamba_denoiser_b200 import workloads as W


class NumpyOps:
    """The two compute steps in plain fp64 numpy: the layer with carries
    (the recurrences of §3.2 Eq. (4)-(6) started from h_in, reporting the
    final states and the step-size sums; the convs reading the halo rows
    outside the segment) and the carry composition."""

    state_dtype = torch.float64

    def layer_carry(self, seg, params, halo, h_in=None, h_out=None, delta_sum=None, out=None):
        x = seg["x"].double().numpy()
        z = seg["z"].double().numpy()
        dt, B, C = (seg[k].double().numpy() for k in ("dt", "B", "C"))
        A, Dk, bias, w, cb = (params[k].double().numpy() for k in ("A", "D", "dt_bias", "conv_w", "conv_b"))
        b, L, D = x.shape
        N = B.shape[-1]
        left, right = ((np.zeros((b, 3, D)), np.zeros((b, 3, D))) if halo is None
                       else (halo[0].double().numpy(), halo[1].double().numpy()))
        xp = np.concatenate([left, x, right], axis=1)
        y = np.zeros((2, b, L, D))
        for r in range(2):
            # forward: tap k on x[t-3+k]; reverse: tap k on x[t+3-k] (xp is x shifted by 3)
            if r == 0:
                pre = sum(w[r][:, k] * xp[:, k:k + L] for k in range(4))
            else:
                pre = sum(w[r][:, k] * xp[:, 6 - k:6 - k + L] for k in range(4))
            u = (pre + cb[r]) / (1.0 + np.exp(-(pre + cb[r])))
            dl = np.logaddexp(0.0, dt[r] + bias[r])  # exactly 0 where dt = -inf
            h = np.zeros((b, D, N)) if h_in is None else h_in[r].double().numpy().copy()
            for t in (range(L) if r == 0 else range(L - 1, -1, -1)):
                h = np.exp(dl[:, t, :, None] * A[r][None]) * h + (dl[:, t] * u[:, t])[:, :, None] * B[r][:, t, None, :]
                y[r][:, t] = (C[r][:, t, None, :] * h).sum(-1) + Dk[r] * u[:, t]
            if h_out is not None:
                h_out[r] = torch.from_numpy(h)
            if delta_sum is not None:
                delta_sum[r] = torch.from_numpy(dl.sum(axis=1))
        res = torch.from_numpy((y[0] + y[1]) * (z / (1.0 + np.exp(-z))))
        if out is not None:
            out.copy_(res)
            return out
        return res

    def compose(self, h_all, ds_all, params, seg):
        A = params["A"].double()
        R = h_all.shape[0]
        hf = torch.zeros_like(h_all[0, 0])
        for j in range(seg):
            hf = torch.exp(A[0][None] * ds_all[j, 0][..., None]) * hf + h_all[j, 0]
        hb = torch.zeros_like(h_all[0, 1])
        for j in range(R - 1, seg, -1):
            hb = torch.exp(A[1][None] * ds_all[j, 1][..., None]) * hb + h_all[j, 1]
        return torch.stack([hf, hb])


def _case(L, seed=11, D=8, b=2):
    inp, par = W.make_case(b, L, D, 16, "fp32", seed)
    inp = {k: v.double() for k, v in inp.items()}
    par = {k: v.double() for k, v in par.items()}
    return inp, par


def test_neighbour_halos_and_extension():
    inp, _ = _case(20)
    segs = SH.split_sequence(inp, [6, 9, 5])
    edges = torch.stack([SH.halo_edges(s) for s in segs])
    left, right = SH.neighbour_halos(edges, 1)
    assert torch.equal(left, inp["x"][:, 3:6]) and torch.equal(right, inp["x"][:, 15:18])
    left0, _ = SH.neighbour_halos(edges, 0)
    _, right2 = SH.neighbour_halos(edges, 2)
    assert not left0.any() and not right2.any()
    assert left.is_contiguous() and right.is_contiguous()
    with pytest.raises(ValueError):
        SH.halo_edges({"x": inp["x"][:, :2]})


@pytest.mark.parametrize("lengths", [[40], [20, 20], [5, 17, 3, 30], [3, 3, 3]])
def test_emulated_segments_match_the_full_layer(lengths):
    inp, par = _case(sum(lengths))
    got = SH.emulate_sharded(inp, par, lengths, ops=NumpyOps())
    want = oracle.layer_fwd(inp, par)
    assert np.abs(got.numpy() - want).max() <= 1e-10 * np.abs(want).max()


@pytest.mark.parametrize("nseg", [2, 5])
def test_chunked_layer_views_and_halos(nseg):
    """ChunkedLayer: one sequence read as nseg batch rows (views, no copy),
    each row's conv halos the neighbouring rows' edge tokens (zeros at the
    ends); two passes and the composition give the full-sequence layer."""
    inp, par = _case(40, b=1)
    plan = SH.ChunkedLayer(inp, par, nseg, ops=NumpyOps())
    assert plan.seg["x"].data_ptr() == inp["x"].data_ptr()
    before, after = plan.halo
    Ls = 40 // nseg
    assert not before[0].any() and not after[-1].any()
    assert torch.equal(before[1], inp["x"][0, Ls - 3:Ls]) and torch.equal(after[0], inp["x"][0, Ls:Ls + 3])
    got = plan.output(plan.run())
    want = oracle.layer_fwd(inp, par)
    assert np.abs(got.numpy() - want).max() <= 1e-10 * np.abs(want).max()


def test_composed_carries_are_the_prefix_and_suffix_states():
    # the forward carry entering a segment is the state of the scan over everything before it
    inp, par = _case(30)
    lengths = [12, 18]
    segs = SH.split_sequence(inp, lengths)
    edges = torch.stack([SH.halo_edges(s) for s in segs])
    ops = NumpyOps()
    aggs = [SH.pass_from_zero(s, SH.neighbour_halos(edges, r), par, ops) for r, s in enumerate(segs)]
    h_in = ops.compose(torch.stack([a[0] for a in aggs]), torch.stack([a[1] for a in aggs]), par, 1)
    head = {k: (v[:, :12] if k in ("x", "z") else v[:, :, :12]) for k, v in inp.items()}
    h_prefix, _ = oracle.prefix_state(head, par)
    assert np.allclose(h_in[0].numpy(), h_prefix, rtol=1e-10, atol=1e-12)
    assert not h_in[1].any()  # the last segment has nothing after it


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, lengths, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp, par = _case(sum(lengths))
        seg = SH.split_sequence(inp, lengths)[rank]
        y = SH.sharded_layer_fwd(seg, par, ops=NumpyOps())
        q.put((rank, y.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("lengths", [[21, 19], [8, 25, 11]])
def test_sharded_layer_over_gloo(lengths):
    world = len(lengths)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, lengths, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp, par = _case(sum(lengths))
    want = oracle.layer_fwd(inp, par)
    full = np.concatenate([got[r] for r in range(world)], axis=1)
    assert np.abs(full - want).max() <= 1e-10 * np.abs(want).max()
