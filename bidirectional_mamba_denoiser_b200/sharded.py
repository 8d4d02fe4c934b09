"""Sequence-sharded bidirectional layer: one long sequence cut into
contiguous segments, one per rank.

The forward scan of segment r needs the state the sequence reaches before
it, and the reverse scan the state it reaches after it ("DiffuMamba:
High-Throughput Diffusion LMs with Mamba Backbone", §3.2 Eq. (4)-(5)).  The
recurrence is affine in the state, so a segment run from state h ends in
exp(A * sum Delta) h + h_end, where h_end is its run from zero: every rank
can scan its segment once from zero, the ranks exchange these small
aggregates ([2, b, D, 16] states and [2, b, D] step-size sums), and each
composes the states entering its own segment and scans again from them.
The causal and anti-causal convs also reach three tokens into the
neighbouring segments, so the ranks first exchange their first and last
three x rows (the halos), which the layer kernels read in place of the zeros
outside the segment: the segment itself is passed as it is.

Per rank, in order (all arithmetic in the CUDA library):
  1. ``halo_edges``: the segment's first and last 3 x rows; all-gathered;
     ``neighbour_halos`` picks the rows before and after this segment.
  2. ``pass_from_zero``: ``bimamba_layer_fwd_carry`` from zero states, for
     h_out and delta_sum (its output is not used); all-gathered.
  3. ``pass_with_carries``: ``bimamba_compose_carries`` for this segment's
     entering states, then ``bimamba_layer_fwd_carry`` from them: the
     segment's layer output.

The collectives are three small all-gathers (the halo rows, the final
states, the step-size sums: a few hundred KB in all), the exchange step of a
scan split along the sequence, and nothing else.  ``sharded_layer_fwd`` runs
the steps under ``torch.distributed``; ``emulate_sharded`` runs them for all
segments in one process (one device), with stacking in place of the
collectives -- the same functions, so the single-device tests check the
arithmetic of the distributed path.  Every segment needs at least 3 tokens.
"""
from __future__ import annotations

from typing import Sequence

import torch

HALO = 3  # conv width - 1


class CudaOps:
    """The compute steps, through the C ABI."""

    state_dtype = torch.float32  # of the carried states and step-size sums

    def __init__(self, flags: int = 0):
        from . import bimamba as bm
        self.bm = bm
        self.flags = flags

    def layer_carry(self, seg: dict, params: dict, halo, h_in=None, h_out=None, delta_sum=None, out=None):
        return self.bm.bimamba_layer_fwd_carry(seg["x"], seg["z"], seg["dt"], seg["B"], seg["C"], params,
                                              h_in=h_in, h_out=h_out, delta_sum=delta_sum, out=out,
                                              flags=self.flags, conv_halo=halo)

    def compose(self, h_all, ds_all, params: dict, seg: int):
        return self.bm.bimamba_compose_carries(h_all, ds_all, params, seg)


def halo_edges(seg: dict) -> torch.Tensor:
    """[2, b, 3, D]: the segment's first and last three x rows."""
    x = seg["x"]
    if x.shape[1] < HALO:
        raise ValueError(f"a segment needs at least {HALO} tokens, got {x.shape[1]}")
    return torch.stack([x[:, :HALO], x[:, x.shape[1] - HALO:]]).contiguous()


def neighbour_halos(all_edges: torch.Tensor, rank: int):
    """From the gathered edges [R, 2, b, 3, D]: the x rows just before the
    segment (rank - 1's last three; zeros at the sequence start) and just
    after it (rank + 1's first three; zeros at the end), as the conv halos
    (before, after) of the segment's layer calls, [b, 3, D] each."""
    R = all_edges.shape[0]
    zeros = torch.zeros_like(all_edges[0, 0])
    left = all_edges[rank - 1, 1] if rank > 0 else zeros
    right = all_edges[rank + 1, 0] if rank < R - 1 else zeros
    return left.contiguous(), right.contiguous()


def pass_from_zero(seg: dict, halo, params: dict, ops) -> tuple[torch.Tensor, torch.Tensor]:
    """The segment scanned from zero states: (h_out [2, b, D, 16],
    delta_sum [2, b, D]) of ops.state_dtype."""
    b, _, D = seg["x"].shape
    N = seg["B"].shape[-1]
    dev = seg["x"].device
    h_out = torch.empty(2, b, D, N, device=dev, dtype=ops.state_dtype)
    ds = torch.empty(2, b, D, device=dev, dtype=ops.state_dtype)
    ops.layer_carry(seg, params, halo, h_out=h_out, delta_sum=ds)
    return h_out, ds


def pass_with_carries(seg: dict, halo, params: dict, h_all: torch.Tensor, ds_all: torch.Tensor, rank: int, ops,
                      out=None) -> torch.Tensor:
    """The segment scanned from the states the other segments hand it: its
    layer output [b, Ls, D] (written to out if given)."""
    h_in = ops.compose(h_all, ds_all, params, rank)
    return ops.layer_carry(seg, params, halo, h_in=h_in, out=out)


def _all_gather(t: torch.Tensor, group=None) -> torch.Tensor:
    import torch.distributed as dist
    parts = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts)


def sharded_layer_fwd(seg: dict, params: dict, group=None, ops=None, out=None) -> torch.Tensor:
    """This rank's segment of the layer output, the segments being the
    ranks' contiguous pieces of one sequence in rank order (any lengths >= 3).
    seg: {"x", "z" [b, Ls, D]; "dt" [2, b, Ls, D]; "B", "C" [2, b, Ls, 16]}."""
    import torch.distributed as dist
    ops = ops or CudaOps()
    rank = dist.get_rank(group)
    halo = neighbour_halos(_all_gather(halo_edges(seg), group), rank)
    h_out, ds = pass_from_zero(seg, halo, params, ops)
    return pass_with_carries(seg, halo, params, _all_gather(h_out, group), _all_gather(ds, group), rank, ops, out=out)


def split_sequence(inputs: dict, lengths: Sequence[int]) -> list[dict]:
    """Cut full-sequence inputs into contiguous segments of the given lengths."""
    segs, t0 = [], 0
    for n in lengths:
        segs.append({"x": inputs["x"][:, t0:t0 + n], "z": inputs["z"][:, t0:t0 + n],
                     "dt": inputs["dt"][:, :, t0:t0 + n], "B": inputs["B"][:, :, t0:t0 + n],
                     "C": inputs["C"][:, :, t0:t0 + n]})
        t0 += n
    assert t0 == inputs["x"].shape[1], "segment lengths must cover the sequence"
    return segs


def emulate_sharded(inputs: dict, params: dict, lengths: Sequence[int], ops=None) -> torch.Tensor:
    """The sharded computation for all segments in this process (stacking in
    place of the all-gathers); returns the full output [b, L, D]."""
    ops = ops or CudaOps()
    segs = [{k: v.contiguous() for k, v in s.items()} for s in split_sequence(inputs, lengths)]
    all_edges = torch.stack([halo_edges(s) for s in segs])
    halos = [neighbour_halos(all_edges, r) for r in range(len(segs))]
    aggs = [pass_from_zero(s, halos[r], params, ops) for r, s in enumerate(segs)]
    h_all = torch.stack([a[0] for a in aggs])
    ds_all = torch.stack([a[1] for a in aggs])
    return torch.cat([pass_with_carries(s, halos[r], params, h_all, ds_all, r, ops) for r, s in enumerate(segs)],
                     dim=1)


class ChunkedLayer:
    """The layer over one long sequence (batch 1) cut into `nseg` equal
    segments that one GPU scans side by side, as the rows of a batch: the
    chunked form of the scan, with carries, inside one device.

    The segments are views of the inputs ([1, L, ...] read as [nseg, L/nseg,
    ...]: no copy); ``__init__`` gathers each segment's conv halos (3 x rows
    on each side) once.  ``run`` is then the scan itself: one layer pass from
    zero states for every segment's final states and step-size sums, the
    composition of the carries entering each segment (nseg small launches),
    and a second layer pass from them, whose output rows are the layer's.  It
    exists to measure this schedule against the single-pass kernels, which
    walk the whole sequence in one chain per (channel, direction) and so need
    no second pass."""

    def __init__(self, inputs: dict, params: dict, nseg: int, ops=None):
        x = inputs["x"]
        if x.shape[0] != 1:
            raise ValueError("the chunked form takes one sequence (batch 1)")
        L = x.shape[1]
        if L % nseg or L // nseg < HALO:
            raise ValueError(f"L = {L} must split into {nseg} equal segments of at least {HALO} tokens")
        self.ops = ops or CudaOps()
        self.params = params
        self.nseg, self.Ls = nseg, L // nseg
        Ls = self.Ls
        D, N = x.shape[2], inputs["B"].shape[-1]
        self.seg = {"x": x.contiguous().view(nseg, Ls, D), "z": inputs["z"].contiguous().view(nseg, Ls, D),
                    "dt": inputs["dt"].contiguous().view(2, nseg, Ls, D),
                    "B": inputs["B"].contiguous().view(2, nseg, Ls, N),
                    "C": inputs["C"].contiguous().view(2, nseg, Ls, N)}
        xs = self.seg["x"]
        before = torch.zeros(nseg, HALO, D, device=x.device, dtype=x.dtype)
        after = torch.zeros_like(before)
        before[1:] = xs[:-1, Ls - HALO:]
        after[:-1] = xs[1:, :HALO]
        self.halo = (before, after)
        dev = x.device
        self.h_out = torch.empty(2, nseg, D, N, device=dev, dtype=self.ops.state_dtype)
        self.ds = torch.empty(2, nseg, D, device=dev, dtype=self.ops.state_dtype)
        self.h_all = torch.empty(nseg, 2, 1, D, N, device=dev, dtype=self.ops.state_dtype)
        self.ds_all = torch.empty(nseg, 2, 1, D, device=dev, dtype=self.ops.state_dtype)
        self.h_in = torch.empty(2, nseg, D, N, device=dev, dtype=self.ops.state_dtype)
        self.y = torch.empty(nseg, Ls, D, device=dev, dtype=x.dtype)

    def run(self) -> torch.Tensor:
        """[nseg, Ls, D]: each segment's rows of the layer output."""
        self.ops.layer_carry(self.seg, self.params, self.halo, h_out=self.h_out, delta_sum=self.ds)
        self.h_all.copy_(self.h_out.permute(1, 0, 2, 3).unsqueeze(2))
        self.ds_all.copy_(self.ds.permute(1, 0, 2).unsqueeze(2))
        for s in range(self.nseg):
            self.h_in[:, s] = self.ops.compose(self.h_all, self.ds_all, self.params, s)[:, 0]
        return self.ops.layer_carry(self.seg, self.params, self.halo, h_in=self.h_in, out=self.y)

    def output(self, y: torch.Tensor) -> torch.Tensor:
        """The layer output [1, L, D] from run()'s result (a view)."""
        return y.view(1, self.nseg * self.Ls, y.shape[-1])
