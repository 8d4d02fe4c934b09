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
three x rows (the halos).

Per rank, in order (all arithmetic in the CUDA library):
  1. ``halo_edges``: the segment's first and last 3 x rows; all-gathered.
  2. ``extend_segment``: the segment with its halo tokens on both sides; the
     halo tokens get dt = -inf, i.e. step size exactly 0, so they only feed
     the conv and leave the state unchanged.
  3. ``pass_from_zero``: ``bimamba_layer_fwd_carry`` from zero states, for
     h_out and delta_sum (its output is not used); all-gathered.
  4. ``pass_with_carries``: ``bimamba_compose_carries`` for this segment's
     entering states, then ``bimamba_layer_fwd_carry`` from them; the
     segment's rows of that output are the result.

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

    def layer_carry(self, ext: dict, params: dict, h_in=None, h_out=None, delta_sum=None, out=None):
        return self.bm.bimamba_layer_fwd_carry(ext["x"], ext["z"], ext["dt"], ext["B"], ext["C"], params,
                                              h_in=h_in, h_out=h_out, delta_sum=delta_sum, out=out,
                                              flags=self.flags)

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
    after it (rank + 1's first three; zeros at the end)."""
    R = all_edges.shape[0]
    zeros = torch.zeros_like(all_edges[0, 0])
    left = all_edges[rank - 1, 1] if rank > 0 else zeros
    right = all_edges[rank + 1, 0] if rank < R - 1 else zeros
    return left, right


def extend_segment(seg: dict, left: torch.Tensor, right: torch.Tensor) -> dict:
    """The segment's inputs with HALO tokens on each side: x from the
    neighbours, dt = -inf (step size 0: the state passes unchanged), z, B, C
    zero.  x, z [b, Ls, D]; dt [2, b, Ls, D]; B, C [2, b, Ls, 16]."""
    def pad(t, dim, value=0.0):
        shape = list(t.shape)
        shape[dim] = HALO
        p = torch.full(shape, value, device=t.device, dtype=t.dtype)
        return torch.cat([p, t, p], dim=dim).contiguous()
    return {
        "x": torch.cat([left.to(seg["x"].dtype), seg["x"], right.to(seg["x"].dtype)], dim=1).contiguous(),
        "z": pad(seg["z"], 1),
        "dt": pad(seg["dt"], 2, float("-inf")),
        "B": pad(seg["B"], 2),
        "C": pad(seg["C"], 2),
    }


def pass_from_zero(ext: dict, params: dict, ops) -> tuple[torch.Tensor, torch.Tensor]:
    """The extended segment scanned from zero states: (h_out [2, b, D, 16],
    delta_sum [2, b, D]) of ops.state_dtype."""
    b, _, D = ext["x"].shape
    N = ext["B"].shape[-1]
    dev = ext["x"].device
    h_out = torch.empty(2, b, D, N, device=dev, dtype=ops.state_dtype)
    ds = torch.empty(2, b, D, device=dev, dtype=ops.state_dtype)
    ops.layer_carry(ext, params, h_out=h_out, delta_sum=ds)
    return h_out, ds


def pass_with_carries(ext: dict, params: dict, h_all: torch.Tensor, ds_all: torch.Tensor, rank: int, ops,
                      out=None) -> torch.Tensor:
    """The extended segment scanned from the states the other segments hand
    it; returns the segment's own rows of the layer output."""
    h_in = ops.compose(h_all, ds_all, params, rank)
    y = ops.layer_carry(ext, params, h_in=h_in)
    seg = y[:, HALO:y.shape[1] - HALO]
    if out is not None:
        out.copy_(seg)
        return out
    return seg


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
    left, right = neighbour_halos(_all_gather(halo_edges(seg), group), rank)
    ext = extend_segment(seg, left, right)
    h_out, ds = pass_from_zero(ext, params, ops)
    return pass_with_carries(ext, params, _all_gather(h_out, group), _all_gather(ds, group), rank, ops, out=out)


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
    segs = split_sequence(inputs, lengths)
    all_edges = torch.stack([halo_edges(s) for s in segs])
    exts = [extend_segment(s, *neighbour_halos(all_edges, r)) for r, s in enumerate(segs)]
    aggs = [pass_from_zero(e, params, ops) for e in exts]
    h_all = torch.stack([a[0] for a in aggs])
    ds_all = torch.stack([a[1] for a in aggs])
    return torch.cat([pass_with_carries(e, params, h_all, ds_all, r, ops) for r, e in enumerate(exts)], dim=1)


class ChunkedLayer:
    """The layer over one long sequence (batch 1) cut into `nseg` equal
    segments that one GPU scans side by side, as the rows of a batch: the
    chunked form of the scan, with carries, inside one device.

    ``__init__`` builds the extended segments once (each with its 3-token
    halos, stacked into [nseg, Ls + 6, D] inputs); ``run`` is then the scan
    itself: one layer pass from zero states for every segment's final states
    and step-size sums, the composition of the carries entering each segment
    (nseg small launches), and a second layer pass from them.  It exists to
    measure this schedule against the single-pass kernels, which walk the
    whole sequence in one chain per (channel, direction) and so need no
    second pass."""

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
        segs = split_sequence(inputs, [self.Ls] * nseg)
        all_edges = torch.stack([halo_edges(s) for s in segs])
        exts = [extend_segment(s, *neighbour_halos(all_edges, r)) for r, s in enumerate(segs)]
        self.ext = {"x": torch.cat([e["x"] for e in exts], 0).contiguous(),
                    "z": torch.cat([e["z"] for e in exts], 0).contiguous(),
                    "dt": torch.cat([e["dt"] for e in exts], 1).contiguous(),
                    "B": torch.cat([e["B"] for e in exts], 1).contiguous(),
                    "C": torch.cat([e["C"] for e in exts], 1).contiguous()}
        D, N = x.shape[2], inputs["B"].shape[-1]
        dev = x.device
        self.h_out = torch.empty(2, nseg, D, N, device=dev, dtype=self.ops.state_dtype)
        self.ds = torch.empty(2, nseg, D, device=dev, dtype=self.ops.state_dtype)
        self.h_all = torch.empty(nseg, 2, 1, D, N, device=dev, dtype=self.ops.state_dtype)
        self.ds_all = torch.empty(nseg, 2, 1, D, device=dev, dtype=self.ops.state_dtype)
        self.h_in = torch.empty(2, nseg, D, N, device=dev, dtype=self.ops.state_dtype)
        self.y = torch.empty(nseg, self.Ls + 2 * HALO, D, device=dev, dtype=x.dtype)

    def run(self) -> torch.Tensor:
        """[nseg, Ls + 6, D]: each segment's extended rows of the layer output."""
        self.ops.layer_carry(self.ext, self.params, h_out=self.h_out, delta_sum=self.ds)
        self.h_all.copy_(self.h_out.permute(1, 0, 2, 3).unsqueeze(2))
        self.ds_all.copy_(self.ds.permute(1, 0, 2).unsqueeze(2))
        for s in range(self.nseg):
            self.h_in[:, s] = self.ops.compose(self.h_all, self.ds_all, self.params, s)[:, 0]
        return self.ops.layer_carry(self.ext, self.params, h_in=self.h_in, out=self.y)

    def output(self, y: torch.Tensor) -> torch.Tensor:
        """The layer output [1, L, D] from run()'s result."""
        return y[:, HALO:HALO + self.Ls].reshape(1, self.nseg * self.Ls, y.shape[-1])
