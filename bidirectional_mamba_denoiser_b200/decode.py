"""Block-cached decoding at the mixer level: per-layer forward caches.

Block-autoregressive denoising ("DiffuMamba: High-Throughput Diffusion LMs
with Mamba Backbone", §4.3; "Training Hybrid Block Diffusion Language Models
with Partial Bidirectionality", abstract) denoises one block of G tokens at a
time.  Each of the K denoising steps of a block runs every layer over the
active block only: the forward direction continues from that layer's cached
state (the state and conv tail after the already generated tokens), the
reverse direction sees the block alone.  Once the block is final, every
layer's cache advances past it (the commit), and the next block starts.

``BlockDecoder`` keeps one cache per layer and runs that schedule through the
C ABI, for either mixer of the library:
  * "mamba1": the d_state-16 layer -- ``bimamba_prefix_state`` once per
    layer, then ``bimamba_block_step`` per step and layer;
  * "mamba2": the Mamba-2 mixer -- ``bimamba2_prefix_state``, then
    ``bimamba2_block_step`` (one workspace shared by the layers' calls, which
    run one after another on one stream);
committing in place on a block's last step.  The block inputs of each step
and layer -- which the layer's in_proj would produce in a full model -- are
supplied by the caller.  ``capture_block`` records one block's K x layers
calls as a CUDA graph, the decoding loop's unit of replay.  All arithmetic
runs in the CUDA library.
"""
from __future__ import annotations

from typing import Callable, Sequence

import torch

from . import bimamba as bm

StepInputs = Callable[[int, int], dict]  # (step, layer) -> the active block's inputs


class BlockDecoder:
    """Per-layer forward caches and the block-cached denoising schedule.

    params: one parameter dict per layer (device tensors as produced by
            ``workloads.make_params`` / ``make_mamba2_params``).
    batch, dtype: the block tensors' batch size and dtype (the conv tail is
            kept in that dtype, the state in fp32).
    mixer "mamba1": d_inner channels with d_state states each; block inputs
            {"x", "z", "dt", "B", "C"}.
    mixer "mamba2": nheads heads of 32 channels, d_state 128, conv over
            d_inner + 2 d_state channels; block inputs {"xbc", "z", "dt"}.
    block_len: the longest block (sizes the Mamba-2 workspace).
    """

    def __init__(self, params: Sequence[dict], batch: int, d_inner: int, dtype: torch.dtype, device,
                 d_state: int = bm.D_STATE, mixer: str = "mamba1", nheads: int = 0, block_len: int = 64):
        if mixer not in ("mamba1", "mamba2"):
            raise ValueError(f"unknown mixer {mixer!r}")
        self.params = list(params)
        self.mixer = mixer
        self.batch, self.d_inner, self.d_state, self.dtype = batch, d_inner, d_state, dtype
        n = len(self.params)
        if mixer == "mamba1":
            self.h = torch.zeros(n, batch, d_inner, d_state, device=device, dtype=torch.float32)
            self.tail = torch.zeros(n, batch, 3, d_inner, device=device, dtype=dtype)
            self.ws = None
        else:
            P = bm.M2_HEADDIM
            assert nheads * P == d_inner, "Mamba-2: d_inner = nheads x 32"
            self.nheads = nheads
            self.h = torch.zeros(n, batch, nheads, P, d_state, device=device, dtype=torch.float32)
            self.tail = torch.zeros(n, batch, 3, d_inner + 2 * d_state, device=device, dtype=dtype)
            self.ws = torch.empty(bm.bimamba2_workspace_bytes(batch, block_len, nheads, P, d_state), device=device,
                                  dtype=torch.uint8)
        self.committed = 0  # tokens behind the caches

    @property
    def layers(self) -> int:
        return len(self.params)

    def cache(self, layer: int):
        return self.h[layer], self.tail[layer]

    def prefill(self, prefix: Callable[[int], dict], length: int, stream=None, workspace=None) -> None:
        """Forward scan of the prompt for every layer: prefix(layer) gives
        that layer's {"x", "dt", "B"} (mamba1) or {"xbc", "dt"} (mamba2) over
        `length` tokens."""
        for layer in range(self.layers):
            inp = prefix(layer)
            h, tail = self.cache(layer)
            if self.mixer == "mamba1":
                bm.bimamba_prefix_state(inp["x"], inp["dt"], inp["B"], self.params[layer], h_out=h, conv_x_out=tail,
                                        stream=stream)
            else:
                bm.bimamba2_prefix_state(inp["xbc"], inp["dt"], self.params[layer], S_out=h, conv_out=tail,
                                         workspace=workspace, stream=stream)
        self.committed = length

    def step(self, step: int, steps: int, inputs: StepInputs, out: torch.Tensor, stream=None) -> None:
        """One denoising step of the active block through every layer; on
        the block's last step (step == steps - 1) each layer commits."""
        commit = step == steps - 1
        for layer in range(self.layers):
            inp = inputs(step, layer)
            cache = self.cache(layer)
            new = cache if commit else None
            if self.mixer == "mamba1":
                bm.bimamba_block_step(cache, inp["x"], inp["z"], inp["dt"], inp["B"], inp["C"], self.params[layer],
                                      out=out[layer], new_state=new, stream=stream)
            else:
                bm.bimamba2_block_step(cache, inp["xbc"], inp["z"], inp["dt"], self.params[layer], out=out[layer],
                                       new_state=new, workspace=self.ws, stream=stream)

    def block(self, steps: int, inputs: StepInputs, out: torch.Tensor, stream=None) -> None:
        """All K steps of one block; the caches advance past it at the end."""
        for s in range(steps):
            self.step(s, steps, inputs, out, stream)
        self.committed += out.shape[2]

    def capture_block(self, steps: int, inputs: StepInputs, out: torch.Tensor, stream) -> torch.cuda.CUDAGraph:
        """Record one block (steps x layers calls, commits included) as a CUDA
        graph on `stream` (not the legacy default stream).  Each replay
        decodes one more block: the caches are updated in place."""
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for s in range(steps):
                self.step(s, steps, inputs, out, stream)
        return graph
