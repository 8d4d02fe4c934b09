"""The block-cached decoding schedule on the host: which calls, in which
order, and when each layer commits (a recording stand-in for the binding;
no kernel runs)."""
import types

import torch

from bidirectional_mamba_denoiser_b200 import decode


class Recorder:
    D_STATE = 16

    def __init__(self):
        self.calls = []

    def bimamba_prefix_state(self, x, dt, B, params, h_out=None, conv_x_out=None, stream=None):
        self.calls.append(("prefix", params["id"]))

    def bimamba_block_step(self, state, x, z, dt, B, C, params, out=None, new_state=None, stream=None):
        self.calls.append(("step", params["id"], int(x.item()), new_state is not None))


def test_schedule_commits_once_per_block_per_layer(monkeypatch):
    rec = Recorder()
    monkeypatch.setattr(decode, "bm", rec)
    layers, steps, blocks = 3, 4, 2
    dec = decode.BlockDecoder([{"id": i} for i in range(layers)], batch=1, d_inner=8, dtype=torch.float32,
                              device="cpu")
    dec.prefill(lambda layer: {"x": None, "dt": None, "B": None}, length=10)
    assert rec.calls == [("prefix", i) for i in range(layers)]
    assert dec.committed == 10
    rec.calls.clear()
    out = torch.zeros(layers, 1, 5, 8)
    for _ in range(blocks):
        dec.block(steps, lambda s, l: {"x": torch.tensor(s), "z": None, "dt": None, "B": None, "C": None}, out)
    want = []
    for _ in range(blocks):
        for s in range(steps):
            for layer in range(layers):
                want.append(("step", layer, s, s == steps - 1))
    assert rec.calls == want
    assert dec.committed == 10 + blocks * 5
