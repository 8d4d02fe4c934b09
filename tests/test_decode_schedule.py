"""The block-cached decoding schedule on the host: which calls, in which
order, and when each layer commits (a recording stand-in for the binding;
no kernel runs)."""

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


class Recorder2:
    """Stand-in for the Mamba-2 mixer's calls."""
    D_STATE = 16
    M2_HEADDIM = 32

    def __init__(self):
        self.calls = []
        self.workspaces = set()

    def bimamba2_workspace_bytes(self, batch, L, nheads, headdim=32, d_state=128):
        return 64

    def bimamba2_prefix_state(self, xbc, dt, params, S_out=None, conv_out=None, workspace=None, stream=None):
        self.calls.append(("prefix", params["id"], tuple(S_out.shape), tuple(conv_out.shape)))

    def bimamba2_block_step(self, state, xbc, z, dt, params, out=None, new_state=None, workspace=None, stream=None):
        self.workspaces.add(workspace.data_ptr())
        self.calls.append(("step", params["id"], int(xbc.item()), new_state is not None))


def test_mamba2_schedule_caches_and_one_shared_workspace(monkeypatch):
    rec = Recorder2()
    monkeypatch.setattr(decode, "bm", rec)
    layers, steps, H, N = 2, 3, 4, 128
    dec = decode.BlockDecoder([{"id": i} for i in range(layers)], batch=2, d_inner=H * 32, dtype=torch.float32,
                              device="cpu", d_state=N, mixer="mamba2", nheads=H, block_len=8)
    # per layer: the state [b][H][32][N] and the xBC conv tail [b][3][H*32 + 2N]
    assert tuple(dec.h.shape) == (layers, 2, H, 32, N) and tuple(dec.tail.shape) == (layers, 2, 3, H * 32 + 2 * N)
    dec.prefill(lambda layer: {"xbc": None, "dt": None}, length=7)
    assert rec.calls == [("prefix", i, (2, H, 32, N), (2, 3, H * 32 + 2 * N)) for i in range(layers)]
    rec.calls.clear()
    out = torch.zeros(layers, 2, 8, H * 32)
    dec.block(steps, lambda s, l: {"xbc": torch.tensor(s), "z": None, "dt": None}, out)
    assert rec.calls == [("step", layer, s, s == steps - 1) for s in range(steps) for layer in range(layers)]
    assert len(rec.workspaces) == 1  # the layers' calls share one workspace
    assert dec.committed == 7 + 8


def test_unknown_mixer_is_rejected():
    import pytest
    with pytest.raises(ValueError):
        decode.BlockDecoder([{}], batch=1, d_inner=8, dtype=torch.float32, device="cpu", mixer="mamba3")
