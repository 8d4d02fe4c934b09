"""Block-cached decoding over several layers (eager and CUDA-graph replay)
against the oracle's own block chain, on a B200."""
import numpy as np
import pytest
import torch

import oracle
from bidirectional_mamba_denoiser_b200 import decode
from bidirectional_mamba_denoiser_b200 import workloads as W
from tests import parity_util as U

pytestmark = pytest.mark.gpu

LAYERS, B, D, P, G, K, BLOCKS = 3, 2, 40, 64, 16, 3, 2


def _case():
    """Per layer: parameters and a token stream long enough for the prefix
    and every (block, step) input; step s of block k uses tokens
    [P + (k*K + s)*G, ... + G) of that layer's stream."""
    cases = [W.make_case(B, P + BLOCKS * K * G, D, 16, "fp32", seed=90 + i) for i in range(LAYERS)]
    return cases


def _slice(inp, lo, hi):
    return {k: (v[:, :, lo:hi] if k in ("dt", "B", "C") else v[:, lo:hi]).contiguous() for k, v in inp.items()}


@pytest.mark.parametrize("graph", [False, True])
def test_block_decoding_matches_oracle_chain(graph):
    cases = _case()
    dev_par = [U.to_device(par) for _, par in cases]
    dev_inp = [U.to_device(inp) for inp, _ in cases]
    dec = decode.BlockDecoder(dev_par, batch=B, d_inner=D, dtype=torch.float32, device="cuda")
    dec.prefill(lambda l: {"x": dev_inp[l]["x"][:, :P].contiguous(), "dt": dev_inp[l]["dt"][0, :, :P].contiguous(),
                           "B": dev_inp[l]["B"][0, :, :P].contiguous()}, P)
    blocks = {}
    for k in range(BLOCKS):
        for s in range(K):
            for l in range(LAYERS):
                lo = P + (k * K + s) * G
                blocks[(k, s, l)] = _slice(dev_inp[l], lo, lo + G)
    state = {"k": 0}
    out = torch.empty(LAYERS, B, G, D, device="cuda")
    outs = []

    def inputs(s, l):
        return blocks[(state["k"], s, l)]

    if not graph:
        for k in range(BLOCKS):
            state["k"] = k
            dec.block(K, inputs, out)
            torch.cuda.synchronize()
            outs.append(out.clone())
    else:
        # inputs are read through fixed buffers that the graph captured
        bufs = [{n: t.clone() for n, t in blocks[(0, s, l)].items()} for s in range(K) for l in range(LAYERS)]
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            g = dec.capture_block(K, lambda s, l: bufs[s * LAYERS + l], out, side)
        torch.cuda.synchronize()
        for k in range(BLOCKS):
            for s in range(K):
                for l in range(LAYERS):
                    for n, t in blocks[(k, s, l)].items():
                        bufs[s * LAYERS + l][n].copy_(t)
            torch.cuda.synchronize()
            g.replay()
            torch.cuda.synchronize()
            outs.append(out.clone())
        del g

    # the oracle's chain, layer by layer
    for l, (inp, par) in enumerate(cases):
        pre = _slice(inp, 0, P)
        h, t = oracle.prefix_state(pre, par)
        for k in range(BLOCKS):
            for s in range(K):
                lo = P + (k * K + s) * G
                blk = _slice(inp, lo, lo + G)
                if s == K - 1:
                    ref, h, t = oracle.block_step(h, t, blk, par, commit=True)
                else:
                    ref = oracle.block_step(h, t, blk, par)
            # the last step's output of block k
            assert U.normwise(U.to_cpu64(outs[k][l]), ref) <= U.TOL_FP32, (l, k)
        assert U.normwise(U.to_cpu64(dec.h[l]), h) <= U.TOL_FP32, l
        assert np.array_equal(U.to_cpu64(dec.tail[l]), t), l


def test_mamba2_block_decoding_matches_layer_oracle():
    """Two layers of the Mamba-2 mixer, prefix of 60 tokens, 2 blocks x 2
    steps of 20: every step's output against the layer oracle by the
    definition of the block step, the conv tails bit-exact."""
    layers, b, H, Pn, G, K = 2, 1, 2, 60, 20, 2
    P, N = 32, 128
    total = Pn + 2 * K * G
    cases = [W.make_mamba2_case(b, total, H, P, N, "fp32", seed=95 + i) for i in range(layers)]
    dev = [(U.to_device(inp), U.to_device(par)) for inp, par in cases]
    dec = decode.BlockDecoder([p for _, p in dev], batch=b, d_inner=H * P, dtype=torch.float32, device="cuda",
                              d_state=N, mixer="mamba2", nheads=H, block_len=G)

    def tok(inp, lo, hi):
        return {"xbc": inp["xbc"][:, :, lo:hi].contiguous(), "z": inp["z"][:, lo:hi].contiguous(),
                "dt": inp["dt"][:, :, lo:hi].contiguous()}

    dec.prefill(lambda l: tok(dev[l][0], 0, Pn), Pn)
    out = torch.empty(layers, b, G, H * P, device="cuda")
    state = {"k": 0}

    def inputs(s, l):
        lo = Pn + (state["k"] * K + s) * G
        return tok(dev[l][0], lo, lo + G)

    for k in range(2):
        state["k"] = k
        for s in range(K):
            dec.step(s, K, inputs, out)
            torch.cuda.synchronize()
            lo = Pn + (k * K + s) * G
            for l, (inp, par) in enumerate(cases):
                # forward from the cache = the full forward over the committed tokens (the prompt
                # and, of each finished block, its last step's tokens) followed by this block
                parts = [tok(inp, 0, Pn)] + [tok(inp, Pn + (kk * K + K - 1) * G, Pn + (kk * K + K) * G)
                                             for kk in range(k)]
                blk = tok(inp, lo, lo + G)
                seq = {n: torch.cat([q[n] for q in parts + [blk]], dim=2 if n != "z" else 1)
                       for n in ("xbc", "z", "dt")}
                _, yf, _ = oracle.mamba2_layer_fwd(seq, par, return_dirs=True)
                _, _, yr = oracle.mamba2_layer_fwd(blk, par, return_dirs=True)
                zz = blk["z"].double().numpy()
                want = (yf[:, -G:] + yr) * (zz / (1.0 + np.exp(-zz)))
                assert U.normwise(U.to_cpu64(out[l]), want) <= U.TOL_FP32, (k, s, l)
    for l, (inp, _) in enumerate(cases):
        # the last commit was block 1's last step: tokens up to Pn + (K + K - 1) G + G
        last = Pn + (K + K - 1) * G + G
        assert np.array_equal(U.to_cpu64(dec.tail[l]), inp["xbc"][0, :, last - 3:last].double().numpy())
