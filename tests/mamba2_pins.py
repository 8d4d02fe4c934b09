"""Pins for the fp64 Mamba-2 oracle: expected values from routes other than
its own loop.

As in ``oracle_pins``, each pin returns the largest discrepancy it saw.  The
expected values come from
  * the d_state-16 layer's oracle (itself pinned independently): a Mamba-2
    head is that recurrence with A and delta constant over the head's
    channels and B, C shared, once B and C have been through the conv, which
    here comes from ``numpy.convolve`` + ``scipy.special.expit``;
  * the materialised L x L dual form of the scan per head
    (M[t, s] = (C_t . B_s) exp(A_h (S_t - S_s)), lower triangle forward,
    upper triangle reverse), a dense ``numpy`` matmul;
  * A = 0, where the state is a running sum of outer products
    (``numpy.cumsum``); B = 0, where only the D skip is left;
  * L = 1 expanded by hand;
  * the method's invariants: the reverse direction is the forward one on the
    flipped sequence with the directions' parameters exchanged, and the gated
    output is additive in the two directions.
"""
from __future__ import annotations

import numpy as np
from scipy.special import expit

import oracle
from bidirectional_mamba_denoiser_b200 import workloads
from tests.oracle_pins import lib_silu, lib_softplus, rel


def np_case2(batch, L, H, P, N, seed=0, shared_xbc=False):
    inp, par = workloads.make_mamba2_case(batch, L, H, P, N, "fp32", seed)
    inp = {k: v.double().numpy().copy() for k, v in inp.items()}
    par = {k: v.double().numpy().copy() for k, v in par.items()}
    if shared_xbc:
        inp["xbc"][1] = inp["xbc"][0]
    return inp, par


def lib_conv_silu(inp, par):
    """v_r = silu(conv_r(xbc_r)) for both directions, [2, b, L, C_conv], by numpy.convolve."""
    xbc = inp["xbc"]
    _, b, L, CH = xbc.shape
    v = np.empty_like(xbc)
    for r in range(2):
        for bi in range(b):
            for c in range(CH):
                w = par["conv_w"][r, c]
                cb = par["conv_b"][r, c] if par.get("conv_b") is not None else 0.0
                col = xbc[r, bi, :, c]
                if r == 0:
                    s = np.convolve(col, w[::-1])[:L]
                else:
                    s = np.convolve(col[::-1], w[::-1])[:L][::-1]
                v[r, bi, :, c] = lib_silu(s + cb)
    return v


def split(v, H, P, N):
    HP = H * P
    return v[..., :HP], v[..., HP:HP + N], v[..., HP + N:HP + 2 * N]


def deltas(inp, par):
    return lib_softplus(inp["dt"] + par["dt_bias"][:, None, None, :])  # [2, b, L, H]


def dims(inp):
    return oracle.mamba2_dims(inp)


# ---------------------------------------------------------------- pins

def pin_reduces_to_dstate16_layer(seed=21, L=40, H=3, P=4, N=6):
    """Per direction, the Mamba-2 mixer is the d_state-16 layer's recurrence
    (with N states) on channels c = h*P + p with A[c, n] = A_h, delta[c] =
    delta_h, D[c] = D_h, B and C taken after their conv.  Both directions'
    outputs come from that oracle with FWD_ONLY / REV_ONLY and are added."""
    inp, par = np_case2(2, L, H, P, N, seed)
    b = inp["z"].shape[0]
    HP = H * P
    v = lib_conv_silu(inp, par)
    _, Bv, Cv = split(v, H, P, N)
    head = np.repeat(np.arange(H), P)
    total = np.zeros((b, L, HP))
    for r, flag in ((0, oracle.FWD_ONLY), (1, oracle.REV_ONLY)):
        m1_inp = {
            "x": inp["xbc"][r][..., :HP],
            "z": inp["z"],
            "dt": inp["dt"][:, :, :, head],
            "B": Bv, "C": Cv,
        }
        m1_par = {
            "A": np.repeat(par["A"][:, head][:, :, None], N, axis=2),
            "D": par["D"][:, head],
            "dt_bias": par["dt_bias"][:, head],
            "conv_w": par["conv_w"][:, :HP],
            "conv_b": par["conv_b"][:, :HP],
        }
        total += oracle.layer_fwd(m1_inp, m1_par, flags=flag)
    return rel(oracle.mamba2_layer_fwd(inp, par), total)


def dual_form_dirs(inp, par):
    """y of both directions per head from the L x L dual form, [2, b, L, H*P]."""
    b, L, H, P, N = dims(inp)
    v = lib_conv_silu(inp, par)
    x, Bv, Cv = split(v, H, P, N)
    dl = deltas(inp, par)
    y = np.empty((2, b, L, H * P))
    tri = np.tril(np.ones((L, L), bool))
    for r in range(2):
        for bi in range(b):
            CB = Cv[r, bi] @ Bv[r, bi].T  # [t, s]
            for h in range(H):
                d = dl[r, bi, :, h]
                if r == 0:
                    S = np.cumsum(d)
                    mask = tri
                else:
                    S = np.cumsum(d[::-1])[::-1]
                    mask = tri.T
                expo = np.where(mask, par["A"][r, h] * (S[:, None] - S[None, :]), -np.inf)
                M = CB * np.exp(expo)
                xh = x[r, bi, :, h * P:(h + 1) * P]
                y[r, bi, :, h * P:(h + 1) * P] = M @ (d[:, None] * xh) + par["D"][r, h] * xh
    return y


def pin_dual_form(seed=22, L=48, H=3, P=4, N=8):
    inp, par = np_case2(2, L, H, P, N, seed)
    y = dual_form_dirs(inp, par)
    want = (y[0] + y[1]) * lib_silu(inp["z"])
    return rel(oracle.mamba2_layer_fwd(inp, par), want)


def pin_zero_decay_running_sum(seed=23, L=30, H=2, P=3, N=5):
    """A = 0: the state is the running sum of delta x B^T (numpy.cumsum)."""
    inp, par = np_case2(1, L, H, P, N, seed)
    par["A"][:] = 0.0
    b, L, H, P, N = dims(inp)
    v = lib_conv_silu(inp, par)
    x, Bv, Cv = split(v, H, P, N)
    dl = deltas(inp, par)
    y = np.zeros((2, b, L, H * P))
    for r in range(2):
        for h in range(H):
            xh = x[r, 0, :, h * P:(h + 1) * P]
            terms = dl[r, 0, :, h][:, None, None] * xh[:, :, None] * Bv[r, 0][:, None, :]  # [L, P, N]
            S = np.cumsum(terms, axis=0) if r == 0 else np.cumsum(terms[::-1], axis=0)[::-1]
            y[r, 0, :, h * P:(h + 1) * P] = np.einsum("tpn,tn->tp", S, Cv[r, 0]) + par["D"][r, h] * xh
    want = (y[0] + y[1]) * lib_silu(inp["z"])
    return rel(oracle.mamba2_layer_fwd(inp, par), want)


def pin_zero_B(seed=24, L=25, H=2, P=3, N=4):
    """Zero conv taps and bias on the B channels make B = silu(0) = 0: y = D x."""
    inp, par = np_case2(1, L, H, P, N, seed)
    HP = H * P
    par["conv_w"][:, HP:HP + N] = 0.0
    par["conv_b"][:, HP:HP + N] = 0.0
    v = lib_conv_silu(inp, par)
    x = v[..., :HP]
    head = np.repeat(np.arange(H), P)
    y = par["D"][:, head][:, None, None, :] * x
    want = (y[0] + y[1]) * lib_silu(inp["z"])
    return rel(oracle.mamba2_layer_fwd(inp, par), want)


def pin_tiny_by_hand(seed=25, H=2, P=2, N=3):
    """L = 1: only tap 3 of either conv sees the token; the state starts at 0,
    so y_r = (C_r . B_r) delta_r x_r + D_r x_r."""
    inp, par = np_case2(1, 1, H, P, N, seed)
    HP = H * P
    y = np.zeros((2, HP))
    for r in range(2):
        raw = inp["xbc"][r, 0, 0]
        u = np.array([lib_silu(par["conv_b"][r, c] + par["conv_w"][r, c, 3] * raw[c]) for c in range(HP + 2 * N)])
        xv, Bv, Cv = u[:HP], u[HP:HP + N], u[HP + N:]
        cb = float(Cv @ Bv)
        for h in range(H):
            d = lib_softplus(inp["dt"][r, 0, 0, h] + par["dt_bias"][r, h])
            for p in range(P):
                y[r, h * P + p] = cb * d * xv[h * P + p] + par["D"][r, h] * xv[h * P + p]
    want = (y[0] + y[1]) * lib_silu(inp["z"][0, 0])
    return rel(oracle.mamba2_layer_fwd(inp, par)[0, 0], want)


def _swap_dirs(inp, par):
    """Flipped sequence with the two directions exchanged."""
    f = {"xbc": inp["xbc"][::-1, :, ::-1].copy(), "z": inp["z"][:, ::-1].copy(),
         "dt": inp["dt"][::-1, :, ::-1].copy()}
    q = {k: (v[::-1].copy() if v is not None else None) for k, v in par.items()}
    return f, q


def pin_flip(seed=26, L=37, H=2, P=3, N=4):
    """The reverse direction is the forward one on the flipped sequence with
    the directions' parameters exchanged (bit-exact: same operations in the
    same order)."""
    inp, par = np_case2(2, L, H, P, N, seed)
    rev = oracle.mamba2_layer_fwd(inp, par, flags=oracle.REV_ONLY)
    f, q = _swap_dirs(inp, par)
    fwd_flipped = oracle.mamba2_layer_fwd(f, q, flags=oracle.FWD_ONLY)
    return float(np.max(np.abs(rev - fwd_flipped[:, ::-1])))


def pin_additive(seed=27, L=29, H=2, P=3, N=4):
    inp, par = np_case2(1, L, H, P, N, seed)
    both = oracle.mamba2_layer_fwd(inp, par)
    f = oracle.mamba2_layer_fwd(inp, par, flags=oracle.FWD_ONLY)
    r = oracle.mamba2_layer_fwd(inp, par, flags=oracle.REV_ONLY)
    return rel(both, f + r)


PINS = {
    "m2_reduces_to_dstate16_layer": (pin_reduces_to_dstate16_layer, 1e-12),
    "m2_dual_form": (pin_dual_form, 1e-10),
    "m2_zero_decay_running_sum": (pin_zero_decay_running_sum, 1e-12),
    "m2_zero_B": (pin_zero_B, 1e-13),
    "m2_tiny_by_hand": (pin_tiny_by_hand, 1e-13),
    "m2_flip": (pin_flip, 0.0),
    "m2_additive": (pin_additive, 1e-15),
}
