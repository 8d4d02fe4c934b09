"""Pins for the fp64 oracle: expected values from routes other than the oracle.

Each pin returns the largest discrepancy it saw, so the same functions serve
the plain pin tests (discrepancy must be ~0) and the planted-mistake test
(some pin must report a large discrepancy).  Nothing here copies the
oracle's loop: the expected values come from library routines
(``numpy.convolve``, ``numpy.logaddexp``, ``scipy.special.expit``,
``numpy.cumsum``), from the materialised L x L quadratic form of the scan,
from hand-expanded formulas for L = 1 and L = 2, or from invariants the
method has (flip symmetry of the reverse layer, additivity of the two
directions, exact block caching).
"""
from __future__ import annotations

import numpy as np
from scipy.special import expit

import oracle
from bidirectional_mamba_denoiser_b200 import workloads


def lib_silu(v):
    return v * expit(v)


def lib_softplus(v):
    return np.logaddexp(0.0, v)


def np_case(batch, L, D, N=16, seed=0, dtype="fp32"):
    inp, par = workloads.make_case(batch, L, D, N, dtype, seed)
    inp = {k: v.double().numpy() for k, v in inp.items()}
    par = {k: v.double().numpy() for k, v in par.items()}
    return inp, par


def lib_features(inp, par):
    """u and delta of both directions from library routines, [2, b, L, D]."""
    x = inp["x"]
    b, L, D = x.shape
    u = np.empty((2, b, L, D))
    dl = np.empty((2, b, L, D))
    for r in range(2):
        for bi in range(b):
            for d in range(D):
                w = par["conv_w"][r, d]
                cb = par["conv_b"][r, d] if par.get("conv_b") is not None else 0.0
                col = x[bi, :, d]
                if r == 0:
                    c = np.convolve(col, w[::-1])[:L] + cb
                else:
                    c = (np.convolve(col[::-1], w[::-1])[:L])[::-1] + cb
                u[r, bi, :, d] = lib_silu(c)
                dl[r, bi, :, d] = lib_softplus(inp["dt"][r, bi, :, d] + par["dt_bias"][r, d])
    return u, dl


def quad_form_dirs(inp, par):
    """y of both directions from the materialised L x L matrices
    M_f[t, s] = sum_n C_f[t,n] B_f[s,n] exp(A_f[n] (S[t] - S[s]))  (s <= t)
    M_b[t, s] = sum_n C_b[t,n] B_b[s,n] exp(A_b[n] (X[s] - X[t]))  (s >= t)
    with S the inclusive and X the exclusive prefix sum of delta."""
    u, dl = lib_features(inp, par)
    b, L, D = inp["x"].shape
    yf = np.empty((b, L, D))
    yb = np.empty((b, L, D))
    tri_lo = np.tril(np.ones((L, L), bool))
    tri_hi = np.triu(np.ones((L, L), bool))
    for bi in range(b):
        for d in range(D):
            for r, y, mask in ((0, yf, tri_lo), (1, yb, tri_hi)):
                A = par["A"][r, d]
                Bm = inp["B"][r, bi]
                Cm = inp["C"][r, bi]
                delta = dl[r, bi, :, d]
                S = np.cumsum(delta)
                X = S - delta
                if r == 0:
                    gap = S[:, None] - S[None, :]          # t, s
                else:
                    gap = X[None, :] - X[:, None]          # t, s
                gap = np.where(mask, gap, 0.0)
                dec = np.exp(A[None, None, :] * gap[:, :, None])   # t, s, n
                M = np.einsum("tn,sn,tsn->ts", Cm, Bm, dec) * mask
                uu = u[r, bi, :, d]
                y[bi, :, d] = M @ (delta * uu) + par["D"][r, d] * uu
    return yf, yb


def rel(a, b):
    scale = max(np.max(np.abs(b)), 1e-300)
    return float(np.max(np.abs(np.asarray(a) - np.asarray(b))) / scale)


# ---------------------------------------------------------------- the pins

def pin_conv_and_delta(seed=3):
    inp, par = np_case(2, 37, 5, seed=seed)
    u, dl = oracle.features(inp, par)
    lu, ldl = lib_features(inp, par)
    return max(rel(u, lu), rel(dl, ldl))


def pin_prefix_sum(seed=4):
    """A = 0, C = 1: y_f[t] = cumsum(delta*u*sum_n B)[t] + D u[t] (and the
    reverse cumulative sum for the reverse direction)."""
    inp, par = np_case(2, 50, 4, seed=seed)
    par["A"][:] = 0.0
    inp["C"][:] = 1.0
    out, yf, yb = oracle.layer_fwd(inp, par, return_dirs=True)
    u, dl = lib_features(inp, par)
    sB = inp["B"].sum(-1)                     # [2, b, L]
    drive0 = dl[0] * u[0] * sB[0][..., None]
    drive1 = dl[1] * u[1] * sB[1][..., None]
    ef = np.cumsum(drive0, axis=1) + par["D"][0] * u[0]
    eb = np.cumsum(drive1[:, ::-1], axis=1)[:, ::-1] + par["D"][1] * u[1]
    eo = (ef + eb) * lib_silu(inp["z"])
    return max(rel(yf, ef), rel(yb, eb), rel(out, eo))


def pin_memoryless(seed=5):
    """A -> -inf: exp(delta*A) = 0, so h_t = delta_t B_t u_t and
    y_t = (C_t . B_t) delta_t u_t + D u_t."""
    inp, par = np_case(1, 29, 6, seed=seed)
    par["A"][:] = -1e300
    out, yf, yb = oracle.layer_fwd(inp, par, return_dirs=True)
    u, dl = lib_features(inp, par)
    cb = np.einsum("rbln,rbln->rbl", inp["C"], inp["B"])[..., None]
    e = cb * dl * u + par["D"][:, None, None, :] * u
    return max(rel(yf, e[0]), rel(yb, e[1]))


def pin_zero_B(seed=6):
    """B = 0: the state never leaves zero and y = D u."""
    inp, par = np_case(1, 33, 6, seed=seed)
    inp["B"][:] = 0.0
    par["D"][:] = np.linspace(0.5, 2.0, par["D"].size).reshape(par["D"].shape)
    out, yf, yb = oracle.layer_fwd(inp, par, return_dirs=True)
    u, _ = lib_features(inp, par)
    return max(rel(yf, par["D"][0] * u[0]), rel(yb, par["D"][1] * u[1]))


def pin_quadratic_form(seed=7, L=48, D=3, random_A=False):
    inp, par = np_case(2, L, D, seed=seed)
    if random_A:
        rng = np.random.default_rng(seed)
        par["A"] = -np.exp(rng.uniform(-3, 2.5, par["A"].shape))
        par["D"] = rng.uniform(-1, 1, par["D"].shape)
    out, yf, yb = oracle.layer_fwd(inp, par, return_dirs=True)
    ef, eb = quad_form_dirs(inp, par)
    eo = (ef + eb) * lib_silu(inp["z"])
    return max(rel(yf, ef), rel(yb, eb), rel(out, eo))


def pin_tiny_by_hand(seed=8):
    """L = 1 and L = 2, expanded by hand."""
    worst = 0.0
    for L in (1, 2):
        inp, par = np_case(1, L, 2, N=3, seed=seed + L)
        out, yf, yb = oracle.layer_fwd(inp, par, return_dirs=True)
        for d in range(2):
            x = inp["x"][0, :, d]
            wf, wb = par["conv_w"][0, d], par["conv_w"][1, d]
            cf, cb = par["conv_b"][0, d], par["conv_b"][1, d]
            Af, Ab = par["A"][0, d], par["A"][1, d]
            Bf, Cf, Bb, Cb = inp["B"][0, 0], inp["C"][0, 0], inp["B"][1, 0], inp["C"][1, 0]
            df = lib_softplus(inp["dt"][0, 0, :, d] + par["dt_bias"][0, d])
            db = lib_softplus(inp["dt"][1, 0, :, d] + par["dt_bias"][1, d])
            Df, Db = par["D"][0, d], par["D"][1, d]
            if L == 1:
                uf = [lib_silu(cf + wf[3] * x[0])]
                ub = [lib_silu(cb + wb[3] * x[0])]
                hf0 = df[0] * Bf[0] * uf[0]
                hb0 = db[0] * Bb[0] * ub[0]
                eyf = [Cf[0] @ hf0 + Df * uf[0]]
                eyb = [Cb[0] @ hb0 + Db * ub[0]]
            else:
                uf = [lib_silu(cf + wf[3] * x[0]), lib_silu(cf + wf[2] * x[0] + wf[3] * x[1])]
                ub = [lib_silu(cb + wb[3] * x[0] + wb[2] * x[1]), lib_silu(cb + wb[3] * x[1])]
                hf0 = df[0] * Bf[0] * uf[0]
                hf1 = np.exp(df[1] * Af) * hf0 + df[1] * Bf[1] * uf[1]
                hb1 = db[1] * Bb[1] * ub[1]
                hb0 = np.exp(db[0] * Ab) * hb1 + db[0] * Bb[0] * ub[0]
                eyf = [Cf[0] @ hf0 + Df * uf[0], Cf[1] @ hf1 + Df * uf[1]]
                eyb = [Cb[0] @ hb0 + Db * ub[0], Cb[1] @ hb1 + Db * ub[1]]
            eo = (np.array(eyf) + np.array(eyb)) * lib_silu(inp["z"][0, :, d])
            worst = max(worst, rel(yf[0, :, d], eyf), rel(yb[0, :, d], eyb), rel(out[0, :, d], eo))
    return worst


def _swap_dirs(inp, par):
    """Inputs for which the forward layer sees what the reverse layer saw,
    on the flipped sequence."""
    fi = {"x": inp["x"][:, ::-1].copy(), "z": inp["z"][:, ::-1].copy(),
          "dt": inp["dt"][::-1, :, ::-1].copy(), "B": inp["B"][::-1, :, ::-1].copy(),
          "C": inp["C"][::-1, :, ::-1].copy()}
    fp = {k: (v[::-1].copy() if v is not None else None) for k, v in par.items()}
    return fi, fp


def pin_flip(seed=9):
    """Eq. (4)/(5): the reverse layer is the forward recurrence in reversed
    index order.  Feeding the flipped sequence with the two directions'
    parameters and inputs exchanged must give the flipped outputs with the
    directions exchanged -- exactly, since the arithmetic is the same."""
    inp, par = np_case(2, 41, 4, seed=seed)
    out, yf, yb = oracle.layer_fwd(inp, par, return_dirs=True)
    fi, fp = _swap_dirs(inp, par)
    out2, yf2, yb2 = oracle.layer_fwd(fi, fp, return_dirs=True)
    return max(float(np.max(np.abs(yf2 - yb[:, ::-1]))), float(np.max(np.abs(yb2 - yf[:, ::-1]))),
               float(np.max(np.abs(out2 - out[:, ::-1]))))


def pin_additive(seed=10):
    """Eq. (6): the directions are added, and the gate is linear in their sum."""
    inp, par = np_case(1, 30, 5, seed=seed)
    out = oracle.layer_fwd(inp, par)
    of = oracle.layer_fwd(inp, par, flags=oracle.FWD_ONLY)
    ob = oracle.layer_fwd(inp, par, flags=oracle.REV_ONLY)
    return rel(of + ob, out)


def _block_cache(seed, P, G, D):
    """§4.3 / follow-up abstract: with the reverse scan kept inside the
    block, the forward part of a block step from the cached prefix state is
    exactly the full-sequence forward over prefix+block, restricted to the
    block; the reverse part is the layer run on the block alone."""
    inp, par = np_case(2, P + G, D, seed=seed)
    _, yf_full, _ = oracle.layer_fwd(inp, par, return_dirs=True)
    pre = {k: (v[:, :, :P] if k in ("dt", "B", "C") else v[:, :P]) for k, v in inp.items()}
    blk = {k: (v[:, :, P:] if k in ("dt", "B", "C") else v[:, P:]) for k, v in inp.items()}
    blk = {k: np.ascontiguousarray(v) for k, v in blk.items()}
    pre = {k: np.ascontiguousarray(v) for k, v in pre.items()}
    h, tail = oracle.prefix_state(pre, par)
    out, yfb, ybb = oracle.block_step(h, tail, blk, par, return_dirs=True)
    _, _, yb_alone = oracle.layer_fwd(blk, par, return_dirs=True)
    e_out = (yf_full[:, P:] + yb_alone) * lib_silu(blk["z"])
    exact = max(float(np.max(np.abs(yfb - yf_full[:, P:]))), float(np.max(np.abs(ybb - yb_alone))))
    return exact, rel(out, e_out)


def pin_block_cache(seed=12, P=45, G=13, D=4):
    """Exact parts of the block-cache identity (bit-for-bit in fp64)."""
    return _block_cache(seed, P, G, D)[0]


def pin_block_cache_gated(seed=12, P=45, G=13, D=4):
    """The gated block output against the two identities' y."""
    return _block_cache(seed, P, G, D)[1]


def pin_block_chain(seed=13, L=96, G=32, D=3):
    """Blocks decoded one after another, committing the state after each,
    reproduce the full forward scan block by block; each block's reverse
    part is the layer on that block alone."""
    inp, par = np_case(1, L, D, seed=seed)
    _, yf_full, _ = oracle.layer_fwd(inp, par, return_dirs=True)
    h = np.zeros((1, D, inp["B"].shape[-1]))
    tail = np.zeros((1, 3, D))
    worst = 0.0
    for s in range(0, L, G):
        blk = {k: np.ascontiguousarray(v[:, :, s:s + G] if k in ("dt", "B", "C") else v[:, s:s + G])
               for k, v in inp.items()}
        out, h, tail, yfb, ybb = oracle.block_step(h, tail, blk, par, commit=True, return_dirs=True)
        _, _, yb_alone = oracle.layer_fwd(blk, par, return_dirs=True)
        worst = max(worst, float(np.max(np.abs(yfb - yf_full[:, s:s + G]))),
                    float(np.max(np.abs(ybb - yb_alone))))
    return worst


PINS = {
    "conv_and_delta": (pin_conv_and_delta, 1e-12),
    "prefix_sum": (pin_prefix_sum, 1e-12),
    "memoryless": (pin_memoryless, 1e-12),
    "zero_B": (pin_zero_B, 1e-13),
    "quadratic_form": (pin_quadratic_form, 1e-10),
    "quadratic_form_random_A": (lambda: pin_quadratic_form(seed=17, random_A=True), 1e-10),
    "tiny_by_hand": (pin_tiny_by_hand, 1e-13),
    "flip": (pin_flip, 0.0),
    "additive": (pin_additive, 1e-15),
    "block_cache": (pin_block_cache, 0.0),
    "block_cache_gated": (pin_block_cache_gated, 1e-14),
    "block_chain": (pin_block_chain, 0.0),
}
