"""Pins of the neighbours' oracle (oracle/proj.py), each by another route:
brute-force loops on tiny inputs, closed forms and one-hot weights.  CPU only."""
import numpy as np
import pytest

import oracle


def _rng(seed=0):
    return np.random.default_rng(seed)


def test_adaln_brute_force():
    # Eq. (10) written out with explicit sums on a tiny input
    r = _rng(1)
    b, L, d = 2, 3, 5
    x, g, be = r.normal(size=(b, L, d)), r.normal(size=(b, d)), r.normal(size=(b, d))
    eps = 1e-3
    got = oracle.adaln(x, g, be, eps)
    for i in range(b):
        for t in range(L):
            mu = sum(x[i, t, k] for k in range(d)) / d
            var = sum((x[i, t, k] - mu) ** 2 for k in range(d)) / d
            for k in range(d):
                want = g[i, k] * (x[i, t, k] - mu) / (var + eps) ** 0.5 + be[i, k]
                assert abs(got[i, t, k] - want) <= 1e-12


def test_adaln_constant_row_gives_beta():
    r = _rng(2)
    x = np.full((1, 4, 16), 3.25)
    g, be = r.normal(size=(1, 16)), r.normal(size=(1, 16))
    assert np.array_equal(oracle.adaln(x, g, be), np.broadcast_to(be[:, None, :], x.shape))


def test_adaln_normalised_moments_and_shift_invariance():
    # with gamma 1, beta 0 the row has mean 0 and variance var / (var + eps) (biased variance, eps inside the root)
    r = _rng(3)
    x = r.normal(size=(2, 5, 64)) * 0.05
    eps = 1e-3
    out = oracle.adaln(x, np.ones((2, 64)), np.zeros((2, 64)), eps)
    var = x.var(axis=-1)
    assert np.allclose(out.mean(axis=-1), 0.0, atol=1e-12)
    assert np.allclose(out.var(axis=-1), var / (var + eps), rtol=1e-12)
    assert np.allclose(oracle.adaln(x + 7.0, np.ones((2, 64)), np.zeros((2, 64)), eps), out, atol=1e-9)


def test_in_proj_split_with_one_hot_weights():
    # row n of w_in picks input column n mod d_model: each output array must be the matching slice
    b, L, dm, D, N = 2, 3, 40, 8, 16
    a = _rng(4).normal(size=(b, L, dm))
    rows = 4 * D + 4 * N
    w = np.zeros((rows, dm))
    w[np.arange(rows), np.arange(rows) % dm] = 1.0
    got = oracle.in_proj(a, w, D, N)
    col = lambda n0, n: a[..., np.arange(n0, n0 + n) % dm]  # noqa: E731
    assert np.array_equal(got["x"], col(0, D)) and np.array_equal(got["z"], col(D, D))
    assert np.array_equal(got["dt"][0], col(2 * D, D)) and np.array_equal(got["dt"][1], col(3 * D, D))
    o = 4 * D
    assert np.array_equal(got["B"][0], col(o, N)) and np.array_equal(got["C"][0], col(o + N, N))
    assert np.array_equal(got["B"][1], col(o + 2 * N, N)) and np.array_equal(got["C"][1], col(o + 3 * N, N))


@pytest.mark.parametrize("which", ["in", "out"])
def test_projections_brute_force(which):
    r = _rng(5)
    b, L, K, D, N = 1, 2, 6, 2, 16
    if which == "in":
        a, w = r.normal(size=(b, L, K)), r.normal(size=(4 * D + 4 * N, K))
        got = oracle.in_proj(a, w, D, N)
        full = np.concatenate([got["x"], got["z"], got["dt"][0], got["dt"][1], got["B"][0], got["C"][0],
                               got["B"][1], got["C"][1]], axis=-1)
    else:
        a, w = r.normal(size=(b, L, K)), r.normal(size=(5, K))
        full = oracle.out_proj(a, w)
    for t in range(L):
        for n in range(w.shape[0]):
            assert abs(full[0, t, n] - sum(a[0, t, k] * w[n, k] for k in range(K))) <= 1e-12
