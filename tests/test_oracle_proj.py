"""Pins of the oracle's projection front-end and output projection (the
steps on either side of the layer): a brute-force loop, one-hot weight rows
that route a chosen hidden coordinate into each field (so a shifted or
swapped field boundary fails), and the identity output projection."""

import numpy as np
import pytest

import oracle


def _brute(x, W):
    T, K = x.shape
    N = W.shape[0]
    y = np.zeros((T, N))
    for t in range(T):
        for n in range(N):
            s = 0.0
            for k in range(K):
                s += x[t, k] * W[n, k]
            y[t, n] = s
    return y


@pytest.mark.parametrize("P", [None, 4, 1])
def test_project_in_equals_brute_force(P):
    rng = np.random.default_rng(5)
    Hq, Hkv, d, HI, dI, Hm, T = 4, 2, 3, 4, 2, 7, 3
    N = sum(oracle.proj_widths(Hq, Hkv, d, HI, dI, P))
    x = rng.standard_normal((T, Hm))
    W = rng.standard_normal((N, Hm))
    got = oracle.project_in(x, W, Hq, Hkv, d, HI, dI, P)
    z = _brute(x, W)
    flat = np.concatenate([got[f].reshape(T, -1) for f in oracle.PROJ_FIELDS], axis=1)
    np.testing.assert_allclose(flat, z, rtol=1e-12, atol=1e-12)
    assert got["q"].shape == (T, Hq, d) and got["k"].shape == (T, Hkv, d)
    assert got["kidx"].shape == (T, Hkv if P is None else P, dI)
    assert got["w"].shape == (T, HI) and got["lam"].shape == (T, Hq)


# the column order the library states for the front-end (lisa.h, lisa_project_in)
DOCUMENTED_ORDER = [("q", lambda Hq, Hkv, d, HI, dI: Hq * d), ("k", lambda Hq, Hkv, d, HI, dI: Hkv * d),
                    ("v", lambda Hq, Hkv, d, HI, dI: Hkv * d), ("qidx", lambda Hq, Hkv, d, HI, dI: HI * dI),
                    ("kidx", lambda Hq, Hkv, d, HI, dI: Hkv * dI), ("w", lambda Hq, Hkv, d, HI, dI: HI),
                    ("lam", lambda Hq, Hkv, d, HI, dI: Hq)]


def test_project_in_field_order():
    """Rows of W_in copy hidden coordinate i into the i-th field of the
    documented order: every entry of that field must equal x[i] (a boundary
    shifted by one column or two fields swapped changes some entry)."""
    Hq, Hkv, d, HI, dI = 2, 1, 4, 2, 3
    widths = [fn(Hq, Hkv, d, HI, dI) for _, fn in DOCUMENTED_ORDER]
    Hm = len(widths)
    W = np.zeros((sum(widths), Hm))
    c = 0
    for i, wd in enumerate(widths):
        W[c:c + wd, i] = 1.0
        c += wd
    x = np.arange(1.0, Hm + 1.0)[None, :] * 10.0
    got = oracle.project_in(x, W, Hq, Hkv, d, HI, dI)
    for i, (name, _) in enumerate(DOCUMENTED_ORDER):
        assert np.all(got[name] == x[0, i]), name


def test_project_out_identity_and_brute_force():
    rng = np.random.default_rng(6)
    Hq, d, T = 3, 4, 2
    o = rng.standard_normal((T, Hq, d))
    np.testing.assert_array_equal(oracle.project_out(o, np.eye(Hq * d)), o.reshape(T, Hq * d))
    W = rng.standard_normal((5, Hq * d))
    np.testing.assert_allclose(oracle.project_out(o, W), _brute(o.reshape(T, -1), W), rtol=1e-12, atol=1e-12)
