"""Pins of the oracle's definition variants (the other readings of the head
mapping the pages leave open: one indexer key per indexer head, one top-M
set shared by all KV heads, linear-branch keys / values per query head).

Each variant is pinned by reducing it to the default definition (pinned in
test_oracle.py against closed forms, library routines and brute force) on
sub-problems built so that a wrong plane, group or head index changes the
result: scores of one indexer head against its own key plane, a problem with a
single KV head, a problem with a single query head.  No GPU is needed.
"""

import numpy as np
import pytest

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- scores
@pytest.mark.parametrize("Hkv,R", [(2, 2), (1, 4), (4, 1), (2, 3)])
def test_key_per_head_scores_are_sums_of_one_head_scores(Hkv, R):
    """With one key plane per indexer head, a group's score is the sum over
    its heads of the one-head score of head j against plane j alone."""
    rng = _rng(11 + Hkv * 7 + R)
    HI, dI, n = Hkv * R, 5, 13
    q = rng.standard_normal((HI, dI))
    w = rng.standard_normal(HI)
    planes = rng.standard_normal((HI, n, dI))
    got = oracle.indexer_scores(q, w, planes, groups=Hkv)
    assert got.shape == (Hkv, n)
    for gs in range(Hkv):
        want = np.zeros(n)
        for r in range(R):
            j = gs * R + r
            want += oracle.indexer_scores(q[j:j + 1], w[j:j + 1], planes[j:j + 1])[0]
        np.testing.assert_allclose(got[gs], want, rtol=1e-13, atol=1e-13)


def test_key_per_head_with_replicated_planes_is_default():
    """Planes that repeat the KV head's key for each of its heads give the
    default scores exactly."""
    rng = _rng(3)
    Hkv, R, dI, n = 2, 3, 4, 9
    q = rng.standard_normal((Hkv * R, dI))
    w = rng.random(Hkv * R)
    kv_planes = rng.standard_normal((Hkv, n, dI))
    per_head = np.repeat(kv_planes, R, axis=0)
    np.testing.assert_array_equal(oracle.indexer_scores(q, w, per_head, groups=Hkv),
                                  oracle.indexer_scores(q, w, kv_planes))


def test_shared_scores_are_sum_over_kv_groups():
    """A shared selection scores every key with all HI heads: with one key
    plane, that is the sum of the default per-KV-head scores over a cache that
    repeats the plane for every KV head."""
    rng = _rng(4)
    Hkv, R, dI, n = 3, 2, 4, 10
    q = rng.standard_normal((Hkv * R, dI))
    w = rng.random(Hkv * R)
    plane = rng.standard_normal((1, n, dI))
    got = oracle.indexer_scores(q, w, plane, groups=1)
    want = oracle.indexer_scores(q, w, np.repeat(plane, Hkv, axis=0)).sum(axis=0)
    np.testing.assert_allclose(got[0], want, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- decode
def _decode_problem(B=2, Hq=6, Hkv=2, d=8, HI=4, dI=4, t=30, P=None, seed=0):
    rng = _rng(seed)
    f = lambda *s: rng.standard_normal(s)
    P = Hkv if P is None else P
    return dict(q=f(B, Hq, d), k=f(B, Hkv, d), v=f(B, Hkv, d), qidx=f(B, HI, dI), kidx=f(B, P, dI),
                w=rng.random((B, HI)), lam=f(B, Hq), k_cache=f(B, Hkv, t, d), v_cache=f(B, Hkv, t, d),
                kidx_cache=f(B, P, t, dI), S=f(B, Hq, d, d), pos=np.array([t, t - 11][:B]))


def _run(pr, M, **kw):
    return oracle.decode_step(pr["q"], pr["k"], pr["v"], pr["qidx"], pr["kidx"], pr["w"], pr["lam"],
                              pr["k_cache"], pr["v_cache"], pr["kidx_cache"], pr["S"], pr["pos"], M, **kw)


def test_shared_set_decode_is_one_kv_head_problem_per_group():
    """With a shared selection, the query heads of KV head g get exactly what
    a default layer with one KV head (g's K/V, all HI indexer heads, the
    shared key plane) gives them; every KV head uses the same set."""
    pr = _decode_problem(P=1, seed=5)
    M = 7
    res = _run(pr, M, shared_set=True)
    Hq, Hkv = pr["q"].shape[1], pr["k"].shape[1]
    G = Hq // Hkv
    assert res["idx"].shape == (2, 1, M)
    for g in range(Hkv):
        hs = slice(g * G, (g + 1) * G)
        sub = _run(dict(q=pr["q"][:, hs], k=pr["k"][:, g:g + 1], v=pr["v"][:, g:g + 1], qidx=pr["qidx"],
                        kidx=pr["kidx"], w=pr["w"], lam=pr["lam"][:, hs], k_cache=pr["k_cache"][:, g:g + 1],
                        v_cache=pr["v_cache"][:, g:g + 1], kidx_cache=pr["kidx_cache"], S=pr["S"][:, hs],
                        pos=pr["pos"]), M)
        np.testing.assert_array_equal(sub["idx"][:, 0], res["idx"][:, 0])
        np.testing.assert_allclose(res["out"][:, hs], sub["out"], rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(res["S"][:, hs], sub["S"], rtol=1e-13, atol=1e-13)


def test_key_per_head_decode_is_sum_of_one_head_scores():
    """Decode with one key plane per indexer head: the scores of KV head g are
    the one-head scores of heads gR .. gR+R-1 summed (each against its own
    plane, new token included); the selection is the top-M of those."""
    pr = _decode_problem(P=4, seed=6)
    M = 9
    res = _run(pr, M)
    Hkv, R = 2, 2
    for b in range(2):
        t = int(pr["pos"][b])
        planes = np.concatenate([pr["kidx_cache"][b, :, :t], pr["kidx"][b][:, None]], axis=1)
        for g in range(Hkv):
            want = np.zeros(t + 1)
            for r in range(R):
                j = g * R + r
                want += oracle.indexer_scores(pr["qidx"][b, j:j + 1], pr["w"][b, j:j + 1], planes[j:j + 1])[0]
            np.testing.assert_allclose(res["scores"][b][g], want, rtol=1e-13, atol=1e-13)
            np.testing.assert_array_equal(res["idx"][b, g], oracle.topm_select(want, M))


def test_key_per_head_shared_set_decode():
    """Both variants together: one set, scored with every indexer head
    against its own plane."""
    pr = _decode_problem(P=4, seed=7)
    M = 6
    res = _run(pr, M, shared_set=True)
    for b in range(2):
        t = int(pr["pos"][b])
        planes = np.concatenate([pr["kidx_cache"][b, :, :t], pr["kidx"][b][:, None]], axis=1)
        want = sum(oracle.indexer_scores(pr["qidx"][b, j:j + 1], pr["w"][b, j:j + 1], planes[j:j + 1])[0]
                   for j in range(4))
        np.testing.assert_allclose(res["scores"][b][0], want, rtol=1e-13, atol=1e-13)
        np.testing.assert_array_equal(res["idx"][b, 0], oracle.topm_select(want, M))


def test_linear_kv_per_head_is_one_head_problem():
    """Linear keys / values per query head: the sparse branch is unchanged,
    and head h's state and linear readout are those of a default layer with
    one query head whose k, v are k_lin[h], v_lin[h]."""
    pr = _decode_problem(seed=8)
    M = 8
    rng = _rng(9)
    B, Hq, d = pr["q"].shape
    k_lin, v_lin = rng.standard_normal((B, Hq, d)), rng.standard_normal((B, Hq, d))
    res = _run(pr, M, k_lin=k_lin, v_lin=v_lin)
    base = _run(pr, M)
    np.testing.assert_allclose(res["o_sp"], base["o_sp"], rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(res["idx"], base["idx"])
    for h in range(Hq):
        sub = _run(dict(q=pr["q"][:, h:h + 1], k=k_lin[:, h:h + 1], v=v_lin[:, h:h + 1], qidx=pr["qidx"][:, :2],
                        kidx=pr["kidx"][:, :1], w=pr["w"][:, :2], lam=pr["lam"][:, h:h + 1],
                        k_cache=pr["k_cache"][:, :1], v_cache=pr["v_cache"][:, :1],
                        kidx_cache=pr["kidx_cache"][:, :1], S=pr["S"][:, h:h + 1], pos=pr["pos"]), M)
        np.testing.assert_allclose(res["S"][:, h], sub["S"][:, 0], rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(res["o_lin"][:, h], sub["o_lin"][:, 0], rtol=1e-13, atol=1e-13)


def test_linear_kv_equal_to_group_kv_is_default():
    pr = _decode_problem(seed=10)
    G = 3
    res = _run(pr, 8, k_lin=np.repeat(pr["k"], G, axis=1), v_lin=np.repeat(pr["v"], G, axis=1))
    base = _run(pr, 8)
    np.testing.assert_array_equal(res["out"], base["out"])
    np.testing.assert_array_equal(res["S"], base["S"])


# ---------------------------------------------------------------- prefill
@pytest.mark.parametrize("P,shared,lin", [(4, False, False), (1, True, False), (4, True, False),
                                          (2, False, True)])
def test_prefill_variant_rows_match_decode(P, shared, lin):
    """Row t of a variant prefill equals the same variant's decode step at
    position t over the first t tokens."""
    rng = _rng(12 + P)
    B, T, Hq, Hkv, d, HI, dI, M = 2, 33, 4, 2, 8, 4, 4, 6
    f = lambda *s: rng.standard_normal(s)
    q, k, v = f(B, T, Hq, d), f(B, T, Hkv, d), f(B, T, Hkv, d)
    qi, ki = f(B, T, HI, dI), f(B, T, P, dI)
    w, lam, S0 = rng.random((B, T, HI)), f(B, T, Hq), f(B, Hq, d, d)
    kl, vl = (f(B, T, Hq, d), f(B, T, Hq, d)) if lin else (None, None)
    full = oracle.prefill(q, k, v, qi, ki, w, lam, S0, M, shared_set=shared, k_lin=kl, v_lin=vl)
    t = T - 1
    head = oracle.prefill(q[:, :t], k[:, :t], v[:, :t], qi[:, :t], ki[:, :t], w[:, :t], lam[:, :t], S0, M,
                          rows=[], shared_set=shared, k_lin=None if kl is None else kl[:, :t],
                          v_lin=None if vl is None else vl[:, :t])
    tr = lambda x: np.transpose(x, (0, 2, 1, 3))
    dec = oracle.decode_step(q[:, t], k[:, t], v[:, t], qi[:, t], ki[:, t], w[:, t], lam[:, t], tr(k[:, :t]),
                             tr(v[:, :t]), tr(ki[:, :t]), head["S"], np.full(B, t), M, shared_set=shared,
                             k_lin=None if kl is None else kl[:, t], v_lin=None if vl is None else vl[:, t])
    np.testing.assert_allclose(dec["out"], full["out"][:, t], rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(dec["idx"], full["idx"][:, t])
    np.testing.assert_allclose(dec["S"], full["S"], rtol=1e-12, atol=1e-12)
    assert full["idx"].shape[2] == (1 if shared else Hkv)
