"""Pins of the fp64 oracle against what the pages and mathematics fix.

Each test checks the oracle against something other than itself: hand-worked
examples (tests/golden), closed forms, a library routine for a special case
(torch scaled-dot-product attention for full causal attention), or brute force
on tiny inputs.  No GPU is needed.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from lisa_inputs import get_config, make_rng, gen_layer, gen_step


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- indexer
def test_indexer_golden(golden_dir):
    g = _load(golden_dir, "indexer_tiny.json")
    got = oracle.indexer_scores(np.array(g["qidx"], float), np.array(g["w"], float),
                                np.array(g["kidx"], float))
    np.testing.assert_array_equal(got, np.array(g["expected"]))


def test_indexer_brute_force_sum():
    """Each score is a sum over (r, c) of w * relu(sum_c q k): check against
    an elementwise triple loop in plain Python on a random tiny case."""
    rng = np.random.default_rng(5)
    Hkv, R, dI, n = 2, 3, 4, 7
    q = rng.standard_normal((Hkv * R, dI))
    w = rng.standard_normal(Hkv * R)          # negative weights allowed
    kk = rng.standard_normal((Hkv, n, dI))
    got = oracle.indexer_scores(q, w, kk)
    for g in range(Hkv):
        for s in range(n):
            acc = 0.0
            for r in range(R):
                dot = 0.0
                for c in range(dI):
                    dot += q[g * R + r, c] * kk[g, s, c]
                acc += w[g * R + r] * (dot if dot > 0 else 0.0)
            assert got[g, s] == pytest.approx(acc, rel=1e-12, abs=1e-14)


# ---------------------------------------------------------------- top-M
def test_topm_golden(golden_dir):
    g = _load(golden_dir, "topm_tiny.json")
    for case in g["cases"]:
        got = oracle.topm_select(np.array(case["scores"], dtype=np.float64), case["M"])
        assert got.tolist() == case["expected"], case["why"]


def _rank_bruteforce(scores):
    n = len(scores)
    return [sum(1 for s2 in range(n) if scores[s2] > scores[s] or (scores[s2] == scores[s] and s2 < s))
            for s in range(n)]


@pytest.mark.parametrize("seed", range(30))
def test_topm_equals_rank_counting(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 40))
    M = int(rng.integers(1, 20))
    # few distinct values -> many exact ties
    scores = rng.integers(-3, 4, size=n).astype(np.float64) * 0.5
    got = oracle.topm_select(scores, M)
    rank = _rank_bruteforce(scores.tolist())
    expect = sorted(s for s in range(n) if rank[s] < M)
    assert got[: len(expect)].tolist() == expect
    assert np.all(got[len(expect):] == -1)
    assert len(expect) == min(M, n)
    assert len(set(expect)) == len(expect)


def test_topm_threshold_and_borderline():
    s = np.array([1.0, 1.00001, 0.5, 2.0])
    assert oracle.topm_threshold(s, 2) == 1.00001
    bl = oracle.borderline_mask(s, 2)
    assert bl.tolist() == [True, True, False, False]
    # prefix <= M: nothing is borderline
    assert not oracle.borderline_mask(s, 4).any()
    # floor when the M-th score is 0: tolerance 1e-4 * 1e-3 * max|I|
    z = np.array([0.0, 0.0, 5.0, 4e-7, 6e-7])
    assert oracle.topm_threshold(z, 4) == 0.0
    assert oracle.borderline_mask(z, 4).tolist() == [True, True, False, True, False]


# ---------------------------------------------------------------- sparse
def test_sparse_golden(golden_dir):
    g = _load(golden_dir, "layer_tiny.json")["sparse"]
    got = oracle.sparse_attention(np.array(g["q"]), np.array(g["K"], float), np.array(g["V"], float))
    np.testing.assert_allclose(got, g["expected"], rtol=1e-12)


def test_sparse_permutation_invariant():
    rng = np.random.default_rng(1)
    q = rng.standard_normal(16)
    K = rng.standard_normal((9, 16))
    V = rng.standard_normal((9, 16))
    p = rng.permutation(9)
    np.testing.assert_allclose(oracle.sparse_attention(q, K, V), oracle.sparse_attention(q, K[p], V[p]),
                               rtol=1e-12, atol=1e-14)


def _small_problem(B=2, T=24, Hq=4, Hkv=2, d=8, HI=4, dI=4, seed=0, S0_normal=True):
    rng = np.random.default_rng(seed)
    f = lambda *s: rng.standard_normal(s)
    q, k, v = f(B, T, Hq, d), f(B, T, Hkv, d), f(B, T, Hkv, d)
    qi, ki = f(B, T, HI, dI), f(B, T, Hkv, dI)
    w = rng.random((B, T, HI))
    lam = f(B, T, Hq)
    S0 = f(B, Hq, d, d) if S0_normal else np.zeros((B, Hq, d, d))
    return q, k, v, qi, ki, w, lam, S0


def test_prefill_full_selection_is_causal_attention():
    """M >= T keeps every prefix token, so with the gate pinned to the sparse
    branch the layer is plain causal GQA softmax attention: compare with
    torch's scaled_dot_product_attention in float64 (a library routine)."""
    q, k, v, qi, ki, w, lam, S0 = _small_problem()
    B, T, Hq, d = q.shape
    lam = np.full_like(lam, 1e4)
    res = oracle.prefill(q, k, v, qi, ki, w, lam, S0, M=T + 3)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).transpose(1, 2), torch.from_numpy(k).transpose(1, 2),
        torch.from_numpy(v).transpose(1, 2), is_causal=True, enable_gqa=True,
    ).transpose(1, 2).numpy()
    np.testing.assert_allclose(res["out"], ref, rtol=1e-10, atol=1e-12)


def test_decode_full_selection_is_causal_attention():
    q, k, v, qi, ki, w, lam, S0 = _small_problem(T=13)
    B, T, Hq, d = q.shape
    t = T - 1
    res = oracle.decode_step(
        q[:, t], k[:, t], v[:, t], qi[:, t], ki[:, t], w[:, t], np.full((B, Hq), 1e4),
        np.transpose(k, (0, 2, 1, 3)), np.transpose(v, (0, 2, 1, 3)), np.transpose(ki, (0, 2, 1, 3)),
        S0, np.full(B, t), M=64)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).transpose(1, 2), torch.from_numpy(k).transpose(1, 2),
        torch.from_numpy(v).transpose(1, 2), is_causal=True, enable_gqa=True,
    ).transpose(1, 2).numpy()[:, t]
    np.testing.assert_allclose(res["out"], ref, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- linear
def test_linear_golden(golden_dir):
    g = _load(golden_dir, "layer_tiny.json")["linear"]
    S1 = oracle.linear_update(np.array(g["S0"], float), np.array(g["k"], float), np.array(g["v"], float))
    np.testing.assert_array_equal(S1, np.array(g["expected_S"], float))
    np.testing.assert_array_equal(oracle.linear_readout(np.array(g["q"], float), S1), g["expected_o"])


def test_linear_recurrence_equals_masked_quadratic_form():
    """o_lin(t) = q_t S_0 + sum_{s<=t} (q_t . k_s) v_s, i.e. Q S_0 + tril(Q K^T) V."""
    q, k, v, qi, ki, w, lam, S0 = _small_problem(T=31, seed=3)
    B, T, Hq, d = q.shape
    G = Hq // k.shape[2]
    lam = np.full_like(lam, -1e4)               # gate pinned to the linear branch
    res = oracle.prefill(q, k, v, qi, ki, w, lam, S0, M=4)
    for b in range(B):
        for h in range(Hq):
            Q, K, V = q[b, :, h], k[b, :, h // G], v[b, :, h // G]
            quad = Q @ S0[b, h] + np.tril(Q @ K.T) @ V
            np.testing.assert_allclose(res["out"][b, :, h], quad, rtol=1e-10, atol=1e-10)
            np.testing.assert_allclose(res["S"][b, h], S0[b, h] + K.T @ V, rtol=1e-10, atol=1e-10)


# ---------------------------------------------------------------- gate
def test_gate_golden(golden_dir):
    g = _load(golden_dir, "layer_tiny.json")["gate"]
    got = oracle.gate_fuse(g["lam"], np.array(g["o_sp"], float), np.array(g["o_lin"], float))
    np.testing.assert_allclose(got, g["expected"], rtol=1e-12)


def test_gate_isolates_branches():
    rng = np.random.default_rng(2)
    a, b = rng.standard_normal(8), rng.standard_normal(8)
    assert np.array_equal(oracle.gate_fuse(1e4, a, b), a)
    assert np.array_equal(oracle.gate_fuse(-1e4, a, b), b)
    np.testing.assert_allclose(oracle.gate_fuse(0.0, a, b), 0.5 * (a + b), rtol=1e-15)


# ---------------------------------------------------------------- whole layer
def test_first_token_closed_form():
    """t = 0: Sel = {0}, o_sp = v_0, o_lin = q_0 (S_0 + k_0^T v_0)."""
    q, k, v, qi, ki, w, lam, S0 = _small_problem(T=1, seed=4)
    B, T, Hq, d = q.shape
    G = Hq // k.shape[2]
    res = oracle.prefill(q, k, v, qi, ki, w, lam, S0, M=4)
    for b in range(B):
        assert res["idx"][b, 0, :, 0].tolist() == [0] * k.shape[2]
        assert np.all(res["idx"][b, 0, :, 1:] == -1)
        for h in range(Hq):
            g = h // G
            o_sp = v[b, 0, g]
            o_lin = q[b, 0, h] @ (S0[b, h] + np.outer(k[b, 0, g], v[b, 0, g]))
            gam = 1 / (1 + math.exp(-lam[b, 0, h]))
            np.testing.assert_allclose(res["out"][b, 0, h], gam * o_sp + (1 - gam) * o_lin, rtol=1e-12, atol=1e-13)


def test_decode_matches_prefill_row():
    """A decode step at position t reproduces row t of a prefill on the same tokens."""
    q, k, v, qi, ki, w, lam, S0 = _small_problem(T=40, seed=6)
    B, T = q.shape[:2]
    M = 8
    full = oracle.prefill(q, k, v, qi, ki, w, lam, S0, M=M)
    t = T - 1
    head = oracle.prefill(q[:, :t], k[:, :t], v[:, :t], qi[:, :t], ki[:, :t], w[:, :t], lam[:, :t], S0, M=M,
                          rows=[])
    tr = lambda x: np.transpose(x, (0, 2, 1, 3))
    dec = oracle.decode_step(q[:, t], k[:, t], v[:, t], qi[:, t], ki[:, t], w[:, t], lam[:, t],
                             tr(k[:, :t]), tr(v[:, :t]), tr(ki[:, :t]), head["S"], np.full(B, t), M)
    np.testing.assert_allclose(dec["out"], full["out"][:, t], rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(dec["idx"], full["idx"][:, t])
    np.testing.assert_allclose(dec["S"], full["S"], rtol=1e-12, atol=1e-12)


def test_selection_is_top_of_scores():
    """Every selected token scores >= every unselected one (sets, not just counts)."""
    q, k, v, qi, ki, w, lam, S0 = _small_problem(T=60, seed=7)
    res = oracle.prefill(q, k, v, qi, ki, w, lam, S0, M=10, rows=[5, 20, 59])
    for (b, t), sc in res["scores"].items():
        for g in range(sc.shape[0]):
            sel = res["idx"][b, t, g]
            sel = sel[sel >= 0]
            assert len(sel) == min(10, t + 1)
            rest = np.setdiff1d(np.arange(t + 1), sel)
            if len(rest):
                assert sc[g, sel].min() >= sc[g, rest].max()


# ---------------------------------------------------------------- inputs
def test_bf16_rounding_matches_torch():
    from lisa_inputs import f32_to_bf16_bits
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * (10.0 ** rng.integers(-8, 8, 100000)),
                        np.array([0.0, -0.0, 1.0, 65504.0, 1e-40, 3.3895313892515355e38], np.float32)])
    x = x.astype(np.float32)
    mine = f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(mine, ref)


def test_generators_deterministic():
    cfg = get_config(1)
    a = gen_step(cfg, make_rng(cfg.seed, 0))
    b = gen_step(cfg, make_rng(cfg.seed, 0))
    np.testing.assert_array_equal(a.q, b.q)
    c = gen_step(cfg, make_rng(cfg.seed, 1))
    assert not np.array_equal(a.q, c.q)


@pytest.mark.parametrize("t,W", [(0, 32), (5, 32), (31, 32), (32, 32), (100, 32), (1000, 256)])
def test_window_is_top_of_position_ordered_scores(t, W):
    """The sliding window is the top-W of scores that grow with the position,
    through the full sort of the top-M selection (an independent route)."""
    scores = np.linspace(0.1, 1.0, t + 1)
    np.testing.assert_array_equal(oracle.window_select(t, W), oracle.topm_select(scores, W))
    w = oracle.window_select(t, W)
    valid = w[w >= 0]
    assert valid.size == min(W, t + 1) and valid[-1] == t and np.all(np.diff(valid) == 1)


def test_window_decode_with_full_window_is_causal_attention():
    """With W >= t + 1 the window variant attends to the whole prefix: the
    sparse branch equals full causal softmax attention (separate loop)."""
    rng = np.random.default_rng(5)
    t, d = 6, 8
    K = rng.standard_normal((t + 1, d))
    V = rng.standard_normal((t + 1, d))
    q = rng.standard_normal(d)
    sel = oracle.window_select(t, 32)
    sel = sel[sel >= 0]
    o = oracle.sparse_attention(q, K[sel], V[sel])
    logits = np.array([q @ K[s] for s in range(t + 1)]) / np.sqrt(d)
    p = np.exp(logits - logits.max())
    p /= p.sum()
    np.testing.assert_allclose(o, sum(p[s] * V[s] for s in range(t + 1)), rtol=1e-12, atol=1e-12)


def _kl_inputs(seed, T=12, Hq=4, Hkv=2, d=8, HI=4, dI=4):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((1, T, Hq, d)), rng.standard_normal((1, T, Hkv, d)),
            rng.standard_normal((1, T, HI, dI)), rng.standard_normal((1, T, Hkv, dI)),
            rng.random((1, T, HI)))


def test_indexer_kl_matches_rel_entr():
    """Against scipy's elementwise relative entropy on the two distributions
    built from the definitions (softmax of scaled dot products; softmax of
    the indexer scores)."""
    from scipy.special import rel_entr, softmax
    q, k, qi, ki, w = _kl_inputs(1)
    kl = oracle.indexer_kl(q, k, qi, ki, w)
    T, Hq, d = q.shape[1], q.shape[2], q.shape[3]
    G = Hq // k.shape[2]
    for t in range(T):
        sc = oracle.indexer_scores(qi[0, t], w[0, t], np.transpose(ki[0, : t + 1], (1, 0, 2)))
        for h in range(Hq):
            p = softmax(np.array([q[0, t, h] @ k[0, s, h // G] for s in range(t + 1)]) / math.sqrt(d))
            r = softmax(sc[h // G])
            assert kl[0, t, h] == pytest.approx(float(np.sum(rel_entr(p, r))), rel=1e-9, abs=1e-12)
    assert np.all(kl >= -1e-12)


def test_indexer_kl_first_token_is_zero_and_uniform_student():
    """t = 0: both distributions are the single token, KL = 0.  w = 0: the
    indexer is uniform over the prefix, KL = log(t+1) - H(teacher)."""
    q, k, qi, ki, w = _kl_inputs(2)
    kl = oracle.indexer_kl(q, k, qi, ki, np.zeros_like(w))
    assert np.allclose(kl[:, 0], 0.0, atol=1e-12)
    T, Hq, d = q.shape[1], q.shape[2], q.shape[3]
    G = Hq // k.shape[2]
    for t in range(1, T):
        for h in range(Hq):
            a = np.array([q[0, t, h] @ k[0, s, h // G] for s in range(t + 1)]) / math.sqrt(d)
            e = np.exp(a - a.max())
            p = e / e.sum()
            entropy = -float(np.sum(p * np.log(p)))
            assert kl[0, t, h] == pytest.approx(math.log(t + 1) - entropy, rel=1e-9, abs=1e-12)


# ---------------------------------------------------------------- KV groups
def _group_problem(seed, B=2, Hq=6, Hkv=2, d=8, HI=4, dI=4, t=30):
    rng = np.random.default_rng(seed)
    f = lambda *s: rng.standard_normal(s)
    return dict(q=f(B, Hq, d), k=f(B, Hkv, d), v=f(B, Hkv, d), qidx=f(B, HI, dI), kidx=f(B, Hkv, dI),
                w=rng.random((B, HI)), lam=f(B, Hq), k_cache=f(B, Hkv, t, d), v_cache=f(B, Hkv, t, d),
                kidx_cache=f(B, Hkv, t, dI), S=f(B, Hq, d, d), pos=np.array([t, t - 11][:B]))


def test_decode_kv_groups_are_independent_problems():
    """KV head g's query heads get what a layer with g's KV head alone gives
    them (its K/V, its R indexer heads and key plane, its query heads): with
    M below the prefix length the groups select different sets, so a wrong
    group index anywhere (selection, cache, heads) changes the result."""
    pr = _group_problem(21)
    M = 7
    run = lambda x: oracle.decode_step(x["q"], x["k"], x["v"], x["qidx"], x["kidx"], x["w"], x["lam"],
                                       x["k_cache"], x["v_cache"], x["kidx_cache"], x["S"], x["pos"], M)
    full = run(pr)
    G, R = 3, 2
    assert not np.array_equal(full["idx"][:, 0], full["idx"][:, 1])     # the sets differ
    for g in range(2):
        hs, rs, gs = slice(g * G, (g + 1) * G), slice(g * R, (g + 1) * R), slice(g, g + 1)
        sub = run(dict(q=pr["q"][:, hs], k=pr["k"][:, gs], v=pr["v"][:, gs], qidx=pr["qidx"][:, rs],
                       kidx=pr["kidx"][:, gs], w=pr["w"][:, rs], lam=pr["lam"][:, hs], k_cache=pr["k_cache"][:, gs],
                       v_cache=pr["v_cache"][:, gs], kidx_cache=pr["kidx_cache"][:, gs], S=pr["S"][:, hs],
                       pos=pr["pos"]))
        np.testing.assert_array_equal(full["idx"][:, g], sub["idx"][:, 0])
        np.testing.assert_allclose(full["out"][:, hs], sub["out"], rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(full["S"][:, hs], sub["S"], rtol=1e-13, atol=1e-13)


def test_prefill_kv_groups_are_independent_problems():
    rng = np.random.default_rng(22)
    B, T, Hq, Hkv, d, HI, dI, M = 1, 25, 4, 2, 8, 4, 4, 5
    f = lambda *s: rng.standard_normal(s)
    q, k, v, qi, ki = f(B, T, Hq, d), f(B, T, Hkv, d), f(B, T, Hkv, d), f(B, T, HI, dI), f(B, T, Hkv, dI)
    w, lam, S0 = rng.random((B, T, HI)), f(B, T, Hq), f(B, Hq, d, d)
    full = oracle.prefill(q, k, v, qi, ki, w, lam, S0, M)
    G, R = 2, 2
    for g in range(Hkv):
        hs, rs, gs = slice(g * G, (g + 1) * G), slice(g * R, (g + 1) * R), slice(g, g + 1)
        sub = oracle.prefill(q[:, :, hs], k[:, :, gs], v[:, :, gs], qi[:, :, rs], ki[:, :, gs], w[:, :, rs],
                             lam[:, :, hs], S0[:, hs], M)
        np.testing.assert_array_equal(full["idx"][:, :, g], sub["idx"][:, :, 0])
        np.testing.assert_allclose(full["out"][:, :, hs], sub["out"], rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(full["S"][:, hs], sub["S"], rtol=1e-13, atol=1e-13)
