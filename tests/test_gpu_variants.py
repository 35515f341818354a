"""GPU parity of the definition variants of the head mapping (one indexer key
per indexer head, one top-M set shared by every KV head, linear-branch keys /
values per query head) through the C ABI, against the fp64 oracle's variant
keyword arguments (pinned in test_oracle_variants.py)."""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from lisa_inputs import get_config, make_rng
from lisa_inputs.gen import round_to_dtype
from harness import check_set, check_out, check_state, f64, dev

pytestmark = pytest.mark.gpu

L = pytest.importorskip("hybrid_linear_top_b200.lisa")

V1 = 1   # LISA_VAR_KEY_PER_INDEXER_HEAD
V2 = 2   # LISA_VAR_SHARED_SET
V3 = 4   # LISA_VAR_LINEAR_KV_PER_QUERY_HEAD
VARIANTS = [V1, V2, V1 | V2, V3, V1 | V3, V1 | V2 | V3]


def _normal(rng, shape, dim, dtype):
    x = rng.standard_normal(size=shape, dtype=np.float32) / np.float32(np.sqrt(dim))
    return round_to_dtype(x, dtype)


def _planes(cfg, variant):
    Gs = 1 if variant & V2 else cfg.Hkv
    P = cfg.HI if variant & V1 else Gs
    return P, Gs


def _layer(cfg, L_max, P, n_rows, kc, vc, kic, S0):
    lay = L.Layer.allocate(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.HI, cfg.dI, cfg.M, L_max,
                           L.LISA_BF16 if cfg.dtype == "bf16" else L.LISA_FP32)
    lay.kidx_cache = torch.full((cfg.B, P, L_max, cfg.dI), float("nan"), dtype=lay.torch_dtype, device="cuda")
    lay.k_cache.fill_(float("nan"))
    lay.v_cache.fill_(float("nan"))
    if n_rows:
        lay.k_cache[:, :, :n_rows] = dev(kc, cfg.dtype)
        lay.v_cache[:, :, :n_rows] = dev(vc, cfg.dtype)
        lay.kidx_cache[:, :, :n_rows] = dev(kic, cfg.dtype)
    lay.state.copy_(torch.from_numpy(S0))
    return lay


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("shape", ["1p5b", "fp32_small"])
def test_decode_variant(variant, shape):
    """Decode step of two sequences at different positions (4095 and 2999
    cached tokens of the 1.5B shape in bf16, or a small fp32 shape)."""
    if shape == "1p5b":
        cfg = dataclasses.replace(get_config("decode_1p5b_16k"), B=2)
        pos = np.array([4095, 2999])
    else:
        cfg = dataclasses.replace(get_config("tiny_fp32"), B=2, Hq=4, Hkv=2, HI=4, M=32)
        pos = np.array([300, 17])
    P, Gs = _planes(cfg, variant)
    rng = make_rng(100 + variant, 0)
    B, Hq, Hkv, d, HI, dI, M = cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.HI, cfg.dI, cfg.M
    n = int(pos.max())
    kc = _normal(rng, (B, Hkv, n, d), d, cfg.dtype)
    vc = _normal(rng, (B, Hkv, n, d), d, cfg.dtype)
    kic = _normal(rng, (B, P, n, dI), dI, cfg.dtype)
    S0 = rng.standard_normal(size=(B, Hq, d, d), dtype=np.float32)
    q = _normal(rng, (B, Hq, d), d, cfg.dtype)
    k = _normal(rng, (B, Hkv, d), d, cfg.dtype)
    v = _normal(rng, (B, Hkv, d), d, cfg.dtype)
    qidx = _normal(rng, (B, HI, dI), dI, cfg.dtype)
    kidx = _normal(rng, (B, P, dI), dI, cfg.dtype)
    w = rng.random(size=(B, HI), dtype=np.float32)
    lam = rng.standard_normal(size=(B, Hq), dtype=np.float32)
    k_lin = _normal(rng, (B, Hq, d), d, cfg.dtype)
    v_lin = _normal(rng, (B, Hq, d), d, cfg.dtype)

    L_max = n + 64
    lay = _layer(cfg, L_max, P, n, kc, vc, kic, S0)
    for b in range(B):   # rows at and beyond pos[b] must not be read before the append
        lay.k_cache[b, :, int(pos[b]):] = float("nan")
        lay.v_cache[b, :, int(pos[b]):] = float("nan")
        lay.kidx_cache[b, :, int(pos[b]):] = float("nan")
    lay.pos.copy_(torch.from_numpy(pos.astype(np.int32)))
    ws = L.alloc_workspace_variant(lay, variant, 1, L.LISA_OP_DECODE)
    out = torch.empty(B, Hq, d, dtype=lay.torch_dtype, device="cuda")
    idx = torch.full((B, Gs, M), -7, dtype=torch.int32, device="cuda")
    lin = variant & V3
    for rep in range(2):   # a repeated call (same state in) gives the same result
        lay.state.copy_(torch.from_numpy(S0))
        L.lisa_decode_step_variant(lay, variant, dev(q, cfg.dtype), dev(k, cfg.dtype), dev(v, cfg.dtype),
                                   dev(kidx, cfg.dtype), dev(qidx, cfg.dtype), dev(w), dev(lam),
                                   dev(k_lin, cfg.dtype) if lin else None, dev(v_lin, cfg.dtype) if lin else None,
                                   1, out, idx, ws)
    torch.cuda.synchronize()
    assert int(lay.err_word.item()) == 0

    a = lambda z: z.astype(np.float64)
    idx_g = idx.cpu().numpy().astype(np.int64)
    ref = oracle.decode_step(a(q), a(k), a(v), a(qidx), a(kidx), a(w), a(lam), a(kc), a(vc), a(kic), a(S0), pos, M,
                             sel_override=idx_g, shared_set=bool(variant & V2),
                             k_lin=a(k_lin) if lin else None, v_lin=a(v_lin) if lin else None)
    for b in range(B):
        for gs in range(Gs):
            check_set(idx_g[b, gs], ref["scores"][b][gs], M, int(pos[b]), where=f"b={b} gs={gs}")
    check_out(f64(out), ref["out"], cfg.dtype, where="out")
    check_state(f64(lay.state), ref["S"], where="state")
    for b in range(B):   # the new token's rows were appended, indexer keys in all P planes
        t = int(pos[b])
        np.testing.assert_array_equal(f64(lay.k_cache[b, :, t]), a(k[b]))
        np.testing.assert_array_equal(f64(lay.v_cache[b, :, t]), a(v[b]))
        np.testing.assert_array_equal(f64(lay.kidx_cache[b, :, t]), a(kidx[b]))


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("shape", ["1p5b", "fp32_small"])
def test_prefill_variant(variant, shape):
    """Causal prefill from an empty cache (T spans several tiles and a ragged
    tail); every output row and the final state are checked."""
    if shape == "1p5b":
        cfg = dataclasses.replace(get_config("prefill_1p5b_16k"), B=1, T=700)
    else:
        cfg = dataclasses.replace(get_config("tiny_fp32"), B=2, Hq=4, Hkv=2, HI=4, M=32, T=200)
    P, Gs = _planes(cfg, variant)
    rng = make_rng(200 + variant, 0)
    B, T, Hq, Hkv, d, HI, dI, M = cfg.B, cfg.T, cfg.Hq, cfg.Hkv, cfg.d, cfg.HI, cfg.dI, cfg.M
    q = _normal(rng, (B, T, Hq, d), d, cfg.dtype)
    k = _normal(rng, (B, T, Hkv, d), d, cfg.dtype)
    v = _normal(rng, (B, T, Hkv, d), d, cfg.dtype)
    qidx = _normal(rng, (B, T, HI, dI), dI, cfg.dtype)
    kidx = _normal(rng, (B, T, P, dI), dI, cfg.dtype)
    w = rng.random(size=(B, T, HI), dtype=np.float32)
    lam = rng.standard_normal(size=(B, T, Hq), dtype=np.float32)
    k_lin = _normal(rng, (B, T, Hq, d), d, cfg.dtype)
    v_lin = _normal(rng, (B, T, Hq, d), d, cfg.dtype)
    S0 = np.zeros((B, Hq, d, d), dtype=np.float32)
    lin = variant & V3

    lay = _layer(cfg, T, P, 0, None, None, None, S0)
    ws = L.alloc_workspace_variant(lay, variant, T, L.LISA_OP_PREFILL)
    out = torch.empty(B, T, Hq, d, dtype=lay.torch_dtype, device="cuda")
    idx = torch.full((B, T, Gs, M), -7, dtype=torch.int32, device="cuda")
    L.lisa_prefill_variant(lay, variant, T, dev(q, cfg.dtype), dev(k, cfg.dtype), dev(v, cfg.dtype),
                           dev(kidx, cfg.dtype), dev(qidx, cfg.dtype), dev(w), dev(lam),
                           dev(k_lin, cfg.dtype) if lin else None, dev(v_lin, cfg.dtype) if lin else None,
                           out, idx, ws)
    torch.cuda.synchronize()
    assert int(lay.err_word.item()) == 0

    a = lambda z: z.astype(np.float64)
    idx_g = idx.cpu().numpy().astype(np.int64)
    rows = sorted(set(range(0, T, 7)) | {T - 1, M - 1, M, M + 1})
    ref = oracle.prefill(a(q), a(k), a(v), a(qidx), a(kidx), a(w), a(lam), a(S0), M, rows=rows,
                         sel_override=lambda b, t: idx_g[b, t], shared_set=bool(variant & V2),
                         k_lin=a(k_lin) if lin else None, v_lin=a(v_lin) if lin else None)
    for b in range(B):
        for t in rows:
            for gs in range(Gs):
                check_set(idx_g[b, t, gs], ref["scores"][(b, t)][gs], M, t, where=f"b={b} t={t} gs={gs}")
    check_out(f64(out)[:, rows], ref["out"][:, rows], cfg.dtype, where="out")
    check_state(f64(lay.state), ref["S"], where="state")
    np.testing.assert_array_equal(f64(lay.kidx_cache[:, :, :T]), a(np.transpose(kidx, (0, 2, 1, 3))))


@pytest.mark.parametrize("variant", [V1, V2, V1 | V2])
def test_indexer_topk_variant_matches_decode(variant):
    """lisa_indexer_topk_variant on appended rows gives the decode step's sets."""
    cfg = dataclasses.replace(get_config("decode_1p5b_16k"), B=1)
    P, Gs = _planes(cfg, variant)
    rng = make_rng(300 + variant, 0)
    n, T = 1500, 3
    lay = L.Layer.allocate(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.HI, cfg.dI, cfg.M, n + T)
    lay.kidx_cache = torch.zeros((cfg.B, P, n + T, cfg.dI), dtype=torch.bfloat16, device="cuda")
    kic = _normal(rng, (cfg.B, P, n + T, cfg.dI), cfg.dI, "bf16")
    lay.kidx_cache.copy_(dev(kic, "bf16"))
    lay.pos.fill_(n)
    qidx = _normal(rng, (cfg.B, T, cfg.HI, cfg.dI), cfg.dI, "bf16")
    w = rng.random(size=(cfg.B, T, cfg.HI), dtype=np.float32)
    ws = L.alloc_workspace_variant(lay, variant, T, L.LISA_OP_INDEXER_TOPK)
    idx = torch.full((cfg.B, T, Gs, cfg.M), -7, dtype=torch.int32, device="cuda")
    L.lisa_indexer_topk_variant(lay, variant, dev(qidx, "bf16"), dev(w), T, idx, ws)
    torch.cuda.synchronize()
    assert int(lay.err_word.item()) == 0
    idx_g = idx.cpu().numpy().astype(np.int64)
    for tau in range(T):
        t = n + tau
        sc = oracle.indexer_scores(qidx[0, tau].astype(np.float64), w[0, tau].astype(np.float64),
                                   kic[0, :, : t + 1].astype(np.float64), groups=Gs)
        for gs in range(Gs):
            check_set(idx_g[0, tau, gs], sc[gs], cfg.M, t, where=f"tau={tau} gs={gs}")
