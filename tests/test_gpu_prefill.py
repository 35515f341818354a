"""GPU parity of lisa_prefill (and prefill followed by decode steps) against
the fp64 oracle, through the C ABI."""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from lisa_inputs import get_config, make_rng, gen_layer, gen_step
from harness import make_layer, step_tensors, check_set, check_out, check_state, f64, dev

pytestmark = pytest.mark.gpu

L = pytest.importorskip("hybrid_linear_top_b200.lisa")


def gpu_prefill(cfg, layer_np, step, T, L_max):
    lay = make_layer(L, cfg, L_max, layer_np, n_rows=0)
    x = step_tensors(step, cfg)
    ws = L.alloc_workspace(lay, T, L.LISA_OP_PREFILL)
    out = torch.empty(cfg.B, T, cfg.Hq, cfg.d, dtype=lay.torch_dtype, device="cuda")
    idx = torch.full((cfg.B, T, cfg.Hkv, cfg.M), -7, dtype=torch.int32, device="cuda")
    L.lisa_prefill(lay, T, x["q"], x["k"], x["v"], x["kidx"], x["qidx"], x["w"], x["lam"], out, idx, ws)
    torch.cuda.synchronize()
    assert int(lay.err_word.item()) == 0
    return lay, out, idx


def check_prefill(cfg, layer_np, step, lay, out, idx, rows=None):
    a = lambda z: z.astype(np.float64)
    idx_g = idx.cpu().numpy().astype(np.int64)
    ref = oracle.prefill(a(step.q), a(step.k), a(step.v), a(step.qidx), a(step.kidx), a(step.w), a(step.lam),
                         a(layer_np.S0), cfg.M, rows=rows, sel_override=lambda b, t: idx_g[b, t])
    T = step.q.shape[1]
    rows = range(T) if rows is None else rows
    for (b, t), sc in ref["scores"].items():
        for g in range(cfg.Hkv):
            check_set(idx_g[b, t, g], sc[g], cfg.M, t, where=f"b={b} t={t} g={g}")
    o = f64(out)
    r = np.asarray(list(rows))
    check_out(o[:, r], ref["out"][:, r], cfg.dtype, where="prefill out")
    check_state(f64(lay.state), ref["S"], where="prefill state")
    # the caches hold the T tokens
    np.testing.assert_array_equal(f64(lay.k_cache[:, :, :T]), np.transpose(a(step.k), (0, 2, 1, 3)))
    np.testing.assert_array_equal(f64(lay.kidx_cache[:, :, :T]), np.transpose(a(step.kidx), (0, 2, 1, 3)))
    return ref


def test_tiny_fp32_prefill_then_decode():
    """Tiny fp32 layer: prefill 512 tokens, then 16 decode steps, each checked."""
    cfg = get_config("tiny_fp32")
    rng = make_rng(cfg.seed, 0)
    layer_np = gen_layer(cfg, rng, 0)
    pre = gen_step(cfg, rng, cfg.T)
    lay, out, idx = gpu_prefill(cfg, layer_np, pre, cfg.T, cfg.L_max)
    ref = check_prefill(cfg, layer_np, pre, lay, out, idx)

    a = lambda z: z.astype(np.float64)
    kc = np.transpose(a(pre.k), (0, 2, 1, 3))
    vc = np.transpose(a(pre.v), (0, 2, 1, 3))
    kic = np.transpose(a(pre.kidx), (0, 2, 1, 3))
    S = ref["S"]
    ws = L.alloc_workspace(lay, 1, L.LISA_OP_DECODE)
    o = torch.empty(cfg.B, cfg.Hq, cfg.d, dtype=lay.torch_dtype, device="cuda")
    ig = torch.empty(cfg.B, cfg.Hkv, cfg.M, dtype=torch.int32, device="cuda")
    lay.pos.fill_(cfg.T)
    for n in range(cfg.n_decode):
        st = gen_step(cfg, rng, 1)
        x = step_tensors(st, cfg, tau=0)
        L.lisa_decode_step(lay, x["q"], x["k"], x["v"], x["kidx"], x["qidx"], x["w"], x["lam"], 1, o, ig, ws)
        lay.pos.add_(1)
        torch.cuda.synchronize()
        s0 = lambda z: a(z[:, 0])
        t = cfg.T + n
        idx_g = ig.cpu().numpy().astype(np.int64)
        r = oracle.decode_step(s0(st.q), s0(st.k), s0(st.v), s0(st.qidx), s0(st.kidx), s0(st.w), s0(st.lam),
                               kc, vc, kic, S, np.array([t]), cfg.M, sel_override=idx_g)
        for g in range(cfg.Hkv):
            check_set(idx_g[0, g], r["scores"][0][g], cfg.M, t, where=f"step {n}")
        check_out(f64(o), r["out"], cfg.dtype, where=f"decode step {n}")
        check_state(f64(lay.state), r["S"], where=f"state step {n}")
        S = r["S"]
        kc = np.concatenate([kc, s0(st.k)[:, :, None]], axis=2)
        vc = np.concatenate([vc, s0(st.v)[:, :, None]], axis=2)
        kic = np.concatenate([kic, s0(st.kidx)[:, :, None]], axis=2)
    assert int(lay.err_word.item()) == 0


@pytest.mark.parametrize("T", [1, 2, 64, 255, 256, 257, 1500])
def test_prefill_1p5b_shape_small(T):
    """1.5B geometry at small T: chunk edges, prefixes around M, two row passes."""
    cfg = dataclasses.replace(get_config("prefill_1p5b_16k"), T=T, B=1 if T > 300 else 2, S0="normal")
    rng = make_rng(200 + T, 0)
    layer_np = gen_layer(cfg, rng, 0)
    step = gen_step(cfg, rng, T)
    lay, out, idx = gpu_prefill(cfg, layer_np, step, T, T + 5)
    check_prefill(cfg, layer_np, step, lay, out, idx)


def _integer_indexer(step, seed):
    """Small-integer indexer inputs (exact in bf16, exact fp32 sums): exact score ties."""
    ir = np.random.default_rng(seed)
    step.kidx = ir.integers(-1, 2, size=step.kidx.shape).astype(np.float32)
    step.qidx = ir.integers(-1, 2, size=step.qidx.shape).astype(np.float32)
    step.w = ir.integers(0, 3, size=step.w.shape).astype(np.float32)
    return step


def test_prefill_exact_ties_integer_inputs():
    """Exact score ties in every row (integer indexer inputs): the selected sets
    must equal the oracle's with no borderline exemption (tie -> lower
    position), through the two-pass select's kept keys, bounds and candidates,
    over two row passes and rows longer and shorter than the bound needs."""
    T = 5000
    cfg = dataclasses.replace(get_config("prefill_1p5b_16k"), T=T, S0="normal")
    rng = make_rng(230, 0)
    layer_np = gen_layer(cfg, rng, 0)
    step = _integer_indexer(gen_step(cfg, rng, T), 5)
    lay, out, idx = gpu_prefill(cfg, layer_np, step, T, T)
    rows = [0, 255, 256, 257, 2047, 2048, 3000, 4095, 4096, 4999]
    a = lambda z: z.astype(np.float64)
    idx_g = idx.cpu().numpy().astype(np.int64)
    for t in rows:
        keys = np.transpose(a(step.kidx[0, :t + 1]), (1, 0, 2))
        sc = oracle.indexer_scores(a(step.qidx[0, t]), a(step.w[0, t]), keys)
        for g in range(cfg.Hkv):
            check_set(idx_g[0, t, g], sc[g], cfg.M, t, exact=True, where=f"t={t} g={g}")
    check_prefill(cfg, layer_np, step, lay, out, idx, rows=rows)


def test_prefill_all_scores_equal():
    """w = 0: every score is 0, so every key of a row ties with the M-th and is
    a candidate (more than the select stages in shared memory for the long
    rows); the first M positions must be selected."""
    T = 6000
    cfg = dataclasses.replace(get_config("prefill_1p5b_16k"), T=T)
    rng = make_rng(231, 0)
    layer_np = gen_layer(cfg, rng, 0)
    step = gen_step(cfg, rng, T)
    step.w = np.zeros_like(step.w)
    lay, out, idx = gpu_prefill(cfg, layer_np, step, T, T)
    idx_g = idx.cpu().numpy()
    for t in [0, 255, 256, 300, 4095, 4500, 5999]:
        want = np.full(cfg.M, -1)
        n = min(cfg.M, t + 1)
        want[:n] = np.arange(n)
        for g in range(cfg.Hkv):
            np.testing.assert_array_equal(idx_g[0, t, g], want, err_msg=f"t={t} g={g}")
    check_prefill(cfg, layer_np, step, lay, out, idx, rows=[0, 256, 4500, 5999])


def test_prefill_largest_m():
    """M = 1024 with two indexer heads per KV head: most rows have fewer kept
    keys than M, so every key is a candidate (bound 0)."""
    T = 3000
    cfg = dataclasses.replace(get_config("prefill_1p5b_16k"), T=T, M=1024, S0="normal")
    rng = make_rng(232, 0)
    layer_np = gen_layer(cfg, rng, 0)
    step = gen_step(cfg, rng, T)
    lay, out, idx = gpu_prefill(cfg, layer_np, step, T, T)
    check_prefill(cfg, layer_np, step, lay, out, idx, rows=[0, 1023, 1024, 1025, 2047, 2999])


@pytest.mark.slow
def test_prefill_1p5b_16k_sampled():
    """Full 16384-token prefill; outputs and sets checked on sampled rows,
    the final state in full."""
    cfg = get_config("prefill_1p5b_16k")
    rng = make_rng(cfg.seed, 0)
    layer_np = gen_layer(cfg, rng, 0)
    step = gen_step(cfg, rng, cfg.T)
    lay, out, idx = gpu_prefill(cfg, layer_np, step, cfg.T, cfg.L_max)
    sr = np.random.default_rng(0)
    rows = sorted(set([0, 1, 63, 64, 255, 256, 1023, 1024, 8191, 16383] + sr.integers(0, cfg.T, 14).tolist()))
    check_prefill(cfg, layer_np, step, lay, out, idx, rows=rows)


def test_prefill_rejects_nonzero_position():
    cfg = dataclasses.replace(get_config("prefill_1p5b_16k"), T=40, B=2)
    rng = make_rng(9, 0)
    layer_np = gen_layer(cfg, rng, 0)
    step = gen_step(cfg, rng, 40)
    lay = make_layer(L, cfg, 100, layer_np, n_rows=0, poison=False)
    lay.pos.copy_(torch.tensor([0, 3], dtype=torch.int32))
    x = step_tensors(step, cfg)
    ws = L.alloc_workspace(lay, 40, L.LISA_OP_PREFILL)
    out = torch.zeros(2, 40, cfg.Hq, cfg.d, dtype=lay.torch_dtype, device="cuda")
    L.lisa_prefill(lay, 40, x["q"], x["k"], x["v"], x["kidx"], x["qidx"], x["w"], x["lam"], out, None, ws)
    torch.cuda.synchronize()
    assert int(lay.err_word.item()) & L.LISA_DEVERR_POS
    assert (out[1] == 0).all()
    assert torch.isfinite(out[0].float()).all()


def test_indexer_topk_rows_match_prefill_sets():
    cfg = dataclasses.replace(get_config("prefill_1p5b_16k"), T=700, B=1)
    rng = make_rng(21, 0)
    layer_np = gen_layer(cfg, rng, 0)
    step = gen_step(cfg, rng, 700)
    lay = make_layer(L, cfg, 800, layer_np, n_rows=0)
    x = step_tensors(step, cfg)
    L.lisa_append_cache(lay, x["k"], x["v"], x["kidx"], 700)
    ws = L.alloc_workspace(lay, 700, L.LISA_OP_INDEXER_TOPK)
    idx = torch.full((1, 700, cfg.Hkv, cfg.M), -7, dtype=torch.int32, device="cuda")
    L.lisa_indexer_topk(lay, x["qidx"], x["w"], 700, idx, ws)
    torch.cuda.synchronize()
    idx_g = idx.cpu().numpy()
    a = lambda z: z.astype(np.float64)
    keys = np.transpose(a(step.kidx[0]), (1, 0, 2))
    for t in [0, 5, 255, 256, 300, 699]:
        sc = oracle.indexer_scores(a(step.qidx[0, t]), a(step.w[0, t]), keys[:, : t + 1])
        for g in range(cfg.Hkv):
            check_set(idx_g[0, t, g], sc[g], cfg.M, t, where=f"t={t} g={g}")


@pytest.mark.parametrize("d,dI,HI,Hq,M", [(64, 32, 8, 8, 64), (128, 64, 2, 8, 128), (128, 32, 16, 32, 64)])
def test_prefill_other_shapes(d, dI, HI, Hq, M):
    """Other head dims, 1..8 indexer heads per KV head (every tcgen05 tile
    width), 4..16 query heads per KV head, M below T."""
    cfg = dataclasses.replace(get_config("prefill_1p5b_16k"), T=700, B=1, Hq=Hq, Hkv=2, d=d, dI=dI, HI=HI, M=M,
                              S0="normal")
    rng = make_rng(300 + d + HI, 0)
    layer_np = gen_layer(cfg, rng, 0)
    step = gen_step(cfg, rng, 700)
    lay, out, idx = gpu_prefill(cfg, layer_np, step, 700, 710)
    check_prefill(cfg, layer_np, step, lay, out, idx)
