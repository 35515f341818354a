"""GPU parity of lisa_decode_step / lisa_indexer_topk / lisa_append_cache
against the fp64 oracle, through the C ABI."""

import numpy as np
import pytest
import torch

import oracle
from lisa_inputs import get_config, make_rng, gen_layer, gen_step, gen_lengths
from lisa_inputs.gen import decode_positions
from harness import make_layer, step_tensors, check_set, check_out, check_state, f64, dev

pytestmark = pytest.mark.gpu

L = pytest.importorskip("hybrid_linear_top_b200.lisa")


def _replace(cfg, **kw):
    import dataclasses
    return dataclasses.replace(cfg, **kw)


def run_decode(cfg, layer_np, step, pos, L_max, fuse_append=True, pre_append=False, exact_sets=False,
               n_rows=None, reps=1, split=0):
    """Run one decode step on the GPU and check it against the oracle
    (split: CTAs per (sequence, KV head), 0 = the library's choice)."""
    B = cfg.B
    n_rows = int(pos.max()) if n_rows is None else n_rows
    lay = make_layer(L, cfg, L_max, layer_np, n_rows=n_rows, decode_split=split)
    # rows >= pos[b] of a shorter sequence must not be read: poison them
    for b in range(B):
        lay.k_cache[b, :, int(pos[b]):] = float("nan")
        lay.v_cache[b, :, int(pos[b]):] = float("nan")
        lay.kidx_cache[b, :, int(pos[b]):] = float("nan")
    lay.pos.copy_(torch.from_numpy(pos.astype(np.int32)))
    x = step_tensors(step, cfg, tau=0)
    if pre_append:
        L.lisa_append_cache(lay, x["k"], x["v"], x["kidx"], 1)
    ws = L.alloc_workspace(lay, 1, L.LISA_OP_DECODE)
    out = torch.empty(B, cfg.Hq, cfg.d, dtype=lay.torch_dtype, device="cuda")
    idx = torch.full((B, cfg.Hkv, cfg.M), -7, dtype=torch.int32, device="cuda")
    S_in = lay.state.clone()
    for _ in range(reps):
        lay.state.copy_(S_in)
        L.lisa_decode_step(lay, x["q"], x["k"], x["v"], x["kidx"], x["qidx"], x["w"], x["lam"], fuse_append,
                           out, idx, ws)
    torch.cuda.synchronize()
    assert int(lay.err_word.item()) == 0

    # oracle on the exact stored values
    kc = layer_np.k_cache.astype(np.float64)
    vc = layer_np.v_cache.astype(np.float64)
    kic = layer_np.kidx_cache.astype(np.float64)
    s0 = lambda a: a[:, 0].astype(np.float64)
    idx_g = idx.cpu().numpy().astype(np.int64)
    ref = oracle.decode_step(s0(step.q), s0(step.k), s0(step.v), s0(step.qidx), s0(step.kidx), s0(step.w),
                             s0(step.lam), kc, vc, kic, layer_np.S0.astype(np.float64), pos, cfg.M,
                             sel_override=idx_g)
    ndiff = 0
    for b in range(B):
        for g in range(cfg.Hkv):
            ndiff += check_set(idx_g[b, g], ref["scores"][b][g], cfg.M, int(pos[b]), exact=exact_sets,
                               where=f"b={b} g={g}")
    errs = check_out(f64(out), ref["out"], cfg.dtype, where="out")
    check_state(f64(lay.state), ref["S"], where="state")
    # the new token was appended at row pos[b]
    if fuse_append or pre_append:
        for b in range(B):
            t = int(pos[b])
            np.testing.assert_array_equal(f64(lay.k_cache[b, :, t]), s0(step.k)[b])
            np.testing.assert_array_equal(f64(lay.v_cache[b, :, t]), s0(step.v)[b])
            np.testing.assert_array_equal(f64(lay.kidx_cache[b, :, t]), s0(step.kidx)[b])
    return dict(ndiff=ndiff, errs=errs, lay=lay)


@pytest.mark.parametrize("split", [0, 4, 8, 16, 32, 64])
def test_decode_1p5b_16k(split):
    """Full-size single-layer decode step at 16384 cached tokens, for every
    CTA split of a (sequence, KV head): the cluster forms (4, 8, 16; the
    library's choice 0 is 16 here) and the wide form (32, 64)."""
    cfg = get_config("decode_1p5b_16k")
    rng = make_rng(cfg.seed, 0)
    lay = gen_layer(cfg, rng, cfg.L - 1)
    step = gen_step(cfg, rng, 1)
    pos = decode_positions(cfg)
    run_decode(cfg, lay, step, pos, cfg.L_max, split=split)


@pytest.mark.parametrize("split", [0, 16, 32])
def test_decode_7b_ragged_batch(split):
    """B=32 ragged lengths in [4096, 16384] (the library's choice is 4 CTAs per
    (sequence, KV head) here)."""
    cfg = get_config("ragged_7b_b32")
    rng = make_rng(cfg.seed, 0)
    lengths = gen_lengths(cfg, rng)
    lay = gen_layer(cfg, rng, cfg.L_hi - 1)
    step = gen_step(cfg, rng, 1)
    pos = decode_positions(cfg, lengths=lengths)
    run_decode(cfg, lay, step, pos, cfg.L_max, n_rows=cfg.L_hi - 1, split=split)


@pytest.mark.parametrize("split", [0, 4, 64])
@pytest.mark.parametrize("L_ctx", [1, 2, 100, 255, 256, 257, 300, 4097])
def test_decode_short_prefixes(L_ctx, split):
    """Prefixes around M (all kept, exactly M, M+1) and t = 0."""
    cfg = _replace(get_config("decode_1p5b_16k"), B=2)
    rng = make_rng(100 + L_ctx, 0)
    lay = gen_layer(cfg, rng, 4096)
    step = gen_step(cfg, rng, 1)
    pos = np.array([L_ctx - 1, max(0, L_ctx // 2 - 1)], dtype=np.int64)
    run_decode(cfg, lay, step, pos, 4200, n_rows=4096, split=split)


def test_decode_twice_reuses_workspace():
    cfg = _replace(get_config("decode_1p5b_16k"), L=3000)
    rng = make_rng(7, 0)
    lay = gen_layer(cfg, rng, 2999)
    step = gen_step(cfg, rng, 1)
    run_decode(cfg, lay, step, np.array([2999]), 3000, reps=3)


@pytest.mark.parametrize("split", [0, 4, 8])
def test_decode_exact_ties_integer_inputs(split):
    """Small-integer indexer inputs make exact score ties (exactly representable
    in bf16 and summed exactly in fp32): the set must equal the oracle's with no
    borderline exemption (tie -> lower position)."""
    cfg = _replace(get_config("decode_1p5b_16k"), B=2, L=5000)
    rng = make_rng(11, 0)
    lay = gen_layer(cfg, rng, 4999)
    step = gen_step(cfg, rng, 1)
    ir = np.random.default_rng(3)
    lay.kidx_cache = ir.integers(-1, 2, size=lay.kidx_cache.shape).astype(np.float32)
    step.kidx = ir.integers(-1, 2, size=step.kidx.shape).astype(np.float32)
    step.qidx = ir.integers(-1, 2, size=step.qidx.shape).astype(np.float32)
    step.w = ir.integers(0, 3, size=step.w.shape).astype(np.float32)
    res = run_decode(cfg, lay, step, np.array([4999, 3000]), 5000, exact_sets=True, split=split)
    assert res["ndiff"] == 0


def test_decode_without_fused_append():
    cfg = _replace(get_config("decode_1p5b_16k"), B=3, L=2048)
    rng = make_rng(12, 0)
    lay = gen_layer(cfg, rng, 2047)
    step = gen_step(cfg, rng, 1)
    run_decode(cfg, lay, step, np.array([2047, 1000, 5]), 2048, fuse_append=False, pre_append=True)


@pytest.mark.parametrize("split", [0, 4, 8])
@pytest.mark.parametrize("dtype,d,dI", [("bf16", 64, 32), ("bf16", 128, 32), ("bf16", 64, 64),
                                        ("fp32", 64, 32), ("fp32", 128, 64)])
def test_decode_other_shapes(dtype, d, dI, split):
    cfg = _replace(get_config("decode_1p5b_16k"), B=2, Hq=8, Hkv=2, HI=2, d=d, dI=dI, M=64, dtype=dtype, L=1500)
    rng = make_rng(13, 0)
    lay = gen_layer(cfg, rng, 1499)
    step = gen_step(cfg, rng, 1)
    run_decode(cfg, lay, step, np.array([1499, 700]), 1500, split=split)


@pytest.mark.parametrize("split", [4, 16, 64])
def test_decode_largest_groups_and_m(split):
    """16 query heads and 8 indexer heads per KV head, M = 1024 (the largest
    supported values)."""
    cfg = _replace(get_config("decode_1p5b_16k"), B=1, Hq=32, Hkv=2, HI=16, M=1024, L=9000)
    rng = make_rng(17, 0)
    lay = gen_layer(cfg, rng, 8999)
    step = gen_step(cfg, rng, 1)
    run_decode(cfg, lay, step, np.array([8999]), 9000, split=split)


def test_decode_bad_position_sets_error_word():
    cfg = _replace(get_config("decode_1p5b_16k"), B=2, L=600)
    rng = make_rng(14, 0)
    lay_np = gen_layer(cfg, rng, 599)
    step = gen_step(cfg, rng, 1)
    lay = make_layer(L, cfg, 600, lay_np, n_rows=599)
    lay.pos.copy_(torch.tensor([599, 600], dtype=torch.int32))   # second is out of range
    x = step_tensors(step, cfg, tau=0)
    ws = L.alloc_workspace(lay, 1, L.LISA_OP_DECODE)
    out = torch.zeros(2, cfg.Hq, cfg.d, dtype=lay.torch_dtype, device="cuda")
    L.lisa_decode_step(lay, x["q"], x["k"], x["v"], x["kidx"], x["qidx"], x["w"], x["lam"], 1, out, None, ws)
    torch.cuda.synchronize()
    assert int(lay.err_word.item()) & L.LISA_DEVERR_POS
    assert torch.isfinite(out[0].float()).all()
    assert (out[1] == 0).all()            # skipped sequence left untouched


def test_indexer_topk_single_token():
    cfg = _replace(get_config("decode_1p5b_16k"), B=2, L=9000)
    rng = make_rng(15, 0)
    lay_np = gen_layer(cfg, rng, 8999)
    step = gen_step(cfg, rng, 1)
    lay = make_layer(L, cfg, 9000, lay_np, n_rows=8999)
    pos = np.array([8999, 4321])
    lay.pos.copy_(torch.from_numpy(pos.astype(np.int32)))
    x = step_tensors(step, cfg)        # [B, 1, ...] layout
    L.lisa_append_cache(lay, x["k"], x["v"], x["kidx"], 1)
    ws = L.alloc_workspace(lay, 1, L.LISA_OP_INDEXER_TOPK)
    idx = torch.full((2, 1, cfg.Hkv, cfg.M), -7, dtype=torch.int32, device="cuda")
    L.lisa_indexer_topk(lay, x["qidx"], x["w"], 1, idx, ws)
    torch.cuda.synchronize()
    idx_g = idx.cpu().numpy()
    for b in range(2):
        t = int(pos[b])
        keys = np.concatenate([lay_np.kidx_cache[b, :, :t], step.kidx[b, 0][:, None]], axis=1).astype(np.float64)
        sc = oracle.indexer_scores(step.qidx[b, 0].astype(np.float64), step.w[b, 0].astype(np.float64), keys)
        for g in range(cfg.Hkv):
            check_set(idx_g[b, 0, g], sc[g], cfg.M, t, where=f"b={b} g={g}")


def test_decode_graph_replays_are_stable():
    """Back-to-back decode steps of independent layers, captured in one CUDA
    graph and replayed many times: every replay must select the same sets and
    no device-side check may fire (guards the barriers of the radix select and
    the ordering of the chained launches)."""
    cfg = get_config("decode_1p5b_16k")
    n_inst = 12
    lays, steps = [], []
    for i in range(n_inst):
        rng = make_rng(cfg.seed, 100 + i)
        lay_np = gen_layer(cfg, rng, cfg.L - 1)
        st = gen_step(cfg, rng, 1)
        lay = make_layer(L, cfg, cfg.L_max, lay_np, n_rows=cfg.L - 1, poison=False)
        lay.pos.fill_(cfg.L - 1)
        lays.append(lay)
        steps.append(step_tensors(st, cfg, tau=0))
    ws = L.alloc_workspace(lays[0], 1, L.LISA_OP_DECODE)
    outs = [torch.empty(1, cfg.Hq, cfg.d, dtype=torch.bfloat16, device="cuda") for _ in range(n_inst)]
    idxs = [torch.empty(1, cfg.Hkv, cfg.M, dtype=torch.int32, device="cuda") for _ in range(n_inst)]
    s = torch.cuda.Stream()

    def run_all():
        for lay, x, o, ix in zip(lays, steps, outs, idxs):
            L.lisa_decode_step(lay, x["q"], x["k"], x["v"], x["kidx"], x["qidx"], x["w"], x["lam"], 1, o, ix, ws,
                               s)

    with torch.cuda.stream(s):
        run_all()
    s.synchronize()
    ref = [ix.clone() for ix in idxs]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        run_all()
    for rep in range(150):
        with torch.cuda.stream(s):
            g.replay()
        if rep % 10 == 9:
            torch.cuda.synchronize()
            assert all(int(l.err_word.item()) == 0 for l in lays), f"replay {rep}"
            assert all(torch.equal(a, b) for a, b in zip(idxs, ref)), f"replay {rep}"
    torch.cuda.synchronize()


@pytest.mark.parametrize("split", [0, 4, 8, 32])
@pytest.mark.parametrize("L_ctx", [16384, 3000])
def test_decode_all_scores_equal(L_ctx, split):
    """w = 0 makes every score 0: the first M positions must be selected (the
    tie rule), and at 16384 tokens every key passes the candidate bound, which
    exercises the cluster-wide radix path."""
    cfg = _replace(get_config("decode_1p5b_16k"), B=1, L=L_ctx)
    rng = make_rng(40 + L_ctx, 0)
    lay = gen_layer(cfg, rng, L_ctx - 1)
    step = gen_step(cfg, rng, 1)
    step.w = np.zeros_like(step.w)
    res = run_decode(cfg, lay, step, np.array([L_ctx - 1]), L_ctx, exact_sets=True, split=split)
    assert res["ndiff"] == 0


def test_decode_inputs_and_output_in_pinned_host_memory():
    """The step's inputs may live in pinned host memory and the output may go
    there (the kernel reads and writes them across the host link)."""
    cfg = _replace(get_config("decode_1p5b_16k"), B=2, L=5000)
    rng = make_rng(23, 0)
    layer_np = gen_layer(cfg, rng, 4999)
    step = gen_step(cfg, rng, 1)
    pos = np.array([4999, 2500])
    lay = make_layer(L, cfg, 5000, layer_np, n_rows=4999)
    lay.pos.copy_(torch.from_numpy(pos.astype(np.int32)))
    x = {k: v.cpu().pin_memory() for k, v in step_tensors(step, cfg, tau=0).items()}
    out = torch.empty(cfg.B, cfg.Hq, cfg.d, dtype=lay.torch_dtype).pin_memory()
    idx = torch.empty(cfg.B, cfg.Hkv, cfg.M, dtype=torch.int32, device="cuda")
    L.lisa_decode_step(lay, x["q"], x["k"], x["v"], x["kidx"], x["qidx"], x["w"], x["lam"], 1, out, idx, None)
    torch.cuda.synchronize()
    assert int(lay.err_word.item()) == 0
    kc, vc, kic = (z.astype(np.float64) for z in (layer_np.k_cache, layer_np.v_cache, layer_np.kidx_cache))
    s0 = lambda a: a[:, 0].astype(np.float64)
    idx_g = idx.cpu().numpy().astype(np.int64)
    ref = oracle.decode_step(s0(step.q), s0(step.k), s0(step.v), s0(step.qidx), s0(step.kidx), s0(step.w),
                             s0(step.lam), kc, vc, kic, layer_np.S0.astype(np.float64), pos, cfg.M,
                             sel_override=idx_g)
    for b in range(cfg.B):
        for g in range(cfg.Hkv):
            check_set(idx_g[b, g], ref["scores"][b][g], cfg.M, int(pos[b]), where=f"b={b} g={g}")
    check_out(f64(out), ref["out"], cfg.dtype, where="out")
    check_state(f64(lay.state), ref["S"], where="state")


@pytest.mark.parametrize("split", [0, 4, 32])
def test_decode_long_context_100k(split):
    """100 000 cached tokens: per-CTA key slices of 6-25K keys, candidate
    segments and the exact select at a long context."""
    cfg = _replace(get_config("decode_1p5b_16k"), B=1, L=100000)
    rng = make_rng(29, 0)
    lay = gen_layer(cfg, rng, 99999)
    step = gen_step(cfg, rng, 1)
    run_decode(cfg, lay, step, np.array([99999]), 100000, split=split)


@pytest.mark.parametrize("split", [4, 64])
def test_decode_bench_launch_configuration(split):
    """The headline workload in the launch configuration the bench times:
    full-size instances (16384 cached tokens, 1.5B shape), one stream, every
    step declared independent of the launch before it, captured in a CUDA
    graph and replayed, each instance with a workspace of its own; the
    cluster form with 4 CTAs and the wide form with 64.  Every instance's
    set, output, state and appended row are checked against the oracle on
    the instance's own data (read back from the device)."""
    import bench
    cfg = get_config("decode_1p5b_16k")
    rng = make_rng(cfg.seed, 0)
    exact = (gen_layer(cfg, rng, cfg.L - 1), gen_step(cfg, rng, 1))
    R = 6
    inst = [bench.Instance(L, cfg, torch, 77 + i, exact if i == 0 else None, split) for i in range(R)]
    for x in inst:
        x.lay.independent = 1
    n = cfg.L - 1
    a = lambda t: t.detach().float().cpu().numpy().astype(np.float64)
    before = [dict(kc=a(x.lay.k_cache[:, :, :n]), vc=a(x.lay.v_cache[:, :, :n]), kic=a(x.lay.kidx_cache[:, :, :n]),
                   S=a(x.lay.state)) for x in inst]
    stream = torch.cuda.Stream()
    per, n_full, tail = bench.plan_graphs(R, R)
    g = bench._capture(torch, stream, [stream], [inst[i % R] for i in range(per)], lambda x, s_: x.step(L, x.ws, s_))
    g.replay()
    torch.cuda.synchronize()
    for i, x in enumerate(inst):
        assert int(x.lay.err_word.item()) == 0, f"instance {i}"
        st = {k: a(getattr(x, k)) for k in ("q", "k", "v", "kidx", "qidx", "w", "lam")}
        idx_g = x.idx.cpu().numpy().astype(np.int64)
        bf = before[i]
        ref = oracle.decode_step(st["q"], st["k"], st["v"], st["qidx"], st["kidx"], st["w"], st["lam"],
                                 bf["kc"], bf["vc"], bf["kic"], bf["S"], np.array([n]), cfg.M, sel_override=idx_g)
        for gg in range(cfg.Hkv):
            check_set(idx_g[0, gg], ref["scores"][0][gg], cfg.M, n, where=f"instance {i} g={gg}")
        check_out(f64(x.out), ref["out"], "bf16", where=f"instance {i} out")
        check_state(f64(x.lay.state), ref["S"], where=f"instance {i} state")
        np.testing.assert_array_equal(a(x.lay.k_cache[:, :, n]), st["k"])
        np.testing.assert_array_equal(a(x.lay.kidx_cache[:, :, n]), st["kidx"])
