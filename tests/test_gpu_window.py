"""GPU parity of the Stage-1 sliding-window variant (lisa_decode_step_window,
lisa_prefill_window) against the fp64 oracle with its window selection."""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from lisa_inputs import get_config, make_rng, gen_layer, gen_step
from lisa_inputs.gen import decode_positions
from harness import make_layer, step_tensors, check_out, check_state, f64

pytestmark = pytest.mark.gpu

L = pytest.importorskip("hybrid_linear_top_b200.lisa")


def _windows(pos, Hkv, W):
    return np.stack([np.stack([oracle.window_select(int(t), W)] * Hkv) for t in pos])


def run_window_decode(cfg, layer_np, step, pos, L_max, n_rows, split=0, kidx=True):
    lay = make_layer(L, cfg, L_max, layer_np, n_rows=n_rows, decode_split=split)
    lay.pos.copy_(torch.from_numpy(pos.astype(np.int32)))
    x = step_tensors(step, cfg, tau=0)
    out = torch.empty(cfg.B, cfg.Hq, cfg.d, dtype=lay.torch_dtype, device="cuda")
    idx = torch.full((cfg.B, cfg.Hkv, cfg.M), -7, dtype=torch.int32, device="cuda")
    L.lisa_decode_step_window(lay, x["q"], x["k"], x["v"], x["kidx"] if kidx else None, x["lam"], 1, out, idx)
    torch.cuda.synchronize()
    assert int(lay.err_word.item()) == 0
    sel = _windows(pos, cfg.Hkv, cfg.M)
    np.testing.assert_array_equal(idx.cpu().numpy(), sel)
    s0 = lambda a: a[:, 0].astype(np.float64)
    ref = oracle.decode_step(s0(step.q), s0(step.k), s0(step.v), s0(step.qidx), s0(step.kidx), s0(step.w),
                             s0(step.lam), layer_np.k_cache.astype(np.float64), layer_np.v_cache.astype(np.float64),
                             layer_np.kidx_cache.astype(np.float64), layer_np.S0.astype(np.float64), pos, cfg.M,
                             sel_override=sel)
    check_out(f64(out), ref["out"], cfg.dtype, where="window out")
    check_state(f64(lay.state), ref["S"], where="window state")
    for b in range(cfg.B):
        t = int(pos[b])
        np.testing.assert_array_equal(f64(lay.k_cache[b, :, t]), s0(step.k)[b])
        np.testing.assert_array_equal(f64(lay.v_cache[b, :, t]), s0(step.v)[b])
    return lay


@pytest.mark.parametrize("split", [0, 4])
def test_window_decode_1p5b_16k(split):
    cfg = get_config("decode_1p5b_16k")
    rng = make_rng(cfg.seed, 0)
    layer_np = gen_layer(cfg, rng, cfg.L - 1)
    step = gen_step(cfg, rng, 1)
    run_window_decode(cfg, layer_np, step, decode_positions(cfg), cfg.L_max, cfg.L - 1, split=split)


@pytest.mark.parametrize("L_ctx", [1, 100, 256, 257, 3000])
def test_window_decode_short_prefixes_without_indexer_key(L_ctx):
    cfg = dataclasses.replace(get_config("decode_1p5b_16k"), B=2)
    rng = make_rng(400 + L_ctx, 0)
    layer_np = gen_layer(cfg, rng, 3000)
    step = gen_step(cfg, rng, 1)
    pos = np.array([L_ctx - 1, max(0, L_ctx // 3 - 1)], dtype=np.int64)
    lay = run_window_decode(cfg, layer_np, step, pos, 3100, 3000, kidx=False)
    # without an indexer key the indexer-key cache row keeps what it held
    for b in range(cfg.B):
        t = int(pos[b])
        np.testing.assert_array_equal(f64(lay.kidx_cache[b, :, t]), layer_np.kidx_cache[b, :, t].astype(np.float64))


@pytest.mark.parametrize("dtype,T,M", [("bf16", 700, 128), ("bf16", 300, 64), ("fp32", 200, 32)])
def test_window_prefill(dtype, T, M):
    base = get_config("prefill_1p5b_16k") if dtype == "bf16" else get_config("tiny_fp32")
    cfg = dataclasses.replace(base, T=T, B=1, M=M, S0="normal")
    rng = make_rng(500 + T, 0)
    layer_np = gen_layer(cfg, rng, 0)
    step = gen_step(cfg, rng, T)
    lay = make_layer(L, cfg, T + 5, layer_np, n_rows=0)
    x = step_tensors(step, cfg)
    ws = L.alloc_workspace(lay, T, L.LISA_OP_PREFILL_WINDOW)
    out = torch.empty(cfg.B, T, cfg.Hq, cfg.d, dtype=lay.torch_dtype, device="cuda")
    idx = torch.full((cfg.B, T, cfg.Hkv, M), -7, dtype=torch.int32, device="cuda")
    L.lisa_prefill_window(lay, T, x["q"], x["k"], x["v"], x["kidx"], x["lam"], out, idx, ws)
    torch.cuda.synchronize()
    assert int(lay.err_word.item()) == 0
    want = np.stack([np.stack([np.stack([oracle.window_select(t, M)] * cfg.Hkv) for t in range(T)])])
    np.testing.assert_array_equal(idx.cpu().numpy(), want)
    a = lambda z: z.astype(np.float64)
    ref = oracle.prefill(a(step.q), a(step.k), a(step.v), a(step.qidx), a(step.kidx), a(step.w), a(step.lam),
                         a(layer_np.S0), M, sel_override=lambda b, t: want[b, t])
    check_out(f64(out), ref["out"], cfg.dtype, where="window prefill out")
    check_state(f64(lay.state), ref["S"], where="window prefill state")


def test_window_workspace_has_no_key_buffer():
    cfg = get_config("prefill_1p5b_16k")
    lay = make_layer(L, cfg, cfg.T, None, poison=False)
    assert L.lisa_workspace_bytes(lay, cfg.T, L.LISA_OP_PREFILL_WINDOW) < \
        L.lisa_workspace_bytes(lay, cfg.T, L.LISA_OP_PREFILL)
