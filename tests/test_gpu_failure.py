"""Failure path of the decode step on the GPU, without faulting the GPU: a
bounded wait that runs out.

lisa_layer.debug_flags = LISA_DEBUG_FORCE_TIMEOUT makes every CTA of the
decode kernel wait on a ring barrier before any copy has been issued, with a
20-microsecond limit: the wait runs out, the kernel ORs LISA_DEVERR_TIMEOUT
into the error word and every CTA returns with nothing in flight.  The test
checks that the bit is set, that nothing else was written, and that the next
normal call on the same layer matches the fp64 oracle."""

import numpy as np
import pytest
import torch

import oracle
from lisa_inputs import get_config, make_rng, gen_layer, gen_step
from harness import make_layer, step_tensors, check_set, check_out, check_state, f64

pytestmark = pytest.mark.gpu

L = pytest.importorskip("hybrid_linear_top_b200.lisa")


@pytest.mark.parametrize("split", [4, 8, 16, 64])
def test_forced_timeout_then_normal_call(split):
    import dataclasses
    cfg = dataclasses.replace(get_config("decode_1p5b_16k"), B=2, L=2048)
    rng = make_rng(900 + split, 0)
    n = 2047
    lay_np = gen_layer(cfg, rng, n)
    step = gen_step(cfg, rng, 1)
    pos = np.array([n, 1000])
    lay = make_layer(L, cfg, 2048, lay_np, n_rows=n, decode_split=split)
    for b in range(cfg.B):                       # rows at and after pos[b] are not the sequence's
        lay.k_cache[b, :, int(pos[b]):] = float("nan")
        lay.v_cache[b, :, int(pos[b]):] = float("nan")
        lay.kidx_cache[b, :, int(pos[b]):] = float("nan")
    lay.pos.copy_(torch.from_numpy(pos.astype(np.int32)))
    x = step_tensors(step, cfg, tau=0)
    out = torch.full((cfg.B, cfg.Hq, cfg.d), float("nan"), dtype=lay.torch_dtype, device="cuda")
    idx = torch.full((cfg.B, cfg.Hkv, cfg.M), -7, dtype=torch.int32, device="cuda")
    S_in = lay.state.clone()
    k_before = lay.k_cache.clone()
    ws = L.alloc_workspace(lay, 1, L.LISA_OP_DECODE)    # used by the wide form (split 64)

    lay.debug_flags = L.LISA_DEBUG_FORCE_TIMEOUT
    L.lisa_decode_step(lay, x["q"], x["k"], x["v"], x["kidx"], x["qidx"], x["w"], x["lam"], 1, out, idx, ws)
    torch.cuda.synchronize()
    assert int(lay.err_word.item()) == L.LISA_DEVERR_TIMEOUT
    assert torch.isnan(out.float()).all(), "output written after the timeout"
    assert bool((idx == -7).all()), "index list written after the timeout"
    assert torch.equal(lay.state, S_in), "state written after the timeout"
    assert torch.equal(torch.isnan(lay.k_cache.float()), torch.isnan(k_before.float())), "cache appended"

    # the next normal call on the same layer is correct
    lay.debug_flags = 0
    lay.err_word.zero_()
    L.lisa_decode_step(lay, x["q"], x["k"], x["v"], x["kidx"], x["qidx"], x["w"], x["lam"], 1, out, idx, ws)
    torch.cuda.synchronize()
    assert int(lay.err_word.item()) == 0
    a = lambda z: z.astype(np.float64)
    s0 = lambda z: a(z[:, 0])
    idx_g = idx.cpu().numpy().astype(np.int64)
    ref = oracle.decode_step(s0(step.q), s0(step.k), s0(step.v), s0(step.qidx), s0(step.kidx), s0(step.w),
                             s0(step.lam), a(lay_np.k_cache), a(lay_np.v_cache), a(lay_np.kidx_cache),
                             a(lay_np.S0), pos, cfg.M, sel_override=idx_g)
    for b in range(cfg.B):
        for g in range(cfg.Hkv):
            check_set(idx_g[b, g], ref["scores"][b][g], cfg.M, int(pos[b]), where=f"b={b} g={g}")
    check_out(f64(out), ref["out"], cfg.dtype, where="out")
    check_state(f64(lay.state), ref["S"], where="state")
