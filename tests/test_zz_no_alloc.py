"""lisa_indexer_topk_noalloc: the indexer + top-M call for callers that cannot
allocate device memory (its scratch is a fixed array inside the library).

Checked through the C ABI against lisa_indexer_topk (which takes a caller
workspace) on two calls in a row: index sets are integer results, so they must
be identical.  This file is collected last on purpose."""

import numpy as np
import pytest
import torch

from lisa_inputs import get_config, make_rng, gen_layer, gen_step
from harness import make_layer, step_tensors

pytestmark = pytest.mark.gpu

L = pytest.importorskip("hybrid_linear_top_b200.lisa")


def _replace(cfg, **kw):
    import dataclasses
    return dataclasses.replace(cfg, **kw)


def test_noalloc_indexer_matches_workspace_call_twice():
    cfg = _replace(get_config("decode_1p5b_16k"), B=2, L=9000)
    T = 5
    rng = make_rng(31, 0)
    lay_np = gen_layer(cfg, rng, 9000 - T)
    step = gen_step(cfg, rng, T)
    lay = make_layer(L, cfg, 9000, lay_np, n_rows=9000 - T)
    pos = np.array([9000 - T, 4000])
    lay.pos.copy_(torch.from_numpy(pos.astype(np.int32)))
    x = step_tensors(step, cfg)
    L.lisa_append_cache(lay, x["k"], x["v"], x["kidx"], T)

    ws = L.alloc_workspace(lay, T, L.LISA_OP_INDEXER_TOPK)
    ref = torch.full((cfg.B, T, cfg.Hkv, cfg.M), -7, dtype=torch.int32, device="cuda")
    L.lisa_indexer_topk(lay, x["qidx"], x["w"], T, ref, ws)
    torch.cuda.synchronize()
    for call in range(2):
        got = torch.full_like(ref, -9)
        L.lisa_indexer_topk_noalloc(lay, x["qidx"], x["w"], T, got)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), f"call {call}: index sets differ"
    assert int(lay.err_word.item()) == 0
    # sanity: the sets are real selections (M entries per row, ascending, inside the prefix)
    r = ref.cpu().numpy()
    for b in range(cfg.B):
        for tau in range(T):
            for g in range(cfg.Hkv):
                row = r[b, tau, g]
                assert np.all(np.diff(row) > 0) and row[0] >= 0 and row[-1] <= pos[b] + tau


def test_noalloc_indexer_many_passes():
    """Enough rows that the fixed scratch is cycled through several passes."""
    cfg = _replace(get_config("decode_1p5b_16k"), B=4, Hkv=2, L=16384)
    T = 200
    rng = make_rng(32, 0)
    lay_np = gen_layer(cfg, rng, 16384 - T)
    step = gen_step(cfg, rng, T)
    lay = make_layer(L, cfg, 16384, lay_np, n_rows=16384 - T, poison=False)
    lay.pos.fill_(16384 - T)
    x = step_tensors(step, cfg)
    L.lisa_append_cache(lay, x["k"], x["v"], x["kidx"], T)
    per_row = cfg.B * cfg.Hkv * 16384 * 4
    assert L.NOALLOC_SCRATCH_BYTES // per_row < T      # more than one pass
    ws = L.alloc_workspace(lay, T, L.LISA_OP_INDEXER_TOPK)
    ref = torch.empty((cfg.B, T, cfg.Hkv, cfg.M), dtype=torch.int32, device="cuda")
    L.lisa_indexer_topk(lay, x["qidx"], x["w"], T, ref, ws)
    for call in range(2):
        got = torch.full_like(ref, -9)
        L.lisa_indexer_topk_noalloc(lay, x["qidx"], x["w"], T, got)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), f"call {call}"
    assert int(lay.err_word.item()) == 0
