"""lisa_indexer_topk_noalloc: the indexer + top-M call for callers that cannot
allocate device memory (its scratch is a fixed array inside the library).

Checked through the C ABI against lisa_indexer_topk (which takes a caller
workspace) on two calls in a row: index sets are integer results, so they must
be identical.  Sampled rows (the first and the last of every pass over the
fixed scratch) are also checked against the fp64 oracle's scores and top-M,
under the same set rule as every other parity test, so a fault shared by both
calls cannot pass.  This file is collected last on purpose."""

import numpy as np
import pytest
import torch

import oracle
from lisa_inputs import get_config, make_rng, gen_layer, gen_step
from harness import check_set, make_layer, step_tensors

pytestmark = pytest.mark.gpu

L = pytest.importorskip("hybrid_linear_top_b200.lisa")


def _replace(cfg, **kw):
    import dataclasses
    return dataclasses.replace(cfg, **kw)


def _check_rows_vs_oracle(got, lay_np, step, pos, rows, M):
    """got [B, T, Hkv, M] from the GPU; rows: (b, tau) pairs to check against
    the oracle's indexer scores over the causal prefix of token pos[b] + tau
    (cached rows below pos[b] from the generated caches, then the appended
    tokens 0..tau)."""
    a = lambda z: np.asarray(z, dtype=np.float64)
    for b, tau in rows:
        t = int(pos[b]) + tau
        keys = np.concatenate([a(lay_np.kidx_cache[b][:, :pos[b]]),
                               a(step.kidx[b, :tau + 1]).transpose(1, 0, 2)], axis=1)
        sc = oracle.indexer_scores(a(step.qidx[b, tau]), a(step.w[b, tau]), keys)
        for g in range(sc.shape[0]):
            check_set(got[b, tau, g], sc[g], M, t, where=f"b={b} tau={tau} g={g}")


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
        _check_rows_vs_oracle(got.cpu().numpy(), lay_np, step, pos, [(0, 0), (0, T - 1), (1, 0), (1, T - 1)],
                              cfg.M)
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
    rows_per_pass = L.NOALLOC_SCRATCH_BYTES // per_row
    assert rows_per_pass < T      # more than one pass
    # the first and last row of every pass (the last pass is partial), over the batch
    taus = sorted({tau for p0 in range(0, T, rows_per_pass) for tau in (p0, min(T, p0 + rows_per_pass) - 1)})
    sample = [(i % cfg.B, tau) for i, tau in enumerate(taus)]
    pos = np.full(cfg.B, 16384 - T)
    ws = L.alloc_workspace(lay, T, L.LISA_OP_INDEXER_TOPK)
    ref = torch.empty((cfg.B, T, cfg.Hkv, cfg.M), dtype=torch.int32, device="cuda")
    L.lisa_indexer_topk(lay, x["qidx"], x["w"], T, ref, ws)
    for call in range(2):
        got = torch.full_like(ref, -9)
        L.lisa_indexer_topk_noalloc(lay, x["qidx"], x["w"], T, got)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), f"call {call}"
        _check_rows_vs_oracle(got.cpu().numpy(), lay_np, step, pos, sample, cfg.M)
    assert int(lay.err_word.item()) == 0
