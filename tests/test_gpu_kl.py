"""GPU parity of lisa_indexer_kl (Stage-2 per-head KL, forward) against the
fp64 oracle.  Tolerance: max-abs 1e-3 on the KL values (fp32 logits from
exact bf16 inputs, fp32 exponentials and logarithms)."""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from lisa_inputs import get_config, make_rng, gen_layer, gen_step
from harness import make_layer, step_tensors

pytestmark = pytest.mark.gpu

L = pytest.importorskip("hybrid_linear_top_b200.lisa")

KL_ATOL = 1e-3


def run_kl(cfg, T, rows=None, seed=0):
    rng = make_rng(600 + seed, 0)
    layer_np = gen_layer(cfg, rng, 0)
    step = gen_step(cfg, rng, T)
    lay = make_layer(L, cfg, T + 7, layer_np, n_rows=0)
    x = step_tensors(step, cfg)
    L.lisa_append_cache(lay, x["k"], x["v"], x["kidx"], T)
    kl = torch.full((cfg.B, T, cfg.Hq), -1.0, dtype=torch.float32, device="cuda")
    L.lisa_indexer_kl(lay, T, x["q"], x["qidx"], x["w"], kl)
    torch.cuda.synchronize()
    assert int(lay.err_word.item()) == 0
    a = lambda z: z.astype(np.float64)
    ref = oracle.indexer_kl(a(step.q), a(step.k), a(step.qidx), a(step.kidx), a(step.w), rows=rows)
    got = kl.cpu().numpy().astype(np.float64)
    r = np.arange(T) if rows is None else np.asarray(rows)
    err = np.abs(got[:, r] - ref[:, r])
    assert np.isfinite(got[:, r]).all()
    assert err.max() <= KL_ATOL, f"max-abs {err.max():.3g} at {np.unravel_index(err.argmax(), err.shape)}"
    assert np.all(got[:, r] >= -KL_ATOL)
    return got, ref


@pytest.mark.parametrize("T", [1, 17, 300])
def test_kl_1p5b_shape(T):
    cfg = dataclasses.replace(get_config("prefill_1p5b_16k"), T=T, B=2 if T < 100 else 1)
    run_kl(cfg, T, seed=T)


@pytest.mark.parametrize("d,dI,HI,Hq", [(64, 32, 2, 8), (128, 32, 16, 32), (128, 32, 8, 14), (128, 64, 2, 14)])
def test_kl_other_shapes(d, dI, HI, Hq):
    cfg = dataclasses.replace(get_config("prefill_1p5b_16k"), T=200, B=1, d=d, dI=dI, HI=HI, Hq=Hq, Hkv=2)
    run_kl(cfg, 200, seed=d + HI)


def test_kl_two_sequences_ragged_block():
    """Two sequences of 300 tokens: the last 128-token block of sequence 0
    runs into sequence 1's rows (their results must not leak)."""
    cfg = dataclasses.replace(get_config("prefill_1p5b_16k"), T=300, B=2)
    run_kl(cfg, 300, seed=5)


def test_kl_2k_sampled_rows():
    cfg = dataclasses.replace(get_config("prefill_1p5b_16k"), T=2048, B=1)
    rows = [0, 1, 15, 16, 17, 63, 64, 511, 1024, 2047]
    run_kl(cfg, 2048, rows=rows, seed=99)
