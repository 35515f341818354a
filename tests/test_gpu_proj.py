"""GPU parity of the projection front-end and the output projection
(tcgen05 GEMMs) against the fp64 oracle, through the C ABI.

Tolerance, from the arithmetic: products of bf16 values are exact in fp32 and
the tensor cores accumulate K of them in fp32, so the accumulation error is at
most about K * 2^-24 * A with A = sum_k |x_k W_nk| (<= 1e-4 * A for the sizes
here); bf16 outputs are then rounded once (<= 2^-9 relative).  The test allows
|y - y*| <= 2^-8 |y*| + 1e-4 A for bf16 fields and 1e-4 A for the fp32 fields
(w, gate_logit).

The reference value of every field AND the magnitude A come from the oracle
(A = the oracle's projection of |x| with |W|), so the field routing the
oracle defines (q | k | v | qidx | kidx | w | gate logits) is what the GPU
output is compared with; the test slices no weights itself."""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from lisa_inputs import get_config, make_rng
from lisa_inputs.gen import round_to_dtype
from harness import dev, f64

pytestmark = pytest.mark.gpu

L = pytest.importorskip("hybrid_linear_top_b200.lisa")

HIDDEN = {"decode_1p5b_16k": 1536, "ragged_7b_b32": 3584}


def _bf16(rng, shape, scale=1.0):
    return round_to_dtype(rng.standard_normal(size=shape, dtype=np.float32) * np.float32(scale), "bf16")


def _check(got, ref, A, f32, where):
    """got: GPU field; ref: the oracle's value; A: the oracle's value for |x|, |W|."""
    bound = 1e-4 * A + (0.0 if f32 else 2.0 ** -8 * np.abs(ref))
    err = np.abs(got - ref)
    assert got.shape == ref.shape, f"{where}: shape {got.shape} vs {ref.shape}"
    assert np.isfinite(got).all(), f"{where}: non-finite"
    bad = err > bound
    assert not bad.any(), f"{where}: {int(bad.sum())} elements out of bound, worst {float((err - bound).max()):.3g}"


def _oracle_in(x, W, cfg, P):
    """The oracle's front-end of (x, W) and of (|x|, |W|) (the error scale)."""
    a = lambda z: z.astype(np.float64)
    ref = oracle.project_in(a(x), a(W), cfg.Hq, cfg.Hkv, cfg.d, cfg.HI, cfg.dI, P)
    mag = oracle.project_in(np.abs(a(x)), np.abs(a(W)), cfg.Hq, cfg.Hkv, cfg.d, cfg.HI, cfg.dI, P)
    return ref, mag


@pytest.mark.parametrize("cfg_name,B,T,variant", [
    ("decode_1p5b_16k", 1, 1, 0),       # a decode step: narrow column tiles
    ("decode_1p5b_16k", 1, 300, 0),     # several row tiles with a ragged tail
    ("decode_1p5b_16k", 3, 50, 1),      # one indexer key per indexer head (4 planes)
    ("decode_1p5b_16k", 16, 1, 1),      # 16 decode tokens: the weight-streaming path at its row limit
    ("decode_1p5b_16k", 17, 1, 0),      # 17 rows: the tensor-core path
    ("decode_1p5b_16k", 5, 1, 2),       # 5 rows: weights as the M operand, one shared key plane
    ("decode_1p5b_16k", 2, 1, 0),       # 2 rows: the weight-streaming CUDA-core path
    ("ragged_7b_b32", 12, 1, 0),        # 7B shape, 12 rows: K split over a cluster of 3
    ("ragged_7b_b32", 32, 1, 1),        # 7B shape, 32 rows: weights as the M operand with N = 32
    ("ragged_7b_b32", 8, 1, 0),         # 7B shape, batch of 8 decode tokens
    ("ragged_7b_b32", 1, 260, 2),       # 7B shape, one shared key plane
])
def test_project_in(cfg_name, B, T, variant):
    cfg = dataclasses.replace(get_config(cfg_name), B=B)
    Hm = HIDDEN[cfg_name]
    lay = L.Layer.allocate(B, cfg.Hq, cfg.Hkv, cfg.d, cfg.HI, cfg.dI, cfg.M, 16)
    widths = L.proj_widths(lay, variant)
    P = widths[4] // cfg.dI
    rng = make_rng(400 + T, 0)
    x = _bf16(rng, (B, T, Hm))
    W = _bf16(rng, (sum(widths), Hm), 1.0 / np.sqrt(Hm))
    proj = L.Proj(Hm, dev(W, "bf16"), None)
    bf = torch.bfloat16
    outs = dict(q=torch.empty(B, T, cfg.Hq, cfg.d, dtype=bf, device="cuda"),
                k=torch.empty(B, T, cfg.Hkv, cfg.d, dtype=bf, device="cuda"),
                v=torch.empty(B, T, cfg.Hkv, cfg.d, dtype=bf, device="cuda"),
                qidx=torch.empty(B, T, cfg.HI, cfg.dI, dtype=bf, device="cuda"),
                kidx=torch.empty(B, T, P, cfg.dI, dtype=bf, device="cuda"),
                w=torch.empty(B, T, cfg.HI, dtype=torch.float32, device="cuda"),
                lam=torch.empty(B, T, cfg.Hq, dtype=torch.float32, device="cuda"))
    for t in outs.values():
        t.fill_(float("nan"))
    L.lisa_project_in(lay, variant, proj, T, dev(x, "bf16"), outs["q"], outs["k"], outs["v"], outs["qidx"],
                      outs["kidx"], outs["w"], outs["lam"])
    torch.cuda.synchronize()
    assert int(lay.err_word.item()) == 0
    ref, mag = _oracle_in(x, W, cfg, P)
    for name in oracle.PROJ_FIELDS:
        _check(f64(outs[name]), ref[name], mag[name], name in ("w", "lam"), name)


@pytest.mark.parametrize("cfg_name,B,T", [("decode_1p5b_16k", 1, 1), ("decode_1p5b_16k", 2, 300),
                                          ("ragged_7b_b32", 32, 1)])
def test_project_out(cfg_name, B, T):
    cfg = dataclasses.replace(get_config(cfg_name), B=B)
    Hm = HIDDEN[cfg_name]
    lay = L.Layer.allocate(B, cfg.Hq, cfg.Hkv, cfg.d, cfg.HI, cfg.dI, cfg.M, 16)
    rng = make_rng(500 + T, 0)
    o = _bf16(rng, (B, T, cfg.Hq, cfg.d), 1.0 / np.sqrt(cfg.d))
    Wo = _bf16(rng, (Hm, cfg.Hq * cfg.d), 1.0 / np.sqrt(cfg.Hq * cfg.d))
    proj = L.Proj(Hm, None, dev(Wo, "bf16"))
    y = torch.full((B, T, Hm), float("nan"), dtype=torch.bfloat16, device="cuda")
    L.lisa_project_out(lay, proj, T, dev(o, "bf16"), y)
    torch.cuda.synchronize()
    a = lambda z: z.astype(np.float64)
    ref = oracle.project_out(a(o), a(Wo))
    mag = oracle.project_out(np.abs(a(o)), np.abs(a(Wo)))
    _check(f64(y), ref, mag, False, "y")


@pytest.mark.parametrize("which", ["in", "out"])
def test_projections_full_prefill_sampled_rows(which):
    """16384 tokens of the 1.5B shape, as the bench runs them: 1280 tiles over
    one persistent CTA per SM, so every CTA walks several tiles and reuses
    both TMEM buffers.  Sampled rows (every tile row block, the ragged edges)
    are checked in full against the oracle."""
    cfg = dataclasses.replace(get_config("prefill_1p5b_16k"), B=1)
    Hm, T = HIDDEN["decode_1p5b_16k"], 16384
    lay = L.Layer.allocate(1, cfg.Hq, cfg.Hkv, cfg.d, cfg.HI, cfg.dI, cfg.M, 16)
    rng = make_rng(700, 0)
    rows = np.unique(np.concatenate([np.arange(0, T, 127), [1, 127, 128, 129, T - 129, T - 128, T - 1]]))
    a = lambda z: z.astype(np.float64)
    bf = torch.bfloat16
    if which == "in":
        widths = L.proj_widths(lay)
        x = _bf16(rng, (1, T, Hm))
        W = _bf16(rng, (sum(widths), Hm), 1.0 / np.sqrt(Hm))
        proj = L.Proj(Hm, dev(W, "bf16"), None)
        outs = [torch.full((1, T, wd), float("nan"), dtype=torch.float32 if i >= 5 else bf, device="cuda")
                for i, wd in enumerate(widths)]
        L.lisa_project_in(lay, 0, proj, T, dev(x, "bf16"), *outs)
        torch.cuda.synchronize()
        ref, mag = _oracle_in(x[:, rows], W, cfg, None)
        for i, name in enumerate(oracle.PROJ_FIELDS):
            got = f64(outs[i][:, rows]).reshape(ref[name].shape)
            _check(got, ref[name], mag[name], name in ("w", "lam"), name)
    else:
        o = _bf16(rng, (1, T, cfg.Hq, cfg.d), 1.0 / np.sqrt(cfg.d))
        Wo = _bf16(rng, (Hm, cfg.Hq * cfg.d), 1.0 / np.sqrt(cfg.Hq * cfg.d))
        proj = L.Proj(Hm, None, dev(Wo, "bf16"))
        y = torch.full((1, T, Hm), float("nan"), dtype=bf, device="cuda")
        L.lisa_project_out(lay, proj, T, dev(o, "bf16"), y)
        torch.cuda.synchronize()
        ref = oracle.project_out(a(o[:, rows]), a(Wo))
        mag = oracle.project_out(np.abs(a(o[:, rows])), np.abs(a(Wo)))
        _check(f64(y[:, rows]), ref, mag, False, "y")
    assert int(lay.err_word.item()) == 0
