"""Deterministic input generation shared by the oracle and the CUDA path.

Recipe (a stated definition; the LISA pages fix no input distribution):

* Generator: ``numpy.random.Generator(PCG64(SeedSequence([seed, layer])))``,
  one stream per (workload seed, layer), so any layer can be generated alone.
* Draw order inside one stream: [ragged lengths] -> k cache -> v cache ->
  indexer-key cache -> S_0 -> then, per step: q, k, v, indexer q, indexer k,
  indexer weights w, gate logits.
* q, k, v, caches and indexer q/k ~ N(0, 1) / sqrt(dim) (dim = d or dI);
  w ~ U(0, 1); gate logits ~ N(0, 1); S_0 = 0 or ~ N(0, 1).
* Everything is drawn in float32 and then rounded to the storage dtype
  (round-to-nearest-even for bf16).  The arrays returned here are float32
  arrays that hold exactly the stored values, so the oracle (fp64) and the
  device see identical numbers.  w, gate logits and S_0 stay float32.

No LISA arithmetic lives here.
"""

from dataclasses import dataclass
from typing import Optional

import numpy as np

from .configs import LisaConfig


def make_rng(seed: int, layer: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), int(layer)])))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); return the 16-bit patterns.

    Finite inputs only (the generators never produce NaN)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32)
    if dtype == "fp32":
        return x
    if dtype == "bf16":
        return bf16_bits_to_f32(f32_to_bf16_bits(x))
    raise ValueError(dtype)


def _normal(rng, shape, scale, dtype):
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    return round_to_dtype(x, dtype)


@dataclass
class LayerData:
    """Per-layer state before the first step.

    k_cache, v_cache: [B, Hkv, n_rows, d]; kidx_cache: [B, Hkv, n_rows, dI];
    S0: [B, Hq, d, d] float32 (S0[b, h, i, j]: key-dim i, value-dim j)."""
    k_cache: np.ndarray
    v_cache: np.ndarray
    kidx_cache: np.ndarray
    S0: np.ndarray


@dataclass
class StepData:
    """Inputs of T new tokens (T = 1 for a decode step).

    q [B,T,Hq,d]; k, v [B,T,Hkv,d]; qidx [B,T,HI,dI]; kidx [B,T,Hkv,dI];
    w [B,T,HI] float32; lam [B,T,Hq] float32 (gate logits)."""
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    qidx: np.ndarray
    kidx: np.ndarray
    w: np.ndarray
    lam: np.ndarray


def gen_lengths(cfg: LisaConfig, rng: np.random.Generator) -> np.ndarray:
    """Ragged decode: L_b (tokens incl. the new one) uniform over the integers [L_lo, L_hi]."""
    return rng.integers(cfg.L_lo, cfg.L_hi + 1, size=cfg.B).astype(np.int64)


def gen_layer(cfg: LisaConfig, rng: np.random.Generator, n_rows: int) -> LayerData:
    B, Hkv, Hq, d, dI = cfg.B, cfg.Hkv, cfg.Hq, cfg.d, cfg.dI
    k = _normal(rng, (B, Hkv, n_rows, d), 1.0 / np.sqrt(d), cfg.dtype)
    v = _normal(rng, (B, Hkv, n_rows, d), 1.0 / np.sqrt(d), cfg.dtype)
    kidx = _normal(rng, (B, Hkv, n_rows, dI), 1.0 / np.sqrt(dI), cfg.dtype)
    if cfg.S0 == "normal":
        S0 = rng.standard_normal(size=(B, Hq, d, d), dtype=np.float32)
    else:
        S0 = np.zeros((B, Hq, d, d), dtype=np.float32)
    return LayerData(k, v, kidx, S0)


def gen_step(cfg: LisaConfig, rng: np.random.Generator, T: int = 1) -> StepData:
    B, Hq, Hkv, d, HI, dI = cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.HI, cfg.dI
    q = _normal(rng, (B, T, Hq, d), 1.0 / np.sqrt(d), cfg.dtype)
    k = _normal(rng, (B, T, Hkv, d), 1.0 / np.sqrt(d), cfg.dtype)
    v = _normal(rng, (B, T, Hkv, d), 1.0 / np.sqrt(d), cfg.dtype)
    qidx = _normal(rng, (B, T, HI, dI), 1.0 / np.sqrt(dI), cfg.dtype)
    kidx = _normal(rng, (B, T, Hkv, dI), 1.0 / np.sqrt(dI), cfg.dtype)
    w = rng.random(size=(B, T, HI), dtype=np.float32)
    lam = rng.standard_normal(size=(B, T, Hq), dtype=np.float32)
    return StepData(q, k, v, qidx, kidx, w, lam)


def decode_positions(cfg: LisaConfig, rng: Optional[np.random.Generator] = None,
                     lengths: Optional[np.ndarray] = None) -> np.ndarray:
    """pos[b] = index of the new token = tokens already cached."""
    if cfg.kind == "ragged_decode":
        assert lengths is not None
        return (lengths - 1).astype(np.int64)
    if cfg.kind == "decode":
        return np.full(cfg.B, cfg.L - 1, dtype=np.int64)
    if cfg.kind == "long_decode":
        return np.full(cfg.B, cfg.L, dtype=np.int64)
    raise ValueError(cfg.kind)
