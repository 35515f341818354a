"""Shared helpers of the GPU parity tests: device buffers from the seeded
inputs, and the comparison rules against the fp64 oracle.

Comparison rules (numbers from the layer's stated tolerances):
  * index sets: right count, ascending, inside [0, t], -1 padded; the symmetric
    difference with the oracle's set may only contain borderline tokens
    (oracle score within 1e-4 relative of the M-th score);
  * outputs: compared with the oracle evaluated on the GPU's own index sets
    (so a legal borderline swap cannot fail them): max-abs <= 2e-2 and
    mean-abs <= 2e-3 for bf16 storage; fp32 storage uses 1e-4 / 1e-5;
  * fp32 linear state: per (b, h), max|S_gpu - S*| <= 1e-4 * max|S*|.
"""

import numpy as np
import torch

import oracle

OUT_TOL = {"bf16": (2e-2, 2e-3), "fp32": (1e-4, 1e-5)}
STATE_REL = 1e-4
BORDER_REL = 1e-4

TDT = {"bf16": torch.bfloat16, "fp32": torch.float32}


def dev(x, dtype="fp32", device="cuda"):
    """float32 numpy array (holding exact storage values) -> device tensor."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(device=device, dtype=TDT[dtype])


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def make_layer(L, cfg, L_max, layer_np=None, n_rows=0, poison=True, device="cuda", decode_split=0):
    """Allocate a lisa Layer; copy rows [0, n_rows) of the generated caches and
    S_0; fill the unused cache rows with NaN so stray reads show up."""
    lay = L.Layer.allocate(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.HI, cfg.dI, cfg.M, L_max,
                           L.LISA_BF16 if cfg.dtype == "bf16" else L.LISA_FP32, device=device,
                           decode_split=decode_split)
    if poison:
        lay.k_cache.fill_(float("nan"))
        lay.v_cache.fill_(float("nan"))
        lay.kidx_cache.fill_(float("nan"))
    if layer_np is not None:
        if n_rows:
            lay.k_cache[:, :, :n_rows] = dev(layer_np.k_cache[:, :, :n_rows], cfg.dtype)
            lay.v_cache[:, :, :n_rows] = dev(layer_np.v_cache[:, :, :n_rows], cfg.dtype)
            lay.kidx_cache[:, :, :n_rows] = dev(layer_np.kidx_cache[:, :, :n_rows], cfg.dtype)
        lay.state.copy_(torch.from_numpy(layer_np.S0))
    return lay


def step_tensors(step, cfg, tau=None):
    """Device tensors of a StepData; tau selects one token (decode layout)."""
    def pick(x):
        return x[:, tau] if tau is not None else x
    return dict(
        q=dev(pick(step.q), cfg.dtype), k=dev(pick(step.k), cfg.dtype), v=dev(pick(step.v), cfg.dtype),
        kidx=dev(pick(step.kidx), cfg.dtype), qidx=dev(pick(step.qidx), cfg.dtype),
        w=dev(pick(step.w)), lam=dev(pick(step.lam)),
    )


def check_set(idx_row, scores_row, M, t, exact=False, where=""):
    """idx_row: GPU set (int array of M); scores_row: oracle scores of 0..t."""
    n = t + 1
    valid = idx_row[idx_row >= 0]
    cnt = min(M, n)
    assert len(valid) == cnt, f"{where}: {len(valid)} selected, expected {cnt}"
    assert np.all(idx_row[cnt:] == -1), f"{where}: padding"
    assert np.all(np.diff(valid) > 0), f"{where}: not strictly ascending"
    assert valid[0] >= 0 and valid[-1] <= t, f"{where}: out of range"
    ref = oracle.topm_select(scores_row, M)
    ref = ref[ref >= 0]
    diff = np.setxor1d(valid, ref)
    if exact:
        assert diff.size == 0, f"{where}: set differs at {diff[:10]}"
    elif diff.size:
        bl = oracle.borderline_mask(scores_row, M, rel=BORDER_REL)
        bad = diff[~bl[diff]]
        assert bad.size == 0, f"{where}: non-borderline differences {bad[:10]} (of {diff.size})"
    return diff.size


def check_out(out_gpu, out_ref, dtype, where=""):
    err = np.abs(out_gpu - out_ref)
    mx, mean = float(err.max()), float(err.mean())
    tmax, tmean = OUT_TOL[dtype]
    assert np.isfinite(out_gpu).all(), f"{where}: non-finite output"
    assert mx <= tmax and mean <= tmean, f"{where}: max-abs {mx:.3g} (<= {tmax}), mean-abs {mean:.3g} (<= {tmean})"
    return mx, mean


def check_state(S_gpu, S_ref, where=""):
    B, Hq = S_ref.shape[:2]
    worst = 0.0
    for b in range(B):
        for h in range(Hq):
            ref = S_ref[b, h]
            e = float(np.abs(S_gpu[b, h] - ref).max()) / max(float(np.abs(ref).max()), 1e-30)
            worst = max(worst, e)
            assert e <= STATE_REL, f"{where}: state (b={b}, h={h}) rel err {e:.3g}"
    return worst
