"""Long chain-of-thought decode (Qwen2.5-7B shape, 28 independent layers,
B = 8, 16384 prefilled rows, 1024 sequential decode steps that each append
their K / V / indexer key and update the linear state) against the fp64
oracle.

The layers are independent (no hidden state flows between them), so the
check is exact on a subset: layers 0 and 27, all 1024 steps of all 8
sequences on the GPU, and sequences 0 and 5 of both layers compared with the
oracle at every step (index sets, outputs) and at the end (state, caches).
The four (layer, sequence) oracle runs go to a spawn-started process pool.
"""

import multiprocessing as mp
import os

import numpy as np
import pytest
import torch

from lisa_inputs import get_config, make_rng, gen_layer, gen_step
from lisa_inputs.gen import decode_positions
from harness import make_layer, dev, f64, check_state

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

L = pytest.importorskip("hybrid_linear_top_b200.lisa")

LAYERS = (0, 27)
SEQS = (0, 5)


def _gpu_layer(cfg, layer):
    """All decode steps of one layer on the GPU; returns the generated data
    and the GPU's outputs, index sets and final state."""
    rng = make_rng(cfg.seed, layer)
    lay_np = gen_layer(cfg, rng, cfg.L)
    steps = [gen_step(cfg, rng, 1) for _ in range(cfg.n_decode)]
    lay = make_layer(L, cfg, cfg.L_max, lay_np, n_rows=cfg.L)
    lay.pos.copy_(torch.from_numpy(decode_positions(cfg).astype(np.int32)))
    ws = L.alloc_workspace(lay, 1, L.LISA_OP_DECODE)
    n = cfg.n_decode
    outs = torch.empty(n, cfg.B, cfg.Hq, cfg.d, dtype=lay.torch_dtype, device="cuda")
    idxs = torch.empty(n, cfg.B, cfg.Hkv, cfg.M, dtype=torch.int32, device="cuda")
    xs = [dict(q=dev(s.q[:, 0], cfg.dtype), k=dev(s.k[:, 0], cfg.dtype), v=dev(s.v[:, 0], cfg.dtype),
               kidx=dev(s.kidx[:, 0], cfg.dtype), qidx=dev(s.qidx[:, 0], cfg.dtype), w=dev(s.w[:, 0]),
               lam=dev(s.lam[:, 0])) for s in steps]
    for i, x in enumerate(xs):
        L.lisa_decode_step(lay, x["q"], x["k"], x["v"], x["kidx"], x["qidx"], x["w"], x["lam"], 1, outs[i],
                           idxs[i], ws)
        lay.pos.add_(1)
    torch.cuda.synchronize()
    assert int(lay.err_word.item()) == 0
    res = dict(out=f64(outs), idx=idxs.cpu().numpy().astype(np.int64), S=f64(lay.state),
               k_tail=f64(lay.k_cache[:, :, cfg.L:]), kidx_tail=f64(lay.kidx_cache[:, :, cfg.L:]))
    # the generated data of the checked sequences, for the oracle workers
    res["data"] = {b: dict(k_cache=lay_np.k_cache[b], v_cache=lay_np.v_cache[b], kidx_cache=lay_np.kidx_cache[b],
                           S0=lay_np.S0[b],
                           steps=[{f: getattr(st, f)[b, 0] for f in ("q", "k", "v", "qidx", "kidx", "w", "lam")}
                                  for st in steps])
                   for b in SEQS}
    del lay, outs, idxs, xs
    torch.cuda.empty_cache()
    return res


def _oracle_pair(args):
    """Oracle run of one (layer, sequence) over every step, with the GPU's
    index sets for the sparse branch; returns per-step checks."""
    import numpy as np
    import oracle
    from lisa_inputs import get_config
    from harness import check_set, check_out

    layer, b, data, gout, gidx = args
    cfg = get_config("longcot_7b_28l")
    a = lambda z: np.asarray(z, dtype=np.float64)[None]
    kc = np.zeros((1, cfg.Hkv, cfg.L_max, cfg.d))
    vc = np.zeros_like(kc)
    kic = np.zeros((1, cfg.Hkv, cfg.L_max, cfg.dI))
    kc[:, :, :cfg.L] = a(data["k_cache"])
    vc[:, :, :cfg.L] = a(data["v_cache"])
    kic[:, :, :cfg.L] = a(data["kidx_cache"])
    S = a(data["S0"])
    worst_max = worst_mean = 0.0
    ndiff = 0
    for i, st in enumerate(data["steps"]):
        t = cfg.L + i
        ref = oracle.decode_step(a(st["q"]), a(st["k"]), a(st["v"]), a(st["qidx"]), a(st["kidx"]), a(st["w"]),
                                 a(st["lam"]), kc, vc, kic, S, np.array([t]), cfg.M, sel_override=gidx[i][None])
        where = f"layer {layer} seq {b} step {i}"
        for g in range(cfg.Hkv):
            ndiff += check_set(gidx[i][g], ref["scores"][0][g], cfg.M, t, where=f"{where} g={g}")
        mx, mean = check_out(gout[i][None], ref["out"], cfg.dtype, where=where)
        worst_max, worst_mean = max(worst_max, mx), max(worst_mean, mean)
        kc[0, :, t] = st["k"]
        vc[0, :, t] = st["v"]
        kic[0, :, t] = st["kidx"]
        S = ref["S"]
    return dict(layer=layer, b=b, S=S[0], k_tail=kc[0, :, cfg.L:], kidx_tail=kic[0, :, cfg.L:],
                worst_max=worst_max, worst_mean=worst_mean, ndiff=ndiff)


def test_decode_longcot_7b_two_layers():
    cfg = get_config("longcot_7b_28l")
    gpu = {layer: _gpu_layer(cfg, layer) for layer in LAYERS}
    jobs = [(layer, b, gpu[layer]["data"][b], gpu[layer]["out"][:, b], gpu[layer]["idx"][:, b])
            for layer in LAYERS for b in SEQS]
    # the oracle allocates ~150 MB per step: keep freed memory in the heap
    # instead of returning it to the kernel (page faults dominate otherwise)
    os.environ.setdefault("MALLOC_MMAP_THRESHOLD_", str(1 << 32))
    os.environ.setdefault("MALLOC_TRIM_THRESHOLD_", str(1 << 34))
    with mp.get_context("spawn").Pool(len(jobs)) as pool:
        results = pool.map(_oracle_pair, jobs)
    for r in results:
        g = gpu[r["layer"]]
        check_state(g["S"][r["b"]][None], r["S"][None], where=f"layer {r['layer']} seq {r['b']} final state")
        np.testing.assert_array_equal(g["k_tail"][r["b"]], r["k_tail"])
        np.testing.assert_array_equal(g["kidx_tail"][r["b"]], r["kidx_tail"])
