"""LISA decode-attention benchmark on B200.

Workload: the Qwen2.5-1.5B-shaped single-layer decode step (B=1, 12 query /
2 KV heads, d=128, 4 indexer heads of dim 64, M=256) at 16384 cached tokens.
One step = one lisa_decode_step call: indexer over all 16384 keys, top-M,
sparse attention, linear-state update and gate.

The timed region replays CUDA graphs of exactly K steps in ONE stream; the
steps rotate over R independent layer instances whose touched bytes exceed
4x the L2 size, and the L2 is flushed before the region (so the traffic is
HBM traffic).  Each step is declared independent of the launch before it, so
consecutive steps overlap on the device (programmatic dependent launch).
value = tokens/s over all ranks (B tokens per step).  Also reported: the same
stream at steady state, the dependent chain (every step waits for the one
before it), a batch of S concurrent chains, the latency of one step alone,
and the end-to-end rate with every step's inputs read from pinned host memory
and its output written back to it (e2e).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lisa|reference]
                  [--streams S] [--split 0|4|8|16] [--workload prefill_1p5b_16k]

--impl reference times the fp64 CPU oracle on the host cores (bounded
sample), the only reference this method has.
"""

import argparse
import json
import os

# hardware work queues for the concurrent chains (read when CUDA starts)
os.environ.setdefault("CUDA_DEVICE_MAX_CONNECTIONS", "32")
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from lisa_inputs import get_config, make_rng, gen_layer, gen_step  # noqa: E402
from lisa_inputs.gen import decode_positions  # noqa: E402

METRIC = "LISA decode-attn tokens/s @16K ctx, M=256; % of HBM roofline"
WORKLOAD = "decode_1p5b_16k"
# DRAM bytes (read + write) of one decode launch from an ncu capture of this
# kernel on this workload, by CTA split (the ncu summary under profiles/);
# None where no capture of the current kernel exists.
DECODE_TRAFFIC = {4: 5390336, 8: None, 16: 5497856, 0: None, 32: None, 64: None}
# nominal HBM3e bandwidth of a B200 (about 8 TB/s), for the second fraction
NOMINAL_HBM_GBS = 8000.0


def algorithmic_bytes(cfg, L, esize=2):
    """Bytes the method must move per decode step (one sequence):
    indexer keys of every cached token, the M selected K and V rows, the fp32
    state read and write, plus the step's own small tensors."""
    G = cfg.Hq // cfg.Hkv
    M = min(cfg.M, L)
    big = cfg.Hkv * L * cfg.dI * esize + cfg.Hkv * M * 2 * cfg.d * esize + cfg.Hq * cfg.d * cfg.d * 4 * 2
    small = (cfg.Hq * cfg.d * esize            # q
             + 2 * cfg.Hkv * cfg.d * esize      # k, v read
             + 2 * cfg.Hkv * cfg.d * esize      # k, v appended
             + 2 * cfg.Hkv * cfg.dI * esize     # kidx read + appended
             + cfg.HI * cfg.dI * esize          # qidx
             + cfg.HI * 4 + cfg.Hq * 4          # w, gate logits
             + cfg.Hq * cfg.d * esize)          # out
    del G
    return big + small


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []
        self.proc = None
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except FileNotFoundError:
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.t:
            self.t.join(timeout=2)

    def summary(self, t0, t1):
        rows = [s for (ts, s) in self.samples if t0 <= ts <= t1] or [s for (_, s) in self.samples]
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            f = [x.strip() for x in r.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(rows)}


# ---------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle
    cfg = get_config(WORKLOAD)
    rng = make_rng(cfg.seed, 0)
    lay = gen_layer(cfg, rng, cfg.L - 1)
    pos = decode_positions(cfg)
    a = lambda z: z.astype(np.float64)
    kc, vc, kic, S0 = a(lay.k_cache), a(lay.v_cache), a(lay.kidx_cache), a(lay.S0)
    steps = [gen_step(cfg, rng, 1) for _ in range(4)]

    def one(st):
        s0 = lambda z: a(z[:, 0])
        oracle.decode_step(s0(st.q), s0(st.k), s0(st.v), s0(st.qidx), s0(st.kidx), s0(st.w), s0(st.lam),
                           kc, vc, kic, S0, pos, cfg.M)

    for i in range(args.warmup):
        one(steps[i % 4])
    t0 = time.perf_counter()
    for i in range(args.steps):
        one(steps[i % 4])
    dt = time.perf_counter() - t0
    cores = len(os.sched_getaffinity(0))
    value = args.steps * cfg.B / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1)/sqrt(dim) caches and inputs)",
        "config": {"workload": WORKLOAD, "B": cfg.B, "L": cfg.L, "M": cfg.M, "parallelism": "replicas"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{args.steps} fp64 oracle decode steps of the 16384-token workload"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline_sample(seconds=10.0):
    """The fp64 oracle on this host's cores, timed on a bounded sample of
    the same workload (whole decode steps, until `seconds` have passed)."""
    import oracle
    cfg = get_config(WORKLOAD)
    rng = make_rng(cfg.seed, 0)
    lay = gen_layer(cfg, rng, cfg.L - 1)
    st = gen_step(cfg, rng, 1)
    pos = decode_positions(cfg)
    a = lambda z: z.astype(np.float64)
    s0 = lambda z: a(z[:, 0])
    args = (s0(st.q), s0(st.k), s0(st.v), s0(st.qidx), s0(st.kidx), s0(st.w), s0(st.lam), a(lay.k_cache),
            a(lay.v_cache), a(lay.kidx_cache), a(lay.S0), pos, cfg.M)
    oracle.decode_step(*args)
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.decode_step(*args)
        n += 1
        dt = time.perf_counter() - t0
        if dt >= seconds:
            break
    return {"value": n * cfg.B / dt, "unit": "tokens/s", "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
            "sample": f"{n} fp64 oracle decode steps of the 16384-token workload in {dt:.1f} s"}


# ---------------------------------------------------------------- lisa arm
# packed per-step inputs of one instance: (name, elements per sequence, bf16?)
def _input_layout(cfg):
    return [("q", cfg.Hq * cfg.d, True), ("k", cfg.Hkv * cfg.d, True), ("v", cfg.Hkv * cfg.d, True),
            ("kidx", cfg.Hkv * cfg.dI, True), ("qidx", cfg.HI * cfg.dI, True), ("w", cfg.HI, False),
            ("lam", cfg.Hq, False)]


class Instance:
    """One independent layer at 16384 cached tokens, with its step inputs.

    The step inputs live in one device buffer (16-byte aligned segments) so
    that the end-to-end run can refill them with a single host-to-device copy
    per step."""

    def __init__(self, L, cfg, torch, seed, exact=None, split=0):
        dev = "cuda"
        bf = torch.bfloat16
        self.lay = L.Layer.allocate(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.HI, cfg.dI, cfg.M, cfg.L, L.LISA_BF16,
                                    decode_split=split)
        n = cfg.L - 1
        segs, off = {}, 0
        for name, nel, is_bf in _input_layout(cfg):
            nb = cfg.B * nel * (2 if is_bf else 4)
            segs[name] = (off, nb, is_bf)
            off += (nb + 15) // 16 * 16
        self.in_bytes = off
        self.inbuf = torch.zeros(off, dtype=torch.uint8, device=dev)
        shapes = {"q": (cfg.B, cfg.Hq, cfg.d), "k": (cfg.B, cfg.Hkv, cfg.d), "v": (cfg.B, cfg.Hkv, cfg.d),
                  "kidx": (cfg.B, cfg.Hkv, cfg.dI), "qidx": (cfg.B, cfg.HI, cfg.dI), "w": (cfg.B, cfg.HI),
                  "lam": (cfg.B, cfg.Hq)}
        for name, (o, nb, is_bf) in segs.items():
            view = self.inbuf[o:o + nb].view(bf if is_bf else torch.float32).view(shapes[name])
            setattr(self, name, view)
        self._segs, self._shapes = segs, shapes
        if exact is not None:
            lay_np, st = exact
            tb = lambda z: torch.from_numpy(np.ascontiguousarray(z)).to(dev, bf)
            tf = lambda z: torch.from_numpy(np.ascontiguousarray(z)).to(dev, torch.float32)
            self.lay.k_cache[:, :, :n] = tb(lay_np.k_cache)
            self.lay.v_cache[:, :, :n] = tb(lay_np.v_cache)
            self.lay.kidx_cache[:, :, :n] = tb(lay_np.kidx_cache)
            self.lay.state.copy_(tf(lay_np.S0))
            s0 = lambda z: z[:, 0]
            for name in ("q", "k", "v", "kidx", "qidx"):
                getattr(self, name).copy_(tb(s0(getattr(st, name))))
            self.w.copy_(tf(s0(st.w)))
            self.lam.copy_(tf(s0(st.lam)))
        else:
            g = torch.Generator(device=dev)
            g.manual_seed(seed)
            rn = lambda shape, dim: (torch.randn(shape, generator=g, device=dev) / dim ** 0.5).to(bf)
            self.lay.k_cache[:, :, :n] = rn((cfg.B, cfg.Hkv, n, cfg.d), cfg.d)
            self.lay.v_cache[:, :, :n] = rn((cfg.B, cfg.Hkv, n, cfg.d), cfg.d)
            self.lay.kidx_cache[:, :, :n] = rn((cfg.B, cfg.Hkv, n, cfg.dI), cfg.dI)
            self.lay.state.copy_(torch.randn(self.lay.state.shape, generator=g, device=dev))
            for name in ("q", "k", "v"):
                getattr(self, name).copy_(rn(shapes[name], cfg.d))
            self.kidx.copy_(rn(shapes["kidx"], cfg.dI))
            self.qidx.copy_(rn(shapes["qidx"], cfg.dI))
            self.w.copy_(torch.rand(shapes["w"], generator=g, device=dev))
            self.lam.copy_(torch.randn(shapes["lam"], generator=g, device=dev))
        self.lay.pos.fill_(n)
        self.out = torch.empty(cfg.B, cfg.Hq, cfg.d, dtype=bf, device=dev)
        self.idx = torch.empty(cfg.B, cfg.Hkv, cfg.M, dtype=torch.int32, device=dev)
        # a workspace of its own (steps of different instances may run concurrently)
        self.ws = L.alloc_workspace(self.lay, 1, L.LISA_OP_DECODE)
        self.host_in = None

    def step(self, L, ws, stream=None):
        L.lisa_decode_step(self.lay, self.q, self.k, self.v, self.kidx, self.qidx, self.w, self.lam, 1, self.out,
                           self.idx, ws, stream)

    def attach_host(self, torch):
        """Pinned host copies of the step inputs and a pinned host output."""
        self.host_in = self.inbuf.cpu().pin_memory()
        self.host_out = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        self.hv = {}
        for name, (o, nb, is_bf) in self._segs.items():
            self.hv[name] = self.host_in[o:o + nb].view(torch.bfloat16 if is_bf else torch.float32).view(
                self._shapes[name])

    def step_e2e(self, L, ws, stream):
        """The decode call on inputs in pinned host memory, writing its output
        to pinned host memory: the kernel reads the step's inputs across the
        host link and writes the result back (zero-copy, no copy engine)."""
        h = self.hv
        L.lisa_decode_step(self.lay, h["q"], h["k"], h["v"], h["kidx"], h["qidx"], h["w"], h["lam"], 1,
                           self.host_out, None, ws, stream)

    def step_e2e_dma(self, L, ws, stream):
        """Host -> device copy of the step's inputs by the copy engine, the
        decode call, and the output copied back to host memory."""
        self.inbuf.copy_(self.host_in, non_blocking=True)
        L.lisa_decode_step(self.lay, self.q, self.k, self.v, self.kidx, self.qidx, self.w, self.lam, 1, self.out,
                           None, ws, stream)
        self.host_out.copy_(self.out, non_blocking=True)


def _capture(torch, stream, chains, items, fn):
    """CUDA graph of fn(item, chain stream) over items; item i goes to chain
    i % len(chains); the chains are independent and join at the end."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        if len(chains) == 1:
            for it in items:
                fn(it, stream)
        else:
            fork = torch.cuda.Event()
            fork.record(stream)
            for s_ in chains:
                s_.wait_event(fork)
            for i, it in enumerate(items):
                fn(it, chains[i % len(chains)])
            for s_ in chains:
                j = torch.cuda.Event()
                j.record(s_)
                stream.wait_event(j)
    return g


def max_over_ranks(ms, world, device):
    """The slowest rank's time (the job's time) when several replicas run."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_rate(units_per_rank, ms, world):
    """Whole-job units per second: every replica processes units_per_rank in
    the (max-over-ranks) time ms."""
    return world * units_per_rank / (ms / 1e3)


def _timed_replays(torch, stream, graphs, barrier=None, before=None):
    """Device time (ms) of replaying `graphs` once each, in order.  `before`
    (optional) enqueues untimed work ahead of the start event.  A sleep kernel
    then keeps the GPU busy while the host enqueues the start event, the
    graphs and the end event, so the region holds device time only, not the
    host's launch latency."""
    if barrier:
        barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        if before:
            before()
        torch.cuda._sleep(400000)
        e0.record(stream)
        for g in graphs:
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    if barrier:
        barrier()
    return e0.elapsed_time(e1)


def plan_graphs(K, R, cap=2048):
    """How exactly K decode steps that rotate over R instances are laid out in
    CUDA graphs: returns (per, n_full, tail), i.e. n_full replays of one graph
    of `per` steps followed by one graph of `tail` steps (0: none), with
    per * n_full + tail == K.  When K >= R, `per` is a whole number of
    rotations (a multiple of R, at most about `cap` steps), so step j of every
    graph runs instance j % R and the full graphs are identical; when K < R a
    single graph runs instances 0 .. K-1, each once."""
    if K < 1 or R < 1:
        raise ValueError(f"steps={K} and instances={R} must be positive")
    if K < R:
        return K, 1, 0
    per = min(R * max(1, cap // R), K // R * R)
    n_full, tail = divmod(K, per)
    return per, n_full, tail


def instances_needed(step_bytes, l2_bytes, streams=1, minimum=0):
    """Independent instances whose touched bytes exceed 4x the L2 size,
    rounded up to a multiple of `streams` (each instance stays in one chain)."""
    R = max(minimum, int(np.ceil(4 * l2_bytes / step_bytes)), streams)
    return -(-R // streams) * streams


def flush_l2(torch, nbytes):
    """Writes a buffer of nbytes on the current stream (evicts what the L2 holds)."""
    buf = torch.empty(int(nbytes), dtype=torch.uint8, device="cuda")
    buf.fill_(1)
    return buf


def _timed_steps(torch, stream, graphs, l2_bytes, barrier=None):
    """Replays `graphs` once untimed (graph upload, warm caches of the code
    path), then flushes the L2 by writing 4x its size and times one replay of
    every graph in order with CUDA events on `stream`.  Returns ms."""
    with torch.cuda.stream(stream):
        for g in graphs:
            g.replay()
    return _timed_replays(torch, stream, graphs, barrier, before=lambda: flush_l2(torch, 4 * l2_bytes))


def run_lisa(args, rank, world):
    import torch
    import torch.distributed as dist
    from hybrid_linear_top_b200 import lisa as L

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    cfg = get_config(WORKLOAD)
    props = torch.cuda.get_device_properties(local)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20)
    step_bytes = algorithmic_bytes(cfg, cfg.L)
    S = max(1, args.streams)
    R = instances_needed(step_bytes, l2, S, args.instances)
    barrier = dist.barrier if world > 1 else None
    K = args.steps
    K_steady = max(K, 20 * R)            # the extra (steady-state) measurements

    rng = make_rng(cfg.seed, 0)
    exact = (gen_layer(cfg, rng, cfg.L - 1), gen_step(cfg, rng, 1))
    inst = [Instance(L, cfg, torch, 1000 * rank + i, exact if i == 0 else None, args.split) for i in range(R)]
    torch.cuda.synchronize()

    stream = torch.cuda.Stream()
    chains = [torch.cuda.Stream() for _ in range(S)]
    run = lambda x, s_: x.step(L, x.ws, s_)

    def set_mode(independent, split):
        for x in inst:
            x.lay.independent = int(independent)
            x.lay.decode_split = split

    def one_stream(n_steps, fn=run):
        per, n_full, tail = plan_graphs(n_steps, R)
        full = _capture(torch, stream, [stream], [inst[i % R] for i in range(per)], fn)
        graphs = [full] * n_full
        if tail:
            graphs.append(_capture(torch, stream, [stream], [inst[i % R] for i in range(tail)], fn))
        return graphs

    # ---- warm-up: exactly W untimed steps, in the headline's mode
    set_mode(True, args.split)
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            inst[i % R].step(L, inst[i % R].ws, stream)
    stream.synchronize()

    # ---- headline: exactly K steps in ONE stream rotating over the R
    #      independent instances; every step is declared independent of the
    #      launch before it, so consecutive steps overlap on the device through
    #      programmatic dependent launch
    graphs = one_stream(K)
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.2)
    t_wall0 = time.time()
    ms = _timed_steps(torch, stream, graphs, l2, barrier)
    t_wall1 = time.time()
    clk.stop()
    ms = max_over_ranks(ms, world, "cuda")
    ms_per_step = ms / K
    value = replica_rate(K * cfg.B, ms, world)
    del graphs
    # the same stream at steady state (K_steady steps)
    ms_ss = max_over_ranks(_timed_steps(torch, stream, one_stream(K_steady), l2, barrier), world, "cuda")

    # ---- dependent chain: one stream, every step waits for the one before it
    #      (as in a stack of layers whose inputs come from the previous launch);
    #      the library's CTA split for one sequence
    set_mode(False, 0)
    ms_dep = max_over_ranks(_timed_steps(torch, stream, one_stream(K_steady), l2, barrier), world, "cuda")

    # ---- one step alone: a sleep kernel keeps the GPU busy while the events
    #      and the step are enqueued, so no host launch latency is timed
    lat = []
    for i in range(min(R, 16)):
        if barrier:
            barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            flush_l2(torch, 4 * l2)
            torch.cuda._sleep(400000)
            e0.record(stream)
            inst[i].step(L, inst[i].ws, stream)
            e1.record(stream)
        torch.cuda.synchronize()
        lat.append(e0.elapsed_time(e1) * 1e3)
    lat_us = max_over_ranks(statistics.median(lat), world, "cuda")

    # ---- a batch of independent layers: S concurrent streams (chains), each
    #      step waiting for the one before it in its chain
    set_mode(False, args.split)
    per, n_full, tail = plan_graphs(K_steady, R)
    gch = [_capture(torch, stream, chains, [inst[i % R] for i in range(per)], run)] * n_full
    if tail:
        gch.append(_capture(torch, stream, chains, [inst[i % R] for i in range(tail)], run))
    ms_ch = max_over_ranks(_timed_steps(torch, stream, gch, l2, barrier), world, "cuda")
    del gch

    bad = [i for i, x in enumerate(inst) if int(x.lay.err_word.item()) != 0]
    if bad:
        raise RuntimeError(f"device-side checks flagged instances {bad[:8]} "
                           f"(err words {[int(inst[i].lay.err_word.item()) for i in bad[:8]]})")

    # ---- end to end through the public call, in the headline's mode and over
    #      exactly K steps: every step's inputs come from pinned host memory and
    #      its output goes back to pinned host memory.  Zero-copy: the kernel
    #      reads the inputs across the host link itself; also reported: the
    #      same with copy-engine copies.
    set_mode(True, args.split)
    for x in inst:
        x.attach_host(torch)
    h2d = inst[0].in_bytes
    d2h = inst[0].out.numel() * inst[0].out.element_size()
    e2e = {}
    for mode, fn in (("zero_copy", lambda x, s_: x.step_e2e(L, x.ws, s_)),
                     ("copy_engine", lambda x, s_: x.step_e2e_dma(L, x.ws, s_))):
        e_ms = max_over_ranks(_timed_steps(torch, stream, one_stream(K, fn), l2, barrier), world, "cuda")
        e2e[mode] = replica_rate(K * cfg.B, e_ms, world)
    if any(int(x.lay.err_word.item()) for x in inst):
        raise RuntimeError("device-side checks flagged the end-to-end run")

    peak, peak_kind = load_peaks()
    gbs = lambda t_ms, n: step_bytes / (t_ms / n * 1e-3) / 1e9
    achieved = gbs(ms, K)
    if rank != 0:
        return
    cpu = cpu_baseline_sample(args.cpu_seconds) if world == 1 and not args.no_cpu_baseline else None
    clocks = clk.summary(t_wall0, t_wall1)
    rate = lambda t_ms, n: replica_rate(n * cfg.B, t_ms, world)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1)/sqrt(dim) caches and inputs; fp32 state ~ N(0,1))",
        "config": {"workload": WORKLOAD, "B": cfg.B, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "d": cfg.d, "HI": cfg.HI,
                   "dI": cfg.dI, "M": cfg.M, "L": cfg.L, "instances": R, "decode_split": args.split or "library",
                   "timing": "one stream, exactly `steps` steps rotating over independent instances, each "
                             "step declared independent of the launch before it (programmatic dependent "
                             "launch lets consecutive steps overlap)",
                   "l2": f"flushed (a {4 * l2 / 2 ** 20:.0f} MiB write) before every timed region; the steps "
                         f"rotate over instances touching {R * step_bytes / 2 ** 20:.0f} MiB "
                         f"(L2 {l2 / 2 ** 20:.0f} MiB)",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "kernel": "decode_cluster_kernel (whole decode step, one launch)",
                     "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_kind": peak_kind, "nominal_peak": NOMINAL_HBM_GBS,
                     "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
                     "algorithmic_bytes_per_launch": step_bytes,
                     "time_per_launch": "timed region / steps",
                     "traffic": DECODE_TRAFFIC.get(args.split)},
        "steady_state": {"steps": K_steady, "tokens_per_s": rate(ms_ss, K_steady),
                         "us_per_step": ms_ss * 1e3 / K_steady, "frac": gbs(ms_ss, K_steady) / peak,
                         "note": "the headline's stream over more steps (no start-up ramp)"},
        "dependent_chain": {"steps": K_steady, "tokens_per_s": rate(ms_dep, K_steady),
                            "us_per_step": ms_dep * 1e3 / K_steady, "frac": gbs(ms_dep, K_steady) / peak,
                            "decode_split": "library",
                            "note": "one stream, every step waits for the launch before it"},
        "concurrent_chains": {"steps": K_steady, "chains": S, "tokens_per_s": rate(ms_ch, K_steady),
                              "us_per_step": ms_ch * 1e3 / K_steady, "frac": gbs(ms_ch, K_steady) / peak,
                              "note": "a batch of independent layers: S streams, each step waiting for "
                                      "the one before it in its stream"},
        "latency_us_one_step": lat_us,
        "clocks": clocks,
        "e2e": {"value": e2e["zero_copy"], "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": K,
                "mode": "headline's stream; inputs read from pinned host memory by the kernel, output "
                        "written to pinned host memory",
                "copy_engine_value": e2e["copy_engine"]},
        "gpu_launches": K,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def run_prefill(args, rank, world):
    """Timing of the causal prefill workload (16384 tokens, 1.5B shape): not
    the headline metric; used for the prefill kernels' measurements."""
    import torch
    from hybrid_linear_top_b200 import lisa as L
    cfg = get_config("prefill_1p5b_16k")
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    rng = make_rng(cfg.seed, 0)
    st = gen_step(cfg, rng, cfg.T)
    tb = lambda z: torch.from_numpy(np.ascontiguousarray(z)).to("cuda", torch.bfloat16)
    tf = lambda z: torch.from_numpy(np.ascontiguousarray(z)).to("cuda", torch.float32)
    x = dict(q=tb(st.q), k=tb(st.k), v=tb(st.v), kidx=tb(st.kidx), qidx=tb(st.qidx), w=tf(st.w), lam=tf(st.lam))
    lay = L.Layer.allocate(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.HI, cfg.dI, cfg.M, cfg.T, L.LISA_BF16)
    ws = L.alloc_workspace(lay, cfg.T, L.LISA_OP_PREFILL)
    out = torch.empty(cfg.B, cfg.T, cfg.Hq, cfg.d, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(cfg.B, cfg.T, cfg.Hkv, cfg.M, dtype=torch.int32, device="cuda")

    def step():
        L.lisa_prefill(lay, cfg.T, x["q"], x["k"], x["v"], x["kidx"], x["qidx"], x["w"], x["lam"], out, idx, ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    if int(lay.err_word.item()) != 0:
        raise RuntimeError(f"device-side checks flagged the prefill (err word {int(lay.err_word.item())})")
    if rank == 0:
        print(json.dumps({"metric": "LISA prefill tokens/s @16K, M=256", "value": cfg.T * cfg.B / (ms / 1e3),
                          "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                          "ms_per_step": ms, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
                          "config": {"workload": "prefill_1p5b_16k", "T": cfg.T, "M": cfg.M}}), flush=True)


def _decode_bytes(cfg, L, B=None):
    """Algorithmic bytes of one decode step of one layer: algorithmic_bytes()
    per sequence (context L, or the per-sequence lengths L)."""
    Ls = np.broadcast_to(np.asarray(L), (cfg.B if B is None else B,))
    return int(sum(algorithmic_bytes(cfg, int(l)) for l in Ls))


def _fill_layer(L, lay, cfg, n_rows, g, torch):
    bf = torch.bfloat16
    rn = lambda shape, dim: (torch.randn(shape, generator=g, device="cuda") / dim ** 0.5).to(bf)
    lay.k_cache[:, :, :n_rows] = rn((cfg.B, cfg.Hkv, n_rows, cfg.d), cfg.d)
    lay.v_cache[:, :, :n_rows] = rn((cfg.B, cfg.Hkv, n_rows, cfg.d), cfg.d)
    lay.kidx_cache[:, :, :n_rows] = rn((cfg.B, cfg.Hkv, n_rows, cfg.dI), cfg.dI)
    lay.state.copy_(torch.randn(lay.state.shape, generator=g, device="cuda"))


def _step_inputs(cfg, g, torch):
    bf = torch.bfloat16
    rn = lambda shape, dim: (torch.randn(shape, generator=g, device="cuda") / dim ** 0.5).to(bf)
    return dict(q=rn((cfg.B, cfg.Hq, cfg.d), cfg.d), k=rn((cfg.B, cfg.Hkv, cfg.d), cfg.d),
                v=rn((cfg.B, cfg.Hkv, cfg.d), cfg.d), kidx=rn((cfg.B, cfg.Hkv, cfg.dI), cfg.dI),
                qidx=rn((cfg.B, cfg.HI, cfg.dI), cfg.dI), w=torch.rand((cfg.B, cfg.HI), generator=g, device="cuda"),
                lam=torch.randn((cfg.B, cfg.Hq), generator=g, device="cuda"))


def _line(rank, metric, value, unit, args, world, ms_per_step, config, roofline, extra=None):
    if rank != 0:
        return
    line = {"metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1)/sqrt(dim) inputs)",
            "config": config, "roofline": roofline}
    line.update(extra or {})
    print(json.dumps(line), flush=True)


def run_kl(args, rank, world):
    """Stage-2 objective forward (lisa_indexer_kl) over a 16384-token prefix at
    the 1.5B shape: per-head KL of the teacher's attention against the
    indexer's distribution for every token and query head."""
    import torch
    from hybrid_linear_top_b200 import lisa as L
    cfg = get_config("prefill_1p5b_16k")
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    g = torch.Generator(device="cuda")
    g.manual_seed(1000 * rank + 7)
    lay = L.Layer.allocate(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.HI, cfg.dI, cfg.M, cfg.T, L.LISA_BF16)
    _fill_layer(L, lay, cfg, cfg.T, g, torch)
    bf = torch.bfloat16
    q = (torch.randn((cfg.B, cfg.T, cfg.Hq, cfg.d), generator=g, device="cuda") / cfg.d ** 0.5).to(bf)
    qidx = (torch.randn((cfg.B, cfg.T, cfg.HI, cfg.dI), generator=g, device="cuda") / cfg.dI ** 0.5).to(bf)
    w = torch.rand((cfg.B, cfg.T, cfg.HI), generator=g, device="cuda")
    kl = torch.empty(cfg.B, cfg.T, cfg.Hq, dtype=torch.float32, device="cuda")
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            L.lisa_indexer_kl(lay, cfg.T, q, qidx, w, kl, stream)
    gr = _capture(torch, stream, [stream], list(range(args.steps)),
                  lambda i, s_: L.lisa_indexer_kl(lay, cfg.T, q, qidx, w, kl, s_))
    ms = max_over_ranks(_timed_replays(torch, stream, [gr]), world, "cuda") / args.steps
    if int(lay.err_word.item()) or not torch.isfinite(kl).all():
        raise RuntimeError("the KL objective flagged an error")
    pairs = cfg.T * (cfg.T + 1) // 2
    flops = cfg.B * (cfg.Hq * pairs * 2 * cfg.d + cfg.HI * pairs * 2 * cfg.dI)
    tf = flops / (ms * 1e-3) / 1e12
    peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
    peak = float(peaks.get("bf16_tflops", 1590.0))
    _line(rank, "LISA Stage-2 KL objective (forward) tokens/s @16K prefix", replica_rate(cfg.T * cfg.B, ms, world),
          "tokens/s", args, world, ms,
          {"workload": "kl_1p5b_16k", "B": cfg.B, "T": cfg.T, "Hq": cfg.Hq, "HI": cfg.HI,
           "parallelism": f"replicas x{world}"},
          {"bound": "tensor", "kernel": "indexer_kl_kernel (warp MMAs)", "achieved": tf, "peak": peak,
           "unit": "TFLOP/s", "frac": tf / peak, "peak_kind": "measured" if peaks else "fallback",
           "algorithmic_flops_per_call": flops, "traffic": None})


def run_proj(args, rank, world):
    """Projections on either side of the layer at the 1.5B shape (hidden size
    1536): the front-end x -> q, k, v, qidx, kidx, w, gate logits and the
    output projection o -> y, for a 16384-token prefill (tcgen05 GEMMs; the
    headline) and for one decode token (weight streams, reported beside it,
    rotating over weight copies larger than L2)."""
    import torch
    from hybrid_linear_top_b200 import lisa as L
    cfg = get_config("prefill_1p5b_16k")
    Hm = 1536
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    g = torch.Generator(device="cuda")
    g.manual_seed(1000 * rank + 11)
    bf = torch.bfloat16

    def setup(B, T, copies):
        lay = L.Layer.allocate(B, cfg.Hq, cfg.Hkv, cfg.d, cfg.HI, cfg.dI, cfg.M, 16, L.LISA_BF16)
        N = sum(L.proj_widths(lay))
        projs = [L.Proj(Hm, (torch.randn((N, Hm), generator=g, device="cuda") / Hm ** 0.5).to(bf),
                        (torch.randn((Hm, cfg.Hq * cfg.d), generator=g, device="cuda") / (cfg.Hq * cfg.d) ** 0.5).to(bf))
                 for _ in range(copies)]
        x = torch.randn((B, T, Hm), generator=g, device="cuda").to(bf)
        o = {"q": torch.empty(B, T, cfg.Hq, cfg.d, dtype=bf, device="cuda"),
             "k": torch.empty(B, T, cfg.Hkv, cfg.d, dtype=bf, device="cuda"),
             "v": torch.empty(B, T, cfg.Hkv, cfg.d, dtype=bf, device="cuda"),
             "qidx": torch.empty(B, T, cfg.HI, cfg.dI, dtype=bf, device="cuda"),
             "kidx": torch.empty(B, T, cfg.Hkv, cfg.dI, dtype=bf, device="cuda"),
             "w": torch.empty(B, T, cfg.HI, device="cuda"), "lam": torch.empty(B, T, cfg.Hq, device="cuda"),
             "y": torch.empty(B, T, Hm, dtype=bf, device="cuda")}

        def step(i, s_):
            pj = projs[i % copies]
            L.lisa_project_in(lay, 0, pj, T, x, o["q"], o["k"], o["v"], o["qidx"], o["kidx"], o["w"], o["lam"], s_)
            L.lisa_project_out(lay, pj, T, o["q"], o["y"], s_)
        return lay, N, step

    stream = torch.cuda.Stream()
    # prefill-size: T = 16384 rows (inputs and outputs far larger than L2)
    T = cfg.T
    lay, N, step = setup(1, T, 1)
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i, stream)
    gr = _capture(torch, stream, [stream], list(range(args.steps)), step)
    ms = max_over_ranks(_timed_replays(torch, stream, [gr]), world, "cuda") / args.steps
    flops = 2 * T * Hm * N + 2 * T * cfg.Hq * cfg.d * Hm
    tf = flops / (ms * 1e-3) / 1e12
    # decode-size: one token, rotating over weight copies that exceed 4x L2
    wbytes = 2 * (N * Hm + Hm * cfg.Hq * cfg.d)
    copies = int(4 * 126 * 2 ** 20 // wbytes) + 1
    lay1, _, step1 = setup(1, 1, copies)
    n1 = 20 * copies
    g1 = _capture(torch, stream, [stream], list(range(n1)), step1)
    g1.replay()
    ms1 = max_over_ranks(_timed_replays(torch, stream, [g1]), world, "cuda") / n1
    if int(lay.err_word.item()) or int(lay1.err_word.item()):
        raise RuntimeError("a projection flagged an error")
    peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
    peak = float(peaks.get("bf16_tflops", 1590.0))
    hbm, hbm_kind = load_peaks()
    dec_gbs = (wbytes + 2 * (Hm + N + cfg.Hq * cfg.d + Hm)) / (ms1 * 1e-3) / 1e9
    _line(rank, "LISA projection front-end + output projection tokens/s @16K-token prefill",
          replica_rate(T, ms, world), "tokens/s", args, world, ms,
          {"workload": "proj_1p5b_16k", "T": T, "Hm": Hm, "N_in": N, "parallelism": f"replicas x{world}"},
          {"bound": "tensor", "kernel": "proj_tc_kernel<256> (tcgen05), front-end + output projection",
           "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
           "peak_kind": "measured" if peaks else "fallback", "algorithmic_flops_per_step": flops, "traffic": None},
          {"decode_token": {"us_per_token": ms1 * 1e3, "achieved_gbs": dec_gbs, "peak_gbs": hbm,
                            "frac": dec_gbs / hbm, "peak_kind": hbm_kind, "weight_copies": copies,
                            "kernels": "proj_gemv_kernel (TMA weight stream), both projections"}})


def run_window(args, rank, world):
    """Stage-1 sliding-window variant at the 1.5B decode shape: the last 256
    positions instead of the indexer's top-256 (lisa_decode_step_window),
    16384 cached tokens, 32 concurrent chains over independent instances."""
    import torch
    from hybrid_linear_top_b200 import lisa as L
    cfg = get_config(WORKLOAD)
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    l2 = getattr(torch.cuda.get_device_properties(0), "L2_cache_size", 126 * 2 ** 20)
    M = min(cfg.M, cfg.L)
    small = (cfg.Hq * cfg.d * 2 + 4 * cfg.Hkv * cfg.d * 2 + cfg.Hq * 4 + cfg.Hq * cfg.d * 2)
    step_bytes = cfg.Hkv * M * 2 * cfg.d * 2 + cfg.Hq * cfg.d * cfg.d * 4 * 2 + small
    # instances: enough that the step footprint (window rows, state) exceeds 4x L2
    R = instances_needed(step_bytes, l2)
    inst = [Instance(L, cfg, torch, 2000 * rank + i, None, args.split) for i in range(R)]
    for x in inst:
        x.lay.independent = 1            # one stream of independent steps, as the headline
    stream = torch.cuda.Stream()
    run = lambda x, s_: L.lisa_decode_step_window(x.lay, x.q, x.k, x.v, x.kidx, x.lam, 1, x.out, None, s_)
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            run(inst[i % R], stream)
    per, n_full, tail = plan_graphs(args.steps, R)
    graphs = [_capture(torch, stream, [stream], [inst[i % R] for i in range(per)], run)] * n_full
    if tail:
        graphs.append(_capture(torch, stream, [stream], [inst[i % R] for i in range(tail)], run))
    ms = max_over_ranks(_timed_steps(torch, stream, graphs, l2), world, "cuda")
    if any(int(x.lay.err_word.item()) for x in inst):
        raise RuntimeError("device-side checks flagged the window decode")
    peak, kind = load_peaks()
    per = ms / args.steps
    achieved = step_bytes / (per * 1e-3) / 1e9
    _line(rank, "LISA Stage-1 window decode tokens/s @16K ctx, W=256", replica_rate(args.steps * cfg.B, ms, world),
          "tokens/s", args, world, per,
          {"workload": "window_1p5b_16k", "B": cfg.B, "L": cfg.L, "W": M, "instances": R,
           "timing": "one stream of independent steps, as the headline",
           "decode_split": args.split or "library", "parallelism": f"replicas x{world}"},
          {"bound": "hbm", "kernel": "decode_cluster_kernel (window mode)", "achieved": achieved, "peak": peak,
           "unit": "GB/s", "frac": achieved / peak, "peak_kind": kind, "algorithmic_bytes_per_launch": step_bytes,
           "traffic": None})


def run_ragged(args, rank, world):
    """Qwen2.5-7B-shaped batched decode step: B=32 sequences with context
    lengths drawn uniformly in [4096, 16384] (one lisa_decode_step call)."""
    import torch
    from hybrid_linear_top_b200 import lisa as L
    from lisa_inputs.gen import gen_lengths
    cfg = get_config("ragged_7b_b32")
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    lengths = gen_lengths(cfg, make_rng(cfg.seed, 0))
    step_bytes = _decode_bytes(cfg, lengths)
    l2 = getattr(torch.cuda.get_device_properties(0), "L2_cache_size", 126 * 2 ** 20)
    R = max(2, int(np.ceil(4 * l2 / step_bytes)))
    g = torch.Generator(device="cuda")
    g.manual_seed(1000 * rank + 3)
    lays, xs = [], []
    for _ in range(R):
        lay = L.Layer.allocate(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.HI, cfg.dI, cfg.M, cfg.L_max, L.LISA_BF16,
                               decode_split=args.split)
        _fill_layer(L, lay, cfg, cfg.L_max - 1, g, torch)
        lay.pos.copy_(torch.from_numpy((lengths - 1).astype(np.int32)))
        lays.append(lay)
        xs.append(_step_inputs(cfg, g, torch))
    out = torch.empty(cfg.B, cfg.Hq, cfg.d, dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.Stream()

    def one(i, s_):
        x = xs[i % R]
        L.lisa_decode_step(lays[i % R], x["q"], x["k"], x["v"], x["kidx"], x["qidx"], x["w"], x["lam"], 1, out,
                           None, None, s_)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            one(i, stream)
    n_graph = min(args.steps, 64 * R)
    gr = _capture(torch, stream, [stream], list(range(n_graph)), one)
    reps, tail_n = divmod(args.steps, n_graph)
    tail = _capture(torch, stream, [stream], list(range(tail_n)), one) if tail_n else None
    gr.replay()
    ms = _timed_replays(torch, stream, [gr] * reps + ([tail] if tail else []))
    ms = max_over_ranks(ms, world, "cuda")
    if any(int(l.err_word.item()) for l in lays):
        raise RuntimeError("device-side checks flagged the ragged decode")
    peak, kind = load_peaks()
    per = ms / args.steps
    achieved = step_bytes / (per * 1e-3) / 1e9
    _line(rank, "LISA decode tokens/s, 7B shape, B=32 ragged 4K-16K, M=256", replica_rate(args.steps * cfg.B, ms, world),
          "tokens/s", args, world, per,
          {"workload": "ragged_7b_b32", "B": cfg.B, "L_range": [cfg.L_lo, cfg.L_hi], "M": cfg.M, "instances": R,
           "decode_split": args.split or "library", "parallelism": f"replicas x{world}"},
          {"bound": "hbm", "kernel": "decode_cluster_kernel", "achieved": achieved, "peak": peak, "unit": "GB/s",
           "frac": achieved / peak, "peak_kind": kind, "algorithmic_bytes_per_launch": step_bytes, "traffic": None})


def run_longcot(args, rank, world):
    """Qwen2.5-7B-shaped long chain of thought: 28 independent layers, B=8,
    16384 prefilled rows, 1024 sequential decode steps per layer (each
    appending its token); the layers run as 28 concurrent chains."""
    import torch
    from hybrid_linear_top_b200 import lisa as L
    cfg = get_config("longcot_7b_28l")
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    n_steps = cfg.n_decode
    g = torch.Generator(device="cuda")
    g.manual_seed(1000 * rank + 4)
    lays, pools = [], []
    for _ in range(cfg.layers):
        lay = L.Layer.allocate(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.HI, cfg.dI, cfg.M, cfg.L_max, L.LISA_BF16,
                               decode_split=args.split)
        _fill_layer(L, lay, cfg, cfg.L, g, torch)
        lays.append(lay)
        pools.append([_step_inputs(cfg, g, torch) for _ in range(4)])     # step inputs cycle over 4 draws
    # pos of step n = L + n for every sequence: one 16-byte aligned row per step
    pos_all = (torch.arange(n_steps, device="cuda", dtype=torch.int32)[:, None] + cfg.L).repeat(1, cfg.B).contiguous()
    out = torch.empty(cfg.layers, cfg.B, cfg.Hq, cfg.d, dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.Stream()
    chains = [torch.cuda.Stream() for _ in range(cfg.layers)]

    def one(item, s_):
        l, n = item
        lay = lays[l]
        lay.pos = pos_all[n]
        x = pools[l][n % 4]
        L.lisa_decode_step(lay, x["q"], x["k"], x["v"], x["kidx"], x["qidx"], x["w"], x["lam"], 1, out[l], None,
                           None, s_)

    block = 64
    graphs = []
    for n0 in range(0, n_steps, block):
        items = [(l, n) for n in range(n0, min(n_steps, n0 + block)) for l in range(cfg.layers)]
        graphs.append(_capture(torch, stream, chains, items, one))
    # warm-up: one pass over a few steps (rewrites the same rows the timed pass writes)
    graphs[0].replay()
    torch.cuda.synchronize()
    ms = _timed_replays(torch, stream, graphs)
    ms = max_over_ranks(ms, world, "cuda")
    if any(int(l.err_word.item()) for l in lays):
        raise RuntimeError("device-side checks flagged the long-CoT decode")
    total_bytes = cfg.layers * sum(_decode_bytes(cfg, cfg.L + n + 1) for n in range(n_steps))
    peak, kind = load_peaks()
    achieved = total_bytes / (ms * 1e-3) / 1e9
    _line(rank, "LISA long-CoT decode tokens/s, 7B shape, 28 layers, B=8, 16K->17K, M=256",
          replica_rate(cfg.B * n_steps, ms, world), "tokens/s", args, world, ms / n_steps,
          {"workload": "longcot_7b_28l", "B": cfg.B, "layers": cfg.layers, "steps": n_steps, "L0": cfg.L,
           "decode_split": args.split or "library", "concurrent_chains": cfg.layers,
           "parallelism": f"replicas x{world}"},
          {"bound": "hbm", "kernel": "decode_cluster_kernel", "achieved": achieved, "peak": peak, "unit": "GB/s",
           "frac": achieved / peak, "peak_kind": kind, "algorithmic_bytes_total": total_bytes, "traffic": None},
          {"note": "steps = sequential decode steps of every layer; value = B x steps / time of the whole stack"})


def run_stack(args, rank, world):
    """The long-CoT shape as a stack of whole layers: 28 layers of the 7B
    shape (hidden size 3584), B=8, 16384 prefilled rows, sequential decode
    steps, every launch in one stream in layer order.  Per step and layer:
    the projection front-end of a hidden state, the decode step (appending
    its token) and the output projection.  The hidden inputs are drawn
    afresh per layer: a chain of random-init layers without the norm and
    residual the pages do not describe grows without bound (the linear
    branch's state amplifies), so the layers are not chained numerically."""
    import torch
    from hybrid_linear_top_b200 import lisa as L
    cfg = get_config("longcot_7b_28l")
    Hm = 3584
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    n_steps = args.steps
    g = torch.Generator(device="cuda")
    g.manual_seed(1000 * rank + 12)
    bf = torch.bfloat16
    lays, projs = [], []
    for _ in range(cfg.layers):
        lay = L.Layer.allocate(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.HI, cfg.dI, cfg.M, cfg.L + n_steps + 1,
                               L.LISA_BF16, decode_split=0)      # one stream: the library's (latency) choice
        _fill_layer(L, lay, cfg, cfg.L, g, torch)
        lays.append(lay)
        N = sum(L.proj_widths(lay))
        projs.append(L.Proj(Hm, (torch.randn((N, Hm), generator=g, device="cuda") / Hm ** 0.5).to(bf),
                            (torch.randn((Hm, cfg.Hq * cfg.d), generator=g, device="cuda") /
                             (cfg.Hq * cfg.d) ** 0.5).to(bf)))
    x0 = [torch.randn((cfg.B, Hm), generator=g, device="cuda").to(bf) for _ in range(4)]
    hid = torch.empty(cfg.B, Hm, dtype=bf, device="cuda")           # a layer's output projection
    B_, Hq, Hkv, d, HI, dI = cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.HI, cfg.dI
    t_in = {"q": torch.empty(B_, Hq, d, dtype=bf, device="cuda"), "k": torch.empty(B_, Hkv, d, dtype=bf, device="cuda"),
            "v": torch.empty(B_, Hkv, d, dtype=bf, device="cuda"),
            "qidx": torch.empty(B_, HI, dI, dtype=bf, device="cuda"),
            "kidx": torch.empty(B_, Hkv, dI, dtype=bf, device="cuda"),
            "w": torch.empty(B_, HI, device="cuda"), "lam": torch.empty(B_, Hq, device="cuda")}
    out = torch.empty(B_, Hq, d, dtype=bf, device="cuda")
    pos_all = (torch.arange(n_steps, device="cuda", dtype=torch.int32)[:, None] + cfg.L).repeat(1, cfg.B).contiguous()
    stream = torch.cuda.Stream()

    def one(n, s_):
        for l in range(cfg.layers):
            lay, pj = lays[l], projs[l]
            lay.pos = pos_all[n]
            src = x0[(n + l) % 4]
            L.lisa_project_in(lay, 0, pj, 1, src, t_in["q"], t_in["k"], t_in["v"], t_in["qidx"], t_in["kidx"],
                              t_in["w"], t_in["lam"], s_)
            L.lisa_decode_step(lay, t_in["q"], t_in["k"], t_in["v"], t_in["kidx"], t_in["qidx"], t_in["w"],
                               t_in["lam"], 1, out, None, None, s_)
            L.lisa_project_out(lay, pj, 1, out, hid, s_)

    block = 16
    graphs = [_capture(torch, stream, [stream], list(range(n0, min(n_steps, n0 + block))), one)
              for n0 in range(0, n_steps, block)]
    graphs[0].replay()                     # warm-up (rewrites the rows the timed pass writes)
    torch.cuda.synchronize()
    ms = max_over_ranks(_timed_replays(torch, stream, graphs), world, "cuda")
    if any(int(l.err_word.item()) for l in lays) or not torch.isfinite(hid.float()).all():
        raise RuntimeError("the chained stack flagged an error")
    wbytes = cfg.layers * sum(2 * p_.W_in.numel() + 2 * p_.W_o.numel() for p_ in projs[:1])
    lisa_bytes = cfg.layers * sum(_decode_bytes(cfg, cfg.L + n + 1) for n in range(n_steps))
    total_bytes = lisa_bytes + n_steps * wbytes
    peak, kind = load_peaks()
    achieved = total_bytes / (ms * 1e-3) / 1e9
    _line(rank, "LISA 28-layer stack decode tokens/s with projections, 7B shape, B=8, 16K context, M=256",
          replica_rate(cfg.B * n_steps, ms, world), "tokens/s", args, world, ms / n_steps,
          {"workload": "stack_7b_28l", "B": cfg.B, "layers": cfg.layers, "steps": n_steps, "L0": cfg.L, "Hm": Hm,
           "decode_split": "library", "parallelism": f"replicas x{world}"},
          {"bound": "hbm", "kernel": "whole stack: projections + decode_cluster_kernel per layer", "achieved": achieved,
           "peak": peak, "unit": "GB/s", "frac": achieved / peak, "peak_kind": kind,
           "algorithmic_bytes_total": total_bytes, "traffic": None},
          {"note": "per layer: front-end, decode step, output projection; one stream in layer order; "
                   "value = B x steps / time of the stack",
           "us_per_layer": ms * 1e3 / (n_steps * cfg.layers)})


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="lisa", choices=["lisa", "reference"])
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=[WORKLOAD, "prefill_1p5b_16k", "ragged_7b_b32", "longcot_7b_28l", "window_1p5b_16k", "kl_1p5b_16k",
                             "proj_1p5b_16k", "stack_7b_28l"])
    ap.add_argument("--instances", type=int, default=0)
    ap.add_argument("--streams", type=int, default=32)
    ap.add_argument("--split", type=int, default=4, choices=[0, 4, 8, 16, 32, 64])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.steps is None:
        args.steps = {WORKLOAD: 2000, "prefill_1p5b_16k": 20, "ragged_7b_b32": 2000,
                      "longcot_7b_28l": 1024, "window_1p5b_16k": 20000, "kl_1p5b_16k": 5,
                      "proj_1p5b_16k": 50, "stack_7b_28l": 256}[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        elif args.workload == "prefill_1p5b_16k":
            run_prefill(args, rank, world)
        elif args.workload == "ragged_7b_b32":
            run_ragged(args, rank, world)
        elif args.workload == "longcot_7b_28l":
            run_longcot(args, rank, world)
        elif args.workload == "window_1p5b_16k":
            run_window(args, rank, world)
        elif args.workload == "kl_1p5b_16k":
            run_kl(args, rank, world)
        elif args.workload == "proj_1p5b_16k":
            run_proj(args, rank, world)
        elif args.workload == "stack_7b_28l":
            run_stack(args, rank, world)
        else:
            run_lisa(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
