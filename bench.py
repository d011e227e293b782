"""Benchmark of the LiftQuant lift-then-project layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lq|reference]

Workload at N=1: the LQ-24/10 decode layer (in=5120, out=13824, lifted K=12288,
batch 1, 40 orthogonal 128x128 whitening blocks, bf16 activations). One step is
one pass of the decode hot path over one batch through one C call,
lq_lift_gemv: whitening + lift, then the 1-bit GEMV with the row-scale
epilogue (two kernels, the GEMV a programmatic dependent of the lift). The
metric is packed-weight GB/s: packed sign bytes (out*K/8) per step divided by
the step time.

Timing: weights (packed signs, s, T^-1) rotate over enough distinct copies to
exceed 3x the L2 size, so every step reads its weights from HBM. Steps are
replayed from CUDA graphs (16 steps per graph, one per weight copy) so that
host launch overhead does not pace the GPU; the timed region is bracketed by a
barrier and device synchronizes and timed with CUDA events on the launching
stream; the reported time is the max over ranks. With N>1 every rank runs an
independent replica (the layer needs no exchange between GPUs), so scaling is
weak and the value sums all ranks' bytes over the slowest rank's time.

One JSON line is printed by rank 0; it carries the roofline of the dominant
kernel (the GEMV, timed alone right after the step region), the end-to-end
number (pinned-host activations in, output back to the host, inside the timed
region: zero-copy, the lift loading and the GEMV storing the host buffers, with
the copy-engine variant beside it), sampled SM clocks, the float64 oracle timed on the host cores, and
secondary results (prefill GEMM TFLOP/s, the LQ-20/8 batch sweep, the LQ-D/8
bit-width sweep, the Kronecker-whitened lift, the encoder's seconds per
million weights).
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from datagen import CONFIGS, make_layer  # noqa: E402

STEPS_PER_GRAPH = 16
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "decode GEMV packed-weight GB/s (% of HBM) and prefill TFLOP/s, per LQ-D/d"


def workload_config(cfg, name, world, shard=False):
    return {"workload": name, "in": cfg.in_dim, "out": cfg.out, "d": cfg.d, "D": cfg.D, "K": cfg.K,
            "batch": 1, "tblk": cfg.tblk,
            "step": ("lq_lift_gemv on this rank's rows + all-gather of the outputs" if shard
                     else "lq_lift_gemv (lift + gemv)"),
            "parallelism": f"rows{world}" if shard else f"replicas{world}",
            "arith": "lift fp32; u as 32-bit fixed point in four int8 digit planes (quantized inside each "
                     "GEMV CTA); u8 x s8 -> s32 mma.sync (exact); fp32 output"}


# ------------------------------------------------------------------ helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def source_digest(paths):
    """sha256 prefix over the named source files, in order (comma-separated list)."""
    import hashlib
    h = hashlib.sha256()
    for p in paths.split(","):
        with open(os.path.join(ROOT, p), "rb") as src:
            h.update(src.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_key):
    """DRAM bytes per launch from an ncu capture recorded in profiles/traffic.txt, or None
    when absent or when any source the kernel is built from has changed since the
    capture (sha256 prefix over the listed files)."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        with open(path) as f:
            for line in f:
                parts = line.split()
                if len(parts) == 4 and parts[0] == kernel_key:
                    if source_digest(parts[1]) != parts[2]:
                        return None
                    return float(parts[3])
    except OSError:
        pass
    return None


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._reader = threading.Thread(target=self._read, daemon=True)
            self._reader.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, which):
        if which == "begin":
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            rows.append((ts, parts))
        if not rows:
            return None
        inside = [r for r in rows if self.t0 is not None and self.t0 <= r[0] <= (self.t1 or r[0])]
        use = inside if inside else rows
        sm = [float(p[1]) for _, p in use if p[1].replace(".", "").isdigit()]
        smax = max(float(p[2]) for _, p in use if p[2].replace(".", "").isdigit())
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for _, p in use:
            for n, v in zip(names, p[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(use), "samples_in_timed_region": len(inside)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x, world, device=None):
    """Max of a float over all ranks (identity when world == 1)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ------------------------------------------------------------------ GPU workloads

class DecodeLayer:
    """Device buffers of one decode workload, rotated over `copies` weight copies."""

    def __init__(self, lq, cfg, batch, copies, torch):
        L = make_layer(cfg, batch)
        self.cfg, self.batch = cfg, batch
        dev = torch.device("cuda")
        pk = torch.from_numpy(L.packed.view(np.int32)).to(dev)
        s = torch.from_numpy(L.s).to(dev)
        tinv = torch.from_numpy(L.tinv).to(dev) if L.tinv is not None else None
        self.packed = [pk] + [pk.clone() for _ in range(copies - 1)]
        self.s = [s] + [s.clone() for _ in range(copies - 1)]
        self.tinv = [tinv] + [tinv.clone() if tinv is not None else None for _ in range(copies - 1)]
        self.M = torch.from_numpy(L.M).to(dev)
        if L.a_dtype == "bf16":
            a = torch.from_numpy(L.a.view(np.int16)).to(dev).view(torch.bfloat16)
        else:
            a = torch.from_numpy(L.a).to(dev)
        self.a = [a.clone() for _ in range(copies)]
        self.a_host = [x.cpu().pin_memory() for x in self.a]
        self.u = [torch.empty((batch, cfg.K), dtype=torch.float32, device=dev) for _ in range(copies)]
        self.o = [torch.empty((batch, cfg.out), dtype=torch.float32, device=dev) for _ in range(copies)]
        self.o_host = [torch.empty((batch, cfg.out), dtype=torch.float32).pin_memory() for _ in range(copies)]
        # one workspace serves every step: the steps run in stream order
        self.ws = lq.gemv_workspace(cfg.out, cfg.K, batch, dev)
        self.copies = copies
        self.lq = lq

    def step(self, i, with_copies=False):
        lq, c = self.lq, self.cfg
        if with_copies:
            self.a[i].copy_(self.a_host[i], non_blocking=True)
        lq.lift_gemv(self.a[i], self.M, self.packed[i], self.s[i], c.K, tinv=self.tinv[i], u=self.u[i], out=self.o[i],
                     workspace=self.ws)
        if with_copies:
            self.o_host[i].copy_(self.o[i], non_blocking=True)

    def step_zero_copy(self, i):
        """Host buffers in and out, no copy-engine transfers: the lift loads a
        from pinned host memory and the GEMV stores o there."""
        lq, c = self.lq, self.cfg
        lq.lift_gemv(self.a_host[i], self.M, self.packed[i], self.s[i], c.K, tinv=self.tinv[i], u=self.u[i],
                     out=self.o_host[i], workspace=self.ws)

    def gemv_only(self, i):
        self.lq.gemv(self.packed[i], self.s[i], self.u[i], out=self.o[i], workspace=self.ws)

    @property
    def packed_bytes(self):
        return self.cfg.out * self.cfg.K // 8


def shard_rows(out, world, rank):
    from bit_lifted_gemm_b200.sharded import row_range
    r0, r1 = row_range(out, world, rank)
    return r1 - r0


class ShardedLayer:
    """Row-sharded decode (bit_lifted_gemm_b200.sharded.ShardedDecode), one
    instance per weight copy: every rank lifts the whole batch, contracts its
    rows and all-gathers the outputs."""

    def __init__(self, lq, cfg, copies, torch, world, rank):
        from bit_lifted_gemm_b200.sharded import ShardedDecode
        L = make_layer(cfg, 1)
        dev = torch.device("cuda")
        pk = torch.from_numpy(L.packed.view(np.int32))
        s = torch.from_numpy(L.s)
        tinv = torch.from_numpy(L.tinv).to(dev) if L.tinv is not None else None
        M = torch.from_numpy(L.M).to(dev)
        self.parts = [ShardedDecode(pk, s, M, cfg.K, tinv=tinv, batch=1) for _ in range(copies)]
        a = torch.from_numpy(L.a.view(np.int16)).to(dev).view(torch.bfloat16) if L.a_dtype == "bf16" \
            else torch.from_numpy(L.a).to(dev)
        self.a = [a.clone() for _ in range(copies)]

    def step(self, i):
        self.parts[i].step(self.a[i])

    def gemv_only(self, i):
        self.parts[i].gemv_only()


def copies_for(bytes_per_copy, l2_bytes):
    return max(STEPS_PER_GRAPH, int(np.ceil(3 * l2_bytes / bytes_per_copy)))


def capture(torch, fn, n):
    """CUDA graph of fn(0..n-1) on a side stream (each fn launches through the C ABI)."""
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for i in range(n):   # warm-up outside capture (sets kernel attributes once)
            fn(i)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        for i in range(n):
            fn(i)
    torch.cuda.synchronize()
    return g


def time_graph(torch, graph, reps, per_rep):
    """ms per unit: `reps` replays, each doing `per_rep` units, timed with events."""
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(st)
    for _ in range(reps):
        graph.replay()
    e1.record(st)
    e1.synchronize()
    return e0.elapsed_time(e1) / (reps * per_rep)


# ------------------------------------------------------------------ oracle on host cores

def oracle_sample(cfg_name, budget_s, nthreads):
    """The float64 oracle on the host: whitening + lift + contraction of the decode
    layer, on as many output rows as fit in `budget_s`. Returns (GB/s of packed
    weights, description)."""
    import oracle
    cfg = CONFIGS[cfg_name]
    L = make_layer(cfg, 1)
    a = oracle.to_f64(L.a, L.a_dtype)
    t = None if L.tinv is None else oracle.to_f64(L.tinv)
    M = oracle.to_f64(L.M)
    # calibrate on 64 rows
    t0 = time.perf_counter()
    u, _ = oracle.forward(L.packed[:64], L.s[:64], a, t, M, cfg.K, nthreads)
    dt = time.perf_counter() - t0
    rows = int(min(cfg.out, max(64, 64 * budget_s / max(dt, 1e-6))))
    # whole passes over the sample, repeated until they fill most of the budget
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.forward(L.packed[:rows], L.s[:rows], a, t, M, cfg.K, nthreads)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= 0.8 * budget_s or dt / reps * (reps + 1) > budget_s:
            break
    gbs = reps * rows * cfg.K / 8 / dt / 1e9
    return gbs, dt, (f"{cfg_name}: whitening + lift + sign contraction of {rows} of {cfg.out} rows, batch 1, "
                     f"{reps} pass(es)")


def reference_arm(args, world, rank):
    """`--impl reference`: the float64 oracle on the host cores as the reference arm."""
    if rank != 0:
        return
    import oracle
    nthreads = oracle.threads_available()
    total_budget = 90.0
    per_step = total_budget / max(1, args.steps + args.warmup)
    for _ in range(args.warmup):
        oracle_sample(args.workload, per_step, nthreads)
    vals, times = [], []
    for _ in range(args.steps):
        v, dt, desc = oracle_sample(args.workload, per_step, nthreads)
        vals.append(v)
        times.append(dt)
    value = float(np.median(vals))
    cfg = CONFIGS[args.workload]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": float(np.median(times) * 1e3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(cfg, args.workload, args.gpus),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": nthreads, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ main arm

def bench_decode_sweep(torch, lq, name, batches, l2, reps=50):
    cfg = CONFIGS[name]
    res = {}
    for b in batches:
        probe = make_layer(cfg, b, packed=False)
        per_copy = cfg.out * cfg.K // 8 + (probe.tinv.nbytes if probe.tinv is not None else 0)
        layer = DecodeLayer(lq, cfg, b, copies_for(per_copy, l2), torch)
        g = capture(torch, layer.step, STEPS_PER_GRAPH)
        gg = capture(torch, layer.gemv_only, STEPS_PER_GRAPH)
        for _ in range(3):
            g.replay()
        ms_step = time_graph(torch, g, reps, STEPS_PER_GRAPH)
        ms_gemv = time_graph(torch, gg, reps, STEPS_PER_GRAPH)
        res[str(b)] = {"step_us": ms_step * 1e3, "gemv_us": ms_gemv * 1e3,
                       "gemv_GBps": layer.packed_bytes / (ms_gemv * 1e-3) / 1e9,
                       "layer_tokens_per_s": b / (ms_step * 1e-3)}
        traffic = profiled_traffic(f"gemv_{name}_b{b}")
        if traffic is not None:
            # DRAM bytes of one GEMV launch (ncu) over the packed weights it streams
            res[str(b)]["traffic_over_weights"] = traffic / (cfg.out * cfg.K // 8)
        del g, gg, layer
        torch.cuda.empty_cache()
    return res


def bench_kron(torch, lq, l2, reps=50):
    """LQ-24/10 with the Kronecker-factored whitening (64 x 80 factors of T^-1):
    the decode lift alone and lift + GEMV at batch 1 (weights rotating as in the
    main step), and the lift of a 2048-token prefill (L2 flushed before each)."""
    from datagen import make_kron_factors
    cfg = CONFIGS["decode_lq24_10"]
    dev = torch.device("cuda")
    kf = make_kron_factors(cfg.in_dim, 64, cfg.d, cfg.index)
    q1, q2, r1, r2 = (torch.from_numpy(x).to(dev) for x in (kf.q1, kf.q2, kf.r1, kf.r2))
    layer = DecodeLayer(lq, cfg, 1, copies_for(cfg.out * cfg.K // 8, l2), torch)

    def lift(i):
        lq.lift_activations_kron(layer.a[i], q1, q2, layer.M, cfg.K, r1=r1, r2=r2, out=layer.u[i])

    def step(i):
        lift(i)
        layer.gemv_only(i)

    g_l = capture(torch, lift, STEPS_PER_GRAPH)
    g_s = capture(torch, step, STEPS_PER_GRAPH)
    for _ in range(3):
        g_s.replay()
    ms_lift = time_graph(torch, g_l, reps, STEPS_PER_GRAPH)
    ms_step = time_graph(torch, g_s, reps, STEPS_PER_GRAPH)
    del g_l, g_s, layer

    tokens = 2048
    L = make_layer(CONFIGS["prefill_lq24_10"], tokens, packed=False)
    a = torch.from_numpy(L.a.view(np.int16)).to(dev).view(torch.bfloat16)
    M = torch.from_numpy(L.M).to(dev)
    u = torch.empty((tokens, cfg.K), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(int(400e6) // 4, dtype=torch.float32, device=dev)
    st = torch.cuda.current_stream()
    for _ in range(3):
        lq.lift_activations_kron(a, q1, q2, M, cfg.K, r1=r1, r2=r2, u_dtype="bf16", out=u)
    times = []
    for _ in range(10):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        lq.lift_activations_kron(a, q1, q2, M, cfg.K, r1=r1, r2=r2, u_dtype="bf16", out=u)
        e1.record(st)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    ms_pre = float(np.median(times))
    n1, n2 = kf.q1.shape[0], kf.q2.shape[0]
    flop_tok = 2 * cfg.in_dim * (n1 + n2) + 2 * cfg.in_dim // cfg.d * cfg.d * cfg.D
    del flush, u, a
    torch.cuda.empty_cache()
    return {"factors": f"{n1}x{n1} and {n2}x{n2}",
            "decode_b1": {"lift_us": ms_lift * 1e3, "step_us": ms_step * 1e3,
                          "step_GBps": cfg.out * cfg.K // 8 / (ms_step * 1e-3) / 1e9},
            "prefill_2048": {"lift_us": ms_pre * 1e3, "lift_TFLOPs": tokens * flop_tok / (ms_pre * 1e-3) / 1e12}}


def bench_encode(torch, lq):
    """Encoder (offline): seconds per million weights for LQ-24/10, LQ-16/8,
    LQ-32/16 and LQ-32/20 on seeded Gaussian weights and projections, each sample
    sized to a second or less (the cost per block grows as 2^(D-d))."""
    dev = torch.device("cuda")
    res = {}
    for name, d, D, rows, in_dim in (("lq24_10", 10, 24, 26, 5120), ("lq16_8", 8, 16, 256, 4096),
                                     ("lq32_16", 16, 32, 32, 4096), ("lq32_20", 20, 32, 256, 4000)):
        g = np.random.default_rng(0x4C51 + D)
        M = torch.from_numpy((g.standard_normal((d, D)) / np.sqrt(D)).astype(np.float32)).to(dev)
        w = torch.from_numpy(g.standard_normal((rows, in_dim)).astype(np.float32)).to(dev)
        K = lq.lifted_dim(in_dim, d, D)
        lq.encode(w[:1, :d * 64].contiguous(), M, lq.lifted_dim(d * 64, d, D))  # load the module
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        lq.encode(w, M, K)
        e1.record()
        e1.synchronize()
        sec = e0.elapsed_time(e1) * 1e-3
        res[name] = {"weights": rows * in_dim, "seconds": sec, "seconds_per_1M_weights": sec / (rows * in_dim) * 1e6,
                     "patterns_per_block": 1 + 2 ** (D - d)}
    return res


def bench_prefill(torch, lq, name, tokens, reps=10):
    cfg = CONFIGS[name]
    L = make_layer(cfg, tokens)
    dev = torch.device("cuda")
    pk = torch.from_numpy(L.packed.view(np.int32)).to(dev)
    s = torch.from_numpy(L.s).to(dev)
    tinv = torch.from_numpy(L.tinv).to(dev)
    M = torch.from_numpy(L.M).to(dev)
    a = torch.from_numpy(L.a.view(np.int16)).to(dev).view(torch.bfloat16)
    u = torch.empty((tokens, cfg.K), dtype=torch.bfloat16, device=dev)
    o = torch.empty((tokens, cfg.out), dtype=torch.float32, device=dev)
    flush = torch.empty(int(400e6) // 4, dtype=torch.float32, device=dev)
    st = torch.cuda.current_stream()

    def t_of(fn):
        for _ in range(3):
            fn()
        times = []
        for _ in range(reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
            fn()
            e1.record(st)
            e1.synchronize()
            times.append(e0.elapsed_time(e1))
        return float(np.median(times))

    ms_lift = t_of(lambda: lq.lift_activations(a, M, cfg.K, tinv=tinv, u_dtype="bf16", out=u))
    ms_gemm = t_of(lambda: lq.gemm(pk, s, u, out=o))
    flops = 2.0 * tokens * cfg.out * cfg.K
    return {"tokens": tokens, "lift_us": ms_lift * 1e3, "gemm_us": ms_gemm * 1e3,
            "gemm_TFLOPs": flops / (ms_gemm * 1e-3) / 1e12,
            "layer_tokens_per_s": tokens / ((ms_lift + ms_gemm) * 1e-3)}


GRAPH_STEPS = 1024      # steps per CUDA graph of the timed region
GEMV_LAUNCHES = 2048    # GEMV-alone launches behind the roofline, whatever --steps is
# Kernels of this library per timed step: the lift and the GEMV. At one column the
# GEMV is the mma.sync kernel, which quantizes u inside its CTAs and covers K in one
# launch for every decode layer timed here (the ncu launch list of the step shows
# the two); the row-sharded mode runs the same two per rank plus an NCCL all-gather.
LAUNCHES_PER_STEP = 2


def spawn_ranks(args):
    """`--gpus N` with N > 1 outside a launcher: start N ranks with torch.distributed.run."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + sys.argv[1:]
    os.execv(sys.executable, cmd)


class StepPlan:
    """Exactly n steps as replays of one GRAPH_STEPS-step graph and one graph of
    the remainder; step i of the run uses weight copy i % copies."""

    def __init__(self, torch, fn, n, copies, full=None):
        self.n = n
        self.full = full if full is not None else (
            capture(torch, fn, GRAPH_STEPS) if n >= GRAPH_STEPS else None)
        self.nfull, rem = divmod(n, GRAPH_STEPS)
        # the remainder continues the rotation where the full graphs leave it
        off = (self.nfull * GRAPH_STEPS) % copies
        self.rem = capture(torch, lambda i: fn((off + i) % copies), rem) if rem else None

    def replay(self):
        for _ in range(self.nfull):
            self.full.replay()
        if self.rem is not None:
            self.rem.replay()

    def warm(self):
        for g in (self.full, self.rem):
            if g is not None:
                g.replay()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100000)
    ap.add_argument("--warmup", type=int, default=2000)
    ap.add_argument("--impl", default="lq", choices=["lq", "reference"])
    ap.add_argument("--workload", default="decode_lq24_10")
    ap.add_argument("--shard", default="none", choices=["none", "rows"],
                    help="rows: one layer split by output rows over the ranks (strong scaling)")
    ap.add_argument("--no-extra", action="store_true", help="skip the secondary sweeps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.steps < 1:
        raise SystemExit("--steps must be at least 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        spawn_ranks(args)
    world, rank, local = dist_setup()
    if world != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; launch one rank per GPU")

    if args.impl == "reference":
        reference_arm(args, world, rank)
        return

    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    import bit_lifted_gemm_b200 as lq

    peaks, peaks_src = load_peaks()
    props = torch.cuda.get_device_properties(device)
    l2 = getattr(props, "L2_cache_size", 126 * 2**20) or 126 * 2**20
    cfg = CONFIGS[args.workload]
    probe = make_layer(cfg, 1, packed=False)
    shard = args.shard == "rows"
    rows_here = shard_rows(cfg.out, world, rank) if shard else cfg.out
    per_copy = rows_here * cfg.K // 8 + (probe.tinv.nbytes if probe.tinv is not None else 0) + 4 * rows_here
    copies = copies_for(per_copy, l2)
    copies = (copies + STEPS_PER_GRAPH - 1) // STEPS_PER_GRAPH * STEPS_PER_GRAPH
    layer = (ShardedLayer(lq, cfg, copies, torch, world, rank) if shard
             else DecodeLayer(lq, cfg, 1, copies, torch))
    step = layer.step

    plan = StepPlan(torch, lambda i: step(i % copies), args.steps, copies)
    warm = StepPlan(torch, lambda i: step(i % copies), args.warmup, copies, full=plan.full)
    g_gemv = capture(torch, lambda i: layer.gemv_only(i % copies), GEMV_LAUNCHES // 16)
    e_plan = None if shard else StepPlan(torch, lambda i: layer.step_zero_copy(i % copies), args.steps, copies)
    c_plan = None if shard else StepPlan(torch, lambda i: layer.step(i % copies, with_copies=True),
                                         args.steps, copies)

    st = torch.cuda.current_stream()
    warm.replay()
    plan.warm()
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    barrier(world, device)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.mark("begin")
    e0.record(st)
    plan.replay()
    e1.record(st)
    e1.synchronize()
    sampler.mark("end")
    torch.cuda.synchronize()
    barrier(world, device)
    ms_total = max_over_ranks(e0.elapsed_time(e1), world, device)
    clocks = sampler.stop()
    ms_per_step = ms_total / args.steps
    launches = LAUNCHES_PER_STEP * args.steps

    # dominant kernel alone (same stream, after the step region): a fixed number of launches
    g_gemv.replay()
    torch.cuda.synchronize()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(st)
    for _ in range(16):
        g_gemv.replay()
    e3.record(st)
    e3.synchronize()
    gemv_us = max_over_ranks(e2.elapsed_time(e3) * 1e3 / GEMV_LAUNCHES, world, device)

    def time_plan(p):
        p.warm()
        barrier(world, device)
        torch.cuda.synchronize()
        e4, e5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e4.record(st)
        p.replay()
        e5.record(st)
        e5.synchronize()
        return max_over_ranks(e4.elapsed_time(e5), world, device) / p.n

    packed_bytes = cfg.out * cfg.K // 8          # the whole layer's signs, every step
    local_bytes = rows_here * cfg.K // 8         # this rank's share
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    achieved = local_bytes / (gemv_us * 1e-6) / 1e9
    if shard:
        value = packed_bytes / (ms_per_step * 1e-3) / 1e9
        e2e = {"value": None, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0,
               "note": "row-sharded mode times the device path only"}
    else:
        ms_e2e = time_plan(e_plan)
        ms_e2e_copies = time_plan(c_plan)
        torch.cuda.synchronize()
        for i in (0, copies - 1):   # zero-copy output equals the device step's, bit for bit
            layer.step(i)
            layer.step_zero_copy(i)
            torch.cuda.synchronize()
            if not torch.equal(layer.o_host[i], layer.o[i].cpu()):
                raise RuntimeError(f"zero-copy step {i} differs from the device step")
        value = world * packed_bytes / (ms_per_step * 1e-3) / 1e9
        e2e = {"value": world * packed_bytes / (ms_e2e * 1e-3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": int(layer.a[0].numel() * layer.a[0].element_size()),
               "d2h_bytes_per_step": int(layer.o[0].numel() * 4), "ms_per_step": ms_e2e,
               "mode": "zero-copy",
               "note": "CUDA-graph replay of lq_lift_gemv on pinned host buffers: the lift loads the "
                       "activations and the GEMV stores the output across the host link",
               "copy_engine": {"value": world * packed_bytes / (ms_e2e_copies * 1e-3) / 1e9,
                               "ms_per_step": ms_e2e_copies,
                               "note": "H2D copy of the activations, lq_lift_gemv on device buffers, "
                                       "D2H copy of the output"}}
    traffic = profiled_traffic("gemv_decode_lq24_10") if (args.workload == "decode_lq24_10" and not shard) else None
    config = dict(workload_config(cfg, args.workload, world, shard),
                  l2=f"inputs larger than L2: {copies} rotating weight copies "
                     f"({copies * per_copy / 1e6:.0f} MB vs L2 {l2 / 1e6:.0f} MB)",
                  graphs=f"{plan.nfull} x {GRAPH_STEPS}-step graph + {plan.n % GRAPH_STEPS}-step graph")
    result = {
        "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "strong" if shard else "weak", "vs_baseline": None, "dtype": "i8",
        "data": "synthetic", "config": config,
        "roofline": {"bound": "hbm", "kernel": "lq_gemv", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": traffic, "peak_source": peaks_src,
                     "avg_launch_us": gemv_us, "launches_timed": GEMV_LAUNCHES,
                     "algorithmic_bytes_per_launch": local_bytes},
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if shard:
        result["multi_gpu"] = ("unmeasured on hardware beyond one GPU" if world == 1 else
                               f"{world} ranks, all-gather of the outputs over NCCL")

    if rank == 0 and world == 1 and not args.no_extra:
        extra = {}
        pre = bench_prefill(torch, lq, "prefill_lq24_10", 2048)
        bf16 = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        pre["frac_of_bf16_peak"] = pre["gemm_TFLOPs"] / bf16
        extra["prefill_lq24_10"] = pre
        extra["decode_lq20_8"] = bench_decode_sweep(torch, lq, "decode_lq20_8", (1, 2, 4, 8, 16), l2)
        for D in (16, 19, 20, 22, 24):
            n = f"sweep_lq{D}_8"
            extra[n] = {"b1": bench_decode_sweep(torch, lq, n, (1,), l2)["1"],
                        "b64": bench_prefill(torch, lq, n, 64)}
        extra["kron_lq24_10"] = bench_kron(torch, lq, l2)
        extra["encode"] = bench_encode(torch, lq)
        # the bulky record on a line of its own, before the headline
        print(json.dumps({"extra": extra}), flush=True)
        sweep = extra["decode_lq20_8"]
        result["prefill"] = {"tflops": pre["gemm_TFLOPs"], "frac": pre["frac_of_bf16_peak"], "tokens": 2048,
                             "peak_tflops": bf16}
        result["decode_lq20_8_gemv_us"] = {b: round(v["gemv_us"], 2) for b, v in sweep.items()}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        nthreads = oracle.threads_available()
        v, dt, desc = oracle_sample(args.workload, 15.0, nthreads)
        v1, dt1, desc1 = oracle_sample(args.workload, 4.0, 1)
        result["cpu_baseline"] = {"value": v, "unit": "GB/s", "cores": nthreads, "kind": "oracle",
                                  "sample": desc + f" ({dt:.1f} s)",
                                  "single_thread": {"value": v1, "unit": "GB/s", "cores": 1,
                                                    "sample": desc1 + f" ({dt1:.1f} s)"}}

    assert lq.get_device_status() == lq.LQ_OK
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        del plan, warm, g_gemv, layer
        torch.cuda.synchronize()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
