"""Benchmark of the HelixLinear forward on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl hxq|reference]
                    [--workload mamba2|qwen25_3b|vq2d|prefill|tiny] [--no-secondary]

A step is one forward of every layer of the workload (default: the
Mamba2-1.3B-shaped decode pair in_proj 8512x2048 + out_proj 2048x4096, scalar
8-bit codebook, M = 1 token) on seeded synthetic inputs.

value: achieved HBM throughput on algorithmic bytes, GB/s = (indices +
8 B per sidecar entry + codebook + x + y) per step x K / device time of the
K steps. Inputs are resident in HBM when timing starts; each step uses its
own replica of the layers, with enough replicas that their total exceeds 4x
the L2 cache, so every step reads its weights cold from HBM. The K steps are
one CUDA-graph replay timed with CUDA events on the launching stream.

e2e: the same metric through the public call with host buffers: each step
copies x from pinned host memory, runs the forwards and copies y back.

--impl reference times the fp64 CPU oracle (the only reference this method
has) on the host cores over a bounded sample of the same workload.

Multi-GPU: every rank runs its own replica of the workload (the layer does
not shard across GPUs in this build): value = all ranks' bytes / max time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except OSError:
        return FALLBACK_PEAKS, "fallback"


def max_over_ranks(torch, dist, world, value, device):
    """The largest of every rank's `value` (device times: the job ends with the
    slowest rank). All ranks must call it, in the same order."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_step, steps, world, ms_max, scale):
    """Whole-job throughput: the units all `world` replicas processed over the
    slowest rank's time, divided by `scale` (1e9 for GB/s, 1e12 for TFLOP/s)."""
    return units_per_step * steps * world / (ms_max * 1e-3) / scale


def layer_bytes(layer, M):
    N, K, mode = layer["N"], layer["K"], layer["mode"]
    idx = N * K if mode == synthetic.MODE_SCALAR8 else 3 * N * K // 4
    cb = 256 * 4 if mode == synthetic.MODE_SCALAR8 else 4096 * 8
    return idx + 8 * layer["sidecar_pos"].size + cb + 2 * M * K + 4 * M * N


def layer_flops(layer, M):
    return 2.0 * M * layer["N"] * layer["K"]


def workload(name, seed=0, M_override=None):
    """[(label, layer, M)] for one named workload, at the M its bench line uses."""
    out = []
    for lname, layer, Ms in synthetic.config_layers(name, seed):
        Ms_run = Ms if M_override is None else (M_override,)
        for M in Ms_run:
            out.append((f"{lname}/M={M}", layer, M))
    return out


DEFAULT_M = {"mamba2": None, "tiny": 1, "qwen25_3b": 1, "vq2d": 1, "prefill": 2048}

# Layers of a workload that read the same activations (grouped runs: one
# hxq_group_forward per group): attention q, k, v and MLP gate, up.
SHARED_INPUT = {"qwen25_3b": [("q", "k", "v"), ("gate", "up")]}


def item_groups(name, items):
    """Index tuples of the items that share their input, per SHARED_INPUT."""
    names = [lbl.split("/")[0] for lbl, _, _ in items]
    out = []
    for grp in SHARED_INPUT.get(name, []):
        idx = tuple(names.index(n) for n in grp if n in names)
        if len(idx) > 1:
            out.append(idx)
    return out


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"hxq_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            self.proc.wait()
            self.f.close()

    def summary(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = sorted(r[0] for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[2]) if v.lower() == "active"})
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------------------- GPU arm

def _code_only(text):
    """C++ source without comments, trailing blanks and empty lines: what
    the compiler sees of it (the kernel files hold no "//" or "/*" inside
    string literals)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_source_hash():
    """Hash of the kernels' code (comments excluded), recorded with each
    ncu capture so that stale traffic figures are not reported."""
    h = hashlib.sha256()
    for f in ("hxq_gemv.cu", "hxq_tc.cu", "hxq_internal.cuh"):
        with open(os.path.join(ROOT, "vq_compressed_linear_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_key):
    """dram bytes per launch recorded from an ncu capture in profiles/, if the
    kernel sources are unchanged since (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path)).get(kernel_key)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_sha") != kernel_source_hash():
        return None
    return rec.get("dram_bytes_per_launch")


def dominant_kernel(layer, M):
    if M <= 4:
        return "gemv_scalar" if layer["mode"] == synthetic.MODE_SCALAR8 else "gemv_vq2d"
    return ("tc_skinny_" if M <= 32 else "tc_prefill_") + \
        ("scalar" if layer["mode"] == synthetic.MODE_SCALAR8 else "vq2d")


def time_workload(hxq, torch, items, steps, warmup, l2_bytes, stream, soak_s=0.0, max_replica_bytes=48 << 30,
                  groups=()):
    """Device time of `steps` steps (CUDA graph, rotating replicas). `groups`
    (index tuples into items) run as one grouped forward each, on one shared x.
    Returns (ms total, bytes per step, flops per step, launches per step, replicas)."""
    step_bytes = sum(layer_bytes(l, M) for _, l, M in items)
    # a group reads its activations once
    step_bytes -= sum(2 * items[j][2] * items[j][1]["K"] for g in groups for j in g[1:])
    grouped = {j for g in groups for j in g}
    step_flops = sum(layer_flops(l, M) for _, l, M in items)
    dev_bytes_step = sum(l["indices"].size + 8 * l["sidecar_pos"].size for _, l, _ in items)
    R = max(1, math.ceil(4 * l2_bytes / max(1, dev_bytes_step)))
    R = min(R, max(1, max_replica_bytes // max(1, dev_bytes_step)), steps + warmup)
    reps, greps = [], []
    for _ in range(R):
        lins = [hxq.HelixLinear.from_layer(l) for _, l, _ in items]
        reps.append(lins)
        greps.append([hxq.HelixGroup([lins[j] for j in g]) for g in groups])
    xs = [torch.from_numpy(synthetic.activations(M, l["K"], 1).view(np.int16)).cuda() for _, l, M in items]
    ys = [torch.empty((M, l["N"]), dtype=torch.float32, device="cuda") for _, l, M in items]

    def step(i):
        for gi, g in enumerate(groups):
            greps[i % R][gi].forward(xs[g[0]], ys=[ys[j] for j in g], stream=stream)
        for j, lin in enumerate(reps[i % R]):
            if j not in grouped:
                lin.forward(xs[j], ys[j], stream=stream)

    with torch.cuda.stream(stream):
        step(0)  # first launches set kernel attributes outside capture
    torch.cuda.synchronize()
    g_warm, g_run = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_warm, stream=stream):
        for i in range(warmup):
            step(i)
    with torch.cuda.graph(g_run, stream=stream):
        for i in range(steps):
            step(warmup + i)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        g_warm.replay()
        t_end = time.time() + soak_s
        while time.time() < t_end:
            g_run.replay()
            stream.synchronize()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):          # replay() launches on the current stream
        e0.record(stream)
        g_run.replay()
        e1.record(stream)
    e1.synchronize()
    ms = e0.elapsed_time(e1)
    for lin in reps[0]:
        lin.check()
    del g_warm, g_run
    for grep in greps:
        for grp in grep:
            grp.close()
    for rep in reps:
        for lin in rep:
            lin.close()
    return ms, step_bytes, step_flops, len(items) - len(grouped) + len(groups), R


def e2e_workload(hxq, torch, items, steps, warmup, stream, groups=()):
    """Same metric through the host-buffer call (HelixLinear.forward_host,
    i.e. hxq_linear_forward_host: pinned host x in, y out, on the stream) for
    every layer of every step (grouped layers: one x copy per group and
    HelixGroup.forward). Returns (ms, h2d bytes/step, d2h bytes/step)."""
    lins = [hxq.HelixLinear.from_layer(l) for _, l, _ in items]
    grps = [hxq.HelixGroup([lins[j] for j in g]) for g in groups]
    grouped = {j for g in groups for j in g}
    skip_x = {j for g in groups for j in g[1:]}
    xh = [torch.from_numpy(synthetic.activations(M, l["K"], 2).view(np.int16)).pin_memory() for _, l, M in items]
    yh = [torch.empty((M, l["N"]), dtype=torch.float32).pin_memory() for _, l, M in items]
    xd = [torch.empty_like(x, device="cuda") for x in xh]
    yd = [torch.empty_like(y, device="cuda") for y in yh]

    def step():
        for gi, g in enumerate(groups):
            xd[g[0]].copy_(xh[g[0]], non_blocking=True)
            grps[gi].forward(xd[g[0]], ys=[yd[j] for j in g], stream=stream)
            for j in g:
                yh[j].copy_(yd[j], non_blocking=True)
        for j, lin in enumerate(lins):
            if j in grouped:
                continue
            lin.forward_host(xh[j], yh[j], xd[j], yd[j], stream=stream, sync=False)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        e1.synchronize()
    ms = e0.elapsed_time(e1)
    for grp in grps:
        grp.close()
    for lin in lins:
        lin.close()
    h2d = sum(x.numel() * 2 for j, x in enumerate(xh) if j not in skip_x)
    d2h = sum(y.numel() * 4 for y in yh)
    return ms, h2d, d2h


# ----------------------------------------------------------------------------- CPU oracle arm

_X_CACHE = {}


def _x_for(layer, M):
    key = (M, layer["K"])
    if key not in _X_CACHE:
        _X_CACHE[key] = synthetic.activations(M, layer["K"], 1)
    return _X_CACHE[key]


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _timing_oracle():
    """The plain C++ oracle compiled for this host (-O3 -march=native, no
    fused multiply-add), in a temporary directory."""
    import tempfile
    from oracle import hxq_oracle_cpp
    return hxq_oracle_cpp, hxq_oracle_cpp.load_timing_build(tempfile.mkdtemp(prefix="hxq_oracle_"))


def _oracle_pass(cpp, lib, items, frac, threads, offset=0):
    """One pass of the C++ oracle (decode with the sidecar, float64 dot
    products) over `frac` of each layer's output rows (a contiguous slice
    that rotates with `offset`). Returns the (bytes, flops) credited, scaled
    by the fraction of rows done."""
    b = f = 0.0
    for _, layer, M in items:
        N = layer["N"]
        nr = max(1, min(N, int(round(frac * N))))
        r0 = (offset * nr) % N if nr < N else 0
        r1 = min(N, r0 + nr)
        cpp.forward_rows(layer, _x_for(layer, M), r0, r1, threads, lib)
        b += layer_bytes(layer, M) * (r1 - r0) / N
        f += layer_flops(layer, M) * (r1 - r0) / N
    return b, f


def oracle_rate(items, threads, budget_s, cpp=None, lib=None):
    """The C++ oracle's rate on `threads` host threads: repeated passes over
    the workload (a row slice per pass, sized so that one pass takes about
    budget_s / 20) until budget_s of wall time. Returns (GB/s, TFLOP/s,
    passes, fraction of rows per pass, seconds)."""
    if lib is None:
        cpp, lib = _timing_oracle()
    for _, layer, M in items:
        _x_for(layer, M)
    frac = 1.0
    t0 = time.perf_counter()
    _oracle_pass(cpp, lib, items, 0.01, threads)  # size the slice on 1 % of the rows
    one = max(1e-6, (time.perf_counter() - t0) / 0.01)
    frac = min(1.0, budget_s / 20 / one)
    passes, tb, tf, tt = 0, 0.0, 0.0, 0.0
    while tt < budget_s:
        t1 = time.perf_counter()
        b, f = _oracle_pass(cpp, lib, items, frac, threads, passes)
        tt += time.perf_counter() - t1
        tb, tf, passes = tb + b, tf + f, passes + 1
    return tb / tt / 1e9, tf / tt / 1e12, passes, frac, tt


def oracle_sample(items, budget_s=6.0):
    """cpu_baseline: the plain C++ oracle timed on one host thread and on
    all host threads, each for about budget_s."""
    cpp, lib = _timing_oracle()
    n_all = os.cpu_count() or 1
    r1 = oracle_rate(items, 1, budget_s, cpp, lib)
    ra = oracle_rate(items, n_all, budget_s, cpp, lib)
    names = ", ".join(lbl for lbl, _, _ in items)
    desc = (f"plain C++ oracle (decode with sidecar + fp64 dot, -O3 -march=native) over {names}: "
            f"1 thread {r1[2]} passes of {r1[3]:.1%} of the rows ({r1[4]:.1f} s); "
            f"{n_all} threads {ra[2]} passes of {ra[3]:.1%} of the rows ({ra[4]:.1f} s)")
    return r1, ra, n_all, desc


def oracle_reference_arm(items, steps, warmup, budget_s=60.0):
    """--impl reference: the plain C++ oracle on all host threads; W warm-up
    passes, then K timed passes, each on a row slice sized so that the K
    passes take about budget_s in total."""
    cpp, lib = _timing_oracle()
    n_all = os.cpu_count() or 1
    for _, layer, M in items:
        _x_for(layer, M)
    t0 = time.perf_counter()
    _oracle_pass(cpp, lib, items, 0.01, n_all)
    one = max(1e-6, (time.perf_counter() - t0) / 0.01)
    frac = min(1.0, budget_s / max(1, steps) / one)
    for i in range(warmup):
        _oracle_pass(cpp, lib, items, frac, n_all, i)
    t0 = time.perf_counter()
    tb = tf = 0.0
    for i in range(steps):
        b, f = _oracle_pass(cpp, lib, items, frac, n_all, warmup + i)
        tb += b
        tf += f
    tt = time.perf_counter() - t0
    desc = (f"plain C++ oracle (-O3 -march=native), {steps} passes over " + ", ".join(lbl for lbl, _, _ in items) +
            f", {frac:.2%} of output rows per pass, {n_all} threads, {cpu_model()}")
    return tb / tt / 1e9, tf / tt / 1e12, desc, n_all, tt


def _oracle_threads():
    """Threads the numpy oracle's BLAS uses (encoder reference arm)."""
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


def profile_run(hxq, torch, items, steps, warmup, groups=()):
    """Small, eager run for ncu: replicas just past 1.25x L2, W + K steps;
    `groups` (index tuples into items) run as one grouped forward each."""
    props = torch.cuda.get_device_properties(0)
    l2 = getattr(props, "L2_cache_size", 126 << 20)
    dev_bytes = sum(l["indices"].size for _, l, _ in items)
    R = max(1, math.ceil(1.25 * l2 / dev_bytes))
    reps = [[hxq.HelixLinear.from_layer(l) for _, l, _ in items] for _ in range(R)]
    grps = [[hxq.HelixGroup([rep[j] for j in g]) for g in groups] for rep in reps]
    grouped = {j for g in groups for j in g}
    xs = [torch.from_numpy(synthetic.activations(M, l["K"], 1).view(np.int16)).cuda() for _, l, M in items]
    ys = [torch.empty((M, l["N"]), dtype=torch.float32, device="cuda") for _, l, M in items]
    for i in range(warmup + steps):
        for gi, g in enumerate(groups):
            grps[i % R][gi].forward(xs[g[0]], ys=[ys[j] for j in g])
        for j, lin in enumerate(reps[i % R]):
            if j not in grouped:
                lin.forward(xs[j], ys[j])
    torch.cuda.synchronize()
    for rep, gs in zip(reps, grps):
        for grp in gs:
            grp.close()
        for lin in rep:
            lin.check()
            lin.close()
    return 0


def run_env(torch, device):
    """What the numbers were taken on: GPU, SM count, torch and CUDA versions."""
    try:
        props = torch.cuda.get_device_properties(device)
        return {"gpu": props.name, "sms": props.multi_processor_count, "torch": torch.__version__,
                "cuda": torch.version.cuda}
    except Exception as e:  # the record must not cost the measurement
        return {"error": type(e).__name__}


# ----------------------------------------------------------------------------- encoder

ENCODER_ROUNDS = 10
# fp32 instructions per point-centroid comparison in the assignment loop
# (subtract, compare, two selects; pairs: two subtracts, two multiplies, add,
# compare, two selects) -- the count the ALU roofline below rests on
ENCODER_OPS = {1: 4, 2: 8}


# (mode, N, K, codebook entries, sidecar threshold)
ENCODER_SHAPES = {"scalar": (0, 8512, 2048, 256, 0.002), "vq2d": (1, 11008, 4096, 4096, 0.006),
                  "tiny": (0, 256, 256, 256, 0.002)}


def encoder_layer(name):
    """The encoder workload: W ~ N(0, 0.02) fp32 [N][K] and k start centroids
    drawn from its points (seeded), the same for both arms."""
    mode, N, K, k, tau = ENCODER_SHAPES[name]
    dim = 1 if mode == 0 else 2
    rng = np.random.default_rng(0)
    W = rng.normal(0, 0.02, size=(N, K)).astype(np.float32)
    pts = W.reshape(-1, dim)
    init = pts[rng.choice(pts.shape[0], k, replace=False)].copy()
    return mode, N, K, k, tau, dim, W, init


def encoder_workload_name(name):
    mode, N, K, k, tau = ENCODER_SHAPES[name]
    return f"encode {N}x{K} mode {mode}, k={k}, {ENCODER_ROUNDS} k-means rounds, threshold {tau}"


def oracle_encoder_arm(name, steps, warmup, budget_s=60.0):
    """--impl reference --encoder: the oracle's k-means rounds and encode on
    the first rows of the same layer, sized so that W + K steps take about
    budget_s. Returns (weights/s, description, threads, seconds)."""
    import oracle
    enc = oracle.hxq_encoder_oracle
    mode, N, K, k, tau, dim, W, init = encoder_layer(name)
    est_s = (ENCODER_ROUNDS + 2) * (W.size // dim) * k * 3e-9  # ~3 ns per point-centroid cell
    rows = max(1, min(N, int(N * budget_s / max(1, steps + warmup) / max(est_s, 1e-9))))
    Ws = W[:rows]
    pts = Ws.reshape(-1, dim)
    start = init if dim == 2 else init[:, 0]

    def step():
        c, _ = enc.kmeans(pts, start, ENCODER_ROUNDS)
        enc.encode(Ws, mode, c.reshape(-1), tau)

    for _ in range(warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(steps):
        step()
    tt = time.perf_counter() - t0
    desc = f"{steps} oracle steps on the first {rows} of {N} rows"
    return rows * K * steps / tt, desc, _oracle_threads(), tt


def encoder_run(hxq, torch, args):
    """One step = ENCODER_ROUNDS k-means rounds on one layer's weights plus
    its encode (indices + sidecar); metric: weights per second."""
    mode, N, K, k, tau, dim, W_h, init_h = encoder_layer(args.encoder)
    W = torch.from_numpy(W_h).cuda()
    pts = W.view(-1, dim) if dim == 2 else W.view(-1)
    n = pts.shape[0]
    init = torch.from_numpy(init_h if dim == 2 else init_h[:, 0].copy()).cuda()
    cent = torch.empty_like(init)
    labels = torch.empty(n, dtype=torch.int16, device="cuda")
    idx = torch.empty(N * K if mode == 0 else 3 * N * K // 4, dtype=torch.uint8, device="cuda")
    cap = N * K // 50
    pos = torch.empty(cap, dtype=torch.int64, device="cuda")
    val = torch.empty(cap, dtype=torch.float32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
    stream = torch.cuda.Stream()

    def step():
        cent.copy_(init)
        hxq.hxq_kmeans(pts, n, dim, k, ENCODER_ROUNDS, cent, labels, stream)
        hxq.hxq_encode(W, mode, N, K, cent.view(-1), tau, idx, pos, val, cap, cnt, stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        e1.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    # comparisons per step: (rounds + final assignment + encode) x n x k
    evals = (ENCODER_ROUNDS + 2) * n * k
    props = torch.cuda.get_device_properties(0)
    clock_ghz = 1.965  # clocks.max.sm of this part
    peak = props.multi_processor_count * 128 * clock_ghz * 1e9 / ENCODER_OPS[dim]
    achieved = evals / (ms * 1e-3)
    line = {"metric": "HXQ encoder weights/s", "value": N * K / (ms * 1e-3), "unit": "weights/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": encoder_workload_name(args.encoder), "sidecar_entries": int(cnt.item())},
            "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "comparisons/s",
                         "frac": achieved / peak, "traffic": None,
                         "peak_kind": f"derived: SMs x 128 fp32 lanes x {clock_ghz} GHz / {ENCODER_OPS[dim]} "
                                      "instructions per comparison"}}
    print(json.dumps(line))
    return 0


# ----------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="hxq", choices=["hxq", "reference"])
    ap.add_argument("--workload", default="mamba2", choices=list(synthetic.CONFIGS))
    ap.add_argument("--M", type=int, default=None, help="token count (default: the workload's bench M)")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--grouped", action="store_true",
                    help="run the layers that share their input as one grouped forward each")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--encoder", choices=sorted(ENCODER_SHAPES), default=None,
                    help="time the encoder instead (k-means rounds + encode of one layer): "
                         "scalar = in_proj 8512x2048, k=256; vq2d = 11008x4096 pairs, k=4096; "
                         "tiny = 256x256, k=256")
    ap.add_argument("--ncu", action="store_true",
                    help="minimal run for profilers: enough layer replicas to exceed L2, then "
                         "W + K eager steps; prints nothing")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference" and rank != 0:
        return 0  # the oracle arm runs on rank 0 alone; the other ranks do no work
    items = workload(args.workload, 0, args.M if args.M else DEFAULT_M[args.workload])
    is_prefill = all(M > 32 for _, _, M in items)
    metric = ("HelixLinear prefill GEMM TFLOP/s" if is_prefill else "HelixLinear GEMV achieved HBM GB/s")
    unit = "TFLOP/s" if is_prefill else "GB/s"
    wl_name = {"mamba2": "mamba2_1.3b_decode_scalar8_M1 (in_proj 8512x2048 + out_proj 2048x4096)"}.get(
        args.workload, args.workload + ":" + ",".join(lbl for lbl, _, _ in items))
    if args.grouped:
        wl_name += " grouped " + "|".join(",".join(items[j][0].split("/")[0] for j in g)
                                          for g in item_groups(args.workload, items))

    if args.impl == "reference":
        if rank != 0:
            return 0
        if args.encoder:
            v, sample, threads, secs = oracle_encoder_arm(args.encoder, args.steps, args.warmup)
            print(json.dumps({
                "impl": "reference", "metric": "HXQ encoder weights/s", "value": v, "unit": "weights/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": encoder_workload_name(args.encoder)},
                "cpu_baseline": {"value": v, "unit": "weights/s", "cores": threads, "kind": "oracle",
                                 "sample": sample + f" ({secs:.1f} s)"},
                "e2e": {"value": v, "unit": "weights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
            return 0
        gbs, tfs, sample, threads, secs = oracle_reference_arm(items, args.steps, args.warmup)
        v = tfs if is_prefill else gbs
        line = {"impl": "reference", "metric": metric, "value": v, "unit": unit, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": wl_name},
                "cpu_baseline": {"value": v, "unit": unit, "cores": threads, "kind": "oracle",
                                 "sample": sample + f" ({secs:.1f} s)", "cpu_model": cpu_model()},
                "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    import torch
    import torch.distributed as dist

    import vq_compressed_linear_b200 as hxq

    if args.ncu:
        return profile_run(hxq, torch, items, args.steps, args.warmup,
                           item_groups(args.workload, items) if args.grouped else ())
    if args.encoder:
        return encoder_run(hxq, torch, args)

    if world > 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local_rank)
    props = torch.cuda.get_device_properties(local_rank)
    l2 = getattr(props, "L2_cache_size", 126 << 20)
    stream = torch.cuda.Stream()
    pk, pk_kind = peaks()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    with ClockSampler(local_rank) as clk:
        barrier()
        ms, step_bytes, step_flops, launches, R = time_workload(
            hxq, torch, items, args.steps, args.warmup, l2, stream, soak_s=1.5,
            groups=item_groups(args.workload, items) if args.grouped else ())
        barrier()
    clocks = clk.summary()
    ms_max = max_over_ranks(torch, dist, world, ms, "cuda")
    units, scale = (step_flops, 1e12) if is_prefill else (step_bytes, 1e9)
    value = job_rate(units, args.steps, world, ms_max, scale)

    # e2e through the public call, host buffers
    e_ms, h2d, d2h = e2e_workload(hxq, torch, items, args.steps, args.warmup, stream,
                                  groups=item_groups(args.workload, items) if args.grouped else ())
    e_ms = max_over_ranks(torch, dist, world, e_ms, "cuda")
    e_val = job_rate(units, args.steps, world, e_ms, scale)

    # roofline of the dominant kernel (all launches of this workload are one kernel)
    _, l0, M0 = items[0]
    kkey = dominant_kernel(l0, M0)
    per_launch_ms = ms / (args.steps * launches)
    if is_prefill:
        peak = float(pk["bf16_tflops"])
        achieved = step_flops / launches / (per_launch_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": profiled_traffic(kkey), "kernel": kkey,
                "peak_kind": f"{pk_kind} bf16 burst"}
    else:
        peak = float(pk["hbm_gbs"])
        achieved = step_bytes / launches / (per_launch_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": profiled_traffic(kkey), "kernel": kkey,
                "peak_kind": f"{pk_kind} copy"}

    line = {"metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if is_prefill else "f32", "data": "synthetic",
            "config": {"workload": wl_name, "tokens_M": sorted({M for _, _, M in items}),
                       "bytes_per_step": step_bytes, "flops_per_step": step_flops,
                       "l2": f"{R} rotating layer replicas per rank ({R * sum(l['indices'].size for _, l, _ in items) / 2**20:.0f} MiB of indices) > 4x L2",
                       "timing": "one CUDA-graph replay of K steps, CUDA events on the launch stream",
                       "parallelism": f"replicas x{world}"},
            "roofline": roof,
            "e2e": {"value": e_val, "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps * launches,
            "clocks": clocks,
            "env": run_env(torch, local_rank)}

    if not args.no_secondary and world == 1:
        sec = []
        runs = [(wl, M, False) for wl in ("qwen25_3b", "vq2d", "prefill") for M in synthetic.CONFIGS[wl][0][4]]
        runs.insert(1, ("qwen25_3b", 1, True))  # q|k|v and gate|up as grouped forwards
        for wl, M, grp in runs:
            its = workload(wl, 0, M)
            s_ms, sb, sf, sl, sR = time_workload(hxq, torch, its, 20, 3, l2, stream,
                                                 groups=item_groups(wl, its) if grp else ())
            pre = M > 32
            v = (sf * 20 / (s_ms * 1e-3) / 1e12) if pre else (sb * 20 / (s_ms * 1e-3) / 1e9)
            pkv = float(pk["bf16_tflops"]) if pre else float(pk["hbm_gbs"])
            # roofline time: slower of bytes at HBM peak and flops at tensor peak
            t_roof = max(sb / (float(pk["hbm_gbs"]) * 1e9), sf / (float(pk["bf16_tflops"]) * 1e12))
            sec.append({"workload": f"{wl} M={M}" + (" grouped" if grp else ""), "value": round(v, 1),
                        "unit": "TFLOP/s" if pre else "GB/s",
                        "frac_of_peak": round(v / pkv, 3),
                        "frac_of_roofline": round(t_roof / (s_ms * 1e-3 / 20), 3),
                        "us_per_step": round(s_ms * 1e3 / 20, 2), "launches_per_step": sl})
        line["secondary"] = sec

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r1, ra, n_all, sample = oracle_sample(items)
        pick = (lambda r: r[1]) if is_prefill else (lambda r: r[0])
        line["cpu_baseline"] = {"value": pick(ra), "unit": unit, "cores": n_all, "kind": "oracle",
                                "sample": sample, "cores_1": pick(r1), "cores_all": pick(ra),
                                "cpu_model": cpu_model()}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
