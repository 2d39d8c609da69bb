"""Benchmark of the weight-only-quantized GEMV on B200.

One step = one pass of the hot path over the six Llama-shaped W4A16 g128 decode
layers at M = 1: (K, N) = (4096, 12288), (4096, 4096), (4096, 28672), (14336, 4096),
(8192, 28672), (28672, 8192), each a separate call of qlinear_w4a16 on its own
resident packed weights (379 MB in total, cycled every step, so no layer is
L2-resident when it is read again).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--no-configs]

Prints one JSON line.  `value` is the achieved algorithmic bandwidth of the whole
job (packed codes + scales/zeros + x + y bytes of every layer of every step on every
rank, divided by the slowest rank's device time).  At one GPU the line also carries a
`configs` table: every layer of the five workloads (W4 4096 x 4096; the six W4 layers;
W2 on the six shapes and W8 on two; LUT4 on two; the outlier variant at M = 1..16 on
two), each timed alone over enough weight copies to defeat L2, next to the CPU oracle
timed on a column sample of the same layer, single-threaded and on all host cores.
`--impl reference` times the CPU oracle on a bounded sample of the headline workload
instead.  Under torchrun every rank runs an independent replica (the layer does not
shard across GPUs in this workload).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import platform
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A16-g128 dequant-GEMV µs/layer at M=1; achieved HBM GB/s vs B200 peak"
SHAPES = [(4096, 12288), (4096, 4096), (4096, 28672), (14336, 4096), (8192, 28672), (28672, 8192)]
WORKLOAD = 1  # seeds 1000 * workload + layer
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024
OUTLIER_M = (1, 2, 4, 8, 16)
BITS = {"w2": 2, "w4": 4, "w8": 8}
KERNEL_SOURCES = ["weight_only_quantized_gemv_b200/csrc/kernels.cuh",
                  "weight_only_quantized_gemv_b200/csrc/layout.h",
                  "weight_only_quantized_gemv_b200/csrc/qlinear.cu"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "qgemv_w4_llama_m1_traffic.txt")


def algorithmic_bytes(K, N, M=1):
    """Packed codes + fp16 scales and zeros + fp16 x + fp16 y, each counted once."""
    return K * N // 2 + 2 * (K // 128) * N * 2 + M * K * 2 + M * N * 2


def format_bytes(kind, K, N, M=1, nnz=0):
    """Algorithmic bytes of one launch of any format: codes, parameters (fp16 scale and
    zero per 128 x 1 group; LUT4: fp32 absmax per 64 x 1 block and the 32-byte table),
    the Tile-COO arrays (2-byte (row, col) and 2-byte value per outlier, 4-byte offset per
    tile), x and y, each counted once."""
    xy = M * K * 2 + M * N * 2
    if kind == "lut4":
        return K * N // 2 + (K // 64) * N * 4 + 32 + xy
    bits = 4 if kind == "outlier" else BITS[kind]
    b = K * N * bits // 8 + 2 * (K // 128) * N * 2 + xy
    if kind == "outlier":
        b += 4 * nnz + 4 * ((K // 128) * (N // 128) + 1)
    return b


def config_specs():
    """The layers of the five workloads: (config, kind, layer index, seed, K, N, [M...])."""
    from synth import gen
    out = [(0, "w4", 0, gen.workload_seed(0, 0), 4096, 4096, [1])]
    for j, (K, N) in enumerate(gen.LLAMA_SHAPES):
        out.append((1, "w4", j, gen.workload_seed(1, j), K, N, [1]))
    for j, (K, N) in enumerate(gen.LLAMA_SHAPES):
        out.append((2, "w2", j, gen.workload_seed(2, j), K, N, [1]))
    for j, (K, N) in enumerate(gen.WORKLOADS[2]["w8_shapes"]):
        out.append((2, "w8", 10 + j, gen.workload_seed(2, 10 + j), K, N, [1]))
    for j, (K, N) in enumerate(gen.WORKLOADS[3]["shapes"]):
        out.append((3, "lut4", j, gen.workload_seed(3, j), K, N, [1]))
    for j, (K, N) in enumerate(gen.WORKLOADS[4]["shapes"]):
        out.append((4, "outlier", j, gen.workload_seed(4, j), K, N, list(OUTLIER_M)))
    return out


def generate_layer(spec):
    """One workload layer from the seeded generator (runs in a worker process); arrays
    that neither the packer nor the oracle reads are dropped before the layer is sent."""
    kind, seed, K, N = spec
    from synth import gen
    if kind == "lut4":
        lay = gen.lut4_layer(seed, K, N)
        lay.codes = None
    elif kind == "outlier":
        lay = gen.outlier_layer(seed, K, N)
        lay.w_full = None
        lay.positions = None
        lay.dense.codes = None
        lay.dense.scales32 = None
    else:
        lay = gen.uniform_layer(seed, K, N, BITS[kind])
        lay.codes = None
        lay.scales32 = None
    return lay


def generate_all(specs, procs):
    """Generate the layers of `specs` ((kind, seed, K, N) tuples) in `procs` spawned worker
    processes (started before this process touches CUDA); dict spec -> layer."""
    specs = list(dict.fromkeys(specs))
    if procs <= 1 or len(specs) == 1:
        return {sp: generate_layer(sp) for sp in specs}
    import multiprocessing as mp
    # largest first, so the pool does not end on one long layer
    order = sorted(specs, key=lambda sp: -sp[2] * sp[3])
    with mp.get_context("spawn").Pool(min(procs, len(order))) as pool:
        layers = pool.map(generate_layer, order, chunksize=1)
    return dict(zip(order, layers))


def replay_plan(n):
    """Graph sizes (steps per replay) that run exactly n steps: a one-step graph first (it
    launches fastest, so the device starts almost at once while the host enqueues the rest),
    then ten-step graphs, then one-step graphs for the remainder."""
    if n <= 0:
        return []
    return [1] + [10] * ((n - 1) // 10) + [1] * ((n - 1) % 10)


def kernel_source_hash():
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def read_traffic():
    """Per-layer DRAM bytes from the committed ncu summary, if taken on this kernel source."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    kv = {}
    with open(TRAFFIC_FILE) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
    if kv.get("kernel_source_hash") != kernel_source_hash():
        return None
    try:
        return {tuple(int(t) for t in k[len("traffic_bytes_"):].split("x")): float(v)
                for k, v in kv.items() if k.startswith("traffic_bytes_")}
    except ValueError:
        return None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------
# clocks sampled during the timed region


class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": float(np.median(loaded)), "sm_max_mhz": max(smax),
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas)


def dist_setup(n_gpus):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    return rank, world, local


def init_pg(local, world, backend="nccl"):
    """Process group of the N replicas (none for one).  Only the timing barriers and the
    max over ranks of the device times use it: the replicas share no data."""
    if world == 1:
        return None
    import datetime

    import torch
    import torch.distributed as dist
    kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return dist


def max_over_ranks(value, dist, device):
    """The slowest rank's time (every rank gets it); the value itself with one rank."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(bytes_per_step_per_rank, world, ms, steps):
    """Whole-job throughput: the bytes all ranks moved over the slowest rank's time."""
    return bytes_per_step_per_rank * world / (ms * 1e-3 / steps) / 1e9


# ---------------------------------------------------------------------------


def host_cores():
    return len(os.sched_getaffinity(0))


def oracle_gemv(kind, lay, x, cols):
    """The fp64 oracle's y[:, cols] for one workload layer."""
    import oracle
    if kind == "lut4":
        return oracle.gemv_lut4(x, lay.qbytes, lay.lut, lay.absmax, 64, cols=cols)
    if kind == "outlier":
        d = lay.dense
        return oracle.gemv_outlier(x, d.qweight, d.scales, d.zeros, lay.tile_offsets, lay.tile_rc,
                                   lay.tile_vals, 4, 128, cols=cols)
    return oracle.gemv_uniform(x, lay.qweight, lay.scales, lay.zeros, lay.bits, 128, cols=cols)


def time_oracle(jobs, seconds, threads, cols):
    """Oracle throughput (GB/s of algorithmic bytes) on column samples.

    `jobs`: (kind, layer, x, K, N, nnz) tuples, taken in turn; each oracle call computes
    `cols` random output columns of one of them (fp64 unpack + eager dequantization +
    dot) and counts the algorithmic bytes of those columns (their codes and parameters,
    their share of the outliers, x and their y).  `threads` Python threads run calls side
    by side (NumPy releases the GIL in its array loops; BLAS is held to one thread each).
    Returns (GB/s, calls, seconds)."""
    from concurrent.futures import ThreadPoolExecutor
    try:
        from threadpoolctl import threadpool_limits
        limiter = threadpool_limits(1)
    except ImportError:
        limiter = None

    def work(seed):
        rs = np.random.default_rng(seed)
        done_bytes, calls, t0 = 0.0, 0, time.perf_counter()
        while time.perf_counter() - t0 < seconds:
            kind, lay, x, K, N, nnz = jobs[calls % len(jobs)]
            c = rs.choice(N, size=min(cols, N), replace=False)
            oracle_gemv(kind, lay, x, c)
            done_bytes += format_bytes(kind, K, len(c), x.shape[0], nnz * len(c) / N)
            calls += 1
        return done_bytes, calls

    t0 = time.perf_counter()
    if threads <= 1:
        res = [work(0)]
    else:
        with ThreadPoolExecutor(threads) as ex:
            res = list(ex.map(work, range(threads)))
    el = time.perf_counter() - t0
    if limiter is not None:
        limiter.unregister()
    return sum(r[0] for r in res) / el / 1e9, sum(r[1] for r in res), el


def cpu_oracle_sample(layers, seconds=5.0, cols=64):
    """The oracle on random column slices of the six headline layers: all host cores (the
    reported value) and one thread.  `layers`: (UniformLayer, x, K, N)."""
    jobs = [("w4", u, x, K, N, 0) for u, x, K, N in layers]
    cores = host_cores()
    all_gbs, all_calls, all_s = time_oracle(jobs, seconds, cores, cols)
    one_gbs, one_calls, one_s = time_oracle(jobs, seconds, 1, cols)
    return {"value": all_gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{cols} random columns of one of the six layers per oracle call (fp64 "
                      f"unpack + eager dequant + dot): {all_calls} calls on {cores} threads in "
                      f"{all_s:.1f} s; single thread {one_calls} calls in {one_s:.1f} s",
            "single_thread_value": one_gbs,
            "cpu": platform.processor() or platform.machine()}


def run_reference(args):
    rank, world, local = dist_setup(args.gpus)
    if rank != 0:
        return
    # the oracle on the host cores: each step is a bounded sample of the workload
    import oracle
    from synth import gen
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except ImportError:
        pass
    cols = args.ref_cols
    layers = []
    for j, (K, N) in enumerate(SHAPES):
        seed = gen.workload_seed(WORKLOAD, j)
        u = gen.uniform_layer(seed, K, N, 4)
        x = gen.activations(seed, 1, K)
        layers.append((u, x, K, N))
    rs = np.random.default_rng(1)

    def step():
        b = 0
        for u, x, K, N in layers:
            c = rs.choice(N, size=cols, replace=False)
            oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, 4, 128, cols=c)
            b += algorithmic_bytes(K, cols)
        return b

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    total = 0
    for _ in range(args.steps):
        total += step()
    el = time.perf_counter() - t0
    value = total / el / 1e9
    sample = f"{cols} random columns of each of the six layers per step (fp64 unpack + eager dequant + dot)"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "W4A16 g128 M=1, six Llama-shaped decode layers (CPU oracle sample)",
                   "layers": [list(s) for s in SHAPES], "M": 1, "columns_per_layer": cols},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def time_layer_gpu(lay, xd, yd, stream, reps=5):
    """Mean device time (us) of one launch of `lay`, alone: a CUDA graph of R launches that
    cycle through enough copies of the layer's packed arrays (codes, parameters, Tile-COO)
    to exceed 3 x L2, so that no launch finds its weights in L2; CUDA events around
    `reps` replays.  Returns (us, copies, R)."""
    import torch
    tensors = [lay.qweight, lay.p0, lay.p1] + (list(lay.tile) if lay.tile is not None else [])
    wbytes = sum(t.numel() * t.element_size() for t in tensors)
    copies = max(2, -(-3 * L2_BYTES // wbytes))
    sets = [tensors] + [[t.clone() for t in tensors] for _ in range(copies - 1)]
    R = max(30, copies)

    def assign(ts):
        lay.qweight, lay.p0, lay.p1 = ts[0], ts[1], ts[2]
        if lay.tile is not None:
            lay.tile = tuple(ts[3:])

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for r in range(R):
            assign(sets[r % copies])
            lay.forward(xd, yd, stream)
    assign(tensors)
    g.replay()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (reps * R)
    del g, sets
    return us, copies, R


def config_rows(specs, host, head_lays, dev, stream, peak, oracle_seconds, cols):
    """One row per (layer, M) of the five workloads: the GPU launch time and bandwidth,
    the oracle's throughput on a column sample (one thread, all host cores), and the
    parity of the GPU output against the oracle on a column sample."""
    import torch
    import oracle
    from synth import gen
    from weight_only_quantized_gemv_b200 import layers as qlayers
    cores = host_cores()
    rows = []
    for cfg, kind, j, seed, K, N, Ms in specs:
        hl = host[(kind, seed, K, N)]
        if cfg == 1:
            lay = head_lays[j]
        elif kind == "lut4":
            lay = qlayers.from_lut4(hl, dev)
        elif kind == "outlier":
            lay = qlayers.from_outlier(hl, dev)
        else:
            lay = qlayers.from_uniform(hl, dev)
        nnz = int(hl.tile_offsets[-1]) if kind == "outlier" else 0
        for M in Ms:
            x = gen.activations(seed + 100 * M if kind == "outlier" else seed, M, K)
            xd = torch.from_numpy(x).to(dev)
            yd = torch.empty((M, N), dtype=torch.float16, device=dev)
            us, copies, R = time_layer_gpu(lay, xd, yd, stream)
            lay.forward(xd, yd, stream)
            torch.cuda.synchronize()
            err = lay.read_error()
            c = np.random.default_rng(seed + M).choice(N, size=min(cols, N), replace=False)
            ref = oracle_gemv(kind, hl, x, c)
            rel, mabs = oracle.parity_errors(yd.float().cpu().numpy()[:, c], ref)
            job = [(kind, hl, x, K, N, nnz)]
            one, _, _ = time_oracle(job, oracle_seconds, 1, cols)
            allc, _, _ = time_oracle(job, oracle_seconds, cores, cols)
            nb = format_bytes(kind, K, N, M, nnz)
            gbs = nb / (us * 1e-6) / 1e9
            rows.append({"config": cfg, "format": kind, "K": K, "N": N, "M": M,
                         "us": round(us, 3), "bytes": nb, "GBs": round(gbs, 1),
                         "frac": round(gbs / peak, 4), "weight_copies": copies, "launches": R,
                         "oracle_GBs_1_thread": round(one, 4),
                         "oracle_GBs_all_cores": round(allc, 4), "oracle_cores": cores,
                         "oracle_sample_cols": int(min(cols, N)),
                         "parity_relL2": float(f"{rel:.3e}"), "parity_maxabs": float(f"{mabs:.3e}"),
                         "error_flags": int(err)})
            del xd, yd
        if cfg != 1:
            del lay
        torch.cuda.empty_cache()
    return rows


def run_gpu(args):
    rank, world, local = dist_setup(args.gpus)
    from synth import gen
    # the layers, generated in spawned worker processes before this process touches CUDA:
    # the six headline layers on every rank; the five workloads' other layers at N = 1
    with_configs = world == 1 and not args.no_configs
    specs = config_specs() if with_configs else []
    gen_specs = [("w4", gen.workload_seed(WORKLOAD, j), K, N) for j, (K, N) in enumerate(SHAPES)]
    gen_specs += [(kind, seed, K, N) for _, kind, _, seed, K, N, _ in specs]
    procs = max(1, min(8, host_cores() // world))
    host = generate_all(gen_specs, procs)

    import torch
    torch.cuda.set_device(local)
    dist = init_pg(local, world)
    dev = torch.device("cuda", local)
    from weight_only_quantized_gemv_b200 import layers as qlayers
    import weight_only_quantized_gemv_b200 as ql

    lays, xs, ys, byts, host_layers = [], [], [], [], []
    for j, (K, N) in enumerate(SHAPES):
        seed = gen.workload_seed(WORKLOAD, j)
        u = host[("w4", seed, K, N)]
        lays.append(qlayers.from_uniform(u, dev, max_m=1))
        x = gen.activations(seed, 1, K)
        xs.append(torch.from_numpy(x).to(dev))
        ys.append(torch.empty((1, N), dtype=torch.float16, device=dev))
        byts.append(algorithmic_bytes(K, N))
        host_layers.append((u, x, K, N))
    step_bytes = float(sum(byts))
    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)

    def eager_step():
        for j, lay in enumerate(lays):
            lay.forward(xs[j], ys[j], stream)

    # warm-up outside any graph (the library's one-time per-kernel set-up happens here)
    for _ in range(3):
        eager_step()
    torch.cuda.synchronize()

    def capture(nsteps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(nsteps):
                eager_step()
        return g
    # The timed region replays graphs of whole steps, so the host never gates the device:
    # one graph holds 10 steps (60 launches), a one-step graph covers the remainder.
    g10, g1 = capture(10), capture(1)
    torch.cuda.synchronize()
    # both graphs run once before the warm-up steps: a graph's first launch uploads it to
    # the device, which must not land in the timed region (with few steps it would)
    g10.replay()
    g1.replay()
    torch.cuda.synchronize()

    def steps(n):
        for size in replay_plan(n):
            (g10 if size == 10 else g1).replay()

    # The other measurements run before the timed region: they bring the GPU from idle to
    # its steady clocks and power state, which a short timed region (a few ms) would
    # otherwise partly run through.
    peak, peak_src = measured_peaks()
    # every layer of the five workloads, each timed alone
    rows = []
    if with_configs:
        rows = config_rows(specs, host, lays, dev, stream, peak, args.oracle_seconds,
                           args.oracle_cols)
    else:  # the headline layers only
        for j, ((K, N), lay) in enumerate(zip(SHAPES, lays)):
            us, copies, R = time_layer_gpu(lay, xs[j], ys[j], stream)
            b = algorithmic_bytes(K, N)
            rows.append({"config": 1, "format": "w4", "K": K, "N": N, "M": 1, "us": round(us, 3),
                         "bytes": b, "GBs": round(b / (us * 1e-6) / 1e9, 1),
                         "frac": round(b / (us * 1e-6) / 1e9 / peak, 4),
                         "weight_copies": copies, "launches": R})


    # end to end through the public API: the step's six x rows host->device in one copy from
    # pinned memory, the six calls, the six y rows device->host in one copy
    kx = [x.numel() for x in xs]
    ny = [y.numel() for y in ys]
    dx = torch.empty(sum(kx), dtype=torch.float16, device=dev)
    dy = torch.empty(sum(ny), dtype=torch.float16, device=dev)
    hx = torch.cat([x.reshape(-1).cpu() for x in xs]).pin_memory()
    hy = torch.empty(sum(ny), dtype=torch.float16).pin_memory()
    xv = [t.view(1, -1) for t in torch.split(dx, kx)]
    yv = [t.view(1, -1) for t in torch.split(dy, ny)]
    e2e_steps = max(3, min(args.steps, 1000))

    def e2e_step():
        dx.copy_(hx, non_blocking=True)
        for j, lay in enumerate(lays):
            lay.forward(xv[j], yv[j], stream)
        hy.copy_(dy, non_blocking=True)
        stream.synchronize()
    # The clock sampler starts here (its start-up pause leaves the GPU idle for a moment);
    # from then on the GPU stays busy: the end-to-end pass (at least 0.2 s of untimed steps,
    # then its timed steps), the W warm-up steps and the timed region.
    with ClockSampler(local) as clk:
        t_warm = time.perf_counter()
        while True:
            e2e_step()
            if time.perf_counter() - t_warm >= 0.2:
                break
        if dist is not None:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / e2e_steps
        e2e_ms = max_over_ranks(e2e_ms, dist, dev)

        steps(args.warmup)
        torch.cuda.synchronize()
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        start.record(stream)
        steps(args.steps)
        stop.record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ms = start.elapsed_time(stop)
    err = max(ql.qlinear_read_error(lay.workspace) for lay in lays)
    ms = max_over_ranks(ms, dist, dev)
    del g10, g1

    if rank == 0:
        # every launch in the timed region is the GEMV kernel: its average launch duration is
        # the region's device time over the launches, bytes per launch the step's over six
        launch_ms = ms / args.steps
        achieved = step_bytes / (launch_ms * 1e-3) / 1e9
        traffic = read_traffic()
        traffic_per_launch = None
        if traffic is not None and all(s in traffic for s in SHAPES):
            traffic_per_launch = float(np.mean([traffic[s] for s in SHAPES]))
        layers_out = [{k: r[k] for k in ("K", "N", "us", "bytes", "GBs", "frac")}
                      for r in rows if r["config"] == 1]
        clocks = clk.summary()
        out = {
            "metric": METRIC,
            "value": job_gbs(step_bytes, world, ms, args.steps),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms / args.steps,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f16",
            "data": "synthetic",
            "config": {
                "workload": "W4A16 asymmetric g128 GEMV, M=1, six Llama-shaped decode layers",
                "layers": [list(s) for s in SHAPES], "M": 1, "group": 128,
                "l2": "inputs larger than L2: 379 MB of packed weights cycled every step",
                "parallelism": f"replicas x{world}",
                "us_per_layer": round(ms * 1e3 / args.steps / len(SHAPES), 3),
            },
            "layers": layers_out,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic_per_launch,
                         "peak_source": peak_src,
                         "kernel": "qgemv_kernel<W4, M<=8> (one launch per layer)",
                         "timing": "CUDA events around the timed region (graph replays of whole steps); "
                                   "the per-layer rows come from a separate pass per layer over "
                                   "enough weight copies to exceed 3 x L2"},
            "e2e": {"value": job_gbs(step_bytes, world, e2e_ms, 1), "unit": "GB/s",
                    "h2d_bytes_per_step": int(dx.numel() * dx.element_size()),
                    "d2h_bytes_per_step": int(dy.numel() * dy.element_size()),
                    "ms_per_step": e2e_ms},
            "gpu_launches": args.steps * len(SHAPES),
            "clocks": clocks,
            "error_flags": err,
        }
        if with_configs:
            out["configs"] = rows
        if not args.no_cpu_baseline and world == 1:
            out["cpu_baseline"] = cpu_oracle_sample(host_layers, seconds=args.cpu_seconds)
        print(json.dumps(out))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    # default: about a second of timed GPU work (enough clock samples), and a bounded
    # number of oracle samples for the reference arm
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--ref-cols", type=int, default=16)
    ap.add_argument("--cpu-seconds", type=float, default=5.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-layer table of the five workloads")
    ap.add_argument("--oracle-seconds", type=float, default=0.5,
                    help="oracle timing per row of the workload table, per thread setting")
    ap.add_argument("--oracle-cols", type=int, default=64)
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.steps is None:
        args.steps = 2000 if args.impl == "reference" else 10000
    if args.steps < 1:
        raise SystemExit("--steps must be at least 1")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
