"""Run one quantized-GEMV configuration repeatedly (for timing and profiler captures).

    python -m weight_only_quantized_gemv_b200.run_layer --fmt w4 --K 8192 --N 28672 --M 1 \
        --launches 4 [--copies 3] [--time] [--outliers 0.005]

The packed codes and parameters are random bytes of the right sizes (the kernel's
speed does not depend on their values), allocated in `--copies` copies that the
launches cycle through so that no launch finds its weights in L2.  With `--outliers F`
(W4 only) every 128 x 128 tile also carries round(F * 16384) Tile-COO entries at random
in-tile positions, and the outlier-aware entry point runs.  With `--time` the launches
are replayed from a CUDA graph and the mean device time per launch is printed as JSON.
"""
from __future__ import annotations

import argparse
import json

import torch

from . import (FORMATS, QL_FMT_LUT4, qlinear_lut4, qlinear_plan, qlinear_read_error,
               qlinear_w2a16, qlinear_w3a16, qlinear_w4a16, qlinear_w4a16_outlier,
               qlinear_w8a16, qlinear_workspace_bytes)

_UNIFORM = {2: qlinear_w2a16, 3: qlinear_w3a16, 4: qlinear_w4a16, 8: qlinear_w8a16}


def algorithmic_bytes(fmt: int, K: int, N: int, M: int, nnz: int = 0, group: int = 128) -> int:
    """Bytes a launch must move at least: codes, parameters, x and y (and the Tile-COO
    arrays: 2-byte (row, col) and 2-byte value per outlier, 4-byte offset per tile).
    Per-channel parameters (group = K) count once per column."""
    if fmt == QL_FMT_LUT4:
        return K * N // 2 + (K // 64) * N * 4 + 32 + M * K * 2 + M * N * 2
    b = K * N * fmt // 8 + 2 * (K // group) * N * 2 + M * K * 2 + M * N * 2
    if nnz:
        b += 4 * nnz + 4 * ((K // 128) * (N // 128) + 1)
    return b


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--fmt", choices=sorted(FORMATS), default="w4")
    ap.add_argument("--K", type=int, default=8192)
    ap.add_argument("--N", type=int, default=28672)
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--launches", type=int, default=4)
    ap.add_argument("--copies", type=int, default=3)
    ap.add_argument("--time", action="store_true")
    ap.add_argument("--outliers", type=float, default=0.0)
    ap.add_argument("--group", type=int, default=128,
                    help="W2/W4/W8 group size: 128, 64, 32, or K (per-channel)")
    a = ap.parse_args()
    fmt, K, N, M = FORMATS[a.fmt], a.K, a.N, a.M
    if a.outliers and (a.fmt != "w4" or N % 128):
        raise SystemExit("--outliers needs --fmt w4 and N % 128 == 0")
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    bits = 4 if fmt == QL_FMT_LUT4 else fmt
    G = K // 128
    gen = torch.Generator(device=dev).manual_seed(0)
    q = [torch.randint(0, 256, (K * N * bits // 8,), dtype=torch.uint8, device=dev, generator=gen)
         for _ in range(a.copies)]
    if fmt == QL_FMT_LUT4:
        p0 = [torch.linspace(-1, 1, 16, device=dev).half().view(torch.int16)] * a.copies
        p1 = [torch.rand((K // 64) * N, device=dev, generator=gen) * 0.05 for _ in range(a.copies)]
    else:
        # packed parameter entries: one per (sub-group, column); per-channel ones repeat per 128
        PG = G * (128 // a.group if a.group < 128 else 1)
        p0 = [(torch.rand(PG * N, device=dev, generator=gen) * 0.01).half().view(torch.int16)
              for _ in range(a.copies)]
        p1 = [torch.randint(0, 1 << bits, (PG * N,), device=dev, generator=gen).half().view(torch.int16)
              for _ in range(a.copies)]
    x = torch.randn(M, K, device=dev, generator=gen).half().view(torch.int16)
    y = torch.empty(M, N, device=dev, dtype=torch.int16)
    ws = torch.zeros(qlinear_workspace_bytes(fmt, M, N, K) // 4 + 64, dtype=torch.int32, device=dev)
    nnz = 0
    outl = a.outliers > 0  # the outlier-aware entry, even if the density rounds to no entries
    if outl:
        T = (K // 128) * (N // 128)
        per = int(round(a.outliers * 128 * 128))
        nnz = per * T
        toff = (torch.arange(T + 1, device=dev, dtype=torch.int64) * per).to(torch.int32)
        trc = [torch.randint(0, 128, (max(nnz, 1) * 2,), dtype=torch.uint8, device=dev, generator=gen)
               for _ in range(a.copies)]  # in-tile (row, col) pairs
        tval = [(torch.randn(max(nnz, 1), device=dev, generator=gen) * 0.2).half().view(torch.int16)
                for _ in range(a.copies)]

    def call(i):  # on the current stream (the capture stream inside the graph below)
        c = i % a.copies
        if outl:
            qlinear_w4a16_outlier(x, q[c], p0[c], p1[c], toff, trc[c], tval[c], y, M, N, K, ws)
        elif fmt == QL_FMT_LUT4:
            qlinear_lut4(x, q[c], p0[c], p1[c], y, M, N, K, ws)
        else:
            _UNIFORM[fmt](x, q[c], p0[c], p1[c], y, M, N, K, ws, group=a.group)

    if not a.time:
        for i in range(a.launches):
            call(i)
        torch.cuda.synchronize()
        print(json.dumps({"launches": a.launches, "error_flags": qlinear_read_error(ws)}))
        return
    for i in range(2 * a.copies):
        call(i)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for i in range(a.launches):
            call(i)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 10
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (reps * a.launches)
    b = algorithmic_bytes(fmt, K, N, M, nnz, group=a.group) + \
        (4 * ((K // 128) * (N // 128) + 1) if outl and not nnz else 0)
    print(json.dumps({"fmt": a.fmt, "group": a.group, "K": K, "N": N, "M": M, "nnz": nnz,
                      "us": round(us, 3), "bytes": b,
                      "GBs": round(b / us / 1e3, 1), "ctas": qlinear_plan(fmt, M, N, K).ctas,
                      "error_flags": qlinear_read_error(ws)}))


if __name__ == "__main__":
    main()
