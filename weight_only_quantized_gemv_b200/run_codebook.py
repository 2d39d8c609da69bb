"""Time the codebook GEMV (Psumbook, m1v4g128) on one layer.

    python -m weight_only_quantized_gemv_b200.run_codebook --K 8192 --N 28672 --M 1 \
        [--launches 30] [--time]

Codes, scales and codebook are random of the right sizes (the kernel's speed does not
depend on their values beyond the spread of the codes, which random codes maximize),
in enough copies that no launch finds its codes in L2.  With `--time` the launches are
replayed from a CUDA graph and the mean device time per launch is printed as JSON with
the algorithmic bytes: codes K N / 4, scales 2 N K / 128, the 2 KB codebook, x and y.
"""
from __future__ import annotations

import argparse
import json
import math

import torch

from . import (QL_FMT_CB, qlinear_codebook, qlinear_codebook_tc, qlinear_codebook_workspace_bytes,
                qlinear_workspace_bytes)

L2_BYTES = 126 * 2 ** 20


def algorithmic_bytes(K: int, N: int, M: int) -> int:
    return K * N // 4 + 2 * (K // 128) * N + 256 * 4 * 2 + 2 * M * K + 2 * M * N


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--K", type=int, default=8192)
    ap.add_argument("--N", type=int, default=28672)
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--launches", type=int, default=30)
    ap.add_argument("--time", action="store_true")
    ap.add_argument("--tc", action="store_true",
                    help="the tensor-core form (qlinear_codebook_tc) instead of the Psumbook")
    a = ap.parse_args()
    K, N, M = a.K, a.N, a.M
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    gen = torch.Generator(device=dev).manual_seed(0)
    per_copy = K * N // 4 + 2 * (K // 128) * N
    copies = max(3, math.ceil(2 * L2_BYTES / per_copy))
    codes = [torch.randint(0, 256, (K * N // 4,), dtype=torch.uint8, device=dev, generator=gen)
             for _ in range(copies)]
    scales = [(0.05 + 0.02 * torch.rand((K // 128) * N, device=dev, generator=gen)).half()
              .view(torch.int16) for _ in range(copies)]
    cb = (torch.rand(256 * 4, device=dev, generator=gen) * 2 - 1).half().view(torch.int16)
    x = torch.randn(M, K, device=dev, generator=gen).half().view(torch.int16)
    y = torch.empty(M, N, device=dev, dtype=torch.int16)
    need = (qlinear_workspace_bytes(QL_FMT_CB, M, N, K) if a.tc
            else qlinear_codebook_workspace_bytes(M, N, K))
    ws = torch.zeros(max(need, 256) // 4 + 64, dtype=torch.int32, device=dev)
    entry = qlinear_codebook_tc if a.tc else qlinear_codebook

    def call(i):
        c = i % copies
        entry(x, codes[c], scales[c], cb, y, M, N, K, ws)

    if not a.time:
        for i in range(a.launches):
            call(i)
        torch.cuda.synchronize()
        print(json.dumps({"launches": a.launches}))
        return
    for i in range(2 * copies):
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
    b = algorithmic_bytes(K, N, M)
    print(json.dumps({"fmt": "cb2", "form": "tensor-core" if a.tc else "psumbook", "K": K, "N": N, "M": M, "us": round(us, 3), "bytes": b,
                      "GBs": round(b / us / 1e3, 1), "lookups": M * K * N // 4,
                      "Glookups_s": round(M * K * N / 4 / us / 1e3, 1)}))


if __name__ == "__main__":
    main()
