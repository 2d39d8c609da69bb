"""Time the prefill paths of one layer: stand-alone dequantization to fp16, the dense
tensor-core GEMM after it, the GEMM with the dequantization fused into it, and (for
comparison) the fused GEMV run over 16-row slices of x.

    python -m weight_only_quantized_gemv_b200.run_prefill --fmt w4 --K 8192 --N 28672 \
        --M 512 [--launches 4] [--time] [--only dequant|prefill|fused|gemv]

Packed codes and parameters are random bytes of the right sizes, and each copy has its
own fp16 weight buffer; the copies (enough of them to exceed twice the L2 size) are
cycled so that no launch finds its inputs or its output lines in L2.  Without `--time`
the chosen entry runs `--launches` times (for profiler captures).  With `--time` each
part is timed with CUDA events on the launching stream after warm-up and printed as
one JSON line:

* dequant: algorithmic bytes = codes + parameters + the fp16 output (2 N K);
* gemm: 2 M N K flops, its time taken as prefill minus dequant;
* fused: 2 M N K flops over the fused kernel's time;
* gemv: ceil(M / 16) launches of the fused GEMV (fp16 out) for the same M rows.
"""
from __future__ import annotations

import argparse
import json
import math

import torch

from . import (FORMATS, QL_FMT_LUT4, qlinear_dequant_fp16, qlinear_lut4, qlinear_prefill,
               qlinear_prefill_fused, qlinear_prefill_read_error,
               qlinear_prefill_workspace_bytes, qlinear_w2a16,
               qlinear_w4a16, qlinear_w8a16, qlinear_workspace_bytes)

_UNIFORM = {2: qlinear_w2a16, 4: qlinear_w4a16, 8: qlinear_w8a16}
L2_BYTES = 126 * 2 ** 20


def dequant_bytes(fmt: int, K: int, N: int) -> int:
    """Bytes the dequantization must move: codes, parameters and the fp16 weights."""
    if fmt == QL_FMT_LUT4:
        return K * N // 2 + (K // 64) * N * 4 + 32 + 2 * N * K
    return K * N * fmt // 8 + 2 * (K // 128) * N * 2 + 2 * N * K


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--fmt", choices=sorted(FORMATS), default="w4")
    ap.add_argument("--K", type=int, default=8192)
    ap.add_argument("--N", type=int, default=28672)
    ap.add_argument("--M", type=int, default=512)
    ap.add_argument("--launches", type=int, default=4)
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--time", action="store_true")
    ap.add_argument("--only", choices=["dequant", "prefill", "fused", "gemv"], default=None)
    ap.add_argument("--stream-k", type=int, default=1, help="fused: 1 = stream-K, 0 = whole tiles")
    a = ap.parse_args()
    fmt, K, N, M = FORMATS[a.fmt], a.K, a.N, a.M
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    bits = 4 if fmt == QL_FMT_LUT4 else fmt
    G = K // 128
    per_copy = K * N * bits // 8 + 2 * N * K
    copies = max(2, math.ceil(2 * L2_BYTES / per_copy))
    gen = torch.Generator(device=dev).manual_seed(0)
    q = [torch.randint(0, 256, (K * N * bits // 8,), dtype=torch.uint8, device=dev, generator=gen)
         for _ in range(copies)]
    if fmt == QL_FMT_LUT4:
        p0 = [torch.linspace(-1, 1, 16, device=dev).half().view(torch.int16)] * copies
        p1 = [torch.rand((K // 64) * N, device=dev, generator=gen) * 0.05 for _ in range(copies)]
    else:
        p0 = [(torch.rand(G * N, device=dev, generator=gen) * 0.01).half().view(torch.int16)
              for _ in range(copies)]
        p1 = [torch.randint(0, 1 << bits, (G * N,), device=dev, generator=gen).half()
              .view(torch.int16) for _ in range(copies)]
    w = [torch.empty(N * K, dtype=torch.int16, device=dev) for _ in range(copies)]
    x = torch.randn(M, K, device=dev, generator=gen).half().view(torch.int16)
    y = torch.empty(M, N, device=dev, dtype=torch.int16)
    ws = torch.zeros(qlinear_workspace_bytes(fmt, 16, N, K) // 4 + 64, dtype=torch.int32,
                     device=dev)

    def dequant(i):
        c = i % copies
        qlinear_dequant_fp16(fmt, q[c], p0[c], p1[c], w[c], N, K)

    def prefill(i):
        c = i % copies
        qlinear_prefill(fmt, x, q[c], p0[c], p1[c], w[c], y, M, N, K)

    pf_ws = torch.zeros(qlinear_prefill_workspace_bytes(M, N, K) // 4 + 64, dtype=torch.int32,
                        device=dev) if a.stream_k else None

    def fused(i):
        c = i % copies
        qlinear_prefill_fused(fmt, x, q[c], p0[c], p1[c], y, M, N, K, pf_ws)

    def gemv(i):
        c = i % copies
        for m0 in range(0, M, 16):
            m = min(16, M - m0)
            if fmt == QL_FMT_LUT4:
                qlinear_lut4(x[m0:], q[c], p0[c], p1[c], y[m0:], m, N, K, ws)
            else:
                _UNIFORM[fmt](x[m0:], q[c], p0[c], p1[c], y[m0:], m, N, K, ws)

    parts = {"dequant": dequant, "prefill": prefill, "fused": fused, "gemv": gemv}
    chosen = [a.only] if a.only else list(parts)
    if not a.time:
        for name in chosen:
            for i in range(a.launches):
                parts[name](i)
        torch.cuda.synchronize()
        print(json.dumps({"launches": a.launches, "parts": chosen}))
        return

    def timed(fn):
        for i in range(2 * copies):
            fn(i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(a.reps):
            fn(i)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e3 / a.reps

    out = {"fmt": a.fmt, "K": K, "N": N, "M": M, "copies": copies}
    t = {name: timed(parts[name]) for name in chosen}
    if "dequant" in t:
        b = dequant_bytes(fmt, K, N)
        out.update(dequant_us=round(t["dequant"], 2), dequant_bytes=b,
                   dequant_GBs=round(b / t["dequant"] / 1e3, 1))
    if "prefill" in t:
        out["prefill_us"] = round(t["prefill"], 2)
        if "dequant" in t:
            g = t["prefill"] - t["dequant"]
            out.update(gemm_us=round(g, 2), gemm_TFLOPs=round(2 * M * N * K / g / 1e6, 1))
    if "fused" in t:
        out.update(fused_us=round(t["fused"], 2),
                   fused_TFLOPs=round(2 * M * N * K / t["fused"] / 1e6, 1))
    if "gemv" in t:
        out["gemv_slices_us"] = round(t["gemv"], 2)
    out["error_flags"] = qlinear_prefill_read_error()
    print(json.dumps(out))


if __name__ == "__main__":
    main()
