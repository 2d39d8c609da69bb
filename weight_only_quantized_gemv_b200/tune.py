"""Offline tuner that builds the measured policy map.

    python -m weight_only_quantized_gemv_b200.tune --fmts w4,w2 \
        --shapes 4096x4096,8192x28672 --M 1-16,32,64,128,512 --out policy.json

Follows the ADAngel page (awesome-system-papers, OSDI'26, core method): for every
(format, K x N layer, M) it runs each candidate of the strategy set through the library's
dispatcher (`qlinear_matmul`), times it with CUDA events (the calls replayed from a CUDA
graph, so the figure is device time), and keeps the fastest.  Candidates:

* the fused GEMV with the planner's rules;
* for M <= 16, the GEMV with a fixed grid of 1, 2 or 3 CTAs per SM, and for W4 at
  2 <= M <= 8 with 1, 2 or 4 warps per work unit;
* the prefill path (dequantization to fp16 + dense GEMM).

Each candidate is installed as a one-entry table, so the timed call is exactly the call a
user makes.  A candidate other than the planner's rule must beat the rule by `--margin`
(default 2%) to be chosen, so timing noise does not pick variants.  With `--validate` the
finished table is then timed again against the built-in rule alone on fresh launches (the
winners' own timings are biased low by the choice); a choice that loses there by the margin
is replaced by the rule's, and the pairs are stored too.

Packed codes and parameters are random bytes of the right sizes, in enough copies (each
with its own fp16 weight buffer) that every launch misses L2.  The measured
M values become ranges: the choice at M_i covers (M_{i-1}, M_i], the last one every larger M.
The JSON file holds the entries (for `load_policy`) and every timing.
"""
from __future__ import annotations

import argparse
import json
import math
from typing import Dict, List, Sequence, Tuple

FMT_CODES = {"w2": 2, "w4": 4, "w8": 8, "lut4": 16}
M_MAX = 2 ** 31 - 1
L2_BYTES = 126 * 2 ** 20

Candidate = Tuple[int, int, int]  # (strategy, warps_per_unit, ctas)


def parse_m_list(text: str) -> List[int]:
    """'1-4,8,16' -> [1, 2, 3, 4, 8, 16] (sorted, unique)."""
    out = set()
    for part in text.split(","):
        part = part.strip()
        if not part:
            continue
        if "-" in part:
            a, b = part.split("-")
            out.update(range(int(a), int(b) + 1))
        else:
            out.add(int(part))
    if not out or min(out) < 1:
        raise ValueError(f"bad M list {text!r}")
    return sorted(out)


def parse_shapes(text: str) -> List[Tuple[int, int]]:
    """'4096x4096,8192x28672' -> [(K, N), ...]."""
    shapes = []
    for part in text.split(","):
        k, n = part.lower().split("x")
        shapes.append((int(k), int(n)))
    return shapes


def candidates(fmt: int, M: int, sms: int) -> List[Candidate]:
    c: List[Candidate] = [(0, 0, 0)]
    if M <= 16:
        c += [(0, 0, k * sms) for k in (1, 2, 3)]
        if fmt == 4 and 2 <= M <= 8:
            c += [(0, w, 0) for w in (1, 2, 4)]
    c.append((1, 0, 0))
    return c


def build_entries(fmt: int, N: int, K: int, best: Dict[int, Candidate]) -> List[dict]:
    """Turn the winner at each measured M into M ranges (merged when neighbours agree)."""
    ms = sorted(best)
    entries: List[dict] = []
    lo = 1
    for i, m in enumerate(ms):
        hi = M_MAX if i == len(ms) - 1 else m
        s, w, c = best[m]
        if entries and (entries[-1]["strategy"], entries[-1]["warps_per_unit"],
                        entries[-1]["ctas"]) == (s, w, c):
            entries[-1]["m_hi"] = hi
        else:
            entries.append(dict(fmt=fmt, N=N, K=K, m_lo=lo, m_hi=hi, strategy=s,
                                warps_per_unit=w, ctas=c))
        lo = m + 1
    return entries


def rule_choice(M: int) -> Candidate:
    """The library's built-in decision (no table entry): GEMV up to M = 64, prefill above."""
    return (1, 0, 0) if M > 64 else (0, 0, 0)


def pick(results: Sequence[Tuple[float, Candidate]], margin: float) -> Tuple[float, Candidate]:
    """The fastest candidate; results[0] is the planner's rule, kept unless beaten by margin."""
    rule = results[0]
    us, cand = min(results)
    if cand != rule[1] and cand[0] == 0 and us * (1 + margin) > rule[0]:
        return rule
    return us, cand


def tune_layer(fmt: int, K: int, N: int, m_list: Sequence[int], reps: int, log,
               margin: float = 0.02, validate: bool = False):
    import torch

    from . import (QL_FMT_LUT4, qlinear_matmul, qlinear_policy_set, qlinear_workspace_bytes)

    dev = torch.device("cuda:0")
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    bits = 4 if fmt == QL_FMT_LUT4 else fmt
    G = K // 128
    per_copy = K * N * bits // 8 + 2 * N * K
    copies = max(2, math.ceil(2 * L2_BYTES / per_copy))
    gen = torch.Generator(device=dev).manual_seed(K * 7 + N)
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
    Mmax = max(m_list)
    x = torch.randn(Mmax, K, device=dev, generator=gen).half().view(torch.int16)
    y = torch.empty(Mmax, N, device=dev, dtype=torch.int16)
    ws_cache: Dict[int, torch.Tensor] = {}

    def time_call(M: int) -> float:
        """Mean device time of qlinear_matmul at M under the installed table."""
        need = qlinear_workspace_bytes(fmt, min(M, 16), N, K)
        if need not in ws_cache:
            ws_cache[need] = torch.zeros(max(need, 256) // 4 + 64, dtype=torch.int32,
                                         device=dev)
        ws = ws_cache[need]

        def call(i):
            j = i % copies
            qlinear_matmul(fmt, x, q[j], p0[j], p1[j], y, M, N, K, ws, None)

        for i in range(2 * copies):
            call(i)
        torch.cuda.synchronize()
        # device time: the calls are replayed from a CUDA graph, so host launch cost (which
        # at a few microseconds per call would swamp small layers) stays out of the number
        side = torch.cuda.Stream()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for i in range(reps):
                call(i)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(3):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) * 1e3 / (3 * reps)

    timings, best = [], {}
    for M in m_list:
        results = []
        for cand in candidates(fmt, M, sms):
            s, w, c = cand
            qlinear_policy_set([dict(fmt=fmt, N=N, K=K, m_lo=1, m_hi=M_MAX, strategy=s,
                                     warps_per_unit=w, ctas=c)])
            us = time_call(M)
            results.append((us, cand))
            timings.append(dict(fmt=fmt, K=K, N=N, M=M, strategy=s, warps_per_unit=w, ctas=c,
                                us=round(us, 3)))
        us, cand = pick(results, margin)
        best[M] = cand
        log(f"fmt={fmt} K={K} N={N} M={M}: best {cand} {us:.2f} us "
            f"(rule {results[0][0]:.2f} us)")
    entries = build_entries(fmt, N, K, best)
    checks = []
    if validate:
        reverted = False
        for M in m_list:
            qlinear_policy_set(entries)
            t_table = time_call(M)
            qlinear_policy_set([])
            t_rule = time_call(M)
            # a choice that loses to the built-in rule on fresh launches was noise: drop it
            drop = t_table > t_rule * (1 + margin)
            if drop:
                best[M] = rule_choice(M)
                reverted = True
            checks.append(dict(fmt=fmt, K=K, N=N, M=M, table_us=round(t_table, 3),
                               rule_us=round(t_rule, 3), reverted=drop))
        if reverted:
            entries = build_entries(fmt, N, K, best)
    qlinear_policy_set([])
    del q, p0, p1, x, y, ws_cache
    torch.cuda.empty_cache()
    return entries, timings, checks


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--fmts", default="w4")
    ap.add_argument("--shapes", default="4096x4096")
    ap.add_argument("--M", default="1-16,24,32,48,64,96,128,256,512")
    ap.add_argument("--reps", type=int, default=10)
    ap.add_argument("--margin", type=float, default=0.02)
    ap.add_argument("--validate", action="store_true")
    ap.add_argument("--out", required=True)
    a = ap.parse_args()
    import sys

    import torch

    from . import qlinear_policy_set

    torch.cuda.set_device(0)
    m_list = parse_m_list(a.M)
    entries, timings, checks = [], [], []
    for name in a.fmts.split(","):
        for K, N in parse_shapes(a.shapes):
            e, t, c = tune_layer(FMT_CODES[name], K, N, m_list, a.reps,
                                 lambda s: print(s, file=sys.stderr, flush=True),
                                 margin=a.margin, validate=a.validate)
            entries += e
            timings += t
            checks += c
    qlinear_policy_set(entries)  # validates the table
    qlinear_policy_set([])
    props = torch.cuda.get_device_properties(0)
    with open(a.out, "w") as f:
        json.dump(dict(device=props.name, sms=props.multi_processor_count, M=m_list,
                       reps=a.reps, margin=a.margin, entries=entries, timings=timings,
                       validation=checks), f, indent=1)
    summary = dict(out=a.out, entries=len(entries), timings=len(timings))
    if checks:
        summary["table_us"] = round(sum(c["table_us"] for c in checks), 1)
        summary["rule_us"] = round(sum(c["rule_us"] for c in checks), 1)
    print(json.dumps(summary))


if __name__ == "__main__":
    main()
