"""Host-side parts of bench.py on the CPU: algorithmic byte counts (hand-computed figures
of the workload table), the workload list, the layer generation in spawned workers, and the
oracle timing helper."""
import numpy as np
import pytest

import bench
from synth import gen


def test_algorithmic_bytes_of_the_workloads():
    # W4 g128 4096 x 4096, M = 1: codes 8 MiB + scales/zeros 2 * 32 * 4096 * 2 + x 8 KB + y 8 KB
    assert bench.format_bytes("w4", 4096, 4096) == 8_929_280
    assert bench.algorithmic_bytes(4096, 4096) == 8_929_280
    # the target layer and the other formats on 8192 x 28672 (M = 1)
    assert bench.format_bytes("w4", 8192, 28672) == 124_854_272
    assert bench.format_bytes("w2", 8192, 28672) == 66_134_016
    assert bench.format_bytes("w8", 8192, 28672) == 242_294_784
    assert bench.format_bytes("lut4", 8192, 28672) == 132_194_336
    # outliers: 4 bytes per entry + 4 bytes per tile offset (T + 1 of them)
    nnz = gen.outlier_count(8192, 28672)
    assert nnz == 1_174_405
    assert bench.format_bytes("outlier", 8192, 28672, 1, nnz) == 129_609_240
    assert bench.format_bytes("outlier", 8192, 28672, 16, nnz) == 130_715_160


def test_workload_list_covers_the_five_configs():
    specs = bench.config_specs()
    assert sorted({s[0] for s in specs}) == [0, 1, 2, 3, 4]
    rows = sum(len(s[6]) for s in specs)
    # 1 + 6 (W4) + 6 (W2) + 2 (W8) + 2 (LUT4) + 2 layers x 5 batch sizes (outliers)
    assert rows == 27
    assert [s[4:6] for s in specs if s[0] == 1] == [tuple(x) for x in gen.LLAMA_SHAPES]
    assert {tuple(s[6]) for s in specs if s[0] == 4} == {(1, 2, 4, 8, 16)}
    # seeds: 1000 * workload + layer (W8 layers of workload 2 at 10, 11)
    assert {s[3] for s in specs if s[1] == "w8"} == {2010, 2011}


def test_spawned_generation_matches_direct_generation():
    specs = [("w4", 11, 256, 64), ("w2", 12, 128, 32), ("lut4", 13, 128, 32),
             ("outlier", 14, 256, 128)]
    got = bench.generate_all(specs, procs=2)
    for sp in specs:
        want = bench.generate_layer(sp)
        g = got[sp]
        if sp[0] == "lut4":
            assert np.array_equal(g.qbytes, want.qbytes) and np.array_equal(g.absmax, want.absmax)
        elif sp[0] == "outlier":
            assert np.array_equal(g.dense.qweight, want.dense.qweight)
            assert np.array_equal(g.tile_offsets, want.tile_offsets)
            assert np.array_equal(g.tile_vals.view(np.uint16), want.tile_vals.view(np.uint16))
        else:
            assert np.array_equal(g.qweight, want.qweight)
            assert np.array_equal(g.scales.view(np.uint16), want.scales.view(np.uint16))


def test_oracle_timing_counts_sample_bytes():
    u = gen.uniform_layer(21, 256, 128, 4)
    x = gen.activations(21, 2, 256)
    gbs, calls, secs = bench.time_oracle([("w4", u, x, 256, 128, 0)], 0.05, 2, 16)
    assert calls >= 2 and secs > 0 and gbs > 0
    # the bytes of one call: 16 columns' codes and parameters, x (2 rows) and 16 y columns
    per_call = bench.format_bytes("w4", 256, 16, 2)
    assert gbs == pytest.approx(calls * per_call / secs / 1e9, rel=1e-9)


def test_replay_plan_runs_exactly_n_steps():
    """The timed region replays graphs of 10 and 1 steps; the plan must add up to exactly the
    requested steps, start with the one-step graph and use few replays."""
    for n in range(0, 200):
        plan = bench.replay_plan(n)
        assert sum(plan) == n
        assert set(plan) <= {1, 10}
        if n:
            assert plan[0] == 1
            assert len(plan) <= 1 + n // 10 + 9
