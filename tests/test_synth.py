"""The seeded input generator: determinism and the workload recipes."""
import numpy as np

from synth import gen


def test_deterministic_per_seed():
    a = gen.uniform_layer(7, 256, 32, 4)
    b = gen.uniform_layer(7, 256, 32, 4)
    c = gen.uniform_layer(8, 256, 32, 4)
    assert np.array_equal(a.qweight, b.qweight) and np.array_equal(a.scales, b.scales)
    assert not np.array_equal(a.qweight, c.qweight)
    assert np.array_equal(gen.activations(7, 2, 256), gen.activations(7, 2, 256))
    assert np.array_equal(gen.lut16(9), gen.lut16(9))


def test_distributions():
    w = gen.weights(1000, 1024, 512)
    assert w.dtype == np.float32
    assert abs(float(w.std()) - 0.02) < 5e-4 and abs(float(w.mean())) < 5e-4
    x = gen.activations(1000, 4, 4096)
    assert x.dtype == np.float16 and abs(float(x.astype(np.float32).std()) - 1) < 0.03


def test_outlier_count_and_positions():
    assert gen.outlier_count(4096, 14336) == 293601
    assert gen.outlier_count(8192, 28672) == 1174405
    lay = gen.outlier_layer(4000, 256, 256)
    assert len(lay.positions) == gen.outlier_count(256, 256)
    assert len(np.unique(lay.positions)) == len(lay.positions)


def test_workload_table():
    assert gen.WORKLOADS[1]["shapes"][4] == (8192, 28672)
    assert gen.workload_seed(4, 1) == 4001
