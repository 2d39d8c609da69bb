"""The measured policy map on the GPU, through the C ABI: qlinear_matmul against the
oracle for every strategy and M from 1 to a few hundred, table entries that change the
GEMV's grid and warps per unit (visible in qlinear_plan, results unchanged), the
workspace check under a larger grid, and the tuner end to end on a small layer."""
import numpy as np
import pytest

import oracle
from synth import gen
from tests.helpers import assert_parity, lut4_layer, uniform_layer

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import weight_only_quantized_gemv_b200 as ql
    from weight_only_quantized_gemv_b200 import layers, tune

DEV = "cuda:0"
M_MAX = 2 ** 31 - 1


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    ql.qlinear_policy_set([])
    yield
    ql.qlinear_policy_set([])


def _layer(fmt, K, N):
    if fmt == "lut4":
        lt = lut4_layer(811, K, N)
        ref = lambda x: oracle.gemv_lut4(x, lt.qbytes, lt.lut, lt.absmax, 64)  # noqa: E731
        return layers.from_lut4(lt, DEV), ref, 16
    bits = int(fmt[1:])
    u = uniform_layer(820 + bits, K, N, bits)
    ref = lambda x: oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, bits, 128)  # noqa: E731
    return layers.from_uniform(u, DEV), ref, bits


def _run(lay, x):
    y = lay.matmul(torch.from_numpy(x).to(DEV))
    torch.cuda.synchronize()
    return y.float().cpu().numpy()


@pytest.mark.parametrize("strategy", [None, 0, 1])
@pytest.mark.parametrize("M", [1, 7, 16, 17, 40, 100])
@pytest.mark.parametrize("fmt", ["w4", "w2", "lut4"])
def test_matmul_parity_every_strategy(fmt, M, strategy):
    K, N = 1024, 208
    lay, ref, code = _layer(fmt, K, N)
    if strategy is not None:
        ql.qlinear_policy_set([dict(fmt=code, N=N, K=K, m_lo=1, m_hi=M_MAX, strategy=strategy)])
    x = gen.activations(1300 + M, M, K)
    assert_parity(_run(lay, x), ref(x), what=f"{fmt} M={M} strategy={strategy}")


def test_table_sets_grid_and_warps_per_unit():
    K, N = 2048, 1152
    lay, ref, _ = _layer("w4", K, N)
    units = (N // 128) * (K // 128)
    default = ql.qlinear_plan(4, 4, N, K)
    ql.qlinear_policy_set([
        dict(fmt=4, N=N, K=K, m_lo=1, m_hi=1, ctas=37),
        dict(fmt=4, N=N, K=K, m_lo=2, m_hi=8, ctas=23, warps_per_unit=4),
        dict(fmt=4, N=N, K=K, m_lo=9, m_hi=16, ctas=10 * units),
    ])
    assert ql.qlinear_plan(4, 1, N, K).ctas == 37
    p = ql.qlinear_plan(4, 4, N, K)
    assert p.ctas == 23 and p.warps_per_unit == 4
    assert (p.ctas, p.warps_per_unit) != (default.ctas, default.warps_per_unit)
    assert ql.qlinear_plan(4, 12, N, K).ctas == units        # clamped to the work units
    for M in (1, 4, 12):
        need = ql.qlinear_workspace_bytes(4, M, N, K)
        ws = torch.zeros(need // 4 + 64, dtype=torch.int32, device=DEV)
        x = gen.activations(1400 + M, M, K)
        y = torch.empty((M, N), dtype=torch.float16, device=DEV)
        ql.qlinear_matmul(4, torch.from_numpy(x).to(DEV).view(torch.int16), lay.qweight, lay.p0,
                          lay.p1, y.view(torch.int16), M, N, K, ws)
        torch.cuda.synchronize()
        assert_parity(y.float().cpu().numpy(), ref(x), what=f"table M={M}")
        assert ql.qlinear_read_error(ws) == 0


def test_larger_grid_needs_a_larger_workspace():
    K, N = 4096, 4096
    lay, _, _ = _layer("w4", K, N)
    small = ql.qlinear_workspace_bytes(4, 16, N, K)
    ql.qlinear_policy_set([dict(fmt=4, N=N, K=K, m_lo=1, m_hi=16, ctas=1024)])
    assert ql.qlinear_workspace_bytes(4, 16, N, K) > small
    ws = torch.zeros(small // 4, dtype=torch.int32, device=DEV)
    x = torch.zeros((16, K), dtype=torch.float16, device=DEV)
    y = torch.empty((16, N), dtype=torch.float16, device=DEV)
    with pytest.raises(ql.QLinearError) as ei:
        ql.qlinear_matmul(4, x.view(torch.int16), lay.qweight, lay.p0, lay.p1,
                          y.view(torch.int16), 16, N, K, ws)
    assert ei.value.status == 5


def test_tuner_end_to_end_small_layer():
    K, N = 1024, 512
    m_list = [1, 4, 17, 80]
    entries, timings, checks = tune.tune_layer(4, K, N, m_list, reps=3, log=lambda s: None,
                                               validate=True)
    assert [c["M"] for c in checks] == m_list and all(c["table_us"] > 0 for c in checks)
    assert len(timings) == sum(len(tune.candidates(4, m, torch.cuda.get_device_properties(0)
                                                   .multi_processor_count)) for m in m_list)
    assert all(t["us"] > 0 for t in timings)
    assert entries[0]["m_lo"] == 1 and entries[-1]["m_hi"] == M_MAX
    ql.qlinear_policy_set(entries)
    lay, ref, _ = _layer("w4", K, N)
    need = max(ql.qlinear_workspace_bytes(4, m, N, K) for m in range(1, 17))
    lay.workspace = torch.zeros(need // 4 + 64, dtype=torch.int32, device=DEV)
    for M in (1, 3, 4, 16, 17, 80, 200):
        x = gen.activations(1500 + M, M, K)
        assert_parity(_run(lay, x), ref(x), what=f"tuned M={M}")
