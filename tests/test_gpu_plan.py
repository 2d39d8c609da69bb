"""Launch plans of the W4 GEMV on the six Llama-shaped layers: grid size, warps per unit,
and the block alignment of the small-layer grids (the planner's rules, restated)."""
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

SHAPES = [(4096, 12288), (4096, 4096), (4096, 28672), (14336, 4096), (8192, 28672),
          (28672, 8192)]


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


@pytest.mark.parametrize("K,N", SHAPES)
def test_m1_plan(K, N):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import weight_only_quantized_gemv_b200 as ql
    p = ql.qlinear_plan(4, 1, N, K)
    G, nblocks = K // 128, (N // 16 + 7) // 8
    U = G * nblocks
    assert p.units == U and p.m_bucket == 1 and p.warps_per_unit == 1
    assert 1 <= p.ctas <= U
    c2 = 2 * _sms()
    kmax = c2 // nblocks
    if kmax >= 1 and U <= 16 * nblocks * kmax:
        # small layer: a block-aligned grid of at most two CTAs per SM
        assert p.ctas % nblocks == 0 and p.ctas <= c2
        k = p.ctas // nblocks
        kd = max(d for d in range(1, kmax + 1) if G % d == 0)
        assert k == (kd if nblocks * kd * 5 >= c2 * 4 else kmax)
    else:
        # large layer: stream-K over every resident slot (three CTAs per SM)
        assert p.ctas == min(U, 3 * _sms())


@pytest.mark.parametrize("K,N", SHAPES)
@pytest.mark.parametrize("M", [2, 5, 8])
def test_m2_to_8_warps_per_unit(K, N, M):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import weight_only_quantized_gemv_b200 as ql
    p = ql.qlinear_plan(4, M, N, K)
    per_cta = -(-p.units // p.ctas)
    assert p.warps_per_unit == (4 if per_cta <= 4 else 2 if per_cta <= 24 else 1)


@pytest.mark.parametrize("M", [9, 16])
def test_m9_to_16_bucket(M):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import weight_only_quantized_gemv_b200 as ql
    for fmt in (2, 4, 8, 16):
        p = ql.qlinear_plan(fmt, M, 28672, 8192)
        assert p.m_bucket == 2 and p.warps_per_unit == 2
