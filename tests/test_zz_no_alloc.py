"""The allocation-free W4A16 entry point (qlinear_w4a16_noalloc) against qlinear_w4a16
and against the fp64 oracle.

qlinear_w4a16_noalloc serves callers that may not allocate device memory (a plug-in
whose device memory belongs to someone else, code that must not call cudaMalloc or
cudaFree): its split-K scratch is a fixed array inside the library, shared by every call
on the device.  This file runs last in the suite so that a stop-at-first-failure run has
already run every other test; it must also pass on its own in a fresh process.
"""
import numpy as np
import pytest

import oracle
from synth import gen
from tests.helpers import assert_parity

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CASES = [(2048, 1152, 1), (1408, 416, 5), (4096, 4096, 16), (8192, 28672, 1)]


@pytest.mark.parametrize("K,N,M", CASES)
def test_noalloc_matches_workspace_entry_on_two_calls(K, N, M):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import weight_only_quantized_gemv_b200 as ql
    from weight_only_quantized_gemv_b200 import layers

    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    seed = 9000 + K + M
    u = gen.uniform_layer(seed, K, N, 4)
    lay = layers.from_uniform(u, dev)
    x = torch.from_numpy(gen.activations(seed, M, K)).to(dev)
    y_ref = lay.forward(x)  # the entry point with a caller-provided workspace
    torch.cuda.synchronize()
    ref = y_ref.float().cpu().numpy()
    # the oracle on every output (the two smaller layers) or on a column sample
    cols = None if K * N <= 4096 * 4096 else np.random.default_rng(seed).choice(N, 256, replace=False)
    x_h = gen.activations(seed, M, K)
    y_oracle = oracle.gemv_uniform(x_h, u.qweight, u.scales, u.zeros, 4, 128, cols=cols)
    assert ql.qlinear_w4a16_noalloc_read_error() == 0  # flags of earlier calls, now cleared
    for call in range(2):  # the second call runs on the scratch the first one left behind
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device=dev)
        ql.qlinear_w4a16_noalloc(x.view(torch.int16), lay.qweight, lay.p0, lay.p1,
                                 y.view(torch.int16), M, N, K)
        torch.cuda.synchronize()
        got = y.float().cpu().numpy()
        assert np.isfinite(got).all(), f"call {call}: unwritten outputs"
        assert_parity(got, ref, what=f"noalloc call {call} K={K} N={N} M={M}")
        assert_parity(got if cols is None else got[:, cols], y_oracle,
                      what=f"noalloc call {call} vs oracle K={K} N={N} M={M}")
        assert ql.qlinear_w4a16_noalloc_read_error() == 0, f"call {call}: a device wait gave up"


def test_noalloc_rejects_before_enqueueing():
    """A misaligned x is rejected with QL_ERR_ALIGN before anything reaches the stream."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import weight_only_quantized_gemv_b200 as ql
    from weight_only_quantized_gemv_b200 import layers

    dev = torch.device("cuda:0")
    K, N = 1024, 256
    u = gen.uniform_layer(9100, K, N, 4)
    lay = layers.from_uniform(u, dev)
    x = torch.from_numpy(gen.activations(9100, 1, K + 8)).to(dev)
    y = torch.empty((1, N), dtype=torch.float16, device=dev)
    xm = x.view(torch.int16).reshape(-1)[1:K + 1]  # 2-byte offset: not 16-byte aligned
    with pytest.raises(ql.QLinearError) as err:
        ql.qlinear_w4a16_noalloc(xm, lay.qweight, lay.p0, lay.p1, y.view(torch.int16), 1, N, K)
    assert err.value.status == 3  # QL_ERR_ALIGN
    assert ql.qlinear_w4a16_noalloc_read_error() == 0
