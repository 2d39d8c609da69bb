"""Failure detection of the GEMV kernels' bounded waits, on the GPU, without a fault.

Every wait of the kernels' shared-memory ring (a stage's copies landing, a stage being
released) is bounded: past its limit it sets a flag in the workspace error word, then waits
at most 2^22 more rounds.  qlinear_debug_wait_test shortens the limit to one round and
makes one wait run out on purpose:
  * a delayed producer (its first copy late by 5 ms) -> flag 1, copy landed late;
  * a consumer that holds its first stage for 5 ms -> the producer's wait to refill it
    runs out -> flag 2.
The delays are far below the 2^22-round second wait, so the flagged calls still finish
with correct results; the next call with normal settings reports no flag.  The hooks are
compiled into the W4 kernels for M = 1 and M = 9..16 only, which these cases use.
"""
import os

import numpy as np
import pytest

import oracle
from synth import gen
from tests.helpers import assert_parity

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    import weight_only_quantized_gemv_b200 as ql
    yield
    ql.qlinear_debug_wait_test()  # defaults again, whatever the test did
    os.environ.pop("QLINEAR_MAX_CTAS", None)


def _case(seed, K, N, M):
    from weight_only_quantized_gemv_b200 import layers
    u = gen.uniform_layer(seed, K, N, 4)
    x = gen.activations(seed, M, K)
    ref = oracle.gemv_uniform(x, u.qweight, u.scales, u.zeros, 4, 128)
    return layers.from_uniform(u, DEV), torch.from_numpy(x).to(DEV), ref


def _forward(lay, xd):
    y = lay.forward(xd)
    torch.cuda.synchronize()
    return y.float().cpu().numpy(), lay.read_error()


@pytest.mark.parametrize("M", [1, 12])
def test_late_copy_sets_full_flag(M):
    import weight_only_quantized_gemv_b200 as ql
    lay, xd, ref = _case(3100 + M, 1024, 256, M)
    assert _forward(lay, xd)[1] == 0
    ql.qlinear_debug_wait_test(1, 5000, 0)
    y, flags = _forward(lay, xd)
    assert flags & 1, f"flags={flags}: the late copy was not reported"
    assert_parity(y, ref, what=f"late copy M={M}")  # the second wait let it land
    ql.qlinear_debug_wait_test()
    y, flags = _forward(lay, xd)
    assert flags == 0
    assert_parity(y, ref, what=f"after late copy M={M}")


@pytest.mark.parametrize("M", [1, 12])
def test_held_stage_sets_empty_flag(M):
    import weight_only_quantized_gemv_b200 as ql
    # one CTA, 16 units through a ring of 4 or 8 stages: the producer must wait for a
    # stage to be released before it refills it
    os.environ["QLINEAR_MAX_CTAS"] = "1"
    lay, xd, ref = _case(3200 + M, 1024, 256, M)
    assert _forward(lay, xd)[1] == 0
    ql.qlinear_debug_wait_test(1, 0, 5000)
    y, flags = _forward(lay, xd)
    assert flags & 2, f"flags={flags}: the held stage was not reported"
    assert_parity(y, ref, what=f"held stage M={M}")
    ql.qlinear_debug_wait_test()
    y, flags = _forward(lay, xd)
    assert flags == 0
    assert_parity(y, ref, what=f"after held stage M={M}")


def test_settings_are_checked():
    import weight_only_quantized_gemv_b200 as ql
    with pytest.raises(ql.QLinearError):
        ql.qlinear_debug_wait_test(1, 70000, 0)
    with pytest.raises(ql.QLinearError):
        ql.qlinear_debug_wait_test(1, 0, 70000)
