"""The bounded barrier wait behind mxfp8_gemm's error_flag, made to run out on
the GPU: a wait on a barrier that nothing arrives on gives up after its
limit and reports it, a wait on a completed phase returns, and the context
stays usable (a quantize launched afterwards is exact)."""
import numpy as np
import pytest

import nvfp4_block_scaled_sm_b200 as mxq
import oracle
import workloads as W
from gpu_util import assert_same, dev, host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("timeout_ns", [1_000, 2_000_000, 20_000_000])
def test_wait_gives_up_after_its_limit(timeout_ns):
    r = mxq.check_bounded_wait(timeout_ns)
    assert r["gave_up"], r
    assert r["completed"], r
    assert timeout_ns <= r["waited_ns"] < timeout_ns + 50_000_000, r


def test_context_usable_after_a_wait_gave_up():
    assert mxq.check_bounded_wait(2_000_000)["gave_up"]
    x = W.activation(seed=71, M=130, N=256)
    q, s = mxq.mxfp8_quantize(dev(x))
    qo, so = oracle.mxfp8_quantize(x)
    assert_same(host(q), qo, "codes after a timed-out wait")
    assert_same(host(s), so, "scales after a timed-out wait")
