"""Device-side failure path without faulting the GPU: a bounded wait that
nothing signals gives up, the kernel reports FFTCONV_ERR_TIMEOUT through the
plan's status word, and the context stays usable."""
import numpy as np
import pytest

import oracle
import workloads as W
from parity_util import assert_close, run_cuda

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports_timeout():
    import long_sequence_fft_b200 as lsf
    plan = lsf.Plan(4096, 2, "bf16")
    lib = lsf.library()
    # signalled: the wait succeeds
    assert lib.fftconv_selftest_bounded_wait(plan.handle, 1024, 1, None) == lsf.OK
    assert plan.device_status() == lsf.OK
    # never signalled: the wait runs out after its poll limit
    assert lib.fftconv_selftest_bounded_wait(plan.handle, 1024, 0, None) == lsf.OK
    assert plan.device_status() == lsf.ERR_TIMEOUT
    assert plan.device_status() == lsf.OK          # the read resets the word
    # the context is still usable: a forward on the same device is exact
    w = W.WORKLOADS["gated_bf16_n4k"].with_shape(B=3, H=2)
    inp = W.make_all(w)
    y, p2 = run_cuda(inp, "bf16")
    assert_close(y, oracle.fftconv(inp["u"], inp["k"], w=inp["w"], v=inp["v"]), "bf16", "after a timeout")
    assert np.isfinite(y).all()
