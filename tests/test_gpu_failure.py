"""Failure detection on the GPU without a fault: the kernels' bounded waits run out on
conditions that never come true, report KDN_ERR_TIMEOUT through the device error word, and
leave the context usable."""
import pytest

import oracle
from kalman_delta_rule_b200 import inputs
from tests.kdn_testutil import assert_rel, max_rel_err
from tests.test_gpu_recurrent import TOL_F32, run_forward

pytestmark = pytest.mark.gpu


def test_bounded_waits_report_timeout_and_the_context_survives(kdn):
    kdn.last_device_error()                       # start from a clear error word
    kdn.selftest_bounded_wait(2_000_000)          # about a millisecond per wait
    with pytest.raises(kdn.KdnError) as err:
        kdn.last_device_error()
    assert err.value.code == kdn.KDN_ERR_TIMEOUT
    kdn.last_device_error()                       # reading cleared it
    w = inputs.tiny_fp32()                        # and the device still computes correctly
    ref = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens)
    o, S, P = run_forward(kdn, w, chunk=0)
    assert_rel(o, ref["o"], TOL_F32, 'o')
