"""kdn_gain_scan_noalloc, the gain scan for callers that cannot allocate device memory
when they call it (a plugin whose host framework owns all device buffers and offers no
allocator, or a serving loop that forbids cudaMalloc/cudaFree after start-up).

It runs the same kernel as kdn_gain_scan with a caller-provided workspace, only with its
scratch in the library's fixed device array.  Two calls in a row with different mu (so the
second call finds the first one's leftovers in the shared array, and any of them read as its
own would change its result), each compared with the workspace call on the same problem, for
both scan kernels: the TMA kernel (bf16, d_k = 128) and the generic one (fp32, d_k = 64, a
ragged tail).  The decoupled look-back forms a chunk's starting uncertainty by the same
operations whichever predecessors have published by then, so the scan is bit-reproducible and
the two entry points must agree bit for bit.  The device's free memory must not change across a
call.  This file is collected last, so a stop-at-first-failure run has run every other test.
"""
import numpy as np
import pytest

from kalman_delta_rule_b200 import inputs
from tests.kdn_testutil import dense_shape, to_dev, to_host

pytestmark = pytest.mark.gpu


CASES = {
    # 64 chunks x 64 (sequence, head) pairs: fits the fixed scratch
    "bf16_dk128_tma_kernel": lambda: inputs.prefill_4x4096(),
    "fp32_dk64_generic_kernel": lambda: inputs.dense("noalloc_fp32", 41, 3, 5, 1000, 64, 64, bf16=False),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_noalloc_gain_scan_matches_the_workspace_version_twice(kdn, case):
    import torch
    w = CASES[case]()
    k, al, sg, r = [to_dev(dense_shape(w, getattr(w, n))) for n in ("k", "alpha", "sigma", "r")]
    stream = torch.cuda.current_stream()
    for call, mu in enumerate((1.0, 2.0)):
        g_ref, be_ref, P_ref = kdn.gain_scan(k, al, sg, r, mu=mu)
        torch.cuda.synchronize()
        kdn.last_device_error()
        p = kdn.make_problem(k, k, mu=mu)
        g = torch.full_like(g_ref, float("nan"))
        be = torch.full_like(be_ref, float("nan"))
        P = torch.full_like(P_ref, float("nan"))
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        st = kdn.kdn_gain_scan_noalloc(p, k.data_ptr(), al.data_ptr(), sg.data_ptr(), r.data_ptr(), None,
                                       g.data_ptr(), be.data_ptr(), P.data_ptr(), stream.cuda_stream or None)
        assert st == kdn.KDN_OK, kdn.kdn_status_string(st)
        torch.cuda.synchronize()
        free_after = torch.cuda.mem_get_info()[0]
        kdn.last_device_error()
        if call == 1:   # the first call on a device may load the library's module with its fixed array
            assert free_after == free_before, (free_before, free_after)
        np.testing.assert_array_equal(to_host(g), to_host(g_ref), err_msg=f"g, call {call}")
        np.testing.assert_array_equal(to_host(be), to_host(be_ref), err_msg=f"k^T g, call {call}")
        np.testing.assert_array_equal(to_host(P), to_host(P_ref), err_msg=f"P, call {call}")


def test_noalloc_gain_scan_rejects_a_problem_larger_than_its_scratch(kdn):
    import torch
    # 32 heads x 1024 chunks of a 65536-token sequence need about 128 MiB of scratch
    k = torch.empty((1, 65536, 32, 128), dtype=torch.bfloat16, device="cuda")
    p = kdn.make_problem(k, k)
    ptr = k.data_ptr()
    st = kdn.kdn_gain_scan_noalloc(p, ptr, ptr, ptr, ptr, None, ptr, None, None, None)
    assert st == kdn.KDN_ERR_UNSUPPORTED
