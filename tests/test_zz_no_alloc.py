"""kdn_gain_scan_noalloc, the gain scan for callers that cannot allocate device memory
when they call it (a plugin whose host framework owns all device buffers and offers no
allocator, or a serving loop that forbids cudaMalloc/cudaFree after start-up).

It must give what kdn_gain_scan gives with a caller-provided workspace, on two calls in
a row (the second call reuses the library's scratch array left over from the first).
This file is collected last, so a stop-at-first-failure run has run every other test.
"""
import numpy as np
import pytest

from kalman_delta_rule_b200 import inputs
from tests.kdn_testutil import dense_shape, max_rel_err, to_dev, to_host

pytestmark = pytest.mark.gpu

TOL = 1e-3   # the gain-scan tolerance on bf16-rounded inputs


def test_noalloc_gain_scan_matches_the_workspace_version_twice(kdn):
    import torch
    w = inputs.prefill_4x4096()          # 64 chunks x 64 (sequence, head) pairs: fits the fixed scratch
    k, al, sg, r = [to_dev(dense_shape(w, getattr(w, n))) for n in ("k", "alpha", "sigma", "r")]
    g_ref, be_ref, P_ref = kdn.gain_scan(k, al, sg, r, mu=2.0)
    torch.cuda.synchronize()
    kdn.last_device_error()
    p = kdn.make_problem(k, k, mu=2.0)
    stream = torch.cuda.current_stream()
    for call in range(2):
        g = torch.full_like(g_ref, float("nan"))
        be = torch.full_like(be_ref, float("nan"))
        P = torch.full_like(P_ref, float("nan"))
        st = kdn.kdn_gain_scan_noalloc(p, k.data_ptr(), al.data_ptr(), sg.data_ptr(), r.data_ptr(), None,
                                       g.data_ptr(), be.data_ptr(), P.data_ptr(), stream.cuda_stream or None)
        assert st == kdn.KDN_OK, kdn.kdn_status_string(st)
        torch.cuda.synchronize()
        kdn.last_device_error()
        assert max_rel_err(to_host(g), to_host(g_ref)) <= TOL, call
        assert max_rel_err(to_host(be), to_host(be_ref)) <= TOL, call
        assert max_rel_err(to_host(P), to_host(P_ref)) <= TOL, call


def test_noalloc_gain_scan_rejects_a_problem_larger_than_its_scratch(kdn):
    import torch
    # 32 heads x 1024 chunks of a 65536-token sequence need about 128 MiB of scratch
    k = torch.empty((1, 65536, 32, 128), dtype=torch.bfloat16, device="cuda")
    p = kdn.make_problem(k, k)
    ptr = k.data_ptr()
    st = kdn.kdn_gain_scan_noalloc(p, ptr, ptr, ptr, ptr, None, ptr, None, None, None)
    assert st == kdn.KDN_ERR_UNSUPPORTED
