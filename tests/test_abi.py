"""The C ABI on the CPU: the library loads, exports every entry point the header
declares, and rejects bad arguments synchronously, before any CUDA call.

Every call here that passes pointers is built to fail validation: the fake
addresses are never dereferenced on any machine."""
import ctypes
import os
import re

import pytest

from kalman_delta_rule_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced (validation fails first)


def header_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(kdn_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from kalman_delta_rule_b200 import build
    build.build()
    return B.load()


def test_library_exports_every_declared_entry_point(lib):
    names = header_functions()
    assert {"kdn_forward_chunkwise", "kdn_decode_step", "kdn_gain_scan", "kdn_workspace_size",
            "kdn_last_device_error", "kdn_status_string", "kdn_version"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_status_strings_and_version(lib):
    for code in range(7):
        s = B.kdn_status_string(code)
        assert s and s != "unknown status"
    assert B.kdn_status_string(99) == "unknown status"
    assert "sm_100a" in B.kdn_version()


def problem(**kw):
    p = B.kdn_problem_t()
    p.B, p.T, p.H, p.d_k, p.d_v = 2, 128, 4, 128, 128
    p.cu_seqlens, p.num_seqs, p.in_dtype, p.mu, p.chunk = None, 0, B.KDN_DTYPE_BF16, 1.0, 64
    p.max_seqlen = 0
    for k, v in kw.items():
        setattr(p, k, v)
    return p


@pytest.mark.parametrize("kw,code", [
    (dict(d_k=48), B.KDN_ERR_UNSUPPORTED),
    (dict(d_v=96), B.KDN_ERR_UNSUPPORTED),
    (dict(chunk=8), B.KDN_ERR_UNSUPPORTED),
    (dict(mu=0.0), B.KDN_ERR_INVALID_ARG),
    (dict(mu=float("nan")), B.KDN_ERR_INVALID_ARG),
    (dict(H=0), B.KDN_ERR_INVALID_ARG),
    (dict(B=-1), B.KDN_ERR_INVALID_ARG),
    (dict(in_dtype=7), B.KDN_ERR_INVALID_ARG),
    (dict(cu_seqlens=FAKE, B=2, num_seqs=3), B.KDN_ERR_INVALID_ARG),
    (dict(max_seqlen=-1), B.KDN_ERR_INVALID_ARG),
    (dict(variant=2), B.KDN_ERR_INVALID_ARG),
])
def test_problem_validation(lib, kw, code):
    p = problem(**kw)
    n = ctypes.c_size_t(0)
    assert lib.kdn_workspace_size(ctypes.byref(p), ctypes.byref(n)) == code
    st = B.kdn_forward_chunkwise(p, *([FAKE] * 6), None, None, FAKE, None, None, FAKE, 1 << 30, None)
    assert st == code


def test_workspace_size_is_host_only_and_sane(lib):
    for chunk in (0, 16, 32, 64):
        for dt in (B.KDN_DTYPE_F32, B.KDN_DTYPE_BF16):
            n = B.kdn_workspace_size(problem(chunk=chunk, in_dtype=dt))
            assert 0 <= n < (1 << 34)
    # a tighter max_seqlen shrinks the gain scan's work list
    full = B.kdn_workspace_size(problem(B=1, T=4096))
    tight = B.kdn_workspace_size(problem(B=1, T=4096, max_seqlen=512))
    assert tight < full
    assert lib.kdn_workspace_size(None, None) == B.KDN_ERR_INVALID_ARG


def test_forward_rejects_bad_pointers(lib):
    p = problem(chunk=0)  # the token-serial path needs no workspace
    ptrs = [FAKE] * 6
    # a missing input
    assert B.kdn_forward_chunkwise(p, None, *ptrs[1:], None, None, FAKE, None, None, None, 0, None) == B.KDN_ERR_INVALID_ARG
    # a misaligned input
    bad = list(ptrs); bad[2] = FAKE + 2
    assert B.kdn_forward_chunkwise(p, *bad, None, None, FAKE, None, None, None, 0, None) == B.KDN_ERR_INVALID_ARG
    # final state aliasing the initial state
    assert B.kdn_forward_chunkwise(p, *ptrs, FAKE + 4096, None, FAKE, FAKE + 4096, None, None, 0, None) == B.KDN_ERR_INVALID_ARG
    assert B.kdn_forward_chunkwise(p, *ptrs, None, FAKE + 4096, FAKE, None, FAKE + 4096, None, 0, None) == B.KDN_ERR_INVALID_ARG
    # the gain scan rejects a missing, short or misaligned workspace before any CUDA call
    p64 = problem(chunk=64)
    need = B.kdn_workspace_size(p64)
    assert need > 0
    k_a_s_r = [FAKE] * 4
    assert B.kdn_gain_scan(p64, *k_a_s_r, None, FAKE, None, None, None, 0, None) == B.KDN_ERR_WORKSPACE
    assert B.kdn_gain_scan(p64, *k_a_s_r, None, FAKE, None, None, FAKE + 4096, need - 1, None) == B.KDN_ERR_WORKSPACE
    assert B.kdn_gain_scan(p64, *k_a_s_r, None, FAKE, None, None, FAKE + 16, need, None) == B.KDN_ERR_WORKSPACE
    assert B.kdn_gain_scan(p64, None, *k_a_s_r[1:], None, FAKE, None, None, FAKE, need, None) == B.KDN_ERR_INVALID_ARG
    # the scan is built for the diagonal uncertainty only
    piso = problem(chunk=64, variant=1)
    assert B.kdn_gain_scan(piso, *k_a_s_r, None, FAKE, None, None, FAKE, need, None) == B.KDN_ERR_UNSUPPORTED
    assert B.kdn_gain_scan_noalloc(piso, *k_a_s_r, None, FAKE, None, None, None) == B.KDN_ERR_UNSUPPORTED


def test_backward_validates_before_any_cuda_call(lib):
    p = problem(chunk=64)
    need = B.kdn_backward_workspace_size(p)
    # P tape, g, den, den^, u tape, S checkpoints every 16 tokens and the sums of g^, k^_S, alpha^_S
    ntok, H, dk, dv = 2 * 128, 4, 128, 128
    assert need >= 4 * (2 * ntok * H * dk + 2 * ntok * H + ntok * H * dv + (ntok // 16 + 2 + 1) * H * dk * dv + 3 * ntok * H * dk)
    assert need < 4 * (2 * ntok * H * dk + 2 * ntok * H + ntok * H * dv + (ntok // 16 + 2 + 1) * H * dk * dv + 3 * ntok * H * dk) + 7 * 256
    ins = [FAKE] * 6                 # q, k, v, alpha, sigma, r
    outs = [FAKE + 4096 * (i + 1) for i in range(6)]   # dq, dk, dv, dalpha, dsigma, dr
    args = lambda d_o=FAKE, o=outs, ws=FAKE, wb=need: [p, *ins, None, None, d_o, None, None, *o, None, None, ws, wb, None]
    assert B.kdn_backward(*args(ws=None)) == B.KDN_ERR_WORKSPACE
    assert B.kdn_backward(*args(wb=need - 1)) == B.KDN_ERR_WORKSPACE
    assert B.kdn_backward(*args(ws=FAKE + 16)) == B.KDN_ERR_WORKSPACE
    assert B.kdn_backward(*args(d_o=None)) == B.KDN_ERR_INVALID_ARG
    assert B.kdn_backward(*args(d_o=FAKE + 2)) == B.KDN_ERR_INVALID_ARG
    bad = list(outs); bad[5] = None
    assert B.kdn_backward(*args(o=bad)) == B.KDN_ERR_INVALID_ARG
    # both variants, the same workspace; sizes as for the forward
    piso = problem(chunk=64, variant=1)
    assert B.kdn_backward_workspace_size(piso) == need
    assert B.kdn_backward(piso, *args(ws=None)[1:]) == B.KDN_ERR_WORKSPACE
    assert B.kdn_backward(problem(d_k=48), *args()[1:]) == B.KDN_ERR_UNSUPPORTED
    assert B.kdn_backward(problem(num_seqs=0, B=0), *args()[1:]) == B.KDN_OK   # nothing to do


def test_decode_rejects_bad_arguments(lib):
    ptrs = [FAKE] * 9
    assert B.kdn_decode_step(4, 2, 48, 64, B.KDN_DTYPE_BF16, 1.0, *ptrs, None) == B.KDN_ERR_UNSUPPORTED
    assert B.kdn_decode_step(4, 2, 64, 64, B.KDN_DTYPE_BF16, -1.0, *ptrs, None) == B.KDN_ERR_INVALID_ARG
    assert B.kdn_decode_step(-1, 2, 64, 64, B.KDN_DTYPE_BF16, 1.0, *ptrs, None) == B.KDN_ERR_INVALID_ARG
    bad = list(ptrs); bad[6] = None
    assert B.kdn_decode_step(4, 2, 64, 64, B.KDN_DTYPE_BF16, 1.0, *bad, None) == B.KDN_ERR_INVALID_ARG
    bad = list(ptrs); bad[0] = FAKE + 8
    assert B.kdn_decode_step(4, 2, 64, 64, B.KDN_DTYPE_F32, 1.0, *bad, None) == B.KDN_ERR_INVALID_ARG
    assert B.kdn_decode_step(0, 2, 64, 64, B.KDN_DTYPE_F32, 1.0, *ptrs, None) == B.KDN_OK  # empty: no-op
    assert B.kdn_decode_tokens_iso(4, 2, 2, 48, 64, B.KDN_DTYPE_BF16, 1.0, *ptrs, None) == B.KDN_ERR_UNSUPPORTED
    assert B.kdn_decode_tokens_iso(4, -1, 2, 64, 64, B.KDN_DTYPE_BF16, 1.0, *ptrs, None) == B.KDN_ERR_INVALID_ARG
    assert B.kdn_decode_tokens_iso(4, 2, 2, 64, 64, B.KDN_DTYPE_BF16, 1.0, *bad, None) == B.KDN_ERR_INVALID_ARG


def test_product_path_fails_loudly_without_library(tmp_path):
    import importlib
    mod = importlib.import_module("kalman_delta_rule_b200.binding")
    saved = mod._lib
    mod._lib = None
    try:
        with pytest.raises(RuntimeError, match="libkdn.so not found"):
            mod.load(str(tmp_path / "missing.so"))
    finally:
        mod._lib = saved


def test_selftest_rejects_a_bad_wait_bound(lib):
    assert B.load().kdn_selftest_bounded_wait(10, None) == B.KDN_ERR_INVALID_ARG
    assert B.load().kdn_selftest_bounded_wait(1 << 40, None) == B.KDN_ERR_INVALID_ARG
