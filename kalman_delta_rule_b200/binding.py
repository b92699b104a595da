"""Thin Python binding of libkdn.so (the C ABI declared in include/kdn.h).

The raw functions keep the C names (``kdn_forward_chunkwise``, ``kdn_decode_step``,
``kdn_gain_scan``, ``kdn_backward``, ``kdn_workspace_size``, ``kdn_last_device_error``,
``kdn_status_string``, ``kdn_version``) and take plain integers for pointers.
``forward``, ``backward``, ``decode_step`` and ``gain_scan`` marshal torch CUDA tensors into those
calls: they allocate outputs and workspace with torch and pass the current stream.
Every step of the computation runs in the library's kernels; there is no CPU or
PyTorch fallback -- a missing library or device raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libkdn.so")

KDN_OK, KDN_ERR_INVALID_ARG, KDN_ERR_UNSUPPORTED, KDN_ERR_CUDA, KDN_ERR_TIMEOUT, KDN_ERR_RANGE, KDN_ERR_WORKSPACE = range(7)
KDN_DTYPE_F32, KDN_DTYPE_BF16 = 0, 1


class KdnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {kdn_status_string(code)} (status {code})")


class kdn_problem_t(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int), ("d_k", ctypes.c_int),
                ("d_v", ctypes.c_int), ("cu_seqlens", ctypes.c_void_p), ("num_seqs", ctypes.c_int),
                ("in_dtype", ctypes.c_int), ("mu", ctypes.c_float), ("chunk", ctypes.c_int),
                ("max_seqlen", ctypes.c_int), ("variant", ctypes.c_int)]


_lib = None
_lock = threading.Lock()
_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_PP = ctypes.POINTER(kdn_problem_t)

_SIGS = {
    "kdn_workspace_size": (_i, [_PP, ctypes.POINTER(_sz)]),
    "kdn_forward_chunkwise": (_i, [_PP] + [_vp] * 6 + [_vp] * 2 + [_vp] * 3 + [_vp, _sz, _vp]),
    "kdn_decode_step": (_i, [_i, _i, _i, _i, _i, _f] + [_vp] * 6 + [_vp] * 3 + [_vp]),
    "kdn_decode_tokens": (_i, [_i, _i, _i, _i, _i, _i, _f] + [_vp] * 6 + [_vp] * 3 + [_vp]),
    "kdn_decode_tokens_iso": (_i, [_i, _i, _i, _i, _i, _i, _f] + [_vp] * 6 + [_vp] * 3 + [_vp]),
    "kdn_gain_scan": (_i, [_PP] + [_vp] * 4 + [_vp] + [_vp] * 3 + [_vp, _sz, _vp]),
    "kdn_last_device_error": (_i, [_vp]),
    "kdn_selftest_bounded_wait": (_i, [ctypes.c_longlong, _vp]),
    "kdn_status_string": (ctypes.c_char_p, [_i]),
    "kdn_version": (ctypes.c_char_p, []),
    "kdn_execution_path": (_i, [_PP]),
    "kdn_gain_scan_noalloc": (_i, [_PP] + [_vp] * 4 + [_vp] + [_vp] * 3 + [_vp]),
    "kdn_backward_workspace_size": (_i, [_PP, ctypes.POINTER(_sz)]),
    "kdn_backward": (_i, [_PP] + [_vp] * 6 + [_vp] * 2 + [_vp] * 3 + [_vp] * 6 + [_vp] * 2 + [_vp, _sz, _vp]),
}


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libkdn.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(f"libkdn.so not found at {path}; build it with "
                                   "`python -m kalman_delta_rule_b200.build`")
            lib = ctypes.CDLL(path)
            for name, (res, args) in _SIGS.items():
                fn = getattr(lib, name)
                fn.restype, fn.argtypes = res, args
            _lib = lib
    return _lib


# ------------------------------------------------------------------ raw C names
def kdn_workspace_size(problem: kdn_problem_t) -> int:
    n = ctypes.c_size_t(0)
    st = load().kdn_workspace_size(ctypes.byref(problem), ctypes.byref(n))
    if st != KDN_OK:
        raise KdnError(st, "kdn_workspace_size")
    return n.value


def kdn_forward_chunkwise(problem, q, k, v, alpha, sigma, r, S0, P0, o, S_out, P_out, workspace, workspace_bytes, stream):
    return load().kdn_forward_chunkwise(ctypes.byref(problem), q, k, v, alpha, sigma, r, S0, P0, o, S_out, P_out,
                                        workspace, workspace_bytes, stream)


def kdn_decode_step(N, H, d_k, d_v, in_dtype, mu, q, k, v, alpha, sigma, r, S, P, o, stream):
    return load().kdn_decode_step(N, H, d_k, d_v, in_dtype, mu, q, k, v, alpha, sigma, r, S, P, o, stream)


def kdn_decode_tokens(N, n_tokens, H, d_k, d_v, in_dtype, mu, q, k, v, alpha, sigma, r, S, P, o, stream):
    return load().kdn_decode_tokens(N, n_tokens, H, d_k, d_v, in_dtype, mu, q, k, v, alpha, sigma, r, S, P, o, stream)


def kdn_decode_tokens_iso(N, n_tokens, H, d_k, d_v, in_dtype, mu, q, k, v, alpha, sigma, r, S, P, o, stream):
    return load().kdn_decode_tokens_iso(N, n_tokens, H, d_k, d_v, in_dtype, mu, q, k, v, alpha, sigma, r, S, P, o,
                                        stream)


def kdn_gain_scan(problem, k, alpha, sigma, r, P0, g, beta_eff, P_out, workspace, workspace_bytes, stream):
    return load().kdn_gain_scan(ctypes.byref(problem), k, alpha, sigma, r, P0, g, beta_eff, P_out,
                                workspace, workspace_bytes, stream)


def kdn_gain_scan_noalloc(problem, k, alpha, sigma, r, P0, g, beta_eff, P_out, stream):
    """The gain scan on the library's fixed scratch array: for callers that cannot
    allocate device memory when they call (no workspace argument)."""
    return load().kdn_gain_scan_noalloc(ctypes.byref(problem), k, alpha, sigma, r, P0, g, beta_eff, P_out, stream)


def kdn_backward_workspace_size(problem: kdn_problem_t) -> int:
    n = ctypes.c_size_t(0)
    st = load().kdn_backward_workspace_size(ctypes.byref(problem), ctypes.byref(n))
    if st != KDN_OK:
        raise KdnError(st, "kdn_backward_workspace_size")
    return n.value


def kdn_backward(problem, q, k, v, alpha, sigma, r, S0, P0, d_o, dS_T, dP_T, dq, dk, dv, dalpha, dsigma, dr,
                 dS0, dP0, workspace, workspace_bytes, stream):
    return load().kdn_backward(ctypes.byref(problem), q, k, v, alpha, sigma, r, S0, P0, d_o, dS_T, dP_T,
                               dq, dk, dv, dalpha, dsigma, dr, dS0, dP0, workspace, workspace_bytes, stream)


def kdn_last_device_error(stream=None) -> int:
    return load().kdn_last_device_error(stream)


def kdn_execution_path(problem) -> int:
    return load().kdn_execution_path(ctypes.byref(problem))


def kdn_status_string(code: int) -> str:
    return load().kdn_status_string(code).decode()


def kdn_version() -> str:
    return load().kdn_version().decode()


# ------------------------------------------------------------------ torch marshalling
def _torch():
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("kalman_delta_rule_b200 needs a CUDA device (B200, sm_100a)")
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return KDN_DTYPE_BF16
    if t.dtype == torch.float32:
        return KDN_DTYPE_F32
    raise TypeError(f"unsupported input dtype {t.dtype} (float32 or bfloat16)")


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensors must be contiguous CUDA tensors")
    return t.data_ptr()


def _stream_handle(stream) -> Optional[int]:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream or None


def _check(st: int, where: str):
    if st != KDN_OK:
        raise KdnError(st, where)


VARIANTS = {"diagonal": 0, "isotropic": 1}


def make_problem(q, v, H=None, cu_seqlens=None, mu: float = 1.0, chunk: int = 64, max_seqlen: int = 0,
                 variant: str = "diagonal") -> kdn_problem_t:
    B, T, H_, dk = q.shape
    p = kdn_problem_t()
    p.B, p.T, p.H, p.d_k, p.d_v = B, T, H_, dk, v.shape[-1]
    p.cu_seqlens = _ptr(cu_seqlens)
    p.num_seqs = (cu_seqlens.numel() - 1) if cu_seqlens is not None else B
    p.in_dtype = _dtype_code(q)
    p.mu = float(mu)
    p.chunk = int(chunk)
    p.max_seqlen = int(max_seqlen)
    p.variant = VARIANTS[variant]
    return p


def forward(q, k, v, alpha, sigma, r, cu_seqlens=None, S0=None, P0=None, mu: float = 1.0, chunk: int = 64,
            o=None, S_out=None, P_out=None, workspace=None, want_state: bool = True, stream=None,
            variant: str = "diagonal", max_seqlen: int = 0):
    """Run kdn_forward_chunkwise on torch tensors ([B,T,H,d]; varlen: B = 1 with int32 cu_seqlens).

    Returns (o, S_out, P_out); P is [N,H,dk] (diagonal) or [N,H] (isotropic).  Outputs are
    allocated when not given; so is the workspace when ``workspace`` is None (``False``
    passes none: the tensor-core path needs one, so such a call runs the fp32 chunk kernel)."""
    torch = _torch()
    p = make_problem(q, v, cu_seqlens=cu_seqlens, mu=mu, chunk=chunk, variant=variant, max_seqlen=max_seqlen)
    N = p.num_seqs
    dev = q.device
    if o is None:
        o = torch.empty(q.shape[:3] + (p.d_v,), dtype=q.dtype, device=dev)
    if want_state and S_out is None:
        S_out = torch.empty((N, p.H, p.d_k, p.d_v), dtype=torch.float32, device=dev)
    if want_state and P_out is None:
        P_out = torch.empty((N, p.H) + ((p.d_k,) if p.variant == 0 else ()), dtype=torch.float32, device=dev)
    if workspace is False:
        workspace = None
    elif workspace is None:
        need = kdn_workspace_size(p)
        workspace = torch.empty(need, dtype=torch.uint8, device=dev) if need else None
    wbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = kdn_forward_chunkwise(p, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(sigma), _ptr(r), _ptr(S0), _ptr(P0),
                               _ptr(o), _ptr(S_out), _ptr(P_out), _ptr(workspace), wbytes, _stream_handle(stream))
    _check(st, "kdn_forward_chunkwise")
    return o, S_out, P_out


def backward(q, k, v, alpha, sigma, r, d_o, cu_seqlens=None, S0=None, P0=None, dS=None, dP=None, mu: float = 1.0,
             workspace=None, want_initial: bool = True, stream=None, variant: str = "diagonal", max_seqlen: int = 0):
    """Run kdn_backward on torch tensors laid out as for ``forward``.

    Returns a dict of fp32 gradients of <o, d_o> + <S_T, dS> + <P_T, dP>: dq, dk, dv,
    dalpha, dsigma ([B,T,H,d]), dr ([B,T,H]) and, with ``want_initial``, dS0 [N,H,dk,dv]
    and dP0 ([N,H,dk] diagonal, [N,H] isotropic).  The workspace is allocated when not given.
    ``max_seqlen`` (packed sequences; 0 = unknown) bounds the chunk-parallel work lists."""
    torch = _torch()
    if d_o.dtype != q.dtype:
        raise ValueError("d_o must have the dtype of the inputs")
    p = make_problem(q, v, cu_seqlens=cu_seqlens, mu=mu, chunk=0, variant=variant, max_seqlen=max_seqlen)
    N = p.num_seqs
    dev = q.device
    f32 = dict(dtype=torch.float32, device=dev)
    out = dict(dq=torch.empty(q.shape, **f32), dk=torch.empty(k.shape, **f32), dv=torch.empty(v.shape, **f32),
               dalpha=torch.empty(alpha.shape, **f32), dsigma=torch.empty(sigma.shape, **f32),
               dr=torch.empty(r.shape, **f32))
    if want_initial:
        out["dS0"] = torch.empty((N, p.H, p.d_k, p.d_v), **f32)
        out["dP0"] = torch.empty((N, p.H) + ((p.d_k,) if p.variant == 0 else ()), **f32)
    if workspace is None:
        workspace = torch.empty(kdn_backward_workspace_size(p), dtype=torch.uint8, device=dev)
    wbytes = workspace.numel() * workspace.element_size()
    st = kdn_backward(p, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(sigma), _ptr(r), _ptr(S0), _ptr(P0),
                      _ptr(d_o), _ptr(dS), _ptr(dP), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                      _ptr(out["dalpha"]), _ptr(out["dsigma"]), _ptr(out["dr"]), _ptr(out.get("dS0")),
                      _ptr(out.get("dP0")), _ptr(workspace), wbytes, _stream_handle(stream))
    _check(st, "kdn_backward")
    return out


def decode_step(q, k, v, alpha, sigma, r, S, P, mu: float = 1.0, o=None, stream=None, variant: str = "diagonal"):
    """One decode step on [N,H,d] token tensors; S [N,H,dk,dv] and P [N,H,dk] ([N,H] isotropic)
    updated in place."""
    torch = _torch()
    if VARIANTS[variant] == 1:
        o4 = None if o is None else o.unsqueeze(1)
        return decode_tokens(*(x.unsqueeze(1) for x in (q, k, v, alpha, sigma, r)), S, P, mu=mu, o=o4,
                             stream=stream, variant=variant).squeeze(1)
    N, H, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    st = kdn_decode_step(N, H, dk, dv, _dtype_code(q), float(mu), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                         _ptr(sigma), _ptr(r), _ptr(S), _ptr(P), _ptr(o), _stream_handle(stream))
    _check(st, "kdn_decode_step")
    return o


def decode_tokens(q, k, v, alpha, sigma, r, S, P, mu: float = 1.0, o=None, stream=None,
                  variant: str = "diagonal"):
    """n tokens per sequence in one launch on [N, n, H, d] token tensors; S, P updated in place
    (P [N,H,dk] diagonal, [N,H] isotropic)."""
    torch = _torch()
    N, n, H, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((N, n, H, dv), dtype=q.dtype, device=q.device)
    fn = kdn_decode_tokens_iso if VARIANTS[variant] == 1 else kdn_decode_tokens
    st = fn(N, n, H, dk, dv, _dtype_code(q), float(mu), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                           _ptr(sigma), _ptr(r), _ptr(S), _ptr(P), _ptr(o), _stream_handle(stream))
    _check(st, "kdn_decode_tokens")
    return o


def gain_scan(k, alpha, sigma, r, cu_seqlens=None, P0=None, mu: float = 1.0, chunk: int = 64,
              want_g: bool = True, want_beta: bool = True, workspace=None, stream=None, max_seqlen: int = 0):
    """Run kdn_gain_scan; returns (g [B,T,H,dk] fp32 or None, beta_eff [B,T,H] or None, P_out [N,H,dk])."""
    torch = _torch()
    p = make_problem(k, k, cu_seqlens=cu_seqlens, mu=mu, chunk=chunk, max_seqlen=max_seqlen)
    dev = k.device
    g = torch.empty(k.shape, dtype=torch.float32, device=dev) if want_g else None
    be = torch.empty(k.shape[:3], dtype=torch.float32, device=dev) if want_beta else None
    P_out = torch.empty((p.num_seqs, p.H, p.d_k), dtype=torch.float32, device=dev)
    need = kdn_workspace_size(p)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    wbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = kdn_gain_scan(p, _ptr(k), _ptr(alpha), _ptr(sigma), _ptr(r), _ptr(P0), _ptr(g), _ptr(be), _ptr(P_out),
                       _ptr(workspace), wbytes, _stream_handle(stream))
    _check(st, "kdn_gain_scan")
    return g, be, P_out


PATH_NAMES = {0: "recurrent", 1: "chunk_fp32", 3: "chunk_tcgen05_two_phase"}


def execution_path(q, v, cu_seqlens=None, mu: float = 1.0, chunk: int = 64, variant: str = "diagonal",
                   workspace: bool = True) -> str:
    """Name of the kernel path kdn_forward_chunkwise takes for these tensors (``workspace``:
    whether the call gets a workspace of kdn_workspace_size() bytes; the tensor-core path
    needs one, and without it the call runs the fp32 chunk kernel)."""
    p = make_problem(q, v, cu_seqlens=cu_seqlens, mu=mu, chunk=chunk, variant=variant)
    code = kdn_execution_path(p)
    if code == 3 and not workspace:
        code = 1
    return PATH_NAMES.get(code, "invalid")


def selftest_bounded_wait(limit_cycles: int = 2_000_000, stream=None):
    """Launch the failure-detection self-test (bounded waits that run out); the device error
    word then holds KDN_ERR_TIMEOUT, which last_device_error() raises."""
    _check(load().kdn_selftest_bounded_wait(int(limit_cycles), _stream_handle(stream)), "kdn_selftest_bounded_wait")


def last_device_error(stream=None):
    """Synchronise and raise if a kernel recorded a device-side condition."""
    _check(kdn_last_device_error(_stream_handle(stream)), "device")


def available_chunks(dtype=None):
    """The `chunk` values of kdn_forward_chunkwise with a built execution path."""
    return [0, 16, 32, 64]
