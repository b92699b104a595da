"""fp64 CPU oracle of the Diagonal KDN memory recurrence (test infrastructure).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by the package's smoke
check and by the benchmark's CPU-baseline leg -- never by the product path.
It shares no code with the CUDA library.

The arithmetic lives in ``kdn_oracle.c`` (plain C, fp64, token by token);
this module builds it with gcc on first use (``build()``), loads it with ctypes
and marshals numpy arrays.  Inputs of any float dtype (or bf16 bit patterns as
uint16) are widened exactly to fp64.

Entry points
------------
diag_forward   -- Diagonal KDN (predict, Kalman gain, decayed delta write,
                  readout, mean-field uncertainty update with scaling mu).
full_kf        -- the full-covariance Kalman filter on the same model (tiny sizes).
delta_forward  -- the delta family with a given write strength beta.
iso_forward    -- isotropic KDN (one uncertainty per head; trace-keeping predict,
                  exact gain, precision-averaged update scaled by mu).
mobius_matrix  -- the 2x2 matrix of one token's uncertainty map (predict then update),
                  for the associative-scan pins.

Parity status: every function is pinned by the tests in
``tests/test_oracle_pins.py``; no function is "parity unpinned".  What stays a
reading rather than a pin (the exact diagonal equations are not printed on any
page) is stated in the C source header.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kdn_oracle.c")
_LIB = os.path.join(_HERE, "libkdn_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile kdn_oracle.c into libkdn_oracle.so (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _bind(path):
    lib = ctypes.CDLL(path)
    i, d = ctypes.c_int, ctypes.c_double
    lib.kdn_oracle_diag.argtypes = [i, _i64p, i, i, i] + [_dp] * 8 + [d] + [_dp] * 7 + [i]
    lib.kdn_oracle_fullkf.argtypes = [i, _i64p, i, i, i] + [_dp] * 8 + [_dp] * 4 + [i]
    lib.kdn_oracle_delta.argtypes = [i, _i64p, i, i, i] + [_dp] * 6 + [_dp] * 2 + [i]
    lib.kdn_oracle_iso.argtypes = lib.kdn_oracle_diag.argtypes
    for f in (lib.kdn_oracle_diag, lib.kdn_oracle_fullkf, lib.kdn_oracle_delta, lib.kdn_oracle_iso):
        f.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


def build_variant(src_text: str, tag: str) -> ctypes.CDLL:
    """Compile a modified copy of the oracle source (used only by the mutation test,
    which plants mistakes on the CPU to show that the pins catch them)."""
    import tempfile
    d = tempfile.mkdtemp(prefix="kdn_oracle_mut_")
    src, lib = os.path.join(d, f"m_{tag}.c"), os.path.join(d, f"m_{tag}.so")
    with open(src, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                           "-fno-fast-math", "-ffp-contract=off", src, "-o", lib, "-lm"])
    return _bind(lib)


def _f64(x):
    if x is None:
        return None
    x = np.asarray(x)
    if x.dtype == np.uint16:  # bf16 bit patterns: exact widening
        x = (x.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(x):
    return None if x is None else x.ctypes.data_as(_dp)


def _threads(n):
    return int(n) if n else (os.cpu_count() or 1)


def _cu(cu_seqlens, ntok):
    if cu_seqlens is None:
        return np.array([0, ntok], dtype=np.int64)
    return np.ascontiguousarray(cu_seqlens, dtype=np.int64)


def diag_forward(q, k, v, alpha, sigma, r, cu_seqlens=None, S0=None, P0=None, mu: float = 1.0,
                 trace: bool = False, threads: Optional[int] = None):
    """Diagonal KDN over tokens [ntok, H, d] split into sequences by ``cu_seqlens``.

    Returns dict(o [ntok,H,dv], S [nseq,H,dk,dv], P [nseq,H,dk]) and, with
    ``trace``, the per-token P^- ("Pm"), P, gain g and k^T g ("beta_eff").
    """
    q, k, v, alpha, sigma, r = map(_f64, (q, k, v, alpha, sigma, r))
    ntok, H, dk = k.shape
    dv = v.shape[-1]
    cu = _cu(cu_seqlens, ntok)
    nseq = len(cu) - 1
    S0, P0 = _f64(S0), _f64(P0)
    o = np.zeros((ntok, H, dv))
    S = np.zeros((nseq, H, dk, dv))
    P = np.zeros((nseq, H, dk))
    tr = {}
    if trace:
        tr = dict(Pm=np.zeros((ntok, H, dk)), P=np.zeros((ntok, H, dk)), g=np.zeros((ntok, H, dk)),
                  beta_eff=np.zeros((ntok, H)))
    rc = _load().kdn_oracle_diag(nseq, cu.ctypes.data_as(_i64p), H, dk, dv,
                                 _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(sigma), _ptr(r),
                                 _ptr(S0), _ptr(P0), float(mu), _ptr(o), _ptr(S), _ptr(P),
                                 _ptr(tr.get("Pm")), _ptr(tr.get("P")), _ptr(tr.get("g")),
                                 _ptr(tr.get("beta_eff")), _threads(threads))
    if rc:
        raise RuntimeError(f"kdn_oracle_diag failed ({rc})")
    out = dict(o=o, S=S, P=P)
    if trace:
        out.update({("trace_" + n): a for n, a in tr.items()})
    return out


def iso_forward(q, k, v, alpha, sigma, r, cu_seqlens=None, S0=None, P0=None, mu: float = 1.0,
                trace: bool = False, threads: Optional[int] = None):
    """Isotropic KDN over tokens [ntok, H, d]; P0 and the returned P are [nseq, H].

    Returns dict(o, S, P) and, with ``trace``, per-token p^- ("Pm") and p [ntok, H],
    the gain g [ntok, H, dk] and k^T g ("beta_eff")."""
    q, k, v, alpha, sigma, r = map(_f64, (q, k, v, alpha, sigma, r))
    ntok, H, dk = k.shape
    dv = v.shape[-1]
    cu = _cu(cu_seqlens, ntok)
    nseq = len(cu) - 1
    S0, P0 = _f64(S0), _f64(P0)
    o = np.zeros((ntok, H, dv))
    S = np.zeros((nseq, H, dk, dv))
    P = np.zeros((nseq, H))
    tr = {}
    if trace:
        tr = dict(Pm=np.zeros((ntok, H)), P=np.zeros((ntok, H)), g=np.zeros((ntok, H, dk)),
                  beta_eff=np.zeros((ntok, H)))
    rc = _load().kdn_oracle_iso(nseq, cu.ctypes.data_as(_i64p), H, dk, dv,
                                _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(sigma), _ptr(r),
                                _ptr(S0), _ptr(P0), float(mu), _ptr(o), _ptr(S), _ptr(P),
                                _ptr(tr.get("Pm")), _ptr(tr.get("P")), _ptr(tr.get("g")),
                                _ptr(tr.get("beta_eff")), _threads(threads))
    if rc:
        raise RuntimeError(f"kdn_oracle_iso failed ({rc})")
    out = dict(o=o, S=S, P=P)
    if trace:
        out.update({("trace_" + n): a for n, a in tr.items()})
    return out


def full_kf(q, k, v, alpha, sigma, r, cu_seqlens=None, S0=None, Sigma0=None, threads: Optional[int] = None):
    """Full-covariance Kalman filter; returns dict(o, S, Sigma [nseq,H,dk,dk], g)."""
    q, k, v, alpha, sigma, r = map(_f64, (q, k, v, alpha, sigma, r))
    ntok, H, dk = k.shape
    dv = v.shape[-1]
    cu = _cu(cu_seqlens, ntok)
    nseq = len(cu) - 1
    S0, Sigma0 = _f64(S0), _f64(Sigma0)
    o = np.zeros((ntok, H, dv))
    S = np.zeros((nseq, H, dk, dv))
    Sig = np.zeros((nseq, H, dk, dk))
    g = np.zeros((ntok, H, dk))
    rc = _load().kdn_oracle_fullkf(nseq, cu.ctypes.data_as(_i64p), H, dk, dv,
                                   _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(sigma), _ptr(r),
                                   _ptr(S0), _ptr(Sigma0), _ptr(o), _ptr(S), _ptr(Sig), _ptr(g),
                                   _threads(threads))
    if rc:
        raise RuntimeError(f"kdn_oracle_fullkf failed ({rc})")
    return dict(o=o, S=S, Sigma=Sig, g=g)


def delta_forward(q, k, v, alpha, beta, cu_seqlens=None, S0=None, threads: Optional[int] = None):
    """Delta family (write key beta*k) with per-channel decay; returns dict(o, S)."""
    q, k, v, alpha, beta = map(_f64, (q, k, v, alpha, beta))
    ntok, H, dk = k.shape
    dv = v.shape[-1]
    cu = _cu(cu_seqlens, ntok)
    nseq = len(cu) - 1
    S0 = _f64(S0)
    o = np.zeros((ntok, H, dv))
    S = np.zeros((nseq, H, dk, dv))
    rc = _load().kdn_oracle_delta(nseq, cu.ctypes.data_as(_i64p), H, dk, dv,
                                  _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S0),
                                  _ptr(o), _ptr(S), _threads(threads))
    if rc:
        raise RuntimeError(f"kdn_oracle_delta failed ({rc})")
    return dict(o=o, S=S)


def diag_chains(w, chains, mu=None, S0=None, P0=None, threads: Optional[int] = None, trace: bool = False,
                iso: bool = False):
    """Diagonal KDN (isotropic with ``iso``) on selected (sequence, head) chains of a
    workload ``w`` (any object with q, k, v, alpha, sigma, r as [ntok, H, d],
    cu_seqlens and mu).

    The chains are packed as the sequences of a one-head problem and run in one call
    (one thread per chain).  Returns {(s, h): dict(o [len, dv], S [dk, dv], P [dk])}."""
    mu = w.mu if mu is None else mu
    cu = w.cu_seqlens
    pieces = [((s, h), (slice(int(cu[s]), int(cu[s + 1])), slice(h, h + 1))) for s, h in chains]

    def cat(name):
        return np.concatenate([getattr(w, name)[sl] for _, sl in pieces], axis=0)
    lens = [sl[0].stop - sl[0].start for _, sl in pieces]
    cu2 = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    S0s = None if S0 is None else np.stack([S0[s, h] for (s, h), _ in pieces])[:, None]
    P0s = None if P0 is None else np.stack([P0[s, h] for (s, h), _ in pieces])[:, None]
    fwd = iso_forward if iso else diag_forward
    res = fwd(cat("q"), cat("k"), cat("v"), cat("alpha"), cat("sigma"), cat("r"),
              cu_seqlens=cu2, S0=S0s, P0=P0s, mu=mu, threads=threads, trace=trace)
    out = {}
    for i, ((s, h), _) in enumerate(pieces):
        sl = slice(cu2[i], cu2[i + 1])
        out[(s, h)] = dict(o=res["o"][sl, 0], S=res["S"][i, 0], P=res["P"][i, 0])
        if trace:
            out[(s, h)].update(g=res["trace_g"][sl, 0], beta_eff=res["trace_beta_eff"][sl, 0],
                               Pm=res["trace_Pm"][sl, 0])
    return out


def mobius_matrix(alpha, sigma, k, r, mu: float = 1.0):
    """2x2 matrix of one token's map P -> P_new on one key channel.

    The uncertainty recursion is a linear-fractional (Moebius) map (explainer,
    closing paragraph of "各向同性近似"; aifromscratch, "Approximation 1"): predict
    x -> alpha^2 x + sigma is [[alpha^2, sigma], [0, 1]] and the update
    x -> x / (1 + c x), c = mu k^2 / r, is [[1, 0], [c, 1]]; a token is their
    product update @ predict.  A matrix [[a, b], [c, d]] acts as x -> (a x + b)/(c x + d).
    Arrays broadcast; the result has shape (..., 2, 2).
    """
    a = _f64(alpha) ** 2
    sg = _f64(sigma)
    c = mu * _f64(k) ** 2 / _f64(r)
    a, sg, c = np.broadcast_arrays(a, sg, c)
    M = np.zeros(a.shape + (2, 2))
    M[..., 0, 0] = a
    M[..., 0, 1] = sg
    M[..., 1, 0] = c * a
    M[..., 1, 1] = c * sg + 1.0
    return M


def run_decode(S0, P0, steps, mu: float = 1.0, threads: Optional[int] = None, iso: bool = False):
    """Decode over a list of per-step token dicts ([N,H,d] arrays) from states S0, P0.

    One decode step is one token of the recurrence with the state carried; the
    steps of a sequence are run as one sequence of the diagonal recurrence.
    Returns dict(o [steps,N,H,dv], S, P).
    """
    def stack(name):
        return np.stack([_f64(s[name]) for s in steps], axis=1)  # [N, steps, ...]
    N = S0.shape[0]
    n = len(steps)
    arrs = {nm: stack(nm) for nm in ("q", "k", "v", "alpha", "sigma", "r")}
    flat = {nm: a.reshape((N * n,) + a.shape[2:]) for nm, a in arrs.items()}
    cu = np.arange(N + 1, dtype=np.int64) * n
    fwd = iso_forward if iso else diag_forward
    res = fwd(flat["q"], flat["k"], flat["v"], flat["alpha"], flat["sigma"], flat["r"],
              cu_seqlens=cu, S0=S0, P0=P0, mu=mu, threads=threads)
    o = res["o"].reshape((N, n) + res["o"].shape[1:]).transpose(1, 0, 2, 3)
    return dict(o=o, S=res["S"], P=res["P"])
