"""Seeded synthetic inputs for the Diagonal KDN memory recurrence.

This module is the one piece shared by the CUDA path's tests/bench and the CPU
oracle: it only draws random numbers and shapes them.  It holds none of the
method's arithmetic (no gain, no decay, no state update).

Distributions (Kalman Delta Networks explainer, "对角近似" section, and the
KDA article's per-channel decay section, read as a workload recipe):

* q, k ~ N(0, 1), then L2-normalised per (token, head) vector;
* v ~ N(0, 1);
* alpha = sigmoid(N(4, 1)) per (token, head, key channel)  -- decay in [0, 1];
* r = softplus(N(0, 1)) + 1e-3 per (token, head)           -- observation noise variance;
* sigma = softplus(N(-3, 1)) per (token, head, key channel) -- process noise variance;
* P0 = 1 and S0 = 0 unless a workload says otherwise.

Values are drawn in fp32; where a workload is bf16 they are rounded to bf16
(round to nearest even) and returned as ``uint16`` bit patterns, so both the
GPU path and the oracle read the very same numbers.

Every tensor is drawn in fixed blocks of ``_BLOCK`` elements, each block from its
own PCG64 stream keyed by ``(seed, tensor id, block index)``; the result does not
depend on the number of threads used to draw it.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

_BLOCK = 1 << 22

# tensor ids of the sub-streams (fixed forever: changing one changes every workload)
_Q, _K, _V, _ALPHA, _R, _SIGMA, _S0, _P0, _POOL, _POOLIDX, _LENS = range(11)


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def _stream(seed, tid: int, blk: int) -> np.random.Generator:
    key = list(seed) if isinstance(seed, (tuple, list)) else [int(seed)]
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(key + [tid, blk])))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest even) and return the 16-bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def as_f64(x: np.ndarray) -> np.ndarray:
    """Numbers of an input array as fp64 (bf16 patterns are widened exactly)."""
    if x.dtype == np.uint16:
        return bf16_to_f32(x).astype(np.float64)
    return np.asarray(x, dtype=np.float64)


def _normal(seed: int, tid: int, n: int, loc: float = 0.0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    nblk = (n + _BLOCK - 1) // _BLOCK

    def fill(b):
        lo, hi = b * _BLOCK, min(n, (b + 1) * _BLOCK)
        _stream(seed, tid, b).standard_normal(out=out[lo:hi], dtype=np.float32)
        if loc:
            out[lo:hi] += np.float32(loc)

    if nblk == 1:
        fill(0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(nblk)))
    return out


def _rowwise(fn, x: np.ndarray, rows_per_task: int = 1 << 16) -> np.ndarray:
    """Apply ``fn`` to row blocks of a 2-D array in threads (in place friendly)."""
    n = x.shape[0]
    if n <= rows_per_task:
        return fn(x)
    out = [None] * ((n + rows_per_task - 1) // rows_per_task)

    def work(i):
        out[i] = fn(x[i * rows_per_task:(i + 1) * rows_per_task])

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(work, range(len(out))))
    return np.concatenate(out, axis=0)


def _l2norm_rows(x: np.ndarray) -> np.ndarray:
    return x / np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True)).astype(np.float32)


def _sigmoid(x):
    return (1.0 / (1.0 + np.exp(-x.astype(np.float64)))).astype(np.float32)


def _softplus(x):
    return np.logaddexp(0.0, x.astype(np.float64)).astype(np.float32)


def _finish(x: np.ndarray, bf16: bool) -> np.ndarray:
    if not bf16:
        return np.ascontiguousarray(x, dtype=np.float32)
    return _rowwise(bf16_bits, x.reshape(-1, x.shape[-1])).reshape(x.shape)


@dataclass
class Workload:
    """One problem instance: tokens flattened as [Ntok, H, d] plus sequence boundaries.

    For a dense batch [B, T, H, d] the flattening is token = b*T + t and
    ``cu_seqlens = [0, T, 2T, ..., B*T]``.  ``bf16`` tells whether the token
    tensors hold bf16 patterns (uint16) or fp32 numbers.
    """
    name: str
    H: int
    dk: int
    dv: int
    cu_seqlens: np.ndarray          # int32 [N+1]
    q: np.ndarray                   # [Ntok, H, dk]
    k: np.ndarray                   # [Ntok, H, dk]
    v: np.ndarray                   # [Ntok, H, dv]
    alpha: np.ndarray               # [Ntok, H, dk]
    sigma: np.ndarray               # [Ntok, H, dk]
    r: np.ndarray                   # [Ntok, H]
    bf16: bool
    S0: Optional[np.ndarray] = None  # fp32 [N, H, dk, dv] or None (zeros)
    P0: Optional[np.ndarray] = None  # fp32 [N, H, dk] or None (ones)
    B: int = 0                       # dense batch size (0 for varlen)
    T: int = 0                       # dense sequence length (0 for varlen)
    chunk: int = 64
    mu: float = 1.0
    meta: dict = field(default_factory=dict)

    @property
    def ntok(self) -> int:
        return int(self.cu_seqlens[-1])

    @property
    def num_seqs(self) -> int:
        return len(self.cu_seqlens) - 1


def draw_tokens(seed, ntok: int, H: int, dk: int, dv: int, bf16: bool,
                key_pool_segments: Optional[int] = None, pool_size: int = 256):
    """Draw q, k, v, alpha, sigma, r for ``ntok`` tokens (flattened) and H heads."""
    nk = ntok * H * dk
    q = _rowwise(_l2norm_rows, _normal(seed, _Q, nk).reshape(ntok * H, dk))
    k = _rowwise(_l2norm_rows, _normal(seed, _K, nk).reshape(ntok * H, dk))
    v = _normal(seed, _V, ntok * H * dv).reshape(ntok * H, dv)
    alpha = _rowwise(_sigmoid, _normal(seed, _ALPHA, nk, loc=4.0).reshape(ntok * H, dk))
    r = (_softplus(_normal(seed, _R, ntok * H)) + np.float32(1e-3)).astype(np.float32)
    sigma = _rowwise(_softplus, _normal(seed, _SIGMA, nk, loc=-3.0).reshape(ntok * H, dk))
    k = k.reshape(ntok, H, dk)
    if key_pool_segments:
        # repeated-key overwrites: odd segments draw every key from a fixed per-head
        # pool of unit vectors (pool drawn once), even segments keep fresh keys.
        pool = _l2norm_rows(_normal(seed, _POOL, H * pool_size * dk).reshape(H * pool_size, dk))
        pool = pool.reshape(H, pool_size, dk)
        seg = ntok // key_pool_segments
        g = _stream(seed, _POOLIDX, 0)
        for s in range(1, key_pool_segments, 2):
            idx = g.integers(0, pool_size, size=(seg, H))
            k[s * seg:(s + 1) * seg] = pool[np.arange(H)[None, :], idx]
    shape_k = (ntok, H, dk)
    return dict(q=_finish(q.reshape(shape_k), bf16), k=_finish(k, bf16),
                v=_finish(v.reshape(ntok, H, dv), bf16),
                alpha=_finish(alpha.reshape(shape_k), bf16), sigma=_finish(sigma.reshape(shape_k), bf16),
                r=_finish(r.reshape(ntok, H), bf16))


def varlen_lengths(seed: int, total: int = 262144, lo: int = 512, hi: int = 16384) -> np.ndarray:
    """Sequence lengths ~ U{lo..hi} summing exactly to ``total``.

    Draw until the remainder R is at most ``hi``; the last sequence takes R if
    R >= lo, otherwise R is added to the previous sequence.
    """
    g = _stream(seed, _LENS, 0)
    lens, rem = [], total
    while rem > hi:
        L = int(g.integers(lo, hi + 1))
        lens.append(L)
        rem -= L
    if rem >= lo or not lens:
        lens.append(rem)
    else:
        lens[-1] += rem
    return np.asarray(lens, dtype=np.int64)


def dense(name, seed, B, H, T, dk, dv, bf16, chunk=64, key_pool_segments=None) -> Workload:
    tok = draw_tokens(seed, B * T, H, dk, dv, bf16, key_pool_segments=key_pool_segments)
    cu = (np.arange(B + 1, dtype=np.int64) * T).astype(np.int32)
    return Workload(name=name, H=H, dk=dk, dv=dv, cu_seqlens=cu, bf16=bf16, B=B, T=T, chunk=chunk, **tok)


def varlen(name, seed, total, H, dk, dv, bf16, chunk=64, lo=512, hi=16384) -> Workload:
    lens = varlen_lengths(seed, total, lo, hi)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    tok = draw_tokens(seed, total, H, dk, dv, bf16)
    return Workload(name=name, H=H, dk=dk, dv=dv, cu_seqlens=cu, bf16=bf16, B=1, T=total, chunk=chunk,
                    meta=dict(lengths=lens), **tok)


# ---------------------------------------------------------------- the five workloads
def tiny_fp32(seed: int = 0) -> Workload:
    """B=1, H=2, T=256, d_k=d_v=32, fp32 inputs, P0 = 1, S0 = 0."""
    return dense("tiny_fp32_B1_H2_T256_d32", seed, 1, 2, 256, 32, 32, bf16=False)


def prefill_4x4096(seed: int = 1) -> Workload:
    """Chunkwise prefill: B=4, H=16, T=4096, d_k=d_v=128, bf16 inputs, chunk 64."""
    return dense("prefill_B4_H16_T4096_d128_bf16", seed, 4, 16, 4096, 128, 128, bf16=True)


def long_context_65536(seed: int = 3) -> Workload:
    """B=1, H=32, T=65536, d=128, bf16; odd 4096-token segments reuse a 256-key pool."""
    return dense("long_B1_H32_T65536_d128_bf16_keypool", seed, 1, 32, 65536, 128, 128, bf16=True,
                 key_pool_segments=16)


def varlen_262144(seed: int = 4) -> Workload:
    """Packed varlen prefill: 262144 tokens, lengths U{512..16384}, H=16, d_k=128, d_v=256."""
    return varlen("varlen_262144_H16_dk128_dv256_bf16", seed, 262144, 16, 128, 256, bf16=True)


@dataclass
class DecodeWorkload:
    """Fused decode: N sequences x H heads, one token per step, state resident in fp32."""
    name: str
    N: int
    H: int
    dk: int
    dv: int
    seed: int
    S0: np.ndarray   # fp32 [N, H, dk, dv]
    P0: np.ndarray   # fp32 [N, H, dk]
    mu: float = 1.0

    def step(self, s: int) -> dict:
        """bf16 inputs of decode step ``s`` (each step has its own streams)."""
        tok = draw_tokens((self.seed, 1 + s), self.N, self.H, self.dk, self.dv, bf16=True)
        return tok  # arrays [N, H, d] / [N, H]


def decode_256x32(seed: int = 2, with_state: bool = True, N: int = 256, H: int = 32, d: int = 128) -> DecodeWorkload:
    """N=256, H=32, d_k=d_v=128; S0 ~ N(0, std 0.1), P0 = softplus(N(0,1)), fp32 state."""
    if with_state:
        S0 = (_normal(seed, _S0, N * H * d * d) * np.float32(0.1)).reshape(N, H, d, d)
        P0 = _softplus(_normal(seed, _P0, N * H * d)).reshape(N, H, d)
    else:
        S0 = P0 = None
    return DecodeWorkload(name=f"decode_N{N}_H{H}_d{d}_bf16_fp32state", N=N, H=H, dk=d, dv=d, seed=seed,
                          S0=S0, P0=P0)


WORKLOADS = {0: tiny_fp32, 1: prefill_4x4096, 2: decode_256x32, 3: long_context_65536, 4: varlen_262144}


def decode_inputs_device(seed: int, steps: int, N: int = 256, H: int = 32, d: int = 128, device="cuda"):
    """The fused-decode workload drawn on a device with a seeded torch generator, for runs too long
    to draw and copy from the host (1024 steps of 256 x 32 heads are 10.7 GB of bf16 inputs).

    Same distributions as the host workload: S0 ~ N(0, std 0.1) and P0 = softplus(N(0, 1)) in fp32;
    per step q, k ~ N(0, 1) L2-normalised per (sequence, head), v ~ N(0, 1), alpha = sigmoid(N(4, 1)),
    r = softplus(N(0, 1)) + 1e-3, sigma = softplus(N(-3, 1)), each rounded to bf16.  Returns a dict:
    S0 [N, H, d, d], P0 [N, H, d], and q, k, v, alpha, sigma [steps, N, H, d], r [steps, N, H]."""
    import torch
    import torch.nn.functional as F
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    rn = lambda *shape: torch.randn(shape, generator=g, device=device)
    out = {"S0": 0.1 * rn(N, H, d, d), "P0": F.softplus(rn(N, H, d))}
    shape = (steps, N, H, d)
    out["q"] = F.normalize(rn(*shape), dim=-1).bfloat16()
    out["k"] = F.normalize(rn(*shape), dim=-1).bfloat16()
    out["v"] = rn(*shape).bfloat16()
    out["alpha"] = torch.sigmoid(rn(*shape) + 4.0).bfloat16()
    out["r"] = (F.softplus(rn(steps, N, H)) + 1e-3).bfloat16()
    out["sigma"] = F.softplus(rn(*shape) - 3.0).bfloat16()
    return out
