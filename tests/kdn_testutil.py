"""Helpers shared by the tests: host->device marshalling, the error metric, and
running the oracle on sampled (sequence, head) chains of a workload."""
import numpy as np

import oracle


def max_rel_err(x, y):
    """max |x - y| / max(max |y|, 1e-6) over the whole tensor (y is the oracle)."""
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    if y.size == 0:
        return 0.0
    return float(np.max(np.abs(x - y)) / max(float(np.max(np.abs(y))), 1e-6))


def to_dev(a, device="cuda"):
    import torch
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    if a.dtype == np.int32:
        return torch.from_numpy(a).to(device)
    return torch.from_numpy(a.astype(np.float32)).to(device)


def to_host(t):
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy()
    return t.cpu().numpy()


def dense_shape(w, x):
    """[ntok, H, d] -> [B, T, H, d] (varlen: B = 1)."""
    B = w.B if w.B else 1
    T = x.shape[0] // B
    return x.reshape((B, T) + x.shape[1:])


def oracle_chains(w, chains, mu=None, S0=None, P0=None, threads=None):
    """Oracle on the listed (seq, head) chains of workload ``w``.

    Returns {(s, h): dict(o [len, dv], S [dk, dv], P [dk])}."""
    mu = w.mu if mu is None else mu
    out = {}
    cu = w.cu_seqlens
    pieces = []
    for s, h in chains:
        t0, t1 = int(cu[s]), int(cu[s + 1])
        sl = (slice(t0, t1), slice(h, h + 1))
        pieces.append(((s, h), sl))
    # one oracle call over all chains: pack them as sequences of a 1-head problem
    def cat(name):
        return np.concatenate([getattr(w, name)[sl] for _, sl in pieces], axis=0)
    lens = [sl[0].stop - sl[0].start for _, sl in pieces]
    cu2 = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    S0s = None if S0 is None else np.stack([S0[s, h] for (s, h), _ in pieces])[:, None]
    P0s = None if P0 is None else np.stack([P0[s, h] for (s, h), _ in pieces])[:, None]
    res = oracle.diag_forward(cat("q"), cat("k"), cat("v"), cat("alpha"), cat("sigma"), cat("r"),
                              cu_seqlens=cu2, S0=S0s, P0=P0s, mu=mu, threads=threads)
    for i, ((s, h), _) in enumerate(pieces):
        out[(s, h)] = dict(o=res["o"][cu2[i]:cu2[i + 1], 0], S=res["S"][i, 0], P=res["P"][i, 0])
    return out
