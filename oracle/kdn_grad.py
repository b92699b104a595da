"""fp64 gradients of the KDN forward, diagonal and isotropic (test infrastructure).

TEST INFRASTRUCTURE ONLY: imported by ``tests/`` and by the benchmark's CPU-baseline
leg -- never by the product path.  It shares no code with the CUDA library.

The forward is restated token by token with plain PyTorch CPU ops in fp64, in the
order of the explainer's diagonal approximation ("对角近似") and the KDA article's
decayed delta rule ("Delta rule" and "per-channel decay" sections):

    P^-  = alpha^2 * P + sigma                    (predict; the diagonal stays diagonal)
    den  = r + sum_i P^-_i k_i^2,  g = P^- k / den (Kalman gain)
    W    = diag(alpha) S,  u = v - W^T k,  S = W + g u^T   (decayed delta write)
    o    = S^T q                                   (readout after the write)
    P    = P^- / (1 + mu P^- k^2 / r)              (mean-field update, information scaled by mu)

and the gradients are PyTorch's reverse-mode differentiation of that loop.  The isotropic
variant (explainer "各向同性近似") keeps one uncertainty p per head:

    p^-  = mean(alpha^2) p + mean(sigma),  g = p^- k / (r + p^- |k|^2),
    p    = p^- / (1 + mu p^- |k|^2 / (d_k r))

The scalar being differentiated is  <o, d_o> + <S_T, dS_T> + <P_T, dP_T>, so the
results are the vector-Jacobian products a training step needs.

Pins (tests/test_oracle_grad.py): the restated forward equals the C oracle
(kdn_oracle.c, itself pinned), both variants; every gradient equals central finite
differences of the C oracle, both variants; single-token closed forms (diagonal); the
readout gradients at the first token do not depend on mu.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch


def _f64(x):
    if x is None:
        return None
    x = np.asarray(x)
    if x.dtype == np.uint16:   # bf16 bit patterns: exact widening
        x = (x.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64))


def forward_t(q, k, v, alpha, sigma, r, cu, S0, P0, mu: float, iso: bool = False):
    """The KDN forward on fp64 torch tensors (token layout [ntok, H, d]).

    cu: list of sequence boundaries; S0 [nseq,H,dk,dv], P0 [nseq,H,dk] ([nseq,H] isotropic).
    Returns o [ntok,H,dv], S [nseq,H,dk,dv], P (shaped as P0) (differentiable)."""
    outs, Ss, Ps = [], [], []
    dk = k.shape[-1]
    for s in range(len(cu) - 1):
        S, P = S0[s], P0[s]
        for t in range(cu[s], cu[s + 1]):
            a, kk = alpha[t], k[t]                       # [H, dk]
            if iso:
                Pm = (a * a).mean(-1) * P + sigma[t].mean(-1)      # [H]
                K2 = (kk * kk).sum(-1)
                den = r[t] + Pm * K2
                g = Pm[:, None] * kk / den[:, None]
            else:
                Pm = a * a * P + sigma[t]
                den = r[t] + (Pm * kk * kk).sum(-1)      # [H]
                g = Pm * kk / den[:, None]
            W = a[:, :, None] * S
            u = v[t] - torch.einsum("hij,hi->hj", W, kk)
            S = W + g[:, :, None] * u[:, None, :]
            outs.append(torch.einsum("hij,hi->hj", S, q[t]))
            if iso:
                P = Pm / (1.0 + mu * Pm * K2 / (dk * r[t]))
            else:
                P = Pm / (1.0 + mu * Pm * kk * kk / r[t][:, None])
        Ss.append(S)
        Ps.append(P)
    o = torch.stack(outs) if outs else torch.zeros((0,) + v.shape[1:], dtype=torch.float64)
    return o, torch.stack(Ss), torch.stack(Ps)


def diag_grad(q, k, v, alpha, sigma, r, d_o, cu_seqlens=None, S0=None, P0=None, dS=None, dP=None,
              mu: float = 1.0, threads: Optional[int] = None, iso: bool = False):
    """Gradients of <o, d_o> + <S_T, dS> + <P_T, dP> with respect to every input.

    Token tensors [ntok, H, d] (r: [ntok, H]); bf16 bit patterns (uint16) are widened
    exactly.  S0 defaults to 0 and P0 to 1 (their gradients are returned either way);
    with ``iso`` the uncertainty is one scalar per head (P0, dP, P: [nseq, H]).
    Returns numpy fp64 arrays: dq, dk, dv, dalpha, dsigma, dr, dS0, dP0, and the
    forward's o, S, P."""
    if threads:
        torch.set_num_threads(int(threads))
    q, k, v, alpha, sigma, r, d_o = map(_f64, (q, k, v, alpha, sigma, r, d_o))
    ntok, H, dk = k.shape
    dv = v.shape[-1]
    cu = [0, ntok] if cu_seqlens is None else [int(x) for x in np.asarray(cu_seqlens)]
    nseq = len(cu) - 1
    S0 = torch.zeros((nseq, H, dk, dv), dtype=torch.float64) if S0 is None else _f64(S0)
    pshape = (nseq, H) if iso else (nseq, H, dk)
    P0 = torch.ones(pshape, dtype=torch.float64) if P0 is None else _f64(P0)
    leaves = [x.clone().requires_grad_(True) for x in (q, k, v, alpha, sigma, r, S0, P0)]
    o, S, P = forward_t(*leaves[:6], cu, leaves[6], leaves[7], float(mu), iso=iso)
    loss = (o * d_o).sum()
    if dS is not None:
        loss = loss + (S * _f64(dS)).sum()
    if dP is not None:
        loss = loss + (P * _f64(dP)).sum()
    grads = torch.autograd.grad(loss, leaves, allow_unused=True)
    names = ("dq", "dk", "dv", "dalpha", "dsigma", "dr", "dS0", "dP0")
    out = {n: (g.numpy() if g is not None else np.zeros(x.shape)) for n, g, x in zip(names, grads, leaves)}
    out.update(o=o.detach().numpy(), S=S.detach().numpy(), P=P.detach().numpy())
    return out
