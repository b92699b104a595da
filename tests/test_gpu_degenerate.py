"""GPU parity of every forward path in the recurrence's degenerate regimes.

* no decay, no process noise, near-noiseless observations (r = 1e-3) and one-hot keys on every
  other token: the gain saturates and repeated confirmation drives P down;
* very strong decay (alpha in [0.01, 0.1]): a 64-token chunk's decay underflows fp32, so the
  tensor-core path forms its intra-chunk decay factors on the CUDA cores (log-space pairwise
  factors) and references its state operands to the chunk start and end;
* resets: the usual decay (sigmoid(N(4,1))) with alpha = 0 on scattered (token, channel) entries
  and on every channel of a few tokens -- chunks with a reset take the pairwise form, the others
  the factored tensor-core form, in the same launch.
Every path matches the oracle in every regime, and no kernel reports a device-side condition.
The gain scan is checked in the same regimes.  Sequences of 1, 1, 2, 33, 64 and 130 tokens, and
a larger dense batch on the tensor-core path."""
import dataclasses

import numpy as np
import pytest

import oracle
from kalman_delta_rule_b200 import inputs
from tests.kdn_testutil import dense_shape, assert_rel, max_rel_err, to_dev, to_host
from tests.test_gpu_recurrent import TOL_BF16, TOL_F32, ragged

pytestmark = pytest.mark.gpu

LENS = [1, 1, 2, 33, 64, 130]


def regime(name, dk, dv, bf16, seed=700, lens=LENS, H=2):
    w = ragged(seed, lens, H, dk, dv, False)     # fp32 draws, rounded below where bf16
    rng = np.random.default_rng(seed + 1)
    k, alpha, sigma, r = w.k.copy(), w.alpha.copy(), w.sigma.copy(), w.r.copy()
    if name == "no_decay_noiseless_onehot":
        onehot = np.zeros_like(k[1::2])
        idx = rng.integers(0, dk, size=onehot.shape[:2])
        np.put_along_axis(onehot, idx[..., None], 1.0, axis=-1)
        k[1::2] = onehot
        alpha[:] = 1.0
        sigma[:] = 0.0
        r[:] = 1e-3
    elif name == "strong_decay":
        alpha = rng.uniform(0.01, 0.1, alpha.shape).astype(np.float32)
    elif name == "resets":
        alpha[rng.random(alpha.shape) < 0.02] = 0.0           # scattered single-channel resets
        alpha[rng.random(alpha.shape[0]) < 0.01] = 0.0        # whole-token resets (every head, channel)
    else:
        raise ValueError(name)
    fields = dict(k=k, alpha=alpha, sigma=sigma, r=r)
    if bf16:
        fields = {n: inputs.bf16_bits(x) for n, x in dict(q=w.q, v=w.v, **fields).items()}
    return dataclasses.replace(w, bf16=bf16, **fields)


def forward(kdn, w, chunk, workspace=None, mu=4.0):
    import torch
    args = [to_dev(dense_shape(w, getattr(w, n))) for n in ("q", "k", "v", "alpha", "sigma", "r")]
    cu = to_dev(w.cu_seqlens)
    o, S, P = kdn.forward(*args, cu_seqlens=cu, mu=mu, chunk=chunk, workspace=workspace,
                          max_seqlen=int(np.diff(w.cu_seqlens).max()))
    torch.cuda.synchronize()
    return to_host(o).reshape((-1,) + o.shape[2:]), to_host(S), to_host(P)


# (chunk, workspace, bf16, d_k) of each execution path
PATHS = {
    "recurrent_fp32": (0, None, False, 32),
    "recurrent_bf16": (0, None, True, 128),
    "chunk_fp32": (64, None, False, 64),
    "chunk_bf16_no_workspace": (64, False, True, 128),
    "tensor_core_two_launch": (64, None, True, 128),
}
REGIMES = ["no_decay_noiseless_onehot", "strong_decay", "resets"]


@pytest.mark.parametrize("name", REGIMES)
@pytest.mark.parametrize("path", sorted(PATHS))
def test_degenerate_regime_every_path(kdn, path, name):
    chunk, ws, bf16, dk = PATHS[path]
    w = regime(name, dk, 64, bf16)
    ref = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens, mu=4.0)
    o, S, P = forward(kdn, w, chunk, ws)
    kdn.last_device_error()
    tol = TOL_BF16 if bf16 else TOL_F32
    for got, want, n in ((o, ref["o"], "o"), (S, ref["S"], "S"), (P, ref["P"], "P")):
        assert_rel(got, want, tol, f"{path} {name} {n}")


@pytest.mark.parametrize("name", ["strong_decay", "resets"])
@pytest.mark.parametrize("dv", [128, 256])
def test_tensor_core_decay_regimes_larger_batch(kdn, name, dv):
    """Three sequences of 640, 1000 and 64 tokens x 4 heads (tens of 64-token units in flight, a
    ragged tail), d_v 128 and 256 (two state tile widths), carried S0 and P0."""
    w = regime(name, 128, dv, True, seed=720 + dv, lens=[640, 1000, 64], H=4)
    rng = np.random.default_rng(dv)
    S0 = (0.1 * rng.standard_normal((w.num_seqs, w.H, 128, dv))).astype(np.float32)
    P0 = rng.uniform(0.3, 2.0, (w.num_seqs, w.H, 128)).astype(np.float32)
    ref = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens, S0=S0, P0=P0, mu=2.0)
    import torch
    args = [to_dev(dense_shape(w, getattr(w, n))) for n in ("q", "k", "v", "alpha", "sigma", "r")]
    cu = to_dev(w.cu_seqlens)
    assert kdn.execution_path(args[0], args[2], cu_seqlens=cu, chunk=64) == "chunk_tcgen05_two_phase"
    o, S, P = kdn.forward(*args, cu_seqlens=cu, S0=to_dev(S0), P0=to_dev(P0), mu=2.0, chunk=64)
    torch.cuda.synchronize()
    kdn.last_device_error()
    assert_rel(to_host(o).reshape((-1,) + o.shape[2:]), ref["o"], TOL_BF16, f"{name} o")
    assert_rel(to_host(S), ref["S"], TOL_BF16, f"{name} S")
    assert_rel(to_host(P), ref["P"], TOL_BF16, f"{name} P")


@pytest.mark.parametrize("name", REGIMES)
@pytest.mark.parametrize("bf16,dk", [(False, 32), (True, 128)])
def test_gain_scan_edge_regimes(kdn, name, bf16, dk):
    """The Moebius gain scan (generic kernel for fp32, the TMA kernel for bf16 d_k = 128) in the
    edge regimes: the gain, k^T g and the final uncertainty against the oracle's traces.  The scan
    composes 2x2 maps and never factors the decay."""
    from tests.test_gpu_scan import TOL, run_scan
    w = regime(name, dk, 64, bf16)
    ref = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens, mu=4.0, trace=True)
    g, be, P = run_scan(kdn, w, mu=4.0, max_seqlen=max(LENS))
    assert_rel(g, ref["trace_g"], TOL[bf16], 'g')
    assert_rel(be, ref["trace_beta_eff"], TOL[bf16], 'be')
    assert_rel(P, ref["P"], TOL[bf16], 'P')
