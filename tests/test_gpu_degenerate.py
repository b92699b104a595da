"""GPU parity of every forward path in the recurrence's degenerate regimes, and the tensor-core
path's documented range limit.

* no decay, no process noise, near-noiseless observations (r = 1e-3) and one-hot keys on every
  other token: the gain saturates and repeated confirmation drives P down -- every path matches
  the oracle;
* very strong decay (alpha in [0.01, 0.1]): the chunk's cumulative decay underflows fp32 within a
  64-token chunk.  The token-serial and fp32 chunk paths (pairwise decay factors) still match the
  oracle; the tensor-core paths, which factor the decay through the chunk start, report
  KDN_ERR_RANGE through kdn_last_device_error (and the error word is cleared afterwards).
The gain scan is checked in both regimes as well.  Sequences of 1, 1, 2, 33, 64 and 130 tokens."""
import dataclasses

import numpy as np
import pytest

import oracle
from kalman_delta_rule_b200 import inputs
from tests.kdn_testutil import dense_shape, max_rel_err, to_dev, to_host
from tests.test_gpu_recurrent import TOL_BF16, TOL_F32, ragged

pytestmark = pytest.mark.gpu

LENS = [1, 1, 2, 33, 64, 130]


def regime(name, dk, dv, bf16, seed=700):
    w = ragged(seed, LENS, 2, dk, dv, False)     # fp32 draws, rounded below where bf16
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
    else:
        alpha = rng.uniform(0.01, 0.1, alpha.shape).astype(np.float32)
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


# (path, chunk, workspace, bf16, d_k): the four execution paths
PATHS = {
    "recurrent_fp32": (0, None, False, 32),
    "recurrent_bf16": (0, None, True, 128),
    "chunk_fp32": (64, None, False, 64),
    "tensor_core_two_launch": (64, None, True, 128),
    "tensor_core_fused": (64, False, True, 128),
}


@pytest.mark.parametrize("path", sorted(PATHS))
def test_no_decay_noiseless_onehot_every_path(kdn, path):
    chunk, ws, bf16, dk = PATHS[path]
    w = regime("no_decay_noiseless_onehot", dk, 64, bf16)
    ref = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens, mu=4.0)
    o, S, P = forward(kdn, w, chunk, ws)
    kdn.last_device_error()
    tol = TOL_BF16 if bf16 else TOL_F32
    for got, want, n in ((o, ref["o"], "o"), (S, ref["S"], "S"), (P, ref["P"], "P")):
        assert max_rel_err(got, want) <= tol, f"{path} {n}: {max_rel_err(got, want):.3e}"


@pytest.mark.parametrize("path", ["recurrent_fp32", "recurrent_bf16", "chunk_fp32"])
def test_strong_decay_fp32_paths_match(kdn, path):
    chunk, ws, bf16, dk = PATHS[path]
    w = regime("strong_decay", dk, 64, bf16)
    ref = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens, mu=4.0)
    o, S, P = forward(kdn, w, chunk, ws)
    kdn.last_device_error()
    tol = TOL_BF16 if bf16 else TOL_F32
    for got, want, n in ((o, ref["o"], "o"), (S, ref["S"], "S"), (P, ref["P"], "P")):
        assert max_rel_err(got, want) <= tol, f"{path} {n}: {max_rel_err(got, want):.3e}"


@pytest.mark.parametrize("path", ["tensor_core_two_launch", "tensor_core_fused"])
def test_strong_decay_tensor_core_paths_report_range(kdn, path):
    chunk, ws, bf16, dk = PATHS[path]
    w = regime("strong_decay", dk, 64, bf16)
    forward(kdn, w, chunk, ws)
    with pytest.raises(kdn.KdnError) as err:
        kdn.last_device_error()
    assert err.value.code == kdn.KDN_ERR_RANGE
    # the error word was cleared: an in-range call reports nothing
    ok = regime("no_decay_noiseless_onehot", dk, 64, bf16)
    forward(kdn, ok, chunk, ws)
    kdn.last_device_error()


@pytest.mark.parametrize("name", ["no_decay_noiseless_onehot", "strong_decay"])
@pytest.mark.parametrize("bf16,dk", [(False, 32), (True, 128)])
def test_gain_scan_edge_regimes(kdn, name, bf16, dk):
    """The Moebius gain scan (generic kernel for fp32, the TMA kernel for bf16 d_k = 128) in both
    edge regimes: the gain, k^T g and the final uncertainty against the oracle's traces.  The scan
    composes 2x2 maps and never factors the decay, so strong decay is in range."""
    from tests.test_gpu_scan import TOL, run_scan
    w = regime(name, dk, 64, bf16)
    ref = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens, mu=4.0, trace=True)
    g, be, P = run_scan(kdn, w, mu=4.0, max_seqlen=max(LENS))
    assert max_rel_err(g, ref["trace_g"]) <= TOL[bf16]
    assert max_rel_err(be, ref["trace_beta_eff"]) <= TOL[bf16]
    assert max_rel_err(P, ref["P"]) <= TOL[bf16]
