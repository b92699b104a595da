"""GPU parity of the isotropic KDN (one uncertainty per head) on every execution path
-- token-serial recurrence, fp32 CUDA-core chunks, tcgen05 chunks, multi-token decode --
against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest

import oracle
from kalman_delta_rule_b200 import inputs
from tests.kdn_testutil import dense_shape, assert_rel, max_rel_err, to_dev, to_host
from tests.test_gpu_recurrent import ragged

pytestmark = pytest.mark.gpu

TOL_F32, TOL_BF16 = 1e-4, 2e-2


def run_iso(kdn, w, chunk, mu=1.0, S0=None, P0=None, workspace=None):
    """Isotropic forward; ``workspace`` None allocates one (two-launch tensor-core path where
    it applies), False passes none (the fp32 chunk kernel)."""
    import torch
    args = [to_dev(dense_shape(w, getattr(w, n))) for n in ("q", "k", "v", "alpha", "sigma", "r")]
    cu = to_dev(w.cu_seqlens) if w.B == 1 and w.num_seqs > 1 else None
    max_seqlen = int(np.diff(w.cu_seqlens).max()) if cu is not None else 0
    path = kdn.execution_path(args[0], args[2], cu_seqlens=cu, chunk=chunk, variant="isotropic",
                              workspace=workspace is None)
    o, S, P = kdn.forward(*args, cu_seqlens=cu, S0=to_dev(S0), P0=to_dev(P0), mu=mu, chunk=chunk,
                          variant="isotropic", workspace=workspace, max_seqlen=max_seqlen)
    torch.cuda.synchronize()
    kdn.last_device_error()
    return path, to_host(o).reshape((-1,) + o.shape[2:]), to_host(S), to_host(P)


@pytest.mark.parametrize("chunk", [0, 16, 32, 64])
@pytest.mark.parametrize("mu", [1.0, 32.0])
def test_iso_tiny_fp32_every_chunk(kdn, chunk, mu):
    w = inputs.tiny_fp32()
    ref = oracle.iso_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens, mu=mu)
    path, o, S, P = run_iso(kdn, w, chunk, mu=mu)
    assert path == ("recurrent" if chunk == 0 else "chunk_fp32")
    assert P.shape == ref["P"].shape
    assert_rel(o, ref["o"], TOL_F32, 'o')
    assert_rel(S, ref["S"], TOL_F32, 'S')
    assert_rel(P, ref["P"], TOL_F32, 'P')


@pytest.mark.parametrize("dk,dv,chunk,form", [(128, 64, 64, "two_phase"), (128, 128, 64, "two_phase"),
                                              (128, 256, 64, "two_phase"), (128, 128, 64, "no_workspace"),
                                              (128, 256, 64, "no_workspace"), (64, 128, 64, "two_phase"),
                                              (128, 128, 0, "two_phase"), (32, 32, 32, "two_phase")])
def test_iso_ragged_varlen_bf16_with_initial_state(kdn, dk, dv, chunk, form):
    """Ragged sequences (1 token, chunk-1, chunk, chunk+1, several chunks and a tail),
    an empty sequence, carried S0 and p0, mu = 4; tensor-core cases in both forms."""
    w = ragged(700 + dk + dv + chunk, [1, 63, 64, 0, 65, 300], 3, dk, dv, True)
    rng = np.random.default_rng(dk + dv)
    S0 = (0.1 * rng.standard_normal((w.num_seqs, w.H, dk, dv))).astype(np.float32)
    P0 = rng.uniform(0.3, 2.0, (w.num_seqs, w.H)).astype(np.float32)
    ref = oracle.iso_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens, S0=S0, P0=P0, mu=4.0)
    path, o, S, P = run_iso(kdn, w, chunk, mu=4.0, S0=S0, P0=P0, workspace=None if form == "two_phase" else False)
    if chunk == 64 and dk == 128:
        assert path == ("chunk_tcgen05_two_phase" if form == "two_phase" else "chunk_fp32")
    assert_rel(o, ref["o"], TOL_BF16, 'o')
    assert_rel(S, ref["S"], TOL_BF16, 'S')
    assert_rel(P, ref["P"], TOL_BF16, 'P')
    np.testing.assert_array_equal(P[3], P0[3])      # the empty sequence keeps its uncertainty


def test_iso_prefill_full_size_sampled(kdn):
    """The prefill workload (4 x 4096 tokens, 16 heads, d = 128, bf16) on the tcgen05 path;
    sampled chains against the oracle element by element."""
    w = inputs.prefill_4x4096()
    ref = oracle.diag_chains(w, [(0, 0), (2, 7), (3, 15)], iso=True)
    for workspace, name in ((None, "chunk_tcgen05_two_phase"),):
        path, o, S, P = run_iso(kdn, w, 64, workspace=workspace)
        assert path == name
        o = o.reshape(w.B * w.T, w.H, -1)
        for (s, h), rr in ref.items():
            sl = slice(int(w.cu_seqlens[s]), int(w.cu_seqlens[s + 1]))
            assert_rel(o[sl, h], rr["o"], TOL_BF16, ('o[sl, h]', (name, s, h)))
            assert_rel(S[s, h], rr["S"], TOL_BF16, ('S[s, h]', (name, s, h)))
            assert_rel(P[s, h], rr["P"], TOL_BF16, ('P[s, h]', (name, s, h)))


@pytest.mark.parametrize("n", [1, 5])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 256)])
def test_iso_decode_tokens_matches_oracle(kdn, n, dk, dv):
    import torch
    N, H = 5, 3
    rng = np.random.default_rng(n + dk)
    S0 = (0.1 * rng.standard_normal((N, H, dk, dv))).astype(np.float32)
    P0 = np.logaddexp(0, rng.standard_normal((N, H))).astype(np.float32)
    steps = [inputs.draw_tokens((21, n, s), N, H, dk, dv, True) for s in range(n)]
    stacked = {nm: np.stack([st[nm] for st in steps], axis=1) for nm in steps[0]}
    S, P = to_dev(S0).clone(), to_dev(P0).clone()
    o = kdn.decode_tokens(*[to_dev(stacked[nm]) for nm in ("q", "k", "v", "alpha", "sigma", "r")], S, P, mu=3.0,
                          variant="isotropic")
    torch.cuda.synchronize()
    kdn.last_device_error()
    ref = oracle.run_decode(S0, P0, steps, mu=3.0, iso=True)
    assert_rel(to_host(o).transpose(1, 0, 2, 3), ref["o"], TOL_BF16, 'to_host(o).transpose(1, 0, 2, 3)')
    assert_rel(to_host(S), ref["S"], TOL_BF16, 'to_host(S)')
    assert_rel(to_host(P), ref["P"], TOL_BF16, 'to_host(P)')
    if n == 1:   # the single-step wrapper takes the same path
        S2, P2 = to_dev(S0).clone(), to_dev(P0).clone()
        o2 = kdn.decode_step(*[to_dev(steps[0][nm]) for nm in ("q", "k", "v", "alpha", "sigma", "r")], S2, P2,
                             mu=3.0, variant="isotropic")
        torch.cuda.synchronize()
        np.testing.assert_array_equal(to_host(o2), to_host(o)[:, 0])
        np.testing.assert_array_equal(to_host(S2), to_host(S))
