"""GPU parity of the chunkwise forward (kdn_forward_chunkwise) against the oracle:
every chunk size, ragged varlen edges, extreme decays and the split-sequence carry."""
import numpy as np
import pytest

import oracle
from kalman_delta_rule_b200 import inputs
from tests.kdn_testutil import assert_rel, max_rel_err
from tests.test_gpu_recurrent import TOL_BF16, TOL_F32, ragged, run_forward

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("mu", [1.0, 32.0])
def test_tiny_fp32_chunkwise_matches_oracle(kdn, chunk, mu):
    w = inputs.tiny_fp32()
    ref = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens, mu=mu)
    o, S, P = run_forward(kdn, w, chunk=chunk, mu=mu)
    assert_rel(o, ref["o"], TOL_F32, 'o')
    assert_rel(S, ref["S"], TOL_F32, 'S')
    assert_rel(P, ref["P"], TOL_F32, 'P')


@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 128), (128, 256), (128, 64)])
@pytest.mark.parametrize("bf16", [False, True])
def test_ragged_varlen_chunkwise(kdn, chunk, dk, dv, bf16):
    w = ragged(200 + dk + dv + chunk, [1, 63, 64, 65, 130, 17], 2, dk, dv, bf16)
    rng = np.random.default_rng(3)
    S0 = (0.1 * rng.standard_normal((w.num_seqs, w.H, dk, dv))).astype(np.float32)
    P0 = rng.uniform(0.3, 2.0, (w.num_seqs, w.H, dk)).astype(np.float32)
    ref = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens, S0=S0, P0=P0, mu=3.0)
    o, S, P = run_forward(kdn, w, chunk=chunk, mu=3.0, S0=S0, P0=P0)
    tol = TOL_BF16 if bf16 else TOL_F32
    assert_rel(o, ref["o"], tol, 'o')
    assert_rel(S, ref["S"], tol, 'S')
    assert_rel(P, ref["P"], tol, 'P')


def test_extreme_decays_fp32(kdn):
    """alpha = 0 (full reset), alpha = 1 and tiny alphas inside one chunk: the
    chunk algebra must follow the serial recurrence."""
    w = ragged(31, [64, 100], 2, 64, 64, False)
    rng = np.random.default_rng(4)
    a = w.alpha.copy()
    a[5] = 0.0
    a[70] = 1.0
    a[80:90] = rng.uniform(1e-6, 1e-3, a[80:90].shape)
    w.alpha = a.astype(np.float32)
    ref = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens)
    for chunk in (0, 16, 64):
        o, S, P = run_forward(kdn, w, chunk=chunk)
        assert_rel(o, ref["o"], TOL_F32, ('o', chunk))
        assert_rel(S, ref["S"], TOL_F32, ('S', chunk))
        assert_rel(P, ref["P"], TOL_F32, ('P', chunk))


def test_split_sequence_carry_on_gpu(kdn):
    """Running a sequence in two calls, the second starting from the first's final
    (S, P), equals one call (the recurrent state is the checkpoint)."""
    w = inputs.tiny_fp32()
    full_o, full_S, full_P = run_forward(kdn, w, chunk=64)
    cut = 100

    def part(lo, hi):
        return inputs.Workload(name="part", H=w.H, dk=w.dk, dv=w.dv, cu_seqlens=np.array([0, hi - lo], np.int32),
                               bf16=False, B=1, T=hi - lo, q=w.q[lo:hi], k=w.k[lo:hi], v=w.v[lo:hi],
                               alpha=w.alpha[lo:hi], sigma=w.sigma[lo:hi], r=w.r[lo:hi])
    o1, S1, P1 = run_forward(kdn, part(0, cut), chunk=64)
    o2, S2, P2 = run_forward(kdn, part(cut, w.ntok), chunk=64, S0=S1, P0=P1)
    assert_rel(np.concatenate([o1, o2]), full_o, TOL_F32, 'np.concatenate([o1, o2])')
    assert_rel(S2, full_S, TOL_F32, 'S2')
    assert_rel(P2, full_P, TOL_F32, 'P2')
