"""GPU parity of the tcgen05 tensor-core chunk path (bf16 inputs, d_k = 128, chunk 64; two
launches: chunk-parallel prep, chunk-serial state) against the fp64 oracle: ragged tails,
varlen, every d_v tile width, initial states, and the full-size workloads on sampled
(sequence, head) chains.  The same calls without a workspace take the fp32 chunk kernel and
are checked too."""
import numpy as np
import pytest

import oracle
from kalman_delta_rule_b200 import inputs
from tests.kdn_testutil import dense_shape, assert_rel, max_rel_err, oracle_chains, to_dev, to_host
from tests.test_gpu_recurrent import TOL_BF16, ragged, run_forward

pytestmark = pytest.mark.gpu


FORMS = {"two_phase": None, "no_workspace": False}   # workspace argument of run_forward


def path_of(kdn, w, chunk=64):
    p = kdn.kdn_problem_t()
    p.B = w.B or 1
    p.T, p.H, p.d_k, p.d_v = w.ntok // p.B, w.H, w.dk, w.dv
    p.cu_seqlens, p.num_seqs = None, p.B
    p.in_dtype, p.mu, p.chunk = (1 if w.bf16 else 0), 1.0, chunk
    return kdn.PATH_NAMES[kdn.kdn_execution_path(p)]


@pytest.mark.parametrize("form", sorted(FORMS))
@pytest.mark.parametrize("dv", [64, 128, 256])
def test_tc_dense_ragged_tail(kdn, dv, form):
    w = inputs.dense("tc_dense", 300 + dv, 2, 3, 200, 128, dv, bf16=True)   # 200 = 3 chunks + a tail of 8
    assert path_of(kdn, w) == "chunk_tcgen05_two_phase"
    ref = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens)
    o, S, P = run_forward(kdn, w, chunk=64, workspace=FORMS[form])
    assert_rel(o, ref["o"], TOL_BF16, 'o')
    assert_rel(S, ref["S"], TOL_BF16, 'S')
    assert_rel(P, ref["P"], TOL_BF16, 'P')


@pytest.mark.parametrize("H", [20, 80])
def test_tc_two_phase_wider_dv_tiles(kdn, H):
    """Enough (sequence, head) chains that the state kernel takes 64- (H=20) and 128-column
    (H=80) d_v tiles (the small cases above take 32), with a ragged tail."""
    w = inputs.dense("tc_tiles", 40 + H, 2, H, 136, 128, 128, bf16=True)   # 136 = 2 chunks + 8
    ref = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens, mu=2.0)
    o, S, P = run_forward(kdn, w, chunk=64, mu=2.0)
    assert_rel(o, ref["o"], TOL_BF16, 'o')
    assert_rel(S, ref["S"], TOL_BF16, 'S')
    assert_rel(P, ref["P"], TOL_BF16, 'P')


@pytest.mark.parametrize("form", sorted(FORMS))
@pytest.mark.parametrize("mu", [1.0, 128.0])
def test_tc_varlen_with_initial_state(kdn, mu, form):
    """Ragged sequences, an empty one among them, carried S0/P0."""
    w = ragged(77, [1, 63, 64, 0, 65, 200, 130, 7], 2, 128, 128, True)
    rng = np.random.default_rng(8)
    S0 = (0.1 * rng.standard_normal((w.num_seqs, w.H, 128, 128))).astype(np.float32)
    P0 = rng.uniform(0.3, 2.0, (w.num_seqs, w.H, 128)).astype(np.float32)
    ref = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens, S0=S0, P0=P0, mu=mu)
    o, S, P = run_forward(kdn, w, chunk=64, mu=mu, S0=S0, P0=P0, workspace=FORMS[form])
    assert_rel(o, ref["o"], TOL_BF16, 'o')
    assert_rel(S, ref["S"], TOL_BF16, 'S')
    assert_rel(P, ref["P"], TOL_BF16, 'P')
    np.testing.assert_array_equal(S[3], S0[3])     # the empty sequence passes its state through
    np.testing.assert_array_equal(P[3], P0[3])


def sampled_check(kdn, w, picks, tol=TOL_BF16, forms=("two_phase",)):
    ref = oracle_chains(w, picks)
    cu = w.cu_seqlens
    for form in forms:
        o, S, P = run_forward(kdn, w, chunk=64, workspace=FORMS[form])
        for (s, h), rr in ref.items():
            sl = slice(int(cu[s]), int(cu[s + 1]))
            assert_rel(o[sl, h], rr["o"], tol, ('o[sl, h]', (form, s, h)))
            assert_rel(S[s, h], rr["S"], tol, ('S[s, h]', (form, s, h)))
            assert_rel(P[s, h], rr["P"], tol, ('P[s, h]', (form, s, h)))


def test_prefill_4x4096_full_size_sampled(kdn):
    """B=4, H=16, T=4096, d=128, bf16, chunk 64 -- the benchmark's launch configuration."""
    w = inputs.prefill_4x4096()
    assert path_of(kdn, w) == "chunk_tcgen05_two_phase"
    rng = np.random.default_rng(1)
    picks = [(0, 0), (3, 15)] + [(int(a), int(b)) for a, b in zip(rng.integers(0, 4, 6), rng.integers(0, 16, 6))]
    sampled_check(kdn, w, sorted(set(picks)))


def test_long_context_65536_full_size_sampled(kdn):
    """B=1, H=32, T=65536 with repeated-key segments; two whole heads checked."""
    w = inputs.long_context_65536()
    sampled_check(kdn, w, [(0, 0), (0, 31)])


def test_varlen_262144_full_size_sampled(kdn):
    """262144 packed tokens, lengths U{512..16384}, H=16, d_k=128, d_v=256."""
    w = inputs.varlen_262144()
    lens = np.diff(w.cu_seqlens)
    longest = int(np.argmax(lens))
    shortest = int(np.argmin(lens))
    picks = [(longest, 3), (shortest, 0), (w.num_seqs - 1, 15), (0, 7)]
    sampled_check(kdn, w, picks)


@pytest.mark.parametrize("variant", ["diagonal", "isotropic"])
def test_prefill_and_gain_scan_are_bit_reproducible(kdn, variant):
    """The decoupled look-backs form each chunk's starting uncertainty by the same operations
    whichever predecessors had published, so two calls on the prefill workload (4096 units on
    every SM, the look-back paths taken differing from run to run) give identical bits: o, S, P of
    the two-launch forward, and g, k^T g, P of the gain scan."""
    import torch
    w = inputs.prefill_4x4096()
    args = [to_dev(dense_shape(w, getattr(w, n))) for n in ("q", "k", "v", "alpha", "sigma", "r")]
    outs = []
    for _ in range(2):
        o, S, P = kdn.forward(*args, mu=1.0, chunk=64, variant=variant)
        torch.cuda.synchronize()
        kdn.last_device_error()
        outs.append((to_host(o), to_host(S), to_host(P)))
    for a_, b_, n in zip(outs[0], outs[1], ("o", "S", "P")):
        np.testing.assert_array_equal(a_, b_, err_msg=n)
    if variant == "diagonal":
        k, al, sg, r = args[1], args[3], args[4], args[5]
        scans = []
        for _ in range(2):
            g, be, P = kdn.gain_scan(k, al, sg, r, mu=1.0)
            torch.cuda.synchronize()
            kdn.last_device_error()
            scans.append((to_host(g), to_host(be), to_host(P)))
        for a_, b_, n in zip(scans[0], scans[1], ("g", "k^T g", "P")):
            np.testing.assert_array_equal(a_, b_, err_msg=n)
