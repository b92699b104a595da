"""GPU parity of the Moebius gain scan (kdn_gain_scan): the gain g_t, the effective
write strength k^T g_t and the final uncertainty, against the oracle's traces."""
import numpy as np
import pytest

import oracle
from kalman_delta_rule_b200 import inputs
from tests.kdn_testutil import dense_shape, assert_rel, max_rel_err, to_dev, to_host
from tests.test_gpu_recurrent import ragged

pytestmark = pytest.mark.gpu

TOL = {False: 1e-4, True: 1e-3}   # fp32 arithmetic on fp32 / bf16-rounded inputs


def run_scan(kdn, w, mu=1.0, P0=None, max_seqlen=0):
    import torch
    args = [to_dev(dense_shape(w, getattr(w, n))) for n in ("k", "alpha", "sigma", "r")]
    cu = to_dev(w.cu_seqlens) if w.B == 1 and w.num_seqs > 1 else None
    g, be, P = kdn.gain_scan(*args, cu_seqlens=cu, P0=to_dev(P0), mu=mu, max_seqlen=max_seqlen)
    torch.cuda.synchronize()
    kdn.last_device_error()
    return to_host(g).reshape(w.k.shape), to_host(be).reshape(w.r.shape), to_host(P)


@pytest.mark.parametrize("mu", [1.0, 32.0])
def test_scan_tiny_fp32(kdn, mu):
    w = inputs.tiny_fp32()
    ref = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens, mu=mu, trace=True)
    g, be, P = run_scan(kdn, w, mu=mu)
    assert_rel(g, ref["trace_g"], TOL[False], 'g')
    assert_rel(be, ref["trace_beta_eff"], TOL[False], 'be')
    assert_rel(P, ref["P"], TOL[False], 'P')


@pytest.mark.parametrize("dk", [32, 64, 128])
@pytest.mark.parametrize("bf16", [False, True])
def test_scan_ragged_varlen(kdn, dk, bf16):
    lens = [1, 63, 64, 65, 300, 129, 7]
    w = ragged(500 + dk, lens, 3, dk, 32, bf16)
    rng = np.random.default_rng(dk)
    P0 = rng.uniform(0.2, 3.0, (w.num_seqs, w.H, dk)).astype(np.float32)
    ref = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens, P0=P0, mu=4.0,
                              trace=True)
    for ms in (0, max(lens)):
        g, be, P = run_scan(kdn, w, mu=4.0, P0=P0, max_seqlen=ms)
        assert_rel(g, ref["trace_g"], TOL[bf16], 'g')
        assert_rel(be, ref["trace_beta_eff"], TOL[bf16], 'be')
        assert_rel(P, ref["P"], TOL[bf16], 'P')


def test_scan_long_context_full_size_sampled(kdn):
    """T=65536: 1024 chunks per head, so the look-back chains are long."""
    w = inputs.long_context_65536()
    g, be, P = run_scan(kdn, w)
    ref = oracle.diag_chains(w, [(0, 0), (0, 17)], trace=True)
    for (s, h), rr in ref.items():
        assert_rel(g[:, h], rr["g"], TOL[True], 'g[:, h]')
        assert_rel(be[:, h], rr["beta_eff"], TOL[True], 'be[:, h]')
        assert_rel(P[s, h], rr["P"], TOL[True], 'P[s, h]')


def test_scan_prefill_full_size_sampled(kdn):
    w = inputs.prefill_4x4096()
    g, be, P = run_scan(kdn, w)
    picks = [(0, 0), (1, 5), (3, 15)]
    ref = oracle.diag_chains(w, picks, trace=True)
    for (s, h), rr in ref.items():
        sl = slice(int(w.cu_seqlens[s]), int(w.cu_seqlens[s + 1]))
        assert_rel(g[sl, h], rr["g"], TOL[True], 'g[sl, h]')
        assert_rel(be[sl, h], rr["beta_eff"], TOL[True], 'be[sl, h]')
        assert_rel(P[s, h], rr["P"], TOL[True], 'P[s, h]')


def test_scan_reports_a_too_small_max_seqlen(kdn):
    """A sequence longer than max_seqlen is an argument error reported by the device
    error word; chunks past the bound are skipped (no wait depends on them)."""
    import torch
    w = ragged(9, [40, 200], 2, 64, 32, True)
    args = [to_dev(dense_shape(w, getattr(w, n))) for n in ("k", "alpha", "sigma", "r")]
    kdn.gain_scan(*args, cu_seqlens=to_dev(w.cu_seqlens), max_seqlen=64)
    torch.cuda.synchronize()
    with pytest.raises(kdn.KdnError) as ei:
        kdn.last_device_error()
    assert ei.value.code == kdn.KDN_ERR_INVALID_ARG
    kdn.last_device_error()   # the word was cleared


def test_information_scaling_weakens_the_effective_write_strength(kdn):
    """Kalman Delta Networks explainer (techwalker), information scaling: mu = d_k instead of
    1 lowers the mean effective write strength k^T g, also with the inputs held fixed.
    P^- is monotone in mu (every Moebius step is monotone in P) and k^T g = k^T P^- k /
    (r + k^T P^- k) grows with P^-, so the drop holds token by token; both settings are
    also checked against the oracle's traces on one chain."""
    w = inputs.prefill_4x4096()
    means = {}
    for mu in (1.0, 128.0):
        g, be, P = run_scan(kdn, w, mu=mu)
        ref = oracle.diag_chains(w, [(0, 3)], mu=mu, trace=True)[(0, 3)]
        assert_rel(be[:4096, 3], ref["beta_eff"], TOL[True], 'be[:4096, 3]')
        means[mu] = be
    assert np.all(means[128.0] <= means[1.0] * (1 + 1e-5) + 1e-7)
    assert float(np.mean(means[128.0])) < float(np.mean(means[1.0]))
