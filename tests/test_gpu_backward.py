"""GPU parity of the backward pass (kdn_backward) against the fp64 gradient oracle
(oracle/kdn_grad.py): every gradient, element by element, for fp32 and bf16 inputs, ragged
varlen batches with an empty sequence, initial states and final-state gradients, every d_k
and the d_v extremes, both uncertainty variants, and the full-size prefill workload
(B4 H16 T4096 d128 bf16) on sampled (sequence, head) chains -- each chain's gradients depend
on that chain's inputs only."""
import functools

import numpy as np
import pytest

from kalman_delta_rule_b200 import inputs
from oracle import kdn_grad
from tests.kdn_testutil import dense_shape, assert_rel, max_rel_err, to_dev, to_host
from tests.test_gpu_recurrent import ragged

pytestmark = pytest.mark.gpu

# fp32 arithmetic on exactly widened inputs (bf16 inputs are widened without rounding on both
# sides), so bf16 and fp32 inputs share the fp32 tolerance
TOL = 1e-4
NAMES = ("dq", "dk", "dv", "dalpha", "dsigma", "dr", "dS0", "dP0")


def cotangents(seed, w, with_final=True, iso=False):
    rng = np.random.default_rng(seed)
    d_o = rng.standard_normal((w.ntok, w.H, w.dv)).astype(np.float32)
    if w.bf16:
        d_o = inputs.bf16_bits(d_o)
    dS = dP = None
    if with_final:
        dS = rng.standard_normal((w.num_seqs, w.H, w.dk, w.dv)).astype(np.float32)
        dP = rng.standard_normal((w.num_seqs, w.H) + (() if iso else (w.dk,))).astype(np.float32)
    return d_o, dS, dP


def initial_state(seed, w, iso=False):
    rng = np.random.default_rng(seed)
    S0 = (0.1 * rng.standard_normal((w.num_seqs, w.H, w.dk, w.dv))).astype(np.float32)
    P0 = rng.uniform(0.3, 2.0, (w.num_seqs, w.H) + (() if iso else (w.dk,))).astype(np.float32)
    return S0, P0


def run_backward(kdn, w, d_o, S0=None, P0=None, dS=None, dP=None, mu=1.0, iso=False):
    import torch
    args = [to_dev(dense_shape(w, getattr(w, n))) for n in ("q", "k", "v", "alpha", "sigma", "r")]
    cu = to_dev(w.cu_seqlens) if w.B == 1 and w.num_seqs > 1 else None
    g = kdn.backward(*args, to_dev(dense_shape(w, d_o)), cu_seqlens=cu, S0=to_dev(S0), P0=to_dev(P0),
                     dS=to_dev(dS), dP=to_dev(dP), mu=mu, variant="isotropic" if iso else "diagonal")
    torch.cuda.synchronize()
    kdn.last_device_error()
    out = {n: to_host(g[n]) for n in NAMES}
    for n in ("dq", "dk", "dv", "dalpha", "dsigma", "dr"):
        out[n] = out[n].reshape((w.ntok,) + out[n].shape[2:])
    return out


def check(got, ref, tol=TOL):
    for n in NAMES:
        assert_rel(got[n], ref[n], tol, n)


@pytest.mark.parametrize("mu", [1.0, 32.0])
def test_backward_tiny_fp32(kdn, mu):
    w = inputs.tiny_fp32()
    S0, P0 = initial_state(1, w)
    d_o, dS, dP = cotangents(2, w)
    ref = kdn_grad.diag_grad(w.q, w.k, w.v, w.alpha, w.sigma, w.r, d_o, cu_seqlens=w.cu_seqlens,
                             S0=S0, P0=P0, dS=dS, dP=dP, mu=mu)
    check(run_backward(kdn, w, d_o, S0, P0, dS, dP, mu=mu), ref)


@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 256), (128, 128)])
@pytest.mark.parametrize("bf16", [False, True])
def test_backward_ragged_varlen(kdn, dk, dv, bf16):
    """Sequences of 1, 63, 64, 0, 65 and 130 tokens (one empty): partial checkpoint chunks,
    partial sub-checkpoint groups and an empty chain, with S0/P0 and final-state gradients."""
    w = ragged(400 + dk + dv, [1, 63, 64, 0, 65, 130], 2, dk, dv, bf16)
    S0, P0 = initial_state(3, w)
    d_o, dS, dP = cotangents(4, w)
    ref = kdn_grad.diag_grad(w.q, w.k, w.v, w.alpha, w.sigma, w.r, d_o, cu_seqlens=w.cu_seqlens,
                             S0=S0, P0=P0, dS=dS, dP=dP, mu=2.0)
    got = run_backward(kdn, w, d_o, S0, P0, dS, dP, mu=2.0)
    check(got, ref)
    # the empty sequence passes the final-state gradients straight through
    np.testing.assert_array_equal(got["dS0"][3], dS[3])
    np.testing.assert_array_equal(got["dP0"][3], dP[3])


@pytest.mark.parametrize("dk,dv,bf16", [(32, 32, False), (64, 256, True), (128, 128, True)])
def test_backward_isotropic_ragged_varlen(kdn, dk, dv, bf16):
    """The isotropic variant (one uncertainty per head): ragged sequences with an empty one,
    S0/p0 and final-state gradients."""
    w = ragged(500 + dk + dv, [1, 63, 64, 0, 65, 130], 2, dk, dv, bf16)
    S0, P0 = initial_state(7, w, iso=True)
    d_o, dS, dP = cotangents(8, w, iso=True)
    ref = kdn_grad.diag_grad(w.q, w.k, w.v, w.alpha, w.sigma, w.r, d_o, cu_seqlens=w.cu_seqlens,
                             S0=S0, P0=P0, dS=dS, dP=dP, mu=3.0, iso=True)
    got = run_backward(kdn, w, d_o, S0, P0, dS, dP, mu=3.0, iso=True)
    check(got, ref)
    np.testing.assert_array_equal(got["dP0"][3], dP[3])


@pytest.mark.parametrize("regime", ["no_decay_noiseless_onehot", "strong_decay"])
def test_backward_degenerate_regimes(kdn, regime):
    """Edge regimes of the recurrence: (a) alpha = 1, sigma = 0, r = 1e-3 and one-hot keys on every
    other token (the gain saturates, repeated confirmation drives P down); (b) alpha in [0.01, 0.1],
    where the state before a token cannot be recovered by undoing the decay -- the state pass
    re-steps it forward from checkpoints instead.  Many one-token sequences among longer ones."""
    import dataclasses
    w = ragged(600, [1, 1, 2, 33, 64, 97], 2, 32, 32, False)
    rng = np.random.default_rng(11)
    if regime == "no_decay_noiseless_onehot":
        k = w.k.copy()
        onehot = np.zeros_like(k[1::2])
        idx = rng.integers(0, w.dk, size=onehot.shape[:2])
        np.put_along_axis(onehot, idx[..., None], 1.0, axis=-1)
        k[1::2] = onehot
        w = dataclasses.replace(w, k=k.astype(np.float32), alpha=np.ones_like(w.alpha), sigma=np.zeros_like(w.sigma),
                                r=np.full_like(w.r, 1e-3))
    else:
        w = dataclasses.replace(w, alpha=rng.uniform(0.01, 0.1, w.alpha.shape).astype(np.float32))
    S0, P0 = initial_state(9, w)
    d_o, dS, dP = cotangents(10, w)
    ref = kdn_grad.diag_grad(w.q, w.k, w.v, w.alpha, w.sigma, w.r, d_o, cu_seqlens=w.cu_seqlens,
                             S0=S0, P0=P0, dS=dS, dP=dP, mu=32.0)
    check(run_backward(kdn, w, d_o, S0, P0, dS, dP, mu=32.0), ref)


def test_backward_dense_defaults(kdn):
    """Dense batch, S0 = 0 and P0 = 1 by default, no final-state gradients."""
    w = inputs.dense("bwd_dense", 12, 2, 3, 150, 128, 128, bf16=True)
    d_o, _, _ = cotangents(5, w, with_final=False)
    ref = kdn_grad.diag_grad(w.q, w.k, w.v, w.alpha, w.sigma, w.r, d_o, cu_seqlens=w.cu_seqlens)
    check(run_backward(kdn, w, d_o), ref)


def test_backward_full_size_sampled_chains(kdn):
    """The prefill workload at full size (B4 H16 T4096 d128 bf16) through one backward call;
    the oracle recomputes two (sequence, head) chains on their own."""
    w = inputs.prefill_4x4096()
    d_o, dS, dP = cotangents(6, w)
    got = run_backward(kdn, w, d_o, dS=dS, dP=dP)
    T = w.ntok // w.B
    for s, h in ((0, 0), (3, 15)):
        sl = slice(s * T, (s + 1) * T)
        pick = lambda x: x[sl, h:h + 1]
        ref = kdn_grad.diag_grad(pick(w.q), pick(w.k), pick(w.v), pick(w.alpha), pick(w.sigma), w.r[sl, h:h + 1],
                                 d_o[sl, h:h + 1], dS=dS[s:s + 1, h:h + 1], dP=dP[s:s + 1, h:h + 1])
        for n in ("dq", "dk", "dv", "dalpha", "dsigma"):
            assert_rel(got[n][sl, h], ref[n][:, 0], TOL, f"chain ({s},{h}) {n}")
        assert_rel(got["dr"][sl, h], ref["dr"][:, 0], TOL, 'got["dr"][sl, h]')
        assert_rel(got["dS0"][s, h], ref["dS0"][0, 0], TOL, 'got["dS0"][s, h]')
        assert_rel(got["dP0"][s, h], ref["dP0"][0, 0], TOL, 'got["dP0"][s, h]')


@functools.lru_cache(maxsize=1)
def _many_short_case():
    lens = np.random.default_rng(31).integers(1, 25, 200)
    w = ragged(950, list(lens), 2, 128, 128, True)
    S0, P0 = initial_state(33, w)
    d_o, dS, dP = cotangents(34, w)
    ref = kdn_grad.diag_grad(w.q, w.k, w.v, w.alpha, w.sigma, w.r, d_o, cu_seqlens=w.cu_seqlens,
                             S0=S0, P0=P0, dS=dS, dP=dP, mu=1.5)
    return w, S0, P0, d_o, dS, dP, ref


@pytest.mark.parametrize("max_seqlen", [0, 24])
def test_backward_many_short_sequences_both_work_lists(kdn, max_seqlen):
    """200 packed sequences of 1-24 tokens, bf16, d = 128.  Without max_seqlen the chunk-parallel
    work lists (nseq x H x the chunks of the whole packed length) do not fit the checkpoint
    region, so the uncertainty tape and its adjoint take the serial per-chain kernels; with it
    they take the chunk-parallel scans.  Both against the gradient oracle."""
    import torch
    w, S0, P0, d_o, dS, dP, ref = _many_short_case()
    args = [to_dev(dense_shape(w, getattr(w, n))) for n in ("q", "k", "v", "alpha", "sigma", "r")]
    g = kdn.backward(*args, to_dev(dense_shape(w, d_o)), cu_seqlens=to_dev(w.cu_seqlens), S0=to_dev(S0),
                     P0=to_dev(P0), dS=to_dev(dS), dP=to_dev(dP), mu=1.5, max_seqlen=max_seqlen)
    torch.cuda.synchronize()
    kdn.last_device_error()
    got = {n: to_host(g[n]) for n in NAMES}
    for n in ("dq", "dk", "dv", "dalpha", "dsigma", "dr"):
        got[n] = got[n].reshape((w.ntok,) + got[n].shape[2:])
    check(got, ref)


def test_backward_reports_a_sequence_longer_than_max_seqlen(kdn):
    """The chunk-parallel uncertainty work lists are sized by max_seqlen (64-token chunks); a
    longer packed sequence is reported by kdn_last_device_error, and the context stays usable:
    the same call with a sufficient bound then matches the gradient oracle."""
    import torch
    w = ragged(977, [1, 63, 64, 0, 65, 130], 2, 128, 128, True)
    d_o, dS, dP = cotangents(5, w)
    args = [to_dev(dense_shape(w, getattr(w, n))) for n in ("q", "k", "v", "alpha", "sigma", "r")]
    cu = to_dev(w.cu_seqlens)
    kdn.backward(*args, to_dev(dense_shape(w, d_o)), cu_seqlens=cu, max_seqlen=64)
    with pytest.raises(kdn.KdnError):
        kdn.last_device_error()
    ref = kdn_grad.diag_grad(w.q, w.k, w.v, w.alpha, w.sigma, w.r, d_o, cu_seqlens=w.cu_seqlens, dS=dS, dP=dP)
    g = kdn.backward(*args, to_dev(dense_shape(w, d_o)), cu_seqlens=cu, dS=to_dev(dS), dP=to_dev(dP), max_seqlen=130)
    torch.cuda.synchronize()
    kdn.last_device_error()
    got = {n: to_host(g[n]) for n in NAMES}
    for n in ("dq", "dk", "dv", "dalpha", "dsigma", "dr"):
        got[n] = got[n].reshape((w.ntok,) + got[n].shape[2:])
    check(got, ref)
