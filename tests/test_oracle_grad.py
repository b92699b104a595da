"""Pins of the fp64 gradient oracle (oracle/kdn_grad.py) to things other than itself (CPU only).

* its forward restatement equals the C oracle for both variants (an independent implementation, pinned on
  its own in test_oracle_pins.py);
* every gradient equals central finite differences of the C oracle's forward (both variants);
* single-token closed forms, derived by hand from the five steps of the recurrence;
* a readout gradient at the first token does not depend on mu (mu scales only the
  uncertainty update, which acts from the next token on).
A dropped term, a sign error or a swapped gradient slot fails one of these.
"""
import numpy as np
import pytest

import oracle
from oracle import kdn_grad


def rand_problem(rng, ntok, H, dk, dv):
    q = rng.standard_normal((ntok, H, dk))
    k = rng.standard_normal((ntok, H, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((ntok, H, dv))
    alpha = 1.0 / (1.0 + np.exp(-rng.normal(1.5, 1.0, (ntok, H, dk))))
    sigma = np.logaddexp(0, rng.normal(-2.0, 1.0, (ntok, H, dk)))
    r = np.logaddexp(0, rng.normal(0.0, 1.0, (ntok, H))) + 1e-2
    return q, k, v, alpha, sigma, r


def c_loss(x, d_o, dS, dP, cu, mu, iso=False):
    q, k, v, alpha, sigma, r, S0, P0 = x
    fwd = oracle.iso_forward if iso else oracle.diag_forward
    f = fwd(q, k, v, alpha, sigma, r, cu_seqlens=cu, S0=S0, P0=P0, mu=mu, threads=1)
    return float((f["o"] * d_o).sum() + (f["S"] * dS).sum() + (f["P"] * dP).sum())


@pytest.mark.parametrize("iso", [False, True])
def test_restated_forward_equals_c_oracle(iso):
    rng = np.random.default_rng(3)
    cu = np.array([0, 5, 12], dtype=np.int32)
    q, k, v, alpha, sigma, r = rand_problem(rng, 12, 2, 4, 3)
    S0 = 0.3 * rng.standard_normal((2, 2, 4, 3))
    P0 = np.logaddexp(0, rng.standard_normal((2, 2) if iso else (2, 2, 4)))
    fwd = oracle.iso_forward if iso else oracle.diag_forward
    ref = fwd(q, k, v, alpha, sigma, r, cu_seqlens=cu, S0=S0, P0=P0, mu=1.7)
    g = kdn_grad.diag_grad(q, k, v, alpha, sigma, r, np.zeros((12, 2, 3)), cu_seqlens=cu, S0=S0, P0=P0, mu=1.7,
                           iso=iso)
    for n in ("o", "S", "P"):
        np.testing.assert_allclose(g[n], ref[n], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("mu,iso", [(1.0, False), (4.0, False), (1.0, True), (4.0, True)])
def test_gradients_equal_finite_differences_of_the_c_oracle(mu, iso):
    rng = np.random.default_rng(5)
    cu = np.array([0, 3, 7], dtype=np.int32)
    ntok, H, dk, dv = 7, 1, 3, 2
    q, k, v, alpha, sigma, r = rand_problem(rng, ntok, H, dk, dv)
    pshape = (2, H) if iso else (2, H, dk)
    S0 = 0.5 * rng.standard_normal((2, H, dk, dv))
    P0 = np.logaddexp(0, rng.standard_normal(pshape))
    d_o = rng.standard_normal((ntok, H, dv))
    dS = rng.standard_normal((2, H, dk, dv))
    dP = rng.standard_normal(pshape)
    g = kdn_grad.diag_grad(q, k, v, alpha, sigma, r, d_o, cu_seqlens=cu, S0=S0, P0=P0, dS=dS, dP=dP, mu=mu, iso=iso)
    x = [q, k, v, alpha, sigma, r, S0, P0]
    names = ("dq", "dk", "dv", "dalpha", "dsigma", "dr", "dS0", "dP0")
    for i, name in enumerate(names):
        fd = np.zeros(x[i].shape)
        for idx in np.ndindex(x[i].shape):
            h = 1e-6 * max(1.0, abs(x[i][idx]))
            xp = [a.copy() for a in x]
            xm = [a.copy() for a in x]
            xp[i][idx] += h
            xm[i][idx] -= h
            fd[idx] = (c_loss(xp, d_o, dS, dP, cu, mu, iso) - c_loss(xm, d_o, dS, dP, cu, mu, iso)) / (2 * h)
        np.testing.assert_allclose(g[name], fd, rtol=2e-6, atol=2e-7, err_msg=name)


def test_single_token_closed_forms():
    """One token, S0 = 0: S_1 = g v^T, o = v (g.q).  With L = <o, d_o> + <P_1, dP>:
    dL/dv = (g.q) d_o, dL/dq = (v.d_o) g, dL/dr (readout part) = -(v.d_o)(g.q)/den,
    dL/dS0_ij = alpha_i d_o_j (q_i - (g.q) k_i); and with z = 1/(1 + c P^-), c = mu k^2/r,
    dP-part: dL/dsigma_i += dP_i z_i^2, dL/dP0_i = alpha_i^2 dP_i z_i^2 + (readout part),
    dL/dk_i += -dP_i (P^-_i z_i)^2 2 mu k_i / r."""
    rng = np.random.default_rng(9)
    dk, dv, mu = 5, 4, 2.5
    q, k, v, alpha, sigma, r = rand_problem(rng, 1, 1, dk, dv)
    P0 = np.logaddexp(0, rng.standard_normal((1, 1, dk)))
    d_o = rng.standard_normal((1, 1, dv))
    dP = rng.standard_normal((1, 1, dk))
    g = kdn_grad.diag_grad(q, k, v, alpha, sigma, r, d_o, P0=P0, dP=dP, mu=mu)
    a, s, kk, qq, vv, rr, p0, do = alpha[0, 0], sigma[0, 0], k[0, 0], q[0, 0], v[0, 0], r[0, 0], P0[0, 0], d_o[0, 0]
    pm = a * a * p0 + s
    den = rr + np.sum(pm * kk * kk)
    gain = pm * kk / den
    gq, vdo = gain @ qq, vv @ do
    c = mu * kk * kk / rr
    z = 1.0 / (1.0 + c * pm)
    # readout part of dL/dP^-_i: (v.d_o) d(g.q)/dP^-_i = (v.d_o) (q_i k_i - (g.q) k_i^2) / den
    dpm_read = vdo * (qq * kk - gq * kk * kk) / den
    dpm = dpm_read + dP[0, 0] * z * z
    np.testing.assert_allclose(g["dv"][0, 0], gq * do, rtol=1e-12)
    np.testing.assert_allclose(g["dq"][0, 0], vdo * gain, rtol=1e-12)
    np.testing.assert_allclose(g["dS0"][0, 0], a[:, None] * np.outer(qq - gq * kk, do), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(g["dsigma"][0, 0], dpm, rtol=1e-11)
    np.testing.assert_allclose(g["dP0"][0, 0], a * a * dpm, rtol=1e-11)
    np.testing.assert_allclose(g["dalpha"][0, 0], 2 * a * p0 * dpm, rtol=1e-11)
    dr = -vdo * gq / den + np.sum(dP[0, 0] * (pm * z) ** 2 * mu * kk * kk / rr ** 2)
    np.testing.assert_allclose(g["dr"][0, 0], dr, rtol=1e-11)
    # dk: readout through g (P^- fixed): (v.d_o) [q_i P^-_i/den - 2 (g.q) P^-_i k_i/den]; update through c
    dk = vdo * (qq * pm / den - 2 * gq * pm * kk / den) - dP[0, 0] * (pm * z) ** 2 * 2 * mu * kk / rr
    np.testing.assert_allclose(g["dk"][0, 0], dk, rtol=1e-11, atol=1e-14)


def test_first_token_readout_gradients_do_not_depend_on_mu():
    rng = np.random.default_rng(2)
    q, k, v, alpha, sigma, r = rand_problem(rng, 1, 2, 4, 3)
    d_o = rng.standard_normal((1, 2, 3))
    g1 = kdn_grad.diag_grad(q, k, v, alpha, sigma, r, d_o, mu=1.0)
    g2 = kdn_grad.diag_grad(q, k, v, alpha, sigma, r, d_o, mu=7.0)
    for n in ("dq", "dk", "dv", "dalpha", "dsigma", "dr", "dS0", "dP0"):
        np.testing.assert_allclose(g1[n], g2[n], rtol=1e-13, atol=1e-15)
