"""Pins of the fp64 oracle to what the pages and the mathematics fix (CPU only).

Each test ties a part of the oracle to something other than itself: a special
case that reduces to a textbook routine, a closed form, a library linear solve,
a brute-force joint posterior, a worked example printed on a page, or an
invariant.  Together they are chosen so that a dropped term, a wrong sign, a
wrong index or a transposed operand in the oracle fails at least one of them.
"""
import os

import numpy as np
import pytest

import oracle
from kalman_delta_rule_b200 import inputs

HERE = os.path.dirname(os.path.abspath(__file__))


def unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def rand_problem(rng, ntok, H, dk, dv, unit=True):
    q = rng.standard_normal((ntok, H, dk))
    k = rng.standard_normal((ntok, H, dk))
    if unit:
        q, k = unit_rows(q), unit_rows(k)
    v = rng.standard_normal((ntok, H, dv))
    alpha = 1.0 / (1.0 + np.exp(-rng.normal(2.0, 1.0, (ntok, H, dk))))
    sigma = np.logaddexp(0, rng.normal(-3.0, 1.0, (ntok, H, dk)))
    r = np.logaddexp(0, rng.normal(0.0, 1.0, (ntok, H))) + 1e-3
    return q, k, v, alpha, sigma, r


# ------------------------------------------------------------------ delta family
def textbook_gated_delta(q, k, v, alpha_scalar, beta):
    """Gated delta rule for one head, written from the tutorial's three steps
    (read v^ = S^T k, compare e = v - v^, correct S += beta k e^T) with a retention
    gate applied to the whole memory first, and the memory read with the query after
    the write.  alpha_scalar: [T]; beta: [T]."""
    T, dk = k.shape
    S = np.zeros((dk, v.shape[1]))
    outs = []
    for t in range(T):
        S = alpha_scalar[t] * S
        v_hat = S.T @ k[t]
        e = v[t] - v_hat
        S = S + beta[t] * np.outer(k[t], e)
        outs.append(S.T @ q[t])
    return np.array(outs), S


def test_kdn_reduces_to_gated_deltanet_when_uncertainty_is_isotropic():
    """With mu = 0, a scalar decay per token and isotropic sigma and P0, the diagonal
    uncertainty stays isotropic, so the Kalman gain is beta_t k_t with the scalar
    Kalman gain beta_t = p_t / (r_t + p_t |k_t|^2), p_t = a_t^2 p_{t-1} + s_t.
    The KDN oracle must then equal the textbook gated delta rule (explainer: DeltaNet,
    Gated DeltaNet and KDA are KDN with the uncertainty tracking dropped)."""
    rng = np.random.default_rng(11)
    T, dk, dv = 40, 8, 5
    q, k, v, _, _, r = rand_problem(rng, T, 1, dk, dv, unit=False)
    a = rng.uniform(0.6, 1.0, T)
    s = rng.uniform(0.01, 0.3, T)
    alpha = np.repeat(a[:, None, None], dk, axis=2)
    sigma = np.repeat(s[:, None, None], dk, axis=2)
    p0 = 0.7
    res = oracle.diag_forward(q, k, v, alpha, sigma, r, P0=np.full((1, 1, dk), p0), mu=0.0)
    p, beta = p0, np.zeros(T)
    for t in range(T):
        p = a[t] ** 2 * p + s[t]
        beta[t] = p / (r[t, 0] + p * np.dot(k[t, 0], k[t, 0]))
    o_ref, S_ref = textbook_gated_delta(q[:, 0], k[:, 0], v[:, 0], a, beta)
    np.testing.assert_allclose(res["o"][:, 0], o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(res["S"][0, 0], S_ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("kind", ["deltanet", "gated", "kda"])
def test_delta_mode_matches_textbook_loops(kind):
    """Constant-beta mode = DeltaNet (alpha = 1), Gated DeltaNet (scalar alpha) and
    KDA (per-channel alpha, D_t = diag(alpha_t) before the delta write, dothoosh
    section on per-channel forgetting)."""
    rng = np.random.default_rng(3)
    T, H, dk, dv = 30, 2, 6, 4
    q, k, v, _, _, _ = rand_problem(rng, T, H, dk, dv)
    beta = rng.uniform(0.1, 1.0, (T, H))
    if kind == "deltanet":
        alpha = np.ones((T, H, dk))
    elif kind == "gated":
        alpha = np.repeat(rng.uniform(0.5, 1.0, (T, H, 1)), dk, axis=2)
    else:
        alpha = rng.uniform(0.5, 1.0, (T, H, dk))
    res = oracle.delta_forward(q, k, v, alpha, beta)
    for h in range(H):
        S = np.zeros((dk, dv))
        for t in range(T):
            S = alpha[t, h][:, None] * S                       # D_t S
            e = v[t, h] - S.T @ k[t, h]                         # v - v^
            S = S + beta[t, h] * np.outer(k[t, h], e)           # S += beta k e^T
            np.testing.assert_allclose(res["o"][t, h], S.T @ q[t, h], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(res["S"][0, h], S, rtol=1e-12, atol=1e-12)


def test_exact_recall_with_unit_beta_and_orthonormal_keys():
    """beta = 1, no decay, orthonormal keys: the memory returns each stored value
    exactly (dothoosh: with beta_t = 1 the memory returns exactly v_t for that key)."""
    rng = np.random.default_rng(5)
    dk, dv, n = 8, 3, 6
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm[:, :n].T
    vals = rng.standard_normal((n, dv))
    # n write tokens, then n read-only tokens (beta = 0) querying every key
    k = np.concatenate([keys, keys])[:, None, :]
    q = np.concatenate([keys, keys])[:, None, :]
    v = np.concatenate([vals, np.zeros((n, dv))])[:, None, :]
    beta = np.concatenate([np.ones(n), np.zeros(n)])[:, None]
    alpha = np.ones((2 * n, 1, dk))
    res = oracle.delta_forward(q, k, v, alpha, beta)
    np.testing.assert_allclose(res["o"][n:, 0], vals, atol=1e-12)


def test_kdn_write_is_exact_recall_in_the_noiseless_limit():
    """For r -> 0 the Kalman gain gives k^T g -> 1: the token just written is read
    back exactly with q = k (explainer: the gain weighs prediction and observation
    by their reliabilities; a noiseless observation is trusted fully)."""
    rng = np.random.default_rng(6)
    T, dk, dv = 12, 10, 4
    q, k, v, alpha, sigma, r = rand_problem(rng, T, 1, dk, dv)
    r[:] = 1e-13
    res = oracle.diag_forward(k, k, v, alpha, sigma, r, trace=True)
    np.testing.assert_allclose(res["o"][:, 0], v[:, 0], atol=1e-9)
    np.testing.assert_allclose(res["trace_beta_eff"][:, 0], 1.0, atol=1e-9)


def test_overwrite_worked_example():
    """Worked example of the tutorial (one key, "Riga" then "Prague"): additive memory
    returns both values, the delta rule with beta = 1 returns the newest; the KDN with
    a noiseless observation behaves like beta = 1 on a unit key."""
    rows = {}
    for line in open(os.path.join(HERE, "golden", "overwrite_riga_prague.txt")):
        if line.strip() and not line.startswith("#"):
            name, a, b = line.split()
            rows[name] = np.array([float(a), float(b)])
    dk = 4
    key = np.zeros(dk); key[1] = 1.0                  # the "Oleg" address
    riga, prague = np.array([1.0, 0.0]), np.array([0.0, 1.0])
    k = np.stack([key, key, key])[:, None, :]
    v = np.stack([riga, prague, np.zeros(2)])[:, None, :]
    q = k.copy()
    # additive linear attention (the negative example): S += v k^T, read S^T q
    S_sum = np.outer(key, riga) + np.outer(key, prague)
    np.testing.assert_allclose(S_sum.T @ key, rows["sum"])
    # delta rule, beta = 1 for the two writes, beta = 0 for the read token
    res = oracle.delta_forward(q, k, v, np.ones((3, 1, dk)), np.array([[1.0], [1.0], [0.0]]))
    np.testing.assert_allclose(res["o"][2, 0], rows["delta"], atol=1e-15)
    np.testing.assert_allclose(res["o"][1, 0], rows["delta"], atol=1e-15)
    # KDN, noiseless observations: the second write replaces the first
    kd = oracle.diag_forward(q[:2], k[:2], v[:2], np.ones((2, 1, dk)), np.full((2, 1, dk), 0.1),
                             np.full((2, 1), 1e-14))
    np.testing.assert_allclose(kd["o"][1, 0], rows["delta"], atol=1e-10)


# ------------------------------------------------------------------ full covariance
def test_full_kf_equals_weighted_ridge_closed_form():
    """Gated KalmaNet blog, section 2.1: the Kalman recursion solves the weighted ridge
    min lambda |S|^2 + sum eta_i |S k_i - v_i|^2, with readout U_t (H_t + lambda I)^-1 q_t,
    U_t = sum eta_i v_i k_i^T, H_t = sum eta_i k_i k_i^T.  Map: no decay, no process
    noise, Sigma0 = I / lambda, r_i = 1 / eta_i.  Checked with a library dense solve."""
    rng = np.random.default_rng(7)
    T, dk, dv, lam = 20, 6, 3, 0.8
    q = rng.standard_normal((T, 1, dk))
    k = rng.standard_normal((T, 1, dk))
    v = rng.standard_normal((T, 1, dv))
    eta = rng.uniform(0.2, 3.0, T)
    res = oracle.full_kf(q, k, v, np.ones((T, 1, dk)), np.zeros((T, 1, dk)), (1.0 / eta)[:, None],
                         Sigma0=np.eye(dk)[None, None] / lam)
    U = np.zeros((dv, dk))
    Hm = np.zeros((dk, dk))
    for t in range(T):
        U += eta[t] * np.outer(v[t, 0], k[t, 0])
        Hm += eta[t] * np.outer(k[t, 0], k[t, 0])
        y = U @ np.linalg.solve(Hm + lam * np.eye(dk), q[t, 0])
        np.testing.assert_allclose(res["o"][t, 0], y, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(res["Sigma"][0, 0], np.linalg.inv(Hm + lam * np.eye(dk)), rtol=1e-10, atol=1e-12)


def test_full_kf_equals_brute_force_joint_posterior():
    """With decay and process noise the filtered mean and covariance of the state at t
    are those of the joint Gaussian over (x_0..x_t) given the observations 1..t
    (Kalman associative memory as a linear-Gaussian state-space model: explainer,
    "把记忆问题重新想成一个滤波问题"; aifromscratch, "How It Works").  Brute force:
    assemble the joint precision, solve it with a library routine."""
    rng = np.random.default_rng(8)
    T, dk, dv = 6, 3, 2
    q, k, v, alpha, sigma, r = rand_problem(rng, T, 1, dk, dv, unit=False)
    S0 = rng.standard_normal((1, 1, dk, dv))
    A0 = rng.standard_normal((dk, dk))
    Sig0 = A0 @ A0.T + 0.5 * np.eye(dk)
    res = oracle.full_kf(q, k, v, alpha, sigma, r, S0=S0, Sigma0=Sig0[None, None])
    for t in range(1, T + 1):
        n = (t + 1) * dk
        Lam = np.zeros((n, n))
        rhs = np.zeros((n, dv))
        P0i = np.linalg.inv(Sig0)
        Lam[:dk, :dk] += P0i
        rhs[:dk] += P0i @ S0[0, 0]
        for s in range(1, t + 1):
            D = np.diag(alpha[s - 1, 0])
            Qi = np.diag(1.0 / sigma[s - 1, 0])
            a, b = slice((s - 1) * dk, s * dk), slice(s * dk, (s + 1) * dk)
            # transition term (x_s - D x_{s-1})^T Q^-1 (x_s - D x_{s-1})
            Lam[b, b] += Qi
            Lam[a, a] += D.T @ Qi @ D
            Lam[b, a] -= Qi @ D
            Lam[a, b] -= D.T @ Qi
            # observation term (v_s - x_s^T k_s)^2 / r_s per value column
            kk = k[s - 1, 0]
            Lam[b, b] += np.outer(kk, kk) / r[s - 1, 0]
            rhs[b] += np.outer(kk, v[s - 1, 0]) / r[s - 1, 0]
        mean = np.linalg.solve(Lam, rhs)
        cov = np.linalg.inv(Lam)
        xt = mean[t * dk:(t + 1) * dk]
        np.testing.assert_allclose(res["o"][t - 1, 0], xt.T @ q[t - 1, 0], rtol=1e-9, atol=1e-10)
        if t == T:
            np.testing.assert_allclose(res["S"][0, 0], xt, rtol=1e-9, atol=1e-10)
            np.testing.assert_allclose(res["Sigma"][0, 0], cov[t * dk:, t * dk:], rtol=1e-9, atol=1e-11)


# ------------------------------------------------------------------ diagonal vs full
def test_diagonal_equals_full_kf_for_axis_aligned_keys():
    """One-hot keys never correlate channels, so the exact posterior stays diagonal and
    the diagonal KDN (mu = 1) must equal the full Kalman filter at every token
    (explainer, "对角近似": the posterior becomes dense only through the new
    observation's key)."""
    rng = np.random.default_rng(9)
    T, H, dk, dv = 50, 2, 5, 3
    q, _, v, alpha, sigma, r = rand_problem(rng, T, H, dk, dv)
    k = np.zeros((T, H, dk))
    idx = rng.integers(0, dk, (T, H))
    scale = rng.uniform(0.3, 2.0, (T, H))
    for t in range(T):
        for h in range(H):
            k[t, h, idx[t, h]] = scale[t, h]
    P0 = rng.uniform(0.2, 2.0, (1, H, dk))
    S0 = rng.standard_normal((1, H, dk, dv))
    d = oracle.diag_forward(q, k, v, alpha, sigma, r, S0=S0, P0=P0, mu=1.0)
    f = oracle.full_kf(q, k, v, alpha, sigma, r, S0=S0, Sigma0=np.stack([np.diag(p) for p in P0[0]])[None])
    np.testing.assert_allclose(d["o"], f["o"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(d["S"], f["S"], rtol=1e-12, atol=1e-12)
    for h in range(H):
        Sig = f["Sigma"][0, h]
        np.testing.assert_allclose(Sig - np.diag(np.diag(Sig)), 0.0, atol=1e-15)
        np.testing.assert_allclose(np.diag(Sig), d["P"][0, h], rtol=1e-12)


def test_one_step_mean_is_exact_and_uncertainty_is_the_precision_diagonal():
    """From a diagonal prior, one update gives the exact posterior mean (explainer: the
    projection loses nothing of the mean) and the mean-field (KL(q||p)) projection keeps
    the diagonal of the posterior precision.  Checked against the full filter and a
    library inverse of its posterior covariance, for arbitrary keys."""
    rng = np.random.default_rng(10)
    H, dk, dv = 3, 7, 4
    q, k, v, alpha, sigma, r = rand_problem(rng, 1, H, dk, dv, unit=False)
    P0 = rng.uniform(0.2, 2.0, (1, H, dk))
    S0 = rng.standard_normal((1, H, dk, dv))
    d = oracle.diag_forward(q, k, v, alpha, sigma, r, S0=S0, P0=P0, mu=1.0)
    f = oracle.full_kf(q, k, v, alpha, sigma, r, S0=S0, Sigma0=np.stack([np.diag(p) for p in P0[0]])[None])
    np.testing.assert_allclose(d["S"], f["S"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(d["o"], f["o"], rtol=1e-12, atol=1e-12)
    for h in range(H):
        prec = np.linalg.inv(f["Sigma"][0, h])
        np.testing.assert_allclose(1.0 / d["P"][0, h], np.diag(prec), rtol=1e-10)
        # and not the diagonal of the covariance (moment matching), which differs
        assert np.max(np.abs(d["P"][0, h] - np.diag(f["Sigma"][0, h]))) > 1e-6


def test_two_step_diagonal_differs_from_full():
    """After two general updates the projected diagonal filter is an approximation:
    it must differ from the full filter (guards against a 'diagonal' oracle that
    secretly carries the dense covariance)."""
    rng = np.random.default_rng(12)
    q, k, v, alpha, sigma, r = rand_problem(rng, 2, 1, 5, 3)
    d = oracle.diag_forward(q, k, v, alpha, sigma, r)
    f = oracle.full_kf(q, k, v, alpha, sigma, r)
    np.testing.assert_allclose(d["o"][0], f["o"][0], rtol=1e-12)
    assert np.max(np.abs(d["o"][1] - f["o"][1])) > 1e-8


# ------------------------------------------------------------------ information scaling
def test_mu_does_not_change_the_current_write():
    """Explainer, "对角近似", last paragraph: the calibration mu scales the precision
    increment after the update; the current write is unchanged, later writes along the
    same direction get weaker."""
    rng = np.random.default_rng(13)
    T, H, dk, dv = 6, 2, 16, 8
    q, k, v, alpha, sigma, r = rand_problem(rng, T, H, dk, dv)
    k[3] = k[0]  # a reused key
    runs = {mu: oracle.diag_forward(q, k, v, alpha, sigma, r, mu=mu, trace=True) for mu in (1.0, 4.0, float(dk))}
    base = runs[1.0]
    for mu, res in runs.items():
        np.testing.assert_allclose(res["o"][0], base["o"][0], rtol=1e-14)
        np.testing.assert_allclose(res["trace_g"][0], base["trace_g"][0], rtol=1e-14)
    # larger mu: smaller posterior uncertainty, weaker later write along the reused key
    assert np.all(runs[float(dk)]["trace_P"][0] <= runs[1.0]["trace_P"][0] + 1e-15)
    assert np.all(runs[float(dk)]["trace_beta_eff"][3] < runs[1.0]["trace_beta_eff"][3])
    assert np.max(np.abs(runs[float(dk)]["o"][3] - base["o"][3])) > 1e-6


@pytest.mark.parametrize("mu", [1.0, 3.0, 32.0])
def test_repeated_axis_key_precision_closed_form(mu):
    """No decay, no process noise, constant r, the same one-hot key n times: the
    precision of that channel grows by mu / r per token, 1/P_n = 1/P_0 + n mu / r, and
    the other channels keep P_0 (repeated confirmation builds resistance: explainer,
    "对角近似")."""
    dk, dv, n, ch, r0 = 6, 2, 25, 4, 0.37
    rng = np.random.default_rng(14)
    k = np.zeros((n, 1, dk)); k[:, 0, ch] = 1.0
    v = rng.standard_normal((n, 1, dv))
    P0 = rng.uniform(0.5, 2.0, (1, 1, dk))
    res = oracle.diag_forward(k, k, v, np.ones((n, 1, dk)), np.zeros((n, 1, dk)), np.full((n, 1), r0),
                              P0=P0, mu=mu, trace=True)
    t = np.arange(1, n + 1)
    np.testing.assert_allclose(1.0 / res["trace_P"][:, 0, ch], 1.0 / P0[0, 0, ch] + t * mu / r0, rtol=1e-12)
    others = [i for i in range(dk) if i != ch]
    np.testing.assert_allclose(res["trace_P"][:, 0, others], np.broadcast_to(P0[0, 0, others], (n, dk - 1)))
    if mu == 1.0:
        # the mean is the shrunk running mean of the observed values: sum v / (n + r / P0)
        run = np.cumsum(v[:, 0], axis=0) / (t + r0 / P0[0, 0, ch])[:, None]
        np.testing.assert_allclose(res["o"][:, 0], run, rtol=1e-12, atol=1e-14)


def test_uncertainty_fixed_point_closed_form():
    """Constant decay a = alpha^2, process noise s and c = mu k^2 / r: the predicted
    uncertainty converges to the positive root of c x^2 + (1 - a - c s) x - s = 0."""
    dk, T = 3, 400
    alpha = np.array([0.9, 0.99, 0.5])
    s = np.array([0.05, 0.01, 0.2])
    kv = np.array([0.6, 0.3, 0.74])
    r0, mu = 0.8, 2.0
    k = np.broadcast_to(kv, (T, 1, dk)).copy()
    res = oracle.diag_forward(k, k, np.zeros((T, 1, 1)), np.broadcast_to(alpha, (T, 1, dk)),
                              np.broadcast_to(s, (T, 1, dk)), np.full((T, 1), r0), mu=mu, trace=True)
    a, c = alpha ** 2, mu * kv ** 2 / r0
    b = 1 - a - c * s
    x = (-b + np.sqrt(b * b + 4 * c * s)) / (2 * c)
    np.testing.assert_allclose(res["trace_Pm"][-1, 0], x, rtol=1e-10)


# ------------------------------------------------------------------ invariants
def test_uncertainty_invariants_on_workload_like_inputs():
    """P stays positive and never grows in the update step; 0 <= k^T g < 1."""
    w = inputs.tiny_fp32()
    res = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens, trace=True)
    assert np.all(res["trace_P"] > 0)
    assert np.all(res["trace_P"] <= res["trace_Pm"])
    assert np.all(res["trace_beta_eff"] >= 0) and np.all(res["trace_beta_eff"] < 1)
    # and the gain is P^- k / (r + sum P^- k^2) read back from the traces
    k = w.k.astype(np.float64)
    den = w.r[..., None] + np.sum(res["trace_Pm"] * k * k, axis=-1, keepdims=True)
    np.testing.assert_allclose(res["trace_g"], res["trace_Pm"] * k / den, rtol=1e-13)


def test_mobius_tree_scan_equals_serial_recursion():
    """The per-channel uncertainty recursion is a Moebius map; composing the tokens'
    2x2 matrices in any bracketing (here a log-depth prefix doubling) and applying the
    product projectively reproduces the serial recursion (explainer, closing paragraph
    of "各向同性近似"; aifromscratch, "Approximation 1")."""
    rng = np.random.default_rng(15)
    T, dk, mu = 300, 4, 3.0
    q, k, v, alpha, sigma, r = rand_problem(rng, T, 1, dk, 2)
    P0 = rng.uniform(0.5, 2.0, (1, 1, dk))
    res = oracle.diag_forward(q, k, v, alpha, sigma, r, P0=P0, mu=mu, trace=True)
    M = oracle.mobius_matrix(alpha[:, 0], sigma[:, 0], k[:, 0], r[:, 0, None], mu=mu)  # [T, dk, 2, 2]
    pref = M.copy()
    step = 1
    while step < T:  # Hillis-Steele inclusive scan: pref[t] = M[t] @ ... @ M[0]
        new = pref.copy()
        new[step:] = pref[step:] @ pref[:-step]
        # renormalise: a Moebius matrix acts projectively
        new /= np.abs(new).max(axis=(-2, -1), keepdims=True)
        pref = new
        step *= 2
    p0 = P0[0, 0]
    P = (pref[..., 0, 0] * p0 + pref[..., 0, 1]) / (pref[..., 1, 0] * p0 + pref[..., 1, 1])
    np.testing.assert_allclose(P, res["trace_P"][:, 0], rtol=1e-11)


def test_split_sequence_with_carried_state_equals_one_call():
    """Checkpoint/resume: carrying (S, P) across a split reproduces one call."""
    w = inputs.tiny_fp32()
    full = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, mu=2.0)
    for cut in (1, 63, 64, 65, 200):
        a = oracle.diag_forward(w.q[:cut], w.k[:cut], w.v[:cut], w.alpha[:cut], w.sigma[:cut], w.r[:cut], mu=2.0)
        b = oracle.diag_forward(w.q[cut:], w.k[cut:], w.v[cut:], w.alpha[cut:], w.sigma[cut:], w.r[cut:],
                                S0=a["S"], P0=a["P"], mu=2.0)
        np.testing.assert_allclose(np.concatenate([a["o"], b["o"]]), full["o"], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(b["S"], full["S"], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(b["P"], full["P"], rtol=1e-12)


def test_varlen_packing_and_head_independence():
    """Packed sequences (cu_seqlens) equal separate calls; every head is independent."""
    rng = np.random.default_rng(16)
    lens = [5, 1, 17, 9]
    ntok, H, dk, dv = sum(lens), 3, 6, 5
    q, k, v, alpha, sigma, r = rand_problem(rng, ntok, H, dk, dv)
    cu = np.concatenate([[0], np.cumsum(lens)])
    S0 = rng.standard_normal((len(lens), H, dk, dv))
    P0 = rng.uniform(0.5, 2, (len(lens), H, dk))
    packed = oracle.diag_forward(q, k, v, alpha, sigma, r, cu_seqlens=cu, S0=S0, P0=P0)
    for s in range(len(lens)):
        sl = slice(cu[s], cu[s + 1])
        for h in range(H):
            one = oracle.diag_forward(q[sl, h:h + 1], k[sl, h:h + 1], v[sl, h:h + 1], alpha[sl, h:h + 1],
                                      sigma[sl, h:h + 1], r[sl, h:h + 1], S0=S0[s:s + 1, h:h + 1],
                                      P0=P0[s:s + 1, h:h + 1], threads=1)
            np.testing.assert_allclose(packed["o"][sl, h], one["o"][:, 0], rtol=1e-13, atol=1e-14)
            np.testing.assert_allclose(packed["S"][s, h], one["S"][0, 0], rtol=1e-13, atol=1e-14)
            np.testing.assert_allclose(packed["P"][s, h], one["P"][0, 0], rtol=1e-13)


def test_decode_runner_equals_one_sequence():
    """A run of decode steps is the recurrence over a sequence with the state carried."""
    rng = np.random.default_rng(17)
    N, H, dk, dv, n = 3, 2, 5, 4, 7
    steps = []
    for _ in range(n):
        q, k, v, alpha, sigma, r = rand_problem(rng, N, H, dk, dv)
        steps.append(dict(q=q, k=k, v=v, alpha=alpha, sigma=sigma, r=r))
    S0 = rng.standard_normal((N, H, dk, dv))
    P0 = rng.uniform(0.5, 2, (N, H, dk))
    dec = oracle.run_decode(S0, P0, steps, mu=1.5)
    for s in range(N):
        S, P = S0[s:s + 1], P0[s:s + 1]
        for t in range(n):
            st = {nm: a[s:s + 1] for nm, a in steps[t].items()}
            one = oracle.diag_forward(st["q"], st["k"], st["v"], st["alpha"], st["sigma"], st["r"], S0=S, P0=P, mu=1.5)
            np.testing.assert_allclose(dec["o"][t, s], one["o"][0], rtol=1e-13, atol=1e-14)
            S, P = one["S"], one["P"]
        np.testing.assert_allclose(dec["S"][s], S[0], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(dec["P"][s], P[0], rtol=1e-13)


# ------------------------------------------------------------------ isotropic KDN
def uniform_channels(rng, T, H, dk):
    """Decay and process noise equal across the key channels of a token (the predict
    then keeps an isotropic covariance isotropic)."""
    a = 1.0 / (1.0 + np.exp(-rng.normal(2.0, 1.0, (T, H, 1))))
    s = np.logaddexp(0, rng.normal(-3.0, 1.0, (T, H, 1)))
    return np.broadcast_to(a, (T, H, dk)).copy(), np.broadcast_to(s, (T, H, dk)).copy()


def test_iso_one_step_gain_is_exact_and_update_is_the_kl_projection():
    """Explainer "各向同性近似" / aifromscratch "Approximation 2": one uncertainty per head.
    From an isotropic prior the Kalman gain is exact, so one step gives the full
    filter's mean and readout; the scalar posterior is the reverse-KL (mean-field)
    projection of the full posterior onto multiples of the identity, found here by a
    library minimiser of KL(N(0, p I) || N(0, Sigma)) over p."""
    from scipy.optimize import minimize_scalar
    rng = np.random.default_rng(30)
    H, dk, dv = 3, 6, 4
    q, k, v, _, _, r = rand_problem(rng, 1, H, dk, dv, unit=False)
    alpha, sigma = uniform_channels(rng, 1, H, dk)
    p0 = rng.uniform(0.3, 2.0, (1, H))
    S0 = rng.standard_normal((1, H, dk, dv))
    iso = oracle.iso_forward(q, k, v, alpha, sigma, r, S0=S0, P0=p0, mu=1.0)
    f = oracle.full_kf(q, k, v, alpha, sigma, r, S0=S0, Sigma0=(p0[0, :, None, None] * np.eye(dk))[None])
    np.testing.assert_allclose(iso["S"], f["S"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(iso["o"], f["o"], rtol=1e-12, atol=1e-12)
    for h in range(H):
        Sig = f["Sigma"][0, h]
        prec_tr = np.trace(np.linalg.inv(Sig))
        logdet = np.linalg.slogdet(Sig)[1]

        def kl(lp):
            p = np.exp(lp)
            return 0.5 * (p * prec_tr - dk + logdet - dk * lp)
        best = minimize_scalar(kl, bounds=(-12.0, 6.0), method="bounded", options={"xatol": 1e-12})
        np.testing.assert_allclose(iso["P"][0, h], np.exp(best.x), rtol=1e-7)


def test_iso_predict_keeps_the_trace_of_the_diagonal_predict():
    """Reading of the isotropic predict: with no information in the token (k = 0) the
    step is the predict alone, and p equals the mean over channels of the diagonal
    filter's predicted variances alpha_i^2 p + sigma_i (non-uniform alpha, sigma)."""
    rng = np.random.default_rng(31)
    H, dk, dv = 2, 8, 3
    q, k, v, alpha, sigma, r = rand_problem(rng, 1, H, dk, dv)
    k[:] = 0.0
    p0 = rng.uniform(0.3, 2.0, (1, H))
    iso = oracle.iso_forward(q, k, v, alpha, sigma, r, P0=p0, mu=1.0)
    dg = oracle.diag_forward(q, k, v, alpha, sigma, r, P0=np.repeat(p0[..., None], dk, axis=-1), mu=1.0)
    np.testing.assert_allclose(iso["P"], dg["P"].mean(axis=-1), rtol=1e-14)


def test_iso_equals_diagonal_without_information_scaling_on_uniform_channels():
    """mu = 0 and decay / noise uniform across channels: a diagonal uncertainty that
    starts isotropic stays isotropic, so the two approximations coincide for every
    token (and both are gated DeltaNet with the scalar Kalman write strength)."""
    rng = np.random.default_rng(32)
    T, H, dk, dv = 40, 2, 8, 5
    q, k, v, _, _, r = rand_problem(rng, T, H, dk, dv)
    alpha, sigma = uniform_channels(rng, T, H, dk)
    p0 = rng.uniform(0.3, 2.0, (1, H))
    iso = oracle.iso_forward(q, k, v, alpha, sigma, r, P0=p0, mu=0.0, trace=True)
    dg = oracle.diag_forward(q, k, v, alpha, sigma, r, P0=np.repeat(p0[..., None], dk, axis=-1), mu=0.0,
                             trace=True)
    np.testing.assert_allclose(iso["o"], dg["o"], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(iso["S"], dg["S"], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(iso["trace_g"], dg["trace_g"], rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(iso["trace_Pm"], dg["trace_Pm"][..., 0], rtol=1e-12)


@pytest.mark.parametrize("mu", [1.0, 8.0])
def test_iso_repeated_confirmation_closed_form(mu):
    """No decay, no process noise, constant r, unit keys in any directions: the head's
    precision grows by mu / (d_k r) per token, 1/p_n = 1/p_0 + n mu / (d_k r)."""
    rng = np.random.default_rng(33)
    n, dk, dv, r0 = 30, 8, 2, 0.45
    k = unit_rows(rng.standard_normal((n, 1, dk)))
    p0 = np.array([[1.7]])
    res = oracle.iso_forward(k, k, rng.standard_normal((n, 1, dv)), np.ones((n, 1, dk)), np.zeros((n, 1, dk)),
                             np.full((n, 1), r0), P0=p0, mu=mu, trace=True)
    t = np.arange(1, n + 1)
    np.testing.assert_allclose(1.0 / res["trace_P"][:, 0], 1.0 / 1.7 + t * mu / (dk * r0), rtol=1e-12)


def test_iso_fixed_point_closed_form():
    """Constant tokens with channel-varying decay and noise: the predicted uncertainty
    converges to the positive root of c x^2 + (1 - a - c s) x - s = 0 with
    a = mean(alpha^2), s = mean(sigma), c = mu |k|^2 / (d_k r)."""
    dk, T = 4, 600
    alpha = np.array([0.9, 0.99, 0.5, 0.8])
    sg = np.array([0.05, 0.01, 0.2, 0.0])
    kv = np.array([0.6, 0.3, 0.74, -0.2])
    r0, mu = 0.8, 2.0
    k = np.broadcast_to(kv, (T, 1, dk)).copy()
    res = oracle.iso_forward(k, k, np.zeros((T, 1, 1)), np.broadcast_to(alpha, (T, 1, dk)),
                             np.broadcast_to(sg, (T, 1, dk)), np.full((T, 1), r0), mu=mu, trace=True)
    a, s, c = np.mean(alpha ** 2), np.mean(sg), mu * np.sum(kv ** 2) / (dk * r0)
    b = 1 - a - c * s
    x = (-b + np.sqrt(b * b + 4 * c * s)) / (2 * c)
    np.testing.assert_allclose(res["trace_Pm"][-1, 0], x, rtol=1e-10)


def test_iso_is_kda_with_a_derived_write_strength():
    """Explainer "各向同性近似": the isotropic KDN keeps the delta-rule form of KDA and only
    derives the scalar write strength from the uncertainty.  The gain is parallel to
    the key, and the KDA recurrence (delta family, per-channel decay) driven by
    beta_t = k^T g / |k|^2 reproduces the outputs and the memory."""
    w = inputs.tiny_fp32()
    iso = oracle.iso_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens, mu=4.0, trace=True)
    k = w.k.astype(np.float64)
    kk = np.sum(k * k, axis=-1)
    beta = iso["trace_beta_eff"] / kk
    np.testing.assert_allclose(iso["trace_g"], beta[..., None] * k, rtol=1e-12, atol=1e-15)
    kda = oracle.delta_forward(w.q, w.k, w.v, w.alpha, beta, cu_seqlens=w.cu_seqlens)
    np.testing.assert_allclose(iso["o"], kda["o"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(iso["S"], kda["S"], rtol=1e-12, atol=1e-13)
    assert np.all(iso["trace_beta_eff"] >= 0) and np.all(iso["trace_beta_eff"] < 1)
    assert np.all(iso["trace_P"] > 0) and np.all(iso["trace_P"] <= iso["trace_Pm"])


def test_iso_mobius_tree_scan_and_split_with_carried_state():
    """The scalar recursion is a Moebius map per token, [[a, s], [c a, c s + 1]]; a
    log-depth prefix product reproduces the serial run, and carrying (S, p) across a
    split reproduces one call."""
    rng = np.random.default_rng(35)
    T, dk, mu = 257, 16, 5.0
    q, k, v, alpha, sigma, r = rand_problem(rng, T, 1, dk, 3)
    res = oracle.iso_forward(q, k, v, alpha, sigma, r, P0=np.array([[0.6]]), mu=mu, trace=True)
    a = np.mean(alpha[:, 0] ** 2, axis=-1)
    s = np.mean(sigma[:, 0], axis=-1)
    c = mu * np.sum(k[:, 0] ** 2, axis=-1) / (dk * r[:, 0])
    M = np.stack([np.stack([a, s], -1), np.stack([c * a, c * s + 1], -1)], -2)   # [T, 2, 2]
    pref, step = M.copy(), 1
    while step < T:
        new = pref.copy()
        new[step:] = pref[step:] @ pref[:-step]
        pref = new / np.abs(new).max(axis=(-2, -1), keepdims=True)
        step *= 2
    P = (pref[:, 0, 0] * 0.6 + pref[:, 0, 1]) / (pref[:, 1, 0] * 0.6 + pref[:, 1, 1])
    np.testing.assert_allclose(P, res["trace_P"][:, 0], rtol=1e-11)
    cut = 100
    x = oracle.iso_forward(q[:cut], k[:cut], v[:cut], alpha[:cut], sigma[:cut], r[:cut], P0=np.array([[0.6]]), mu=mu)
    y = oracle.iso_forward(q[cut:], k[cut:], v[cut:], alpha[cut:], sigma[cut:], r[cut:], S0=x["S"], P0=x["P"], mu=mu)
    np.testing.assert_allclose(np.concatenate([x["o"], y["o"]]), res["o"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(y["P"], res["P"], rtol=1e-12)
