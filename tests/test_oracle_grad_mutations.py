"""Mutation check of the gradient oracle's pins (CPU only).

Each case plants one plausible mistake in a copy of the restated forward of oracle/kdn_grad.py
(the function its gradients are taken from) and checks that the pins of test_oracle_grad.py --
agreement with the C oracle's forward, and finite differences of the C oracle -- reject it.
The mistakes live only in the copy; the oracle itself is never modified."""
import inspect
import textwrap

import numpy as np
import pytest

import oracle
from oracle import kdn_grad

MUTATIONS = {
    "alpha_not_squared_in_predict": ("Pm = a * a * P + sigma[t]", "Pm = a * P + sigma[t]"),
    "noise_dropped": ("Pm = a * a * P + sigma[t]", "Pm = a * a * P"),
    "gain_without_observation_noise": ("den = r[t] + (Pm * kk * kk).sum(-1)", "den = (Pm * kk * kk).sum(-1)"),
    "gain_from_P_not_Pm": ("g = Pm * kk / den[:, None]", "g = P * kk / den[:, None]"),
    "residual_sign": ('u = v[t] - torch.einsum("hij,hi->hj", W, kk)', 'u = v[t] + torch.einsum("hij,hi->hj", W, kk)'),
    "no_decay_on_memory": ("W = a[:, :, None] * S", "W = S"),
    "readout_before_write": ('outs.append(torch.einsum("hij,hi->hj", S, q[t]))',
                             'outs.append(torch.einsum("hij,hi->hj", W, q[t]))'),
    "mu_ignored": ("P = Pm / (1.0 + mu * Pm * kk * kk / r[t][:, None])", "P = Pm / (1.0 + Pm * kk * kk / r[t][:, None])"),
    "update_from_P": ("P = Pm / (1.0 + mu * Pm * kk * kk / r[t][:, None])", "P = P / (1.0 + mu * Pm * kk * kk / r[t][:, None])"),
    "iso_mean_of_alpha": ("Pm = (a * a).mean(-1) * P + sigma[t].mean(-1)", "Pm = a.mean(-1) * P + sigma[t].mean(-1)"),
    "iso_update_not_averaged": ("P = Pm / (1.0 + mu * Pm * K2 / (dk * r[t]))", "P = Pm / (1.0 + mu * Pm * K2 / r[t])"),
}


def mutated_forward(find, repl):
    src = textwrap.dedent(inspect.getsource(kdn_grad.forward_t))
    assert src.count(find) == 1, find
    ns = dict(kdn_grad.__dict__)
    exec(src.replace(find, repl), ns)
    return ns["forward_t"]


def problem(seed, iso):
    rng = np.random.default_rng(seed)
    ntok, H, dk, dv = 9, 1, 3, 2
    q = rng.standard_normal((ntok, H, dk)); k = rng.standard_normal((ntok, H, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((ntok, H, dv))
    alpha = 1.0 / (1.0 + np.exp(-rng.normal(1.0, 1.0, (ntok, H, dk))))
    sigma = np.logaddexp(0, rng.normal(-1.5, 1.0, (ntok, H, dk)))
    r = np.logaddexp(0, rng.normal(0.0, 1.0, (ntok, H))) + 1e-2
    cu = np.array([0, 4, 9], dtype=np.int32)
    S0 = 0.5 * rng.standard_normal((2, H, dk, dv))
    P0 = np.logaddexp(0, rng.standard_normal((2, H) if iso else (2, H, dk)))
    d_o = rng.standard_normal((ntok, H, dv))
    dS = rng.standard_normal((2, H, dk, dv))
    dP = rng.standard_normal((2, H) if iso else (2, H, dk))
    return q, k, v, alpha, sigma, r, cu, S0, P0, d_o, dS, dP


def pins_hold(iso, mu=2.5):
    """The pins of test_oracle_grad.py on one problem: forward equals the C oracle, and the
    gradients of q, k, alpha, sigma, r equal central finite differences of the C oracle."""
    q, k, v, alpha, sigma, r, cu, S0, P0, d_o, dS, dP = problem(4, iso)
    fwd = oracle.iso_forward if iso else oracle.diag_forward
    g = kdn_grad.diag_grad(q, k, v, alpha, sigma, r, d_o, cu_seqlens=cu, S0=S0, P0=P0, dS=dS, dP=dP, mu=mu, iso=iso)
    ref = fwd(q, k, v, alpha, sigma, r, cu_seqlens=cu, S0=S0, P0=P0, mu=mu, threads=1)
    for n in ("o", "S", "P"):
        if not np.allclose(g[n], ref[n], rtol=1e-10, atol=1e-12):
            return False

    def loss(x):
        f = fwd(*x, cu_seqlens=cu, S0=S0, P0=P0, mu=mu, threads=1)
        return float((f["o"] * d_o).sum() + (f["S"] * dS).sum() + (f["P"] * dP).sum())

    x = [q, k, v, alpha, sigma, r]
    for i, name in ((0, "dq"), (1, "dk"), (3, "dalpha"), (4, "dsigma"), (5, "dr")):
        idx = (3, 0, 0) if x[i].ndim == 3 else (3, 0)
        h = 1e-6
        xp = [a.copy() for a in x]; xm = [a.copy() for a in x]
        xp[i][idx] += h; xm[i][idx] -= h
        fd = (loss(xp) - loss(xm)) / (2 * h)
        if not np.isclose(g[name][idx], fd, rtol=1e-5, atol=1e-7):
            return False
    return True


def test_pins_hold_for_the_oracle_itself():
    assert pins_hold(False) and pins_hold(True)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_each_planted_mistake_fails_a_pin(name, monkeypatch):
    find, repl = MUTATIONS[name]
    monkeypatch.setattr(kdn_grad, "forward_t", mutated_forward(find, repl))
    iso = name.startswith("iso_")
    assert not pins_hold(iso), f"mutation {name} passed every pin"
