"""The pins have teeth: plausible mistakes planted in a copy of the oracle source
(on the CPU, never in the product) must each make at least one pin fail.

Every mutation below keeps all memory accesses in bounds; only the arithmetic or
the wiring changes.
"""
import inspect
import os

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = open(os.path.join(os.path.dirname(oracle.__file__), "kdn_oracle.c")).read()

MUTATIONS = {
    "predict_alpha_not_squared": ("Pm[i] = al[i] * al[i] * P[i] + sg[i];", "Pm[i] = al[i] * P[i] + sg[i];"),
    "predict_drops_process_noise": ("Pm[i] = al[i] * al[i] * P[i] + sg[i];", "Pm[i] = al[i] * al[i] * P[i];"),
    "gain_den_drops_a_key_factor": ("den += Pm[i] * k[i] * k[i];", "den += Pm[i] * k[i];"),
    "gain_uses_posterior_not_predicted": ("g[i] = Pm[i] * k[i] / den;", "g[i] = P[i] * k[i] / den;"),
    "update_ignores_mu": ("P[i] = Pm[i] / (1.0 + J->mu * Pm[i] * k[i] * k[i] / r);",
                          "P[i] = Pm[i] / (1.0 + Pm[i] * k[i] * k[i] / r);"),
    "update_moment_matching": ("P[i] = Pm[i] / (1.0 + J->mu * Pm[i] * k[i] * k[i] / r);",
                               "P[i] = Pm[i] - J->mu * g[i] * k[i] * Pm[i];"),
    "readout_before_write": ("delta_write(S, dk, dv, al, k, g, v, u);\n        readout(S, dk, dv, q, J->o + th * dv);",
                             "readout(S, dk, dv, q, J->o + th * dv);\n        delta_write(S, dk, dv, al, k, g, v, u);"),
    "readout_with_key": ("readout(S, dk, dv, q, J->o + th * dv);", "readout(S, dk, dv, k, J->o + th * dv);"),
    "state_decay_squared": ("S[(size_t)i * dv + j] *= alpha[i];", "S[(size_t)i * dv + j] *= alpha[i] * alpha[i];"),
    "residual_sign": ("u[j] = v[j] - pred;", "u[j] = v[j] + pred;"),
    "full_predict_transposed_decay": ("al[i] * Sig[(size_t)i * dk + j] * al[j]", "al[i] * Sig[(size_t)i * dk + j] * al[i]"),
    "full_update_sign": ("Sm[(size_t)i * dk + j] - Sk[i] * Sk[j] / den", "Sm[(size_t)i * dk + j] + Sk[i] * Sk[j] / den"),
    "initial_state_ignored": ("if (J->S0) memcpy(S,", "if (J->S0 && 0) memcpy(S,"),
    "initial_uncertainty_ignored": ("P[i] = J->P0 ? J->P0[sh * dk + i] : 1.0;", "P[i] = 1.0;"),
    "head_index_dropped": ("const size_t th = (size_t)t * H + h;", "const size_t th = (size_t)t * H;"),
    "noise_indexed_by_token_only": ("const double r = J->r ? J->r[th] : 0.0;", "const double r = J->r ? J->r[t] : 0.0;"),
    "iso_predict_mean_of_alpha_not_alpha_squared": ("a2 += al[i] * al[i];", "a2 += al[i];"),
    "iso_predict_drops_process_noise": ("Pm[0] = (a2 / dk) * P[0] + sm / dk;", "Pm[0] = (a2 / dk) * P[0];"),
    "iso_gain_uses_posterior": ("const double den = r + Pm[0] * kk;", "const double den = r + P[0] * kk;"),
    "iso_update_not_averaged_over_directions": ("P[0] = Pm[0] / (1.0 + J->mu * Pm[0] * kk / (dk * r));",
                                                "P[0] = Pm[0] / (1.0 + J->mu * Pm[0] * kk / r);"),
    "iso_update_ignores_mu": ("P[0] = Pm[0] / (1.0 + J->mu * Pm[0] * kk / (dk * r));",
                              "P[0] = Pm[0] / (1.0 + Pm[0] * kk / (dk * r));"),
    "iso_initial_uncertainty_ignored": ("P[0] = J->P0 ? J->P0[sh] : 1.0;", "P[0] = 1.0;"),
}


def _pin_calls():
    for name, fn in sorted(vars(pins).items()):
        if not name.startswith("test_") or not inspect.isfunction(fn):
            continue
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if marks:
            arg, values = marks[0].args
            for val in values:
                yield f"{name}[{val}]", (lambda f=fn, a=arg, x=val: f(**{a: x}))
        else:
            yield name, fn


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_planted_mistake_is_caught(mutation):
    old, new = MUTATIONS[mutation]
    assert SRC.count(old) == 1, f"mutation anchor not unique/absent: {old!r}"
    lib = oracle.build_variant(SRC.replace(old, new), mutation)
    saved = oracle._lib
    oracle._lib = lib
    caught = []
    try:
        for name, call in _pin_calls():
            try:
                call()
            except (AssertionError, RuntimeError, FloatingPointError, ValueError, ZeroDivisionError):
                caught.append(name)
    finally:
        oracle._lib = saved
    assert caught, f"no pin caught the planted mistake {mutation}"
