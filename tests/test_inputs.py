"""The seeded input generators (CPU): the device-side decode generator draws the workload's
distributions and shapes, reproducibly, and the parity-log helper records what it checks."""
import numpy as np
import pytest

from kalman_delta_rule_b200 import inputs


def test_decode_inputs_device_shapes_ranges_and_seed():
    torch = pytest.importorskip("torch")
    steps, N, H, d = 3, 4, 2, 32
    a = inputs.decode_inputs_device(7, steps, N, H, d, device="cpu")
    b = inputs.decode_inputs_device(7, steps, N, H, d, device="cpu")
    assert a["S0"].shape == (N, H, d, d) and a["S0"].dtype == torch.float32
    assert a["P0"].shape == (N, H, d) and bool((a["P0"] > 0).all())
    for n in ("q", "k", "v", "alpha", "sigma"):
        assert a[n].shape == (steps, N, H, d) and a[n].dtype == torch.bfloat16, n
    assert a["r"].shape == (steps, N, H) and a["r"].dtype == torch.bfloat16
    for n in a:
        assert torch.equal(a[n], b[n]), n                      # same seed, same draws
    kn = a["k"].float().norm(dim=-1)
    assert float((kn - 1).abs().max()) < 1e-2                  # unit keys (bf16 rounding)
    al = a["alpha"].float()
    assert bool((al > 0).all()) and bool((al <= 1).all())
    assert float(al.mean()) > 0.9                              # sigmoid(N(4, 1))
    assert bool((a["sigma"].float() > 0).all()) and bool((a["r"].float() >= 1e-3).all())
    s0 = a["S0"].numpy()
    assert 0.08 < float(s0.std()) < 0.12                       # S0 ~ N(0, std 0.1)
    c = inputs.decode_inputs_device(8, steps, N, H, d, device="cpu")
    assert not torch.equal(a["q"], c["q"])


def test_parity_log_records_each_check():
    from tests import kdn_testutil as tu
    n0 = len(tu.MARGINS)
    err = tu.assert_rel(np.array([1.0, 2.0]), np.array([1.0, 2.0 + 1e-3]), 1e-2, "x")
    assert 0 < err < 1e-2 and len(tu.MARGINS) == n0 + 1
    assert tu.MARGINS[-1]["what"] == "x" and tu.MARGINS[-1]["tol"] == 1e-2
    with pytest.raises(AssertionError):
        tu.assert_rel(np.array([1.0]), np.array([2.0]), 1e-2, "y")
