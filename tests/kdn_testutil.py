"""Helpers shared by the tests: host->device marshalling, the error metric, and
running the oracle on sampled (sequence, head) chains of a workload."""
import os

import numpy as np

import oracle


def max_rel_err(x, y):
    """max |x - y| / max(max |y|, 1e-6) over the whole tensor (y is the oracle)."""
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    if y.size == 0:
        return 0.0
    return float(np.max(np.abs(x - y)) / max(float(np.max(np.abs(y))), 1e-6))


# every parity check's achieved error: (test id, what, error, tolerance); conftest writes them
# to the JSON file named by $KDN_PARITY_LOG at the end of the session
MARGINS = []


def assert_rel(got, want, tol, what=""):
    """Assert max_rel_err(got, want) <= tol and record the achieved error."""
    err = max_rel_err(got, want)
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    MARGINS.append({"test": test, "what": str(what), "err": err, "tol": float(tol)})
    assert err <= tol, f"{what}: max relative error {err:.3e} > {tol:.1e}"
    return err


def to_dev(a, device="cuda"):
    import torch
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    if a.dtype == np.int32:
        return torch.from_numpy(a).to(device)
    return torch.from_numpy(a.astype(np.float32)).to(device)


def to_host(t):
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy()
    return t.cpu().numpy()


def dense_shape(w, x):
    """[ntok, H, d] -> [B, T, H, d] (varlen: B = 1)."""
    B = w.B if w.B else 1
    T = x.shape[0] // B
    return x.reshape((B, T) + x.shape[1:])


def oracle_chains(w, chains, mu=None, S0=None, P0=None, threads=None):
    """Oracle on the listed (seq, head) chains of workload ``w``:
    {(s, h): dict(o [len, dv], S [dk, dv], P [dk])}."""
    return oracle.diag_chains(w, chains, mu=mu, S0=S0, P0=P0, threads=threads)
