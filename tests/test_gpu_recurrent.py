"""GPU parity of the fused recurrent kernel (prefill path chunk=0) and the decode step
against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest

import oracle
from kalman_delta_rule_b200 import inputs
from tests.kdn_testutil import dense_shape, assert_rel, max_rel_err, oracle_chains, to_dev, to_host

pytestmark = pytest.mark.gpu

TOL_F32, TOL_BF16 = 1e-4, 2e-2


def run_forward(kdn, w, chunk, mu=1.0, S0=None, P0=None, workspace=None):
    """Forward through the C ABI; ``workspace`` None allocates one of kdn_workspace_size()
    bytes (two-launch tensor-core path where it applies), False passes none."""
    import torch
    args = [to_dev(dense_shape(w, getattr(w, n))) for n in ("q", "k", "v", "alpha", "sigma")]
    r = to_dev(dense_shape(w, w.r))
    cu = to_dev(w.cu_seqlens) if w.B == 1 and w.num_seqs > 1 else None
    max_seqlen = int(np.diff(w.cu_seqlens).max()) if cu is not None else 0
    o, S, P = kdn.forward(*args, r, cu_seqlens=cu, S0=to_dev(S0), P0=to_dev(P0), mu=mu, chunk=chunk,
                          workspace=workspace, max_seqlen=max_seqlen)
    torch.cuda.synchronize()
    kdn.last_device_error()
    return to_host(o).reshape((-1,) + o.shape[2:]), to_host(S), to_host(P)


@pytest.mark.parametrize("mu", [1.0, 32.0])
def test_tiny_fp32_recurrent_matches_oracle(kdn, mu):
    w = inputs.tiny_fp32()
    ref = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens, mu=mu)
    o, S, P = run_forward(kdn, w, chunk=0, mu=mu)
    assert_rel(o, ref["o"], TOL_F32, 'o')
    assert_rel(S, ref["S"], TOL_F32, 'S')
    assert_rel(P, ref["P"], TOL_F32, 'P')


def ragged(seed, lens, H, dk, dv, bf16):
    tok = inputs.draw_tokens(seed, int(sum(lens)), H, dk, dv, bf16)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return inputs.Workload(name="ragged", H=H, dk=dk, dv=dv, cu_seqlens=cu, bf16=bf16, B=1, T=int(sum(lens)), **tok)


@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 128), (128, 256), (128, 32)])
@pytest.mark.parametrize("bf16", [False, True])
def test_ragged_varlen_recurrent(kdn, dk, dv, bf16):
    w = ragged(100 + dk + dv, [1, 63, 64, 65, 130], 3, dk, dv, bf16)
    rng = np.random.default_rng(1)
    S0 = (0.1 * rng.standard_normal((w.num_seqs, w.H, dk, dv))).astype(np.float32)
    P0 = rng.uniform(0.3, 2.0, (w.num_seqs, w.H, dk)).astype(np.float32)
    ref = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens, S0=S0, P0=P0, mu=2.0)
    o, S, P = run_forward(kdn, w, chunk=0, mu=2.0, S0=S0, P0=P0)
    tol = TOL_BF16 if bf16 else TOL_F32
    assert_rel(o, ref["o"], tol, 'o')
    assert_rel(S, ref["S"], tol, 'S')
    assert_rel(P, ref["P"], tol, 'P')


def test_empty_sequences_and_zero_tokens(kdn):
    w = ragged(7, [5, 0, 3], 2, 32, 32, True)  # an empty sequence in the middle
    S0 = np.random.default_rng(2).standard_normal((3, 2, 32, 32)).astype(np.float32)
    ref = oracle.diag_forward(w.q, w.k, w.v, w.alpha, w.sigma, w.r, cu_seqlens=w.cu_seqlens, S0=S0)
    o, S, P = run_forward(kdn, w, chunk=0, S0=S0)
    assert_rel(o, ref["o"], TOL_BF16, 'o')
    np.testing.assert_array_equal(S[1], S0[1])  # the empty sequence passes its state through
    np.testing.assert_array_equal(P[1], 1.0)
    assert_rel(S, ref["S"], TOL_BF16, 'S')


def decode_run(kdn, S0, P0, steps, bf16=True, mu=1.0):
    import torch
    S = to_dev(S0).clone()
    P = to_dev(P0).clone()
    outs = []
    for st in steps:
        o = kdn.decode_step(*[to_dev(st[n]) for n in ("q", "k", "v", "alpha", "sigma", "r")], S, P, mu=mu)
        outs.append(to_host(o))
    torch.cuda.synchronize()
    kdn.last_device_error()
    return np.stack(outs), to_host(S), to_host(P)


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 256), (32, 64)])
@pytest.mark.parametrize("bf16", [True, False])
def test_decode_small_matches_oracle(kdn, dk, dv, bf16):
    N, H, n = 5, 3, 12
    rng = np.random.default_rng(dk + dv)
    S0 = (0.1 * rng.standard_normal((N, H, dk, dv))).astype(np.float32)
    P0 = np.logaddexp(0, rng.standard_normal((N, H, dk))).astype(np.float32)
    steps = [inputs.draw_tokens((9, s), N, H, dk, dv, bf16) for s in range(n)]
    o, S, P = decode_run(kdn, S0, P0, steps, bf16, mu=1.5)
    ref = oracle.run_decode(S0, P0, steps, mu=1.5)
    tol = TOL_BF16 if bf16 else TOL_F32
    assert_rel(o, ref["o"], tol, 'o')
    assert_rel(S, ref["S"], tol, 'S')
    assert_rel(P, ref["P"], tol, 'P')


def test_decode_full_size_sampled(kdn):
    """The decode workload's launch configuration (256 sequences x 32 heads, d = 128,
    fp32 state, bf16 inputs) for 16 steps; sampled (sequence, head) chains are checked
    against the oracle element by element."""
    w = inputs.decode_256x32()
    n = 16
    steps = [w.step(s) for s in range(n)]
    o, S, P = decode_run(kdn, w.S0, w.P0, steps)
    rng = np.random.default_rng(0)
    picks = [(int(a), int(b)) for a, b in zip(rng.integers(0, w.N, 12), rng.integers(0, w.H, 12))]
    picks += [(0, 0), (w.N - 1, w.H - 1)]
    for (ns, h) in picks:
        sub = [{nm: a[ns:ns + 1, h:h + 1] for nm, a in st.items()} for st in steps]
        ref = oracle.run_decode(w.S0[ns:ns + 1, h:h + 1], w.P0[ns:ns + 1, h:h + 1], sub)
        assert_rel(o[:, ns, h], ref["o"][:, 0, 0], TOL_BF16, 'o[:, ns, h]')
        assert_rel(S[ns, h], ref["S"][0, 0], TOL_BF16, 'S[ns, h]')
        assert_rel(P[ns, h], ref["P"][0, 0], TOL_BF16, 'P[ns, h]')


def test_decode_1024_steps_full_size_sampled(kdn):
    """The decode workload as stated: 256 sequences x 32 heads, d = 128, fp32 state, 1024
    single-token steps through kdn_decode_step, inputs drawn on the device (seeded).  Eight
    sampled (sequence, head) chains: o at every step and the final S and P against the oracle
    run on the same bf16 inputs copied back to the host."""
    import torch
    steps, N, H, d = 1024, 256, 32, 128
    dv = inputs.decode_inputs_device(2, steps, N, H, d)
    S0, P0 = dv["S0"].clone(), dv["P0"].clone()
    S, P = dv["S0"], dv["P0"]
    rng = np.random.default_rng(2)
    picks = [(0, 0), (N - 1, H - 1)] + [(int(a), int(b)) for a, b in zip(rng.integers(0, N, 6), rng.integers(0, H, 6))]
    ni = torch.tensor([p[0] for p in picks], device="cuda")
    hi = torch.tensor([p[1] for p in picks], device="cuda")
    o = torch.empty((N, H, d), dtype=torch.bfloat16, device="cuda")
    o_s = torch.empty((steps, len(picks), d), dtype=torch.float32, device="cuda")
    names = ("q", "k", "v", "alpha", "sigma", "r")
    for s in range(steps):
        kdn.decode_step(*[dv[nm][s] for nm in names], S, P, o=o)
        o_s[s] = o[ni, hi].float()
    torch.cuda.synchronize()
    kdn.last_device_error()
    got_o, got_S, got_P = to_host(o_s), to_host(S[ni, hi]), to_host(P[ni, hi])
    host = {nm: to_host(dv[nm][:, ni, hi]) for nm in names}    # [steps, picks, ...]
    S0h, P0h = to_host(S0[ni, hi]), to_host(P0[ni, hi])
    for i, (ns, h) in enumerate(picks):
        sub = [{nm: host[nm][s, i][None, None] for nm in names} for s in range(steps)]
        ref = oracle.run_decode(S0h[i][None, None], P0h[i][None, None], sub)
        assert_rel(got_o[:, i], ref["o"][:, 0, 0], TOL_BF16, f"o ({ns},{h})")
        assert_rel(got_S[i], ref["S"][0, 0], TOL_BF16, f"S ({ns},{h})")
        assert_rel(got_P[i], ref["P"][0, 0], TOL_BF16, f"P ({ns},{h})")


@pytest.mark.parametrize("n", [1, 4, 7])
def test_decode_tokens_matches_oracle_and_single_steps(kdn, n):
    """n tokens per launch (multi-token decode) = the oracle's n steps, and bit-identical to
    n single-token decode steps (the same per-token arithmetic, the state kept on chip)."""
    import torch
    N, H, dk, dv = 6, 3, 128, 128
    rng = np.random.default_rng(n)
    S0 = (0.1 * rng.standard_normal((N, H, dk, dv))).astype(np.float32)
    P0 = np.logaddexp(0, rng.standard_normal((N, H, dk))).astype(np.float32)
    steps = [inputs.draw_tokens((11, n, s), N, H, dk, dv, True) for s in range(n)]
    stacked = {nm: np.stack([st[nm] for st in steps], axis=1) for nm in steps[0]}   # [N, n, H, ...]
    S, P = to_dev(S0).clone(), to_dev(P0).clone()
    o = kdn.decode_tokens(*[to_dev(stacked[nm]) for nm in ("q", "k", "v", "alpha", "sigma", "r")], S, P, mu=2.0)
    torch.cuda.synchronize()
    kdn.last_device_error()
    ref = oracle.run_decode(S0, P0, steps, mu=2.0)
    o_h = to_host(o).transpose(1, 0, 2, 3)   # [n, N, H, dv]
    assert_rel(o_h, ref["o"], TOL_BF16, 'o_h')
    assert_rel(to_host(S), ref["S"], TOL_BF16, 'to_host(S)')
    assert_rel(to_host(P), ref["P"], TOL_BF16, 'to_host(P)')
    o1, S1, P1 = decode_run(kdn, S0, P0, steps, mu=2.0)
    np.testing.assert_array_equal(to_host(S), S1)
    np.testing.assert_array_equal(to_host(P), P1)
    np.testing.assert_array_equal(o_h, o1)
