"""Anchored APF: the retention pulls d toward its initial value d0 instead of 0,
    d_{t+1} = r_t d_t + (1 - r_t) d0 + eta beta_t (1 - beta_t <d_t, k_t^2>) k_t^2 / ||k_t||^2
("OSDN: Improving Delta Rule with Provable Online Preconditioning in Linear
Attention", APF section, read as refreshing the calibration toward d0; still
affine in d). CPU tests pin the oracle option against closed forms and the chunk
form; GPU tests compare the kernels with it.
"""
import numpy as np
import pytest
import torch

import oracle
from preconditioned_delta_rule_token_b200 import workloads as W
from tests._util import BF16_TOL, FP32_TOL, slice_rel_err
from tests.test_chunk_algebra import chunked_delta


def _case(seed, B=1, T=150, H=2, dk=16, dv=8, eta=0.5):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    k[0, 5, 0] = 0.0
    v = rng.standard_normal((B, T, H, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, T, H))))
    r = rng.uniform(0.6, 1.0, (B, T, H))
    d0 = rng.uniform(0.5, 1.5, (B, H, dk))
    S0 = 0.3 * rng.standard_normal((B, H, dv, dk))
    return q, k, v, beta, r, d0, S0, eta


def test_anchor_without_forgetting_is_plain():
    q, k, v, beta, r, d0, S0, eta = _case(1)
    a = oracle.fwd(q, k, v, beta, None, d0, S0, eta=eta, anchor=True)
    p = oracle.fwd(q, k, v, beta, None, d0, S0, eta=eta)
    for x, y in zip(a, p):
        np.testing.assert_array_equal(x, y)


def test_closed_forms_without_the_hypergradient_step():
    """eta = 0: anchored d stays d0; plain APF decays it to prod_t r_t * d0."""
    q, k, v, beta, r, d0, S0, _ = _case(2)
    _, _, da = oracle.fwd(q, k, v, beta, r, d0, S0, eta=0.0, anchor=True)
    np.testing.assert_allclose(da, d0, rtol=1e-13, atol=0)
    _, _, dp = oracle.fwd(q, k, v, beta, r, d0, S0, eta=0.0)
    np.testing.assert_allclose(dp, np.prod(r, axis=1)[..., None] * d0, rtol=1e-12)
    # beta = 0 (no writes, no d step): the anchor is a fixed point
    _, S, da = oracle.fwd(q, k, v, 0 * beta, r, d0, S0, eta=0.7, anchor=True)
    np.testing.assert_allclose(da, d0, rtol=1e-13)
    np.testing.assert_array_equal(S, S0)


def _chunked_anchored_scan(k, beta, r, d0, eta, L):
    """Chunk form on e = d - d0 (the plain recurrence) with <d0, a_t> added to the
    chunk-start term of c_t. k: [T, dk]. Returns D [T, dk] and d after T."""
    T, dk = k.shape
    e = np.zeros(dk)                                   # e_1 = d_1 - d0 = 0
    D = np.zeros((T, dk))
    for c0 in range(0, T, L):
        kk = k[c0:c0 + L]
        n = len(kk)
        a = kk * kk
        nrm = a.sum(1)
        ok = nrm > 0
        u = np.where(ok[:, None], a / np.where(ok, nrm, 1)[:, None], 0.0)
        g = np.where(ok, eta * beta[c0:c0 + n], 0.0)
        be, rr = beta[c0:c0 + n], r[c0:c0 + n]
        R = np.ones((n + 1, n + 1))
        for t in range(n + 1):
            for j in range(t):
                R[t, j] = np.prod(rr[j:t])
        M = np.zeros((n, n))
        for t in range(n):
            for j in range(t):
                M[t, j] = g[t] * be[t] * R[t, j + 1] * (a[t] @ u[j])
        c = g * (1 - be * (R[np.arange(n), 0] * (a @ e) + a @ d0))
        x = np.linalg.solve(np.eye(n) + M, c)
        for t in range(n):
            D[c0 + t] = d0 + R[t, 0] * e + sum(R[t, j + 1] * x[j] * u[j] for j in range(t))
        e = R[n, 0] * e + sum(R[n, j + 1] * x[j] * u[j] for j in range(n))
    return D, e + d0


@pytest.mark.parametrize("L", [16, 64])
def test_chunk_form_equals_the_recurrence(L):
    q, k, v, beta, r, d0, S0, eta = _case(3)
    ro, rS, rd = oracle.fwd(q, k, v, beta, r, d0, S0, eta=eta, anchor=True)
    for h in range(k.shape[2]):
        D, dT = _chunked_anchored_scan(k[0, :, h], beta[0, :, h], r[0, :, h], d0[0, h], eta, L)
        np.testing.assert_allclose(dT, rd[0, h], rtol=1e-11, atol=1e-12)
        out, S = chunked_delta(q[0, :, h], k[0, :, h], D * k[0, :, h], v[0, :, h], beta[0, :, h], S0[0, h], 64)
        np.testing.assert_allclose(out, ro[0, :, h], rtol=1e-10, atol=1e-10)
        np.testing.assert_allclose(S, rS[0, h], rtol=1e-10, atol=1e-10)


def test_decode_steps_equal_the_forward():
    q, k, v, beta, r, d0, S0, eta = _case(4, T=12)
    ro, rS, rd = oracle.fwd(q, k, v, beta, r, d0, S0, eta=eta, anchor=True)
    S, d = S0.copy(), d0.copy()
    for t in range(q.shape[1]):
        o = oracle.step(q[:, t], k[:, t], v[:, t], beta[:, t], S, d, r=r[:, t], eta=eta, d_anchor=d0)
        np.testing.assert_allclose(o, ro[:, t], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, rS, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(d, rd, rtol=1e-12, atol=1e-12)


GPU_CASES = [
    # dtype, B, H, T, dk, dv, eta
    (W.BF16, 2, 3, 200, 128, 128, 1e-2),
    (W.BF16, 1, 2, 130, 128, 128, 1.0),
    (W.FP32, 2, 2, 130, 128, 64, 0.5),
    (W.BF16, 1, 2, 70, 64, 64, 0.5),
]


def _inputs(case, seed=41):
    dtype, B, H, T, dk, dv, eta = case
    w = W.Workload("anchored", B, H, T, dk, dv, 64, dtype, True, "gaussian", d0="uniform", S0="normal", seed=seed)
    inp = W.make_forward_inputs(w)
    # keep r well below 1 so that the anchor term matters
    inp["r"] = (0.9 + 0.1 * torch.rand(inp["r"].shape, generator=torch.Generator().manual_seed(seed))).to(
        inp["r"].dtype)
    return w, inp


@pytest.mark.gpu
@pytest.mark.parametrize("case", GPU_CASES, ids=lambda c: "%s-B%dH%dT%d-dk%ddv%d-eta%g" % c)
def test_gpu_forward_matches_oracle(case):
    import preconditioned_delta_rule_token_b200 as pk
    w, inp = _inputs(case)
    dev = lambda x: None if x is None else x.cuda()
    out, S, d = pk.forward(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["beta"]), dev(inp["r"]),
                           dev(inp["d0"]), dev(inp["S0"]), eta=w.eta, apf_anchor=True)
    assert pk.osdn_sync_status() == 0
    f = W.to_f64
    ro, rS, rd = oracle.fwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["beta"]), f(inp["r"]), f(inp["d0"]),
                            f(inp["S0"]), eta=w.eta, anchor=True)
    tol = BF16_TOL if w.dtype == W.BF16 else FP32_TOL
    assert slice_rel_err(out.float().cpu().numpy(), ro, (0, 2)) <= tol
    assert slice_rel_err(S.cpu().numpy(), rS, (0, 1)) <= tol
    assert slice_rel_err(d.cpu().numpy(), rd, (0, 1)) <= tol
    # and the anchor changes the result (it is not silently ignored)
    _, _, rd_plain = oracle.fwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["beta"]), f(inp["r"]), f(inp["d0"]),
                                f(inp["S0"]), eta=w.eta)
    assert slice_rel_err(rd_plain, rd, (0, 1)) > 10 * tol


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [W.FP32, W.BF16])
def test_gpu_decode_matches_oracle(dtype):
    import preconditioned_delta_rule_token_b200 as pk
    w, inp = _inputs((dtype, 2, 3, 24, 128, 128, 0.5))
    dev = lambda x: None if x is None else x.cuda()
    S, d = dev(inp["S0"]).clone(), dev(inp["d0"]).clone()
    anchor = dev(inp["d0"]).clone()
    outs = []
    for t in range(w.T):
        tok = {n: dev(inp[n][:, t].contiguous()) for n in ("q", "k", "v", "beta", "r")}
        outs.append(pk.step(tok["q"], tok["k"], tok["v"], tok["beta"], S, d, r=tok["r"], eta=w.eta, d_anchor=anchor))
    assert pk.osdn_sync_status() == 0
    out = torch.stack(outs, 1).float().cpu().numpy()
    f = W.to_f64
    ro, rS, rd = oracle.fwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["beta"]), f(inp["r"]), f(inp["d0"]),
                            f(inp["S0"]), eta=w.eta, anchor=True)
    tol = BF16_TOL if dtype == W.BF16 else FP32_TOL
    assert slice_rel_err(out, ro, (0, 2)) <= tol
    assert slice_rel_err(S.cpu().numpy(), rS, (0, 1)) <= tol
    assert slice_rel_err(d.cpu().numpy(), rd, (0, 1)) <= tol


@pytest.mark.gpu
def test_gpu_residual_ratio_anchored():
    import preconditioned_delta_rule_token_b200 as pk
    w, inp = _inputs((W.BF16, 2, 2, 130, 128, 128, 0.5))
    dev = lambda x: None if x is None else x.cuda()
    rho, qg, d = pk.residual_ratio(dev(inp["k"]), dev(inp["beta"]), dev(inp["r"]), dev(inp["d0"]), eta=w.eta,
                                   apf_anchor=True)
    assert pk.osdn_sync_status() == 0
    f = W.to_f64
    _, _, rd, rrho, rqg = oracle.residual_ratio(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["beta"]), f(inp["r"]),
                                                f(inp["d0"]), f(inp["S0"]), eta=w.eta, anchor=True)
    assert slice_rel_err(rho.cpu().numpy(), rrho, (0, 2)) <= BF16_TOL
    assert np.max(np.abs(qg.cpu().numpy() - rqg) / np.maximum(rqg, 1e-30)) <= BF16_TOL
    assert slice_rel_err(d.cpu().numpy(), rd, (0, 1)) <= BF16_TOL
