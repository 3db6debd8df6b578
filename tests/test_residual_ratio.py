"""Residual-ratio diagnostic rho_t = (1 - beta_t <d_t, k_t^2>)^2 and
q_geo = exp(mean_t log rho_t).

"OSDN: Improving Delta Rule with Provable Online Preconditioning in Linear
Attention", technical summary sections 4-5: the contraction factor of one write,
f_t(S_t) / f_t(S_{t-1}) with f_t(S) = 1/2 ||S k_t - v_t||^2, and its geometric
mean over a sequence. CPU tests pin the oracle's rho against the loss ratio
recomputed from its own S trajectory and against special cases; GPU tests
compare the scan kernels' rho and q_geo with the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from preconditioned_delta_rule_token_b200 import workloads as W
from tests._util import BF16_TOL, FP32_TOL, slice_rel_err


def _case(seed, B=1, T=24, H=2, dk=8, dv=5, eta=0.5, apf=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    k[0, 3, 1] = 0.0                                   # a zero key
    v = rng.standard_normal((B, T, H, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, T, H))))
    r = rng.uniform(0.8, 1.0, (B, T, H)) if apf else None
    d0 = rng.uniform(0.5, 1.5, (B, H, dk))
    S0 = 0.3 * rng.standard_normal((B, H, dv, dk))
    return q, k, v, beta, r, d0, S0, eta


def test_rho_is_the_loss_ratio_of_the_trajectory():
    """rho_t = f_t(S_t)/f_t(S_{t-1}), with both losses computed here from the S
    before and after each oracle step (not from <d, k^2>)."""
    q, k, v, beta, r, d0, S0, eta = _case(1)
    _, _, _, rho, _ = oracle.residual_ratio(q, k, v, beta, r, d0, S0, eta=eta)
    B, T, H, dk = k.shape
    S, d = S0.copy(), d0.copy()
    for t in range(T):
        before = 0.5 * np.sum((np.einsum("bhvk,bhk->bhv", S, k[:, t]) - v[:, t]) ** 2, axis=-1)
        oracle.step(q[:, t], k[:, t], v[:, t], beta[:, t], S, d, r=r[:, t], eta=eta)
        after = 0.5 * np.sum((np.einsum("bhvk,bhk->bhv", S, k[:, t]) - v[:, t]) ** 2, axis=-1)
        np.testing.assert_allclose(rho[:, t], after / before, rtol=1e-9, atol=1e-12)


def test_rho_special_cases():
    q, k, v, beta, r, d0, S0, eta = _case(2)
    # beta = 0: no write, rho = 1 and q_geo = 1
    _, _, _, rho, qg = oracle.residual_ratio(q, k, v, 0 * beta, r, d0, S0, eta=eta)
    np.testing.assert_array_equal(rho, 1.0)
    np.testing.assert_array_equal(qg, 1.0)
    # a zero key writes nothing: rho = 1 at that token
    _, _, _, rho, _ = oracle.residual_ratio(q, k, v, beta, r, d0, S0, eta=eta)
    assert rho[0, 3, 1] == 1.0
    # beta = 1, d = 1, unit keys: the gated Newton step, rho = 0 and q_geo = 0
    k2 = k.copy()
    k2[0, 3, 1] = k2[0, 2, 1]
    _, _, _, rho, qg = oracle.residual_ratio(q, k2, v, np.ones_like(beta), None, None, S0, eta=0.0)
    np.testing.assert_allclose(rho, 0.0, atol=1e-24)
    assert np.all(qg == 0.0)


def test_q_geo_is_the_geometric_mean():
    q, k, v, beta, r, d0, S0, eta = _case(3, T=7)
    _, _, _, rho, qg = oracle.residual_ratio(q, k, v, beta, r, d0, S0, eta=eta)
    for b in range(rho.shape[0]):
        for h in range(rho.shape[2]):
            np.testing.assert_allclose(qg[b, h], np.prod(rho[b, :, h]) ** (1.0 / rho.shape[1]), rtol=1e-12)


CASES = [
    # dtype, B, H, T, dk, apf, eta
    (W.BF16, 2, 3, 200, 128, True, 1e-2),
    (W.BF16, 1, 2, 65, 128, False, 1.0),
    (W.BF16, 2, 2, 130, 128, True, 0.0),
    (W.FP32, 2, 2, 130, 128, True, 1e-2),
    (W.FP32, 1, 3, 70, 64, True, 0.5),
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=lambda c: "%s-B%dH%dT%d-dk%d-apf%d-eta%g" % c)
def test_gpu_residual_ratio_matches_oracle(case):
    import preconditioned_delta_rule_token_b200 as pk
    dtype, B, H, T, dk, apf, eta = case
    w = W.Workload("rho", B, H, T, dk, dk, 64, dtype, apf, "gaussian", d0="uniform", S0="normal", seed=31)
    inp = W.make_forward_inputs(w)
    inp["k"][0, min(5, T - 1), 0] = 0                  # a zero key
    dev = lambda x: None if x is None else x.cuda()
    rho, qg, d = pk.residual_ratio(dev(inp["k"]), dev(inp["beta"]), dev(inp["r"]), dev(inp["d0"]), eta=eta)
    assert pk.osdn_sync_status() == 0
    f = W.to_f64
    _, _, rd, rrho, rqg = oracle.residual_ratio(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["beta"]), f(inp["r"]),
                                                f(inp["d0"]), f(inp["S0"]), eta=eta)
    tol = BF16_TOL if dtype == W.BF16 else FP32_TOL
    assert slice_rel_err(rho.cpu().numpy(), rrho, (0, 2)) <= tol
    assert np.max(np.abs(qg.cpu().numpy() - rqg) / np.maximum(rqg, 1e-30)) <= tol
    assert slice_rel_err(d.cpu().numpy(), rd, (0, 1)) <= tol
