"""Gated OSDN: OSDN on the gated delta rule backbone,
    S_t = alpha_t S_{t-1} (I - beta_t k_t kw_t^T) + beta_t v_t kw_t^T,  kw_t = d_t (.) k_t,
with the preconditioner d unchanged ("OSDN: Improving Delta Rule with Provable
Online Preconditioning in Linear Attention": the pages run OSDN on the gated
DeltaNet backbone; the composition is the plainest one, the OSDN write key in the
gated update). CPU tests pin the oracle option; GPU tests compare the kernels.
"""
import numpy as np
import pytest
import torch

import oracle
from preconditioned_delta_rule_token_b200 import workloads as W
from tests._util import BF16_TOL, slice_rel_err
from tests.test_chunk_algebra import chunked_scan


def _case(seed, B=1, T=150, H=2, dk=16, dv=8, eta=0.5):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    k[0, 5, 0] = 0.0
    v = rng.standard_normal((B, T, H, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, T, H))))
    r = rng.uniform(0.8, 1.0, (B, T, H))
    alpha = rng.uniform(0.85, 1.0, (B, T, H))
    d0 = rng.uniform(0.5, 1.5, (B, H, dk))
    S0 = 0.3 * rng.standard_normal((B, H, dv, dk))
    return q, k, v, beta, r, alpha, d0, S0, eta


def test_alpha_one_is_ungated():
    q, k, v, beta, r, alpha, d0, S0, eta = _case(1)
    g = oracle.fwd(q, k, v, beta, r, d0, S0, eta=eta, alpha=np.ones_like(alpha))
    p = oracle.fwd(q, k, v, beta, r, d0, S0, eta=eta)
    for x, y in zip(g, p):
        np.testing.assert_array_equal(x, y)


def test_alpha_zero_restarts_the_state():
    """alpha_t0 = 0 wipes S before token t0's write: the rest equals a fresh
    forward from S = 0 with the d carried to t0 (d does not depend on S)."""
    q, k, v, beta, r, alpha, d0, S0, eta = _case(2)
    t0 = 60
    alpha[:, t0] = 0.0
    ro, rS, rd = oracle.fwd(q, k, v, beta, r, d0, S0, eta=eta, alpha=alpha)
    _, _, d_mid = oracle.fwd(q[:, :t0], k[:, :t0], v[:, :t0], beta[:, :t0], r[:, :t0], d0, S0, eta=eta,
                             alpha=alpha[:, :t0])
    fo, fS, fd = oracle.fwd(q[:, t0:], k[:, t0:], v[:, t0:], beta[:, t0:], r[:, t0:], d_mid, None, eta=eta,
                            alpha=alpha[:, t0:])
    np.testing.assert_allclose(ro[:, t0:], fo, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(rS, fS, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(rd, fd, rtol=1e-12, atol=1e-12)


def test_unit_preconditioner_is_textbook_gated_deltanet():
    """eta = 0, d0 = 1, no APF: S_t = alpha S (I - beta k k^T) + beta v k^T, o = S q,
    written out here from that definition."""
    q, k, v, beta, _, alpha, _, S0, _ = _case(3, T=40)
    ro, rS, _ = oracle.fwd(q, k, v, beta, None, None, S0, eta=0.0, alpha=alpha)
    B, T, H, dk = k.shape
    for b in range(B):
        for h in range(H):
            S = S0[b, h].copy()
            for t in range(T):
                kt = k[b, t, h]
                S = alpha[b, t, h] * S @ (np.eye(dk) - beta[b, t, h] * np.outer(kt, kt)) + \
                    beta[b, t, h] * np.outer(v[b, t, h], kt)
                np.testing.assert_allclose(S @ q[b, t, h], ro[b, t, h], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(S, rS[b, h], rtol=1e-12, atol=1e-12)


def chunked_gated_delta(q, k, kw, v, beta, alpha, S0, C):
    """Gated chunk form for one unit, as the tensor-core kernel computes it: gamma =
    cumulative alpha within the chunk, A = strict_tril(diag(beta) (K Kw^T) (.) Gamma),
    Gamma_tj = gamma_t / gamma_j, T = (I + A)^{-1}, W = T diag(beta gamma) K,
    U0 = T diag(beta) V, Ut = diag(1/gamma) (U0 - W S^T),
    O = diag(gamma) (Q S^T + tril(Q Kw^T) Ut), S <- gamma_C (S + Ut^T Kw)."""
    T = k.shape[0]
    S = S0.copy()
    out = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        Q, K, Kw, V = q[c0:c0 + C], k[c0:c0 + C], kw[c0:c0 + C], v[c0:c0 + C]
        b, g = beta[c0:c0 + C], np.cumprod(alpha[c0:c0 + C])
        n = len(K)
        Gam = g[:, None] / g[None, :]
        A = np.tril(b[:, None] * (K @ Kw.T) * Gam, -1)
        Tm = np.linalg.inv(np.eye(n) + A)
        Wm = Tm @ ((b * g)[:, None] * K)
        U0 = Tm @ (b[:, None] * V)
        Ut = (U0 - Wm @ S.T) / g[:, None]
        out[c0:c0 + n] = g[:, None] * (Q @ S.T + np.tril(Q @ Kw.T) @ Ut)
        S = g[-1] * (S + Ut.T @ Kw)
    return out, S


def chunked_gated_delta_plain_inverse(q, k, kw, v, beta, alpha, S0, C):
    """The same chunk form with the decay moved out of the triangular solve:
    T = diag(gamma) Th diag(1/gamma) with Th = (I + strict_tril(diag(beta) K Kw^T))^{-1}
    (no decay in it), so Ut = Th diag(beta/gamma) V - Th diag(beta) K S^T; O and the
    state carry as above. It divides by gamma, so it needs gates near 1."""
    T = k.shape[0]
    S = S0.copy()
    out = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        Q, K, Kw, V = q[c0:c0 + C], k[c0:c0 + C], kw[c0:c0 + C], v[c0:c0 + C]
        b, g = beta[c0:c0 + C], np.cumprod(alpha[c0:c0 + C])
        n = len(K)
        Th = np.linalg.inv(np.eye(n) + np.tril(b[:, None] * (K @ Kw.T), -1))
        Ut = Th @ ((b / g)[:, None] * V) - (Th @ (b[:, None] * K)) @ S.T
        out[c0:c0 + n] = g[:, None] * (Q @ S.T + np.tril(Q @ Kw.T) @ Ut)
        S = g[-1] * (S + Ut.T @ Kw)
    return out, S


def chunked_gated_delta_ratio(q, k, kw, v, beta, alpha, S0, C):
    """The chunk form the tensor-core kernel computes, every decay factor a ratio
    gamma_t / gamma_j <= 1 (t >= j) taken as 2^(G_t - G_j) of the in-chunk cumulative
    log2 alpha G (each log2 alpha clamped at -120, so alpha = 0 is allowed):
    A = strict_tril(diag(beta) (K Kw^T) (.) R), T = (I + A)^{-1}, W = T diag(beta gamma) K,
    U0 = T diag(beta) V, U = U0 - W S^T, O = diag(gamma) Q S^T + (tril(Q Kw^T) (.) R) U,
    S <- gamma_C S + (diag(gamma_C / gamma) U)^T Kw, with R_tj = gamma_t / gamma_j."""
    T = k.shape[0]
    S = S0.copy()
    out = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        Q, K, Kw, V = q[c0:c0 + C], k[c0:c0 + C], kw[c0:c0 + C], v[c0:c0 + C]
        b = beta[c0:c0 + C]
        with np.errstate(divide="ignore"):
            G = np.cumsum(np.maximum(np.log2(alpha[c0:c0 + C]), -120.0))
        n = len(K)
        R = np.exp2(np.minimum(G[:, None] - G[None, :], 0.0))
        g = np.exp2(G)
        Tm = np.linalg.inv(np.eye(n) + np.tril(b[:, None] * (K @ Kw.T) * R, -1))
        U = Tm @ (b[:, None] * V) - (Tm @ ((b * g)[:, None] * K)) @ S.T
        out[c0:c0 + n] = g[:, None] * (Q @ S.T) + (np.tril(Q @ Kw.T) * R) @ U
        S = g[-1] * S + (np.exp2(G[-1] - G)[:, None] * U).T @ Kw
    return out, S


@pytest.mark.parametrize("form", [chunked_gated_delta, chunked_gated_delta_plain_inverse, chunked_gated_delta_ratio])
def test_gated_chunk_form_equals_the_recurrence(form):
    q, k, v, beta, r, alpha, d0, S0, eta = _case(4)
    ro, rS, rd = oracle.fwd(q, k, v, beta, r, d0, S0, eta=eta, alpha=alpha)
    for h in range(k.shape[2]):
        D, dT = chunked_scan(k[0, :, h], beta[0, :, h], r[0, :, h], d0[0, h], eta, 64)
        np.testing.assert_allclose(dT, rd[0, h], rtol=1e-11, atol=1e-12)
        out, S = form(q[0, :, h], k[0, :, h], D * k[0, :, h], v[0, :, h], beta[0, :, h], alpha[0, :, h],
                      S0[0, h], 64)
        np.testing.assert_allclose(out, ro[0, :, h], rtol=1e-10, atol=1e-10)
        np.testing.assert_allclose(S, rS[0, h], rtol=1e-10, atol=1e-10)


def _hard_alpha(rng, B, T, H):
    """Gates far from 1: alpha ~ U(0.05, 1), a run of alpha = 0.2 over two whole
    64-token chunks, and alpha = 0 (a restart) at a few tokens, one a chunk start."""
    alpha = rng.uniform(0.05, 1.0, (B, T, H))
    alpha[:, 64:192] = 0.2
    for t in (5, 64 * 3, 64 * 3 + 40):
        if t < T:
            alpha[:, t] = 0.0
    return alpha


def test_ratio_chunk_form_with_gates_far_from_one():
    q, k, v, beta, r, _, d0, S0, eta = _case(8, T=300)
    alpha = _hard_alpha(np.random.default_rng(8), *k.shape[:3])
    ro, rS, rd = oracle.fwd(q, k, v, beta, r, d0, S0, eta=eta, alpha=alpha)
    for h in range(k.shape[2]):
        D, _ = chunked_scan(k[0, :, h], beta[0, :, h], r[0, :, h], d0[0, h], eta, 64)
        out, S = chunked_gated_delta_ratio(q[0, :, h], k[0, :, h], D * k[0, :, h], v[0, :, h], beta[0, :, h],
                                           alpha[0, :, h], S0[0, h], 64)
        np.testing.assert_allclose(out, ro[0, :, h], rtol=1e-9, atol=1e-9)
        np.testing.assert_allclose(S, rS[0, h], rtol=1e-9, atol=1e-9)


def test_decode_steps_equal_the_forward():
    q, k, v, beta, r, alpha, d0, S0, eta = _case(5, T=12)
    ro, rS, rd = oracle.fwd(q, k, v, beta, r, d0, S0, eta=eta, alpha=alpha)
    S, d = S0.copy(), d0.copy()
    for t in range(q.shape[1]):
        o = oracle.step(q[:, t], k[:, t], v[:, t], beta[:, t], S, d, r=r[:, t], eta=eta, alpha=alpha[:, t])
        np.testing.assert_allclose(o, ro[:, t], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, rS, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(d, rd, rtol=1e-12, atol=1e-12)


def _gated_inputs(dtype, B, H, T, dk, dv, eta, lo, seed):
    w = W.Workload("gated", B, H, T, dk, dv, 64, dtype, True, "gaussian", d0="uniform", S0="normal", eta=eta,
                   seed=seed)
    inp = W.make_forward_inputs(w)
    g = torch.Generator().manual_seed(seed + 7)
    alpha = (lo + (1 - lo) * torch.rand((B, T, H), generator=g)).to(inp["k"].dtype)
    return w, inp, alpha


GATED_CASES = [
    # B, H, T, eta, lowest alpha
    (2, 3, 200, 1e-2, 0.9),
    (1, 2, 130, 1.0, 0.5),
    (2, 2, 64, 0.0, 0.8),
    (1, 3, 1, 1e-2, 0.9),
    (2, 3, 300, 1e-2, 0.05),
    (1, 2, 129, 0.5, 0.0),
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", GATED_CASES, ids=lambda c: "B%dH%dT%d-eta%g-alpha%g" % c)
def test_gpu_gated_forward_matches_oracle(case):
    import preconditioned_delta_rule_token_b200 as pk
    B, H, T, eta, lo = case
    w, inp, alpha = _gated_inputs(W.BF16, B, H, T, 128, 128, eta, lo, seed=51)
    dev = lambda x: None if x is None else x.cuda()
    out, S, d = pk.forward(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["beta"]), dev(inp["r"]),
                           dev(inp["d0"]), dev(inp["S0"]), eta=eta, alpha=dev(alpha))
    assert pk.osdn_sync_status() == 0
    f = W.to_f64
    ro, rS, rd = oracle.fwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["beta"]), f(inp["r"]), f(inp["d0"]),
                            f(inp["S0"]), eta=eta, alpha=f(alpha))
    assert slice_rel_err(out.float().cpu().numpy(), ro, (0, 2)) <= BF16_TOL
    assert slice_rel_err(S.cpu().numpy(), rS, (0, 1)) <= BF16_TOL
    assert slice_rel_err(d.cpu().numpy(), rd, (0, 1)) <= BF16_TOL


@pytest.mark.gpu
def test_gpu_gated_forward_with_gates_far_from_one():
    """alpha ~ U(0.05, 1) with a run of alpha = 0.2 over two whole chunks and alpha = 0
    restarts (one at a chunk start): the decay accumulated in a chunk falls far below
    the fp32 range, and the kernel's ratios gamma_t / gamma_j stay in it."""
    import preconditioned_delta_rule_token_b200 as pk
    w, inp, _ = _gated_inputs(W.BF16, 2, 3, 300, 128, 128, 1e-2, 0.5, seed=56)
    alpha = torch.from_numpy(_hard_alpha(np.random.default_rng(56), 2, 300, 3)).to(torch.bfloat16)
    dev = lambda x: None if x is None else x.cuda()
    out, S, d = pk.forward(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["beta"]), dev(inp["r"]),
                           dev(inp["d0"]), dev(inp["S0"]), eta=w.eta, alpha=dev(alpha))
    assert pk.osdn_sync_status() == 0
    f = W.to_f64
    ro, rS, rd = oracle.fwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["beta"]), f(inp["r"]), f(inp["d0"]),
                            f(inp["S0"]), eta=w.eta, alpha=f(alpha))
    assert np.all(np.isfinite(out.float().cpu().numpy()))
    assert slice_rel_err(out.float().cpu().numpy(), ro, (0, 2)) <= BF16_TOL
    assert slice_rel_err(S.cpu().numpy(), rS, (0, 1)) <= BF16_TOL
    assert slice_rel_err(d.cpu().numpy(), rd, (0, 1)) <= BF16_TOL


@pytest.mark.gpu
def test_gpu_gated_with_unit_alpha_is_ungated():
    import preconditioned_delta_rule_token_b200 as pk
    w, inp, alpha = _gated_inputs(W.BF16, 2, 2, 150, 128, 128, 1e-2, 1.0, seed=52)
    dev = lambda x: None if x is None else x.cuda()
    args = (dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["beta"]), dev(inp["r"]), dev(inp["d0"]),
            dev(inp["S0"]))
    g = pk.forward(*args, eta=w.eta, alpha=dev(torch.ones_like(alpha)))
    p = pk.forward(*args, eta=w.eta)
    assert pk.osdn_sync_status() == 0
    for x, y in zip(g, p):
        torch.testing.assert_close(x.float(), y.float(), rtol=1e-6, atol=1e-6)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [W.FP32, W.BF16])
def test_gpu_gated_decode_matches_oracle(dtype):
    import preconditioned_delta_rule_token_b200 as pk
    w, inp, alpha = _gated_inputs(dtype, 2, 3, 24, 128, 128, 0.5, 0.7, seed=53)
    dev = lambda x: None if x is None else x.cuda()
    S, d = dev(inp["S0"]).clone(), dev(inp["d0"]).clone()
    outs = []
    for t in range(w.T):
        tok = {n: dev(inp[n][:, t].contiguous()) for n in ("q", "k", "v", "beta", "r")}
        outs.append(pk.step(tok["q"], tok["k"], tok["v"], tok["beta"], S, d, r=tok["r"], eta=w.eta,
                            alpha=dev(alpha[:, t].contiguous())))
    assert pk.osdn_sync_status() == 0
    f = W.to_f64
    ro, rS, rd = oracle.fwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["beta"]), f(inp["r"]), f(inp["d0"]),
                            f(inp["S0"]), eta=w.eta, alpha=f(alpha))
    from tests._util import FP32_TOL
    tol = BF16_TOL if dtype == W.BF16 else FP32_TOL
    out = torch.stack(outs, 1).float().cpu().numpy()
    assert slice_rel_err(out, ro, (0, 2)) <= tol
    assert slice_rel_err(S.cpu().numpy(), rS, (0, 1)) <= tol
    assert slice_rel_err(d.cpu().numpy(), rd, (0, 1)) <= tol


@pytest.mark.gpu
def test_gpu_gated_forward_unsupported_shapes_are_refused():
    import preconditioned_delta_rule_token_b200 as pk
    for dtype, dk in ((W.FP32, 128), (W.BF16, 64)):
        w, inp, alpha = _gated_inputs(dtype, 1, 1, 70, dk, dk, 1e-2, 0.9, seed=54)
        dev = lambda x: None if x is None else x.cuda()
        with pytest.raises(pk.OsdnError) as e:
            pk.forward(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["beta"]), dev(inp["r"]), None, None,
                       eta=w.eta, alpha=dev(alpha))
        assert e.value.code == pk.OSDN_ERR_UNSUPPORTED


@pytest.mark.gpu
@pytest.mark.parametrize("lo", [0.9, 0.05])
def test_gpu_gated_full_size_layer_every_unit(lo):
    """The 1.3B-shaped layer (B8 H16 T4096) with alpha ~ U(lo, 1), every unit compared
    with the oracle."""
    import preconditioned_delta_rule_token_b200 as pk
    w = W.LAYER_1P3B
    inp = W.make_forward_inputs(w)
    alpha = (lo + (1 - lo) * torch.rand((w.B, w.T, w.H), generator=torch.Generator().manual_seed(55))).to(
        torch.bfloat16)
    dev = lambda x: None if x is None else x.cuda()
    out, S, d = pk.forward(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["beta"]), dev(inp["r"]), None, None,
                           eta=w.eta, alpha=dev(alpha))
    assert pk.osdn_sync_status() == 0
    f = W.to_f64
    ro, rS, rd = oracle.fwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["beta"]), f(inp["r"]), None, None,
                            eta=w.eta, alpha=f(alpha))
    assert slice_rel_err(out.float().cpu().numpy(), ro, (0, 2)) <= BF16_TOL
    assert slice_rel_err(S.cpu().numpy(), rS, (0, 1)) <= BF16_TOL
    assert slice_rel_err(d.cpu().numpy(), rd, (0, 1)) <= BF16_TOL
