"""Pins for the CPU oracle: each test checks the oracle against something the
pages or the mathematics fix, not against a retyped copy of its own formula.

Source: "OSDN: Improving Delta Rule with Provable Online Preconditioning in
Linear Attention" (gist.science technical summary: section 1 loss and DeltaNet
rule; section 2.1 right preconditioning and the scaled write key; section 2.2
hypergradient surrogate and closed form; section 2.3 APF; section 3 Theorem 5.2
gated Newton condition), and the textbook DeltaNet rule as restated, transposed,
in eq. (3) of "Erase-then-Delta Attention" (bittide digest, section 2.2).
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_case(seed, B=2, T=12, H=2, dk=5, dv=3, apf=True, eta=0.3, d0_uniform=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    r = rng.uniform(0.5, 1.0, (B, T, H)) if apf else None
    d0 = rng.uniform(0.5, 1.5, (B, H, dk)) if d0_uniform else np.ones((B, H, dk))
    S0 = 0.3 * rng.standard_normal((B, H, dv, dk))
    return dict(q=q, k=k, v=v, beta=beta, r=r, d0=d0, S0=S0, eta=eta)


def _definition_reference(c):
    """Token loop built from the definitions only, in float64 with autograd:
    f_t(S) = 1/2 ||S k_t - v_t||^2 (section 1); its gradient by autograd;
    S_t(d) = S_{t-1} - beta_t grad f_t(S_{t-1}) diag(d) (section 2.1, explicit
    right-preconditioned form with a dense diagonal matrix);
    h_t(d) = (f_t(S_t(d)) - f_t(S_{t-1})) / ||grad f_t(S_{t-1})||_F^2 (section
    2.2, the definition, not its closed form); d_{t+1} = r_t d_t - eta grad_d
    h_t(d_t) (section 2.3, read as a descent step); o_t = S_t q_t."""
    q, k, v, beta, r, d0, S0, eta = (c[n] for n in ("q", "k", "v", "beta", "r", "d0", "S0", "eta"))
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    out = np.zeros((B, T, H, dv))
    Sf = np.zeros((B, H, dv, dk))
    df = np.zeros((B, H, dk))
    for b in range(B):
        for h in range(H):
            S = torch.tensor(S0[b, h], dtype=torch.float64)
            d = torch.tensor(d0[b, h], dtype=torch.float64)
            for t in range(T):
                kt = torch.tensor(k[b, t, h], dtype=torch.float64)
                vt = torch.tensor(v[b, t, h], dtype=torch.float64)
                qt = torch.tensor(q[b, t, h], dtype=torch.float64)
                bt = float(beta[b, t, h])
                rt = 1.0 if r is None else float(r[b, t, h])

                def f(Sx):
                    res = Sx @ kt - vt
                    return 0.5 * (res * res).sum()

                Sg = S.clone().requires_grad_(True)
                (G,) = torch.autograd.grad(f(Sg), Sg)          # grad f_t(S_{t-1})
                G = G.detach()
                f_prev = f(S).detach()
                gnorm2 = (G * G).sum()

                def S_next(dx):
                    return S - bt * (G @ torch.diag(dx))

                dg = d.clone().requires_grad_(True)
                hval = (f(S_next(dg)) - f_prev) / gnorm2
                (gh,) = torch.autograd.grad(hval, dg)
                S = S_next(d).detach()
                out[b, t, h] = (S @ qt).numpy()
                d = (rt * d - eta * gh).detach()
            Sf[b, h] = S.numpy()
            df[b, h] = d.numpy()
    return out, Sf, df


@pytest.mark.parametrize("apf", [True, False])
def test_oracle_matches_definitions_with_autograd(apf):
    c = _rand_case(1 + int(apf), apf=apf)
    ref = _definition_reference(c)
    got = oracle.fwd(c["q"], c["k"], c["v"], c["beta"], c["r"], c["d0"], c["S0"], eta=c["eta"])
    for a, b in zip(got, ref):
        np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)


def test_hypergradient_closed_form_follows_from_definition():
    """Section 2.2: the surrogate built from f equals ((1 - beta<d,k^2>)^2 - 1) / (2||k||^2)
    for any S and v (the decoupling from S, v and the residual)."""
    rng = np.random.default_rng(7)
    for _ in range(20):
        dk, dv = 6, 4
        k = rng.standard_normal(dk)
        v = rng.standard_normal(dv)
        S = rng.standard_normal((dv, dk))
        d = rng.uniform(0.2, 2.0, dk)
        beta = rng.uniform(0.05, 1.5)
        e = S @ k - v
        G = np.outer(e, k)
        S1 = S - beta * G @ np.diag(d)
        f0 = 0.5 * np.sum((S @ k - v) ** 2)
        f1 = 0.5 * np.sum((S1 @ k - v) ** 2)
        h_def = (f1 - f0) / np.sum(G * G)
        s = np.dot(d, k * k)
        h_closed = ((1 - beta * s) ** 2 - 1) / (2 * np.dot(k, k))
        assert abs(h_def - h_closed) < 1e-12 * max(1.0, abs(h_closed))


def test_reduces_to_deltanet_in_transposed_convention():
    """d == 1, eta = 0, no APF: the update is textbook DeltaNet, written here as
    S'_t = (I - beta k k^T) S'_{t-1} + beta k v^T with S' = S^T (dk x dv) and
    o_t = S'_t^T q_t (eq. (3) of the erase-then-delta digest)."""
    c = _rand_case(3, apf=False, eta=0.0, d0_uniform=False)
    B, T, H, dk = c["k"].shape
    out, Sf, df = oracle.fwd(c["q"], c["k"], c["v"], c["beta"], None, c["d0"], c["S0"], eta=0.0)
    for b in range(B):
        for h in range(H):
            Sp = c["S0"][b, h].T.copy()
            for t in range(T):
                kt, vt, qt, bt = c["k"][b, t, h], c["v"][b, t, h], c["q"][b, t, h], c["beta"][b, t, h]
                Sp = (np.eye(dk) - bt * np.outer(kt, kt)) @ Sp + bt * np.outer(kt, vt)
                np.testing.assert_allclose(out[b, t, h], Sp.T @ qt, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(Sf[b, h], Sp.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(df, np.ones_like(df))


def test_exact_recall_with_orthonormal_keys():
    """beta = 1, d == 1, orthonormal keys: every written pair is recalled exactly, S_T k_i = v_i."""
    rng = np.random.default_rng(4)
    dk, dv = 8, 5
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm.T                                     # rows orthonormal
    vals = rng.standard_normal((dk, dv))
    k = keys[None, :, None, :]
    v = vals[None, :, None, :]
    q = k.copy()
    beta = np.ones((1, dk, 1))
    S0 = rng.standard_normal((1, 1, dv, dk))        # any prior memory is overwritten
    _, Sf, _ = oracle.fwd(q, k, v, beta, None, None, S0, eta=0.0)
    np.testing.assert_allclose(Sf[0, 0] @ keys.T, vals.T, atol=1e-12)


def test_gated_newton_step_writes_exactly():
    """Theorem 5.2's gated Newton condition beta_t <d_t, k_t^2> = 1 makes the
    written pair exact: S_t k_t = v_t, for any preconditioner d_t."""
    rng = np.random.default_rng(5)
    B, H, dk, dv = 1, 3, 7, 4
    S = np.ascontiguousarray(rng.standard_normal((B, H, dv, dk)))
    d = np.ascontiguousarray(rng.uniform(0.5, 1.5, (B, H, dk)))
    for t in range(25):
        k = rng.standard_normal((B, H, dk))
        v = rng.standard_normal((B, H, dv))
        q = rng.standard_normal((B, H, dk))
        beta = 1.0 / np.einsum("bhi,bhi->bh", d, k * k)
        r = rng.uniform(0.8, 1.0, (B, H))
        oracle.step(q, k, v, beta, S, d, r=r, eta=0.4)
        np.testing.assert_allclose(np.einsum("bhvi,bhi->bhv", S, k), v, atol=1e-11)


def test_residual_ratio_invariant():
    """From sections 2.1-2.2: f_t(S_t) / f_t(S_{t-1}) = (1 - beta_t <d_t, k_t^2>)^2 exactly."""
    rng = np.random.default_rng(6)
    B, H, dk, dv = 2, 2, 6, 5
    S = np.ascontiguousarray(rng.standard_normal((B, H, dv, dk)))
    d = np.ascontiguousarray(rng.uniform(0.5, 1.5, (B, H, dk)))
    for t in range(30):
        k = rng.standard_normal((B, H, dk))
        v = rng.standard_normal((B, H, dv))
        q = rng.standard_normal((B, H, dk))
        beta = rng.uniform(0.05, 0.95, (B, H))
        s = np.einsum("bhi,bhi->bh", d, k * k)
        f0 = 0.5 * np.sum((np.einsum("bhvi,bhi->bhv", S, k) - v) ** 2, axis=-1)
        oracle.step(q, k, v, beta, S, d, r=None, eta=0.2)
        f1 = 0.5 * np.sum((np.einsum("bhvi,bhi->bhv", S, k) - v) ** 2, axis=-1)
        np.testing.assert_allclose(f1 / f0, (1 - beta * s) ** 2, rtol=1e-9)


def test_preconditioner_is_decoupled_from_values_and_queries():
    """Section 2.2: the d-update depends only on keys, beta and r, so changing v
    or q leaves the final d bit-identical (and does change S)."""
    c = _rand_case(8)
    o1, S1, d1 = oracle.fwd(c["q"], c["k"], c["v"], c["beta"], c["r"], c["d0"], c["S0"], eta=c["eta"])
    rng = np.random.default_rng(9)
    o2, S2, d2 = oracle.fwd(rng.standard_normal(c["q"].shape), c["k"], rng.standard_normal(c["v"].shape),
                            c["beta"], c["r"], c["d0"], c["S0"], eta=c["eta"])
    np.testing.assert_array_equal(d1, d2)
    assert np.max(np.abs(S1 - S2)) > 1e-3


@pytest.mark.parametrize("beta", [0.9, 1.6])
def test_sign_of_preconditioner_step_drives_gated_newton(beta):
    """A repeated key with eta = 1, r = 1: descent on h drives beta <d_t, k^2> to 1
    monotonically, from below or from above (the gated Newton comparator of
    Theorem 5.2). The literal '+' sign of section 2.3 would push it away from 1,
    so this fixes the sign."""
    rng = np.random.default_rng(10)
    dk, dv = 8, 3
    k = rng.standard_normal(dk)
    k /= np.linalg.norm(k)
    S = np.zeros((1, 1, dv, dk))
    d = np.ones((1, 1, dk))
    prev = None
    for t in range(300):
        gap = abs(beta * float(np.dot(d[0, 0], k * k)) - 1.0)
        if prev is not None:
            assert gap <= prev + 1e-15
        prev = gap
        oracle.step(rng.standard_normal((1, 1, dk)), k[None, None], rng.standard_normal((1, 1, dv)),
                    np.array([[beta]]), S, d, r=None, eta=1.0)
    assert prev < 1e-8


def test_continuation_and_step_equal_one_forward():
    """Checkpoint/resume: fwd(T1) then fwd(T2) from its (S, d) equals fwd(T1 + T2);
    T single-token steps equal one forward."""
    c = _rand_case(11, T=17)
    full = oracle.fwd(c["q"], c["k"], c["v"], c["beta"], c["r"], c["d0"], c["S0"], eta=c["eta"])
    T1 = 6
    sl = lambda x, a, b: None if x is None else x[:, a:b]
    o1, S1, d1 = oracle.fwd(sl(c["q"], 0, T1), sl(c["k"], 0, T1), sl(c["v"], 0, T1), sl(c["beta"], 0, T1),
                            sl(c["r"], 0, T1), c["d0"], c["S0"], eta=c["eta"])
    o2, S2, d2 = oracle.fwd(sl(c["q"], T1, 17), sl(c["k"], T1, 17), sl(c["v"], T1, 17), sl(c["beta"], T1, 17),
                            sl(c["r"], T1, 17), d1, S1, eta=c["eta"])
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), full[0], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(S2, full[1], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(d2, full[2], rtol=1e-13, atol=1e-13)
    S = np.ascontiguousarray(c["S0"].copy())
    d = np.ascontiguousarray(c["d0"].copy())
    for t in range(17):
        o = oracle.step(c["q"][:, t], c["k"][:, t], c["v"][:, t], c["beta"][:, t], S, d, r=c["r"][:, t],
                        eta=c["eta"])
        np.testing.assert_allclose(o, full[0][:, t], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(S, full[1], rtol=1e-13, atol=1e-13)


def test_apf_with_unit_retention_equals_plain_osdn():
    c = _rand_case(12)
    a = oracle.fwd(c["q"], c["k"], c["v"], c["beta"], np.ones_like(c["beta"]), c["d0"], c["S0"], eta=c["eta"])
    b = oracle.fwd(c["q"], c["k"], c["v"], c["beta"], None, c["d0"], c["S0"], eta=c["eta"])
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_zero_key_skips_gradient_and_writes_nothing():
    """||k||^2 = 0: h is undefined (its closed form divides by ||k||^2); the
    reading is to skip the d step. The write term is zero anyway."""
    rng = np.random.default_rng(13)
    S = np.ascontiguousarray(rng.standard_normal((1, 1, 3, 4)))
    d = np.ascontiguousarray(rng.uniform(0.5, 1.5, (1, 1, 4)))
    S_prev, d_prev = S.copy(), d.copy()
    q = rng.standard_normal((1, 1, 4))
    o = oracle.step(q, np.zeros((1, 1, 4)), rng.standard_normal((1, 1, 3)), np.array([[0.7]]), S, d,
                    r=np.array([[0.9]]), eta=0.5)
    np.testing.assert_array_equal(S, S_prev)
    np.testing.assert_allclose(d, 0.9 * d_prev, rtol=0, atol=0)
    np.testing.assert_allclose(o[0, 0], S_prev[0, 0] @ q[0, 0], rtol=1e-14)


def test_hand_worked_example_exact():
    """Two tokens, dk = 2, dv = 1, worked by hand in exact rationals from the
    section 2.1 scaled-key update, o_t = S_t q_t and the section 2.2/2.3 step.
    Inputs and expected values live in tests/golden/hand_worked_two_tokens.json
    with the derivation; every number is a dyadic rational, so float64 is exact."""
    with open(os.path.join(GOLDEN, "hand_worked_two_tokens.json")) as fh:
        g = json.load(fh)
    F = lambda s: float(Fraction(s))
    arr = lambda x: np.array([[F(e) for e in row] for row in x])
    k = arr(g["k"])[None, :, None, :]
    q = arr(g["q"])[None, :, None, :]
    v = np.array([F(e) for e in g["v"]])[None, :, None, None]
    beta = np.array([F(e) for e in g["beta"]])[None, :, None]
    d0 = np.array([F(e) for e in g["d0"]])[None, None, :]
    out, Sf, df = oracle.fwd(q, k, v, beta, None, d0, None, eta=F(g["eta"]))
    np.testing.assert_array_equal(out[0, :, 0, 0], [F(e) for e in g["expected_out"]])
    np.testing.assert_array_equal(Sf[0, 0, 0], [F(e) for e in g["expected_S"][0]])
    np.testing.assert_array_equal(df[0, 0], [F(e) for e in g["expected_d"]])


def test_oracle_golden_regression():
    """The oracle's float64 outputs on a small seeded case, stored by
    tests/golden/make_oracle_golden.py (which calls only the oracle). Any
    change to the oracle's arithmetic shows up here."""
    from tests.golden.make_oracle_golden import CASE, compute
    with open(os.path.join(GOLDEN, "oracle_small_case.json")) as fh:
        stored = json.load(fh)
    got = compute()
    assert stored["case"] == CASE
    for key in ("out", "S", "d"):
        np.testing.assert_allclose(np.array(got[key]), np.array(stored[key]), rtol=1e-12, atol=1e-13)
