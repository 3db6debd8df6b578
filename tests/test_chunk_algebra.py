"""Design checks (CPU, float64): the chunk forms the CUDA kernels compute equal
the token-by-token recurrence of the oracle.

1. Chunk form of the preconditioner recurrence (the affine recurrence of the
   APF section): per block of L tokens with carry d_c,
     s_t = R_{t,0} <d_c, a_t> + sum_{j<t} R_{t,j+1} x_j <u_j, a_t>,
     x_t = g_t (1 - beta_t s_t)   (g_t = eta beta_t, u_t = k_t^2 / ||k_t||^2)
   i.e. (I + M) x = c with M_tj = g_t beta_t R_{t,j+1} <u_j, a_t> (j < t) and
   c_t = g_t (1 - beta_t R_{t,0} <d_c, a_t>); then
     d_t = R_{t,0} d_c + sum_{j<t} R_{t,j+1} x_j u_j,   d_{c+1} = d_L.
2. Chunkwise WY form of the delta rule with the scaled write key Kw = D (.) K:
     A = strict_tril(diag(beta) K Kw^T), U = (I + A)^{-1} diag(beta) (V - K S^T),
     O = Q S^T + tril(Q Kw^T) U, S <- S + U^T Kw.
Both are checked against the oracle for several block sizes and ragged T.
"""
import numpy as np
import pytest

import oracle


def _case(seed, B=1, T=150, H=2, dk=16, dv=8, eta=0.5, apf=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    k[0, 5, 0] = 0.0                                   # a zero key
    v = rng.standard_normal((B, T, H, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, T, H))))
    r = rng.uniform(0.6, 1.0, (B, T, H)) if apf else None
    d0 = rng.uniform(0.5, 1.5, (B, H, dk))
    S0 = 0.3 * rng.standard_normal((B, H, dv, dk))
    return q, k, v, beta, r, d0, S0, eta


def chunked_scan(k, beta, r, d0, eta, L):
    """Preconditioner for every token of one unit by the chunk form. k: [T, dk]."""
    T, dk = k.shape
    r = np.ones(T) if r is None else r
    d = d0.copy()
    D = np.zeros((T, dk))
    for c0 in range(0, T, L):
        kk = k[c0:c0 + L]
        n = len(kk)
        a = kk * kk
        nrm = a.sum(1)
        ok = nrm > 0
        u = np.where(ok[:, None], a / np.where(ok, nrm, 1)[:, None], 0.0)
        g = np.where(ok, eta * beta[c0:c0 + n], 0.0)
        be = beta[c0:c0 + n]
        rr = r[c0:c0 + n]
        R = np.ones((n + 1, n + 1))                    # R[t, j] = prod_{m=j}^{t-1} r_m (t >= j)
        for t in range(n + 1):
            for j in range(t):
                R[t, j] = np.prod(rr[j:t])
        G = a @ u.T                                    # G[t, j] = <a_t, u_j>
        M = np.zeros((n, n))
        for t in range(n):
            for j in range(t):
                M[t, j] = g[t] * be[t] * R[t, j + 1] * G[t, j]
        c = g * (1 - be * R[np.arange(n), 0] * (a @ d))
        x = np.linalg.solve(np.eye(n) + M, c)
        for t in range(n):
            D[c0 + t] = R[t, 0] * d + sum(R[t, j + 1] * x[j] * u[j] for j in range(t))
        d = R[n, 0] * d + sum(R[n, j + 1] * x[j] * u[j] for j in range(n))
    return D, d


def chunked_delta(q, k, kw, v, beta, S0, C):
    """Chunkwise WY form for one unit: q, k, kw [T, dk], v [T, dv], S0 [dv, dk]."""
    T = k.shape[0]
    S = S0.copy()
    out = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        Q, K, Kw, V, b = q[c0:c0 + C], k[c0:c0 + C], kw[c0:c0 + C], v[c0:c0 + C], beta[c0:c0 + C]
        n = len(K)
        A = np.tril(b[:, None] * (K @ Kw.T), -1)
        U = np.linalg.solve(np.eye(n) + A, b[:, None] * (V - K @ S.T))
        out[c0:c0 + n] = Q @ S.T + np.tril(Q @ Kw.T) @ U
        S = S + U.T @ Kw
    return out, S


@pytest.mark.parametrize("L", [16, 64, 128])
@pytest.mark.parametrize("apf", [True, False])
def test_chunk_forms_equal_the_recurrence(L, apf):
    q, k, v, beta, r, d0, S0, eta = _case(20 + L, apf=apf)
    ro, rS, rd = oracle.fwd(q, k, v, beta, r, d0, S0, eta=eta)
    B, T, H, dk = k.shape
    for h in range(H):
        D, dT = chunked_scan(k[0, :, h], beta[0, :, h], None if r is None else r[0, :, h], d0[0, h], eta, L)
        np.testing.assert_allclose(dT, rd[0, h], rtol=1e-11, atol=1e-12)
        out, S = chunked_delta(q[0, :, h], k[0, :, h], D * k[0, :, h], v[0, :, h], beta[0, :, h], S0[0, h], 64)
        np.testing.assert_allclose(out, ro[0, :, h], rtol=1e-10, atol=1e-10)
        np.testing.assert_allclose(S, rS[0, h], rtol=1e-10, atol=1e-10)


def test_transposed_gram_is_wrong():
    """The Gram of the chunk form is diag(beta) K Kw^T (read key rows, write key
    columns); its transpose diag(beta) Kw K^T does not reproduce the recurrence
    once d varies per token."""
    q, k, v, beta, r, d0, S0, eta = _case(3)
    ro, rS, rd = oracle.fwd(q, k, v, beta, r, d0, S0, eta=eta)
    D, _ = chunked_scan(k[0, :, 0], beta[0, :, 0], r[0, :, 0], d0[0, 0], eta, 64)
    kw = D * k[0, :, 0]
    # swap the roles of K and Kw in the Gram only
    T = k.shape[1]
    S = S0[0, 0].copy()
    out = np.zeros((T, v.shape[-1]))
    for c0 in range(0, T, 64):
        K, Kw, V, Q, b = k[0, c0:c0 + 64, 0], kw[c0:c0 + 64], v[0, c0:c0 + 64, 0], q[0, c0:c0 + 64, 0], beta[0, c0:c0 + 64, 0]
        A = np.tril(b[:, None] * (Kw @ K.T), -1)
        U = np.linalg.solve(np.eye(len(K)) + A, b[:, None] * (V - K @ S.T))
        out[c0:c0 + len(K)] = Q @ S.T + np.tril(Q @ Kw.T) @ U
        S = S + U.T @ Kw
    assert np.max(np.abs(out - ro[0, :, 0])) > 1e-3
