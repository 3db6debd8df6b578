"""Design check (CPU, float64): the chunk form of the adjoint that the backward
kernels compute equals the oracle's token-by-token gradients.

The forward per chunk of C tokens with chunk-start state S ("OSDN: Improving Delta
Rule with Provable Online Preconditioning in Linear Attention", technical summary
section 2.1, the DeltaNet chunk pipeline with the scaled write key Kw = D (.) K):
    Kb = diag(beta) K,  A = strict_tril(Kb Kw^T),  T = (I + A)^{-1},  W = T Kb,
    U0 = T diag(beta) V,  Vn = U0 - W S^T,  P = tril(Q Kw^T),
    O = Q S^T + P Vn,  S' = S + Vn^T Kw.
Its reverse, chunk by chunk from the last with dS' = dL/dS':
    dVn = P^T dO + Kw dS'^T,        dS = dS' + dO^T Q - dVn^T W,
    dP = tril(dO Vn^T),             dQ = dO S + dP Kw,
    dW = -dVn S,                    dT = (dW K^T + dVn V^T) diag(beta),
    dA = -strict_tril(T^T dT T^T),  dAb = diag(beta) dA,
    dKw = Vn dS' + dP^T Q + dAb^T K,
    dV = diag(beta) T^T dVn,        dK = diag(beta) T^T dW + dAb Kw + dKw (.) D,
    dbeta = rowdot(T^T dW, K) + rowdot(T^T dVn, V) + rowsum(dA (.) K Kw^T),
    dD = dKw (.) K,
followed by the reverse of the APF recurrence token by token (section 2.3). This is
the algebra written at the top of csrc/bwd.cuh; here it is restated in numpy and
compared with oracle.bwd (itself pinned by finite differences).

The reverse of the APF recurrence also has a chunk form, the transposed counterpart
of the forward scan's: with Ld_j = dL/dd of token j of a block of L tokens,
Ld_L the adjoint entering from the next block, rho(i, j) = prod_{m=i}^{j-1} r_m,
a_j = k_j^2 and c2_j = -eta beta_j^2 / ||k_j||^2 (0 for a zero key), the unknowns
y_j = <a_j, Ld_{j+1}> solve the upper-triangular system
    y_j - sum_{i>j} rho(j+1, i) c2_i <a_j, a_i> y_i
        = rho(j+1, L) <a_j, Ld_L> + sum_{i>j} rho(j+1, i) <a_j, dD_i>,
after which Ld_{j} = rho(j, L) Ld_L + sum_{i>=j} rho(j, i) (dD_i + c2_i y_i a_i) for every j
(Ld_0 leaves the block). Only <a_j, Ld_L> and the last sum depend on the carried
Ld_L; the system's matrix and its inverse do not.
"""
import numpy as np
import pytest

import oracle


def _case(seed, T, dk=8, dv=6, apf=True):
    rng = np.random.default_rng(seed)
    c = dict(q=rng.standard_normal((1, T, 1, dk)), k=rng.standard_normal((1, T, 1, dk)),
             v=rng.standard_normal((1, T, 1, dv)), beta=rng.uniform(0.1, 0.9, (1, T, 1)),
             r=rng.uniform(0.8, 1.0, (1, T, 1)) if apf else None,
             d0=rng.uniform(0.5, 1.5, (1, 1, dk)), S0=0.3 * rng.standard_normal((1, 1, dv, dk)))
    c["k"] /= np.linalg.norm(c["k"], axis=-1, keepdims=True)
    if T > 5:
        c["k"][0, 5, 0] = 0.0                            # a zero key: the d step is skipped
    cot = dict(dout=rng.standard_normal((1, T, 1, dv)), dS_final=rng.standard_normal((1, 1, dv, dk)),
               dd_final=rng.standard_normal((1, 1, dk)))
    return c, cot


def _d_trajectory(k, beta, r, d0, eta, anchor):
    """d_t before each token's own update (the forward recurrence, written out)."""
    T, dk = k.shape
    D = np.zeros((T, dk))
    d = d0.copy()
    for t in range(T):
        D[t] = d
        a = k[t] ** 2
        n = a.sum()
        x = eta * beta[t] * (1 - beta[t] * (d @ a)) / n if n > 0 else 0.0
        d = r[t] * d + ((1 - r[t]) * d0 if anchor else 0.0) + x * a
    return D, d


def chunk_backward(q, k, v, beta, r, d0, S0, dout, dS_final, dd_final, eta, anchor, C, alpha=None,
                   dalpha_form="direct"):
    """Gradients of one (b, h) unit by the chunk-form adjoint. q, k: [T, dk]; v, dout: [T, dv].

    alpha [T] (gated OSDN, the state decayed by alpha_t before token t's write) takes the
    chunk form with every decay factor a ratio of the in-chunk cumulative gate gamma:
    R_tj = gamma_t / gamma_j, rho_j = gamma_C / gamma_j,
        A = strict_tril(Kb Kw^T (.) R), W = T diag(beta gamma) K, P = tril(Q Kw^T) (.) R,
        O = diag(gamma) Q S^T + P Vn, S' = gamma_C S + Vn^T diag(rho) Kw,
    and its reverse
        dVn = P^T dO + diag(rho) Kw dS'^T,  dS = gamma_C dS' + dO^T diag(gamma) Q - dVn^T W,
        dPr = tril(dO Vn^T) (.) R,  dQ = diag(gamma) dO S + dPr Kw,
        dW = -dVn S,  dT = dW (diag(beta gamma) K)^T + dVn (diag(beta) V)^T,
        dA = -strict_tril(T^T dT T^T),  dAr = dA (.) R,
        dKw = diag(rho) Vn dS' + dPr^T Q + dAr^T Kb,
        dK = diag(beta) dAr Kw + diag(beta gamma) T^T dW + dKw (.) D,
        dbeta = rowdot(dAr Kw, K) + gamma (.) rowdot(T^T dW, K) + rowdot(T^T dVn, V),
    with the adjoint of G = log gamma collected from every place gamma enters,
        dG_t = gamma_t <dO_t, (Q S^T)_t> + gamma_t beta_t <(T^T dW)_t, K_t> + sum_j X_tj - sum_j X_jt
               - Y_t + [t = last] (gamma_C <dS', S> + sum_j Y_j),
        X = (dA (.) Kb Kw^T + tril(dO Vn^T) (.) Q Kw^T) (.) R,  Y_j = rho_j <Vn_j, dS' Kw_j>,
    and dalpha_m = (sum_{t >= m} dG_t) / alpha_m (G_t is the sum of log alpha up to t): the
    "cumsum" form, which needs alpha > 0. The "direct" form (the CUDA kernel's) sums only the
    terms whose gate product holds alpha_m and divides alpha_m out in the exponent:
        dalpha_m = sum_{t >= m} a_t 2^(L_t - l_m) + sum_{j < m} y_j 2^(L_C - L_j - l_m)
                   + c 2^(L_C - l_m) + sum_{t >= m > j} X'_tj 2^(L_t - L_j - l_m),
    l = log2 alpha (clamped at -120, so alpha = 0 is allowed), L its in-chunk cumulative sum,
    a_t = <dO_t, (Q S^T)_t> + beta_t <(T^T dW)_t, K_t>, y_j = <Vn_j, dS' Kw_j>, c = <dS', S>,
    X' = X with R divided out. Gamma and every ratio are taken as 2^(differences of L).
    The "factorized" form (the kernel's) splits each exponent into two non-positive parts,
    L_t - L_j - l_m = (L_t - L_m) + (L_{m-1} - L_j), so the pair sums are one matrix product
    Y = X' W^T with W_mj = 2^(L_{m-1} - L_j) (j < m):
        dalpha_m = sum_{t >= m} 2^(L_t - L_m) (Y_tm + a_t 2^L_{m-1})
                   + 2^(L_C - L_m) (sum_{j < m} W_mj y_j + c 2^L_{m-1})."""
    T, dk = k.shape
    dv = v.shape[1]
    r = np.ones(T) if r is None else r
    gated = alpha is not None
    alpha = np.ones(T) if alpha is None else alpha
    D, _ = _d_trajectory(k, beta, r, d0, eta, anchor)
    Kw_all = D * k
    starts = list(range(0, T, C))
    # forward over the chunks: the state at every chunk start and the chunk matrices
    S = S0.copy()
    saved = []
    lg2 = np.maximum(np.log2(np.maximum(alpha, 1e-300)), -120.0)
    for c0 in starts:
        sl = slice(c0, min(T, c0 + C))
        K, Kw, Q, V, be = k[sl], Kw_all[sl], q[sl], v[sl], beta[sl]
        n = len(K)
        L = np.cumsum(lg2[sl])
        g = 2.0 ** L
        R = np.tril(2.0 ** np.minimum(L[:, None] - L[None, :], 0.0))
        rho = 2.0 ** (L[-1] - L)
        Kb = be[:, None] * K
        A = np.tril(Kb @ Kw.T, -1) * R
        Tm = np.linalg.inv(np.eye(n) + A)
        W = Tm @ (g[:, None] * Kb)
        U0 = Tm @ (be[:, None] * V)
        Vn = U0 - W @ S.T
        P = np.tril(Q @ Kw.T) * R
        saved.append((sl, S.copy(), Tm, W, Vn, P, g, R, rho, L))
        S = g[-1] * S + Vn.T @ (rho[:, None] * Kw)
    # reverse over the chunks
    dS = dS_final.copy()
    dq, dk_, dvv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dbeta, dD, dalpha = np.zeros(T), np.zeros((T, dk)), np.zeros(T)
    for sl, Sc, Tm, W, Vn, P, g, R, rho, L in reversed(saved):
        K, Kw, Q, V, be, dO, Dc = k[sl], Kw_all[sl], q[sl], v[sl], beta[sl], dout[sl], D[sl]
        Kb = be[:, None] * K
        dVn = P.T @ dO + (rho[:, None] * Kw) @ dS.T
        dS_prev = g[-1] * dS + dO.T @ (g[:, None] * Q) - dVn.T @ W
        dPm = np.tril(dO @ Vn.T)                  # adjoint of P
        dPr = dPm * R                             # adjoint of the unmasked Q Kw^T
        dq[sl] = g[:, None] * (dO @ Sc) + dPr @ Kw
        dW = -dVn @ Sc
        dT = dW @ (g[:, None] * Kb).T + dVn @ (be[:, None] * V).T
        dA = -np.tril(Tm.T @ dT @ Tm.T, -1)       # adjoint of A
        dAr = dA * R                              # adjoint of the unmasked Kb Kw^T
        dKw = rho[:, None] * (Vn @ dS) + dPr.T @ Q + dAr.T @ Kb
        TdW, TdVn = Tm.T @ dW, Tm.T @ dVn
        dvv[sl] = be[:, None] * TdVn
        dk_[sl] = be[:, None] * (dAr @ Kw) + (be * g)[:, None] * TdW + dKw * Dc
        dbeta[sl] = ((dAr @ Kw) * K).sum(1) + g * (TdW * K).sum(1) + (TdVn * V).sum(1)
        dD[sl] = dKw * K
        if gated and dalpha_form == "cumsum":
            # adjoint of G = log gamma, then of log alpha (reverse cumulative sum), then of alpha
            X = (dA * (Kb @ Kw.T) + dPm * (Q @ Kw.T)) * R
            Yr = rho * ((Vn @ dS) * Kw).sum(1)    # rho_j <Vn_j, dS' Kw_j>
            dG = g * (dO * (Q @ Sc.T)).sum(1) + g * be * (TdW * K).sum(1) + X.sum(1) - X.sum(0) - Yr
            dG[-1] += g[-1] * (dS * Sc).sum() + Yr.sum()
            dalpha[sl] = np.cumsum(dG[::-1])[::-1] / alpha[sl]
        elif gated and dalpha_form == "factorized":
            Xp = np.tril(dA * (Kb @ Kw.T) + dPm * (Q @ Kw.T), -1)
            a = (dO * (Q @ Sc.T)).sum(1) + be * (TdW * K).sum(1)
            y = ((Vn @ dS) * Kw).sum(1)
            cs = (dS * Sc).sum()
            n = len(L)
            Lm1 = np.concatenate([[0.0], L[:-1]])                 # L_{m-1}, with L_{-1} = 0
            Wf = np.tril(2.0 ** np.minimum(Lm1[:, None] - L[None, :], 0.0), -1)
            Y = Xp @ Wf.T
            da = np.zeros(n)
            for m in range(n):
                da[m] = ((2.0 ** (L[m:] - L[m]) * (Y[m:, m] + a[m:] * 2.0 ** Lm1[m])).sum()
                         + 2.0 ** (L[-1] - L[m]) * ((Wf[m, :m] * y[:m]).sum() + cs * 2.0 ** Lm1[m]))
            dalpha[sl] = da
        elif gated:
            Xp = np.tril(dA * (Kb @ Kw.T) + dPm * (Q @ Kw.T), -1)
            a = (dO * (Q @ Sc.T)).sum(1) + be * (TdW * K).sum(1)
            y = ((Vn @ dS) * Kw).sum(1)
            cs = (dS * Sc).sum()
            l = lg2[sl]
            da = np.zeros(len(l))
            for m in range(len(l)):
                da[m] = ((a[m:] * 2.0 ** (L[m:] - l[m])).sum() + (y[:m] * 2.0 ** (L[-1] - L[:m] - l[m])).sum()
                         + cs * 2.0 ** (L[-1] - l[m])
                         + (Xp[m:, :m] * 2.0 ** (L[m:, None] - L[None, :m] - l[m])).sum())
            dalpha[sl] = da
        dS = dS_prev
    # reverse of the preconditioner recurrence
    Ld = dd_final.copy()
    dr = np.zeros(T)
    dd_anchor = np.zeros(dk)
    anc = d0 if anchor else np.zeros(dk)
    for t in range(T - 1, -1, -1):
        a, d = k[t] ** 2, D[t]
        n, s = a.sum(), D[t] @ a
        dr[t] = (d - anc) @ Ld
        if anchor:
            dd_anchor += (1 - r[t]) * Ld
        ds = 0.0
        if n > 0:
            x = eta * beta[t] * (1 - beta[t] * s) / n
            dx = a @ Ld
            dbeta[t] += dx * eta * (1 - 2 * beta[t] * s) / n
            ds = -dx * eta * beta[t] ** 2 / n
            dk_[t] += 2 * k[t] * (x * Ld + ds * d - dx * x / n)
        Ld = r[t] * Ld + dD[t] + ds * a
    return dict(dq=dq, dk=dk_, dv=dvv, dbeta=dbeta, dr=dr, dd0=Ld + dd_anchor, dS0=dS, dalpha=dalpha)


@pytest.mark.parametrize("T,C,anchor,apf", [(150, 64, False, True), (150, 64, True, True), (64, 64, False, True),
                                             (97, 16, True, True), (130, 32, False, False)])
def test_chunk_adjoint_matches_the_token_gradients(T, C, anchor, apf):
    c, cot = _case(T + C, T, apf=apf)
    eta = 0.3
    ref = oracle.bwd(c["q"], c["k"], c["v"], c["beta"], cot["dout"], c["r"], c["d0"], c["S0"], cot["dS_final"],
                     cot["dd_final"], eta=eta, anchor=anchor)
    u = lambda x: None if x is None else x[0, :, 0]
    got = chunk_backward(u(c["q"]), u(c["k"]), u(c["v"]), u(c["beta"]), u(c["r"]), c["d0"][0, 0], c["S0"][0, 0],
                         u(cot["dout"]), cot["dS_final"][0, 0], cot["dd_final"][0, 0], eta, anchor, C)
    pairs = [("dq", u(ref["dq"])), ("dk", u(ref["dk"])), ("dv", u(ref["dv"])), ("dbeta", u(ref["dbeta"])),
             ("dd0", ref["dd0"][0, 0]), ("dS0", ref["dS0"][0, 0])]
    if apf:
        pairs.append(("dr", u(ref["dr"])))
    for name, want in pairs:
        np.testing.assert_allclose(got[name], want, rtol=1e-9, atol=1e-10 * max(1.0, np.abs(want).max()),
                                   err_msg=name)


@pytest.mark.parametrize("T,C,anchor,lo", [(150, 64, False, 0.85), (150, 64, True, 0.3), (97, 16, False, 0.05),
                                            (64, 64, True, 0.6)])
def test_gated_chunk_adjoint_matches_the_token_gradients(T, C, anchor, lo):
    """Gated OSDN: the chunk-form adjoint above, with the decay as ratios of the in-chunk
    cumulative gate, equals the oracle's token-by-token gradients (dalpha included), for
    gates down to 0.05 and a run of small gates over a whole chunk."""
    c, cot = _case(T + C + 1, T)
    rng = np.random.default_rng(T * 3 + C)
    alpha = rng.uniform(lo, 1.0, (1, T, 1))
    alpha[0, C:min(T, 2 * C), 0] = max(lo, 0.2)
    eta = 0.3
    ref = oracle.bwd(c["q"], c["k"], c["v"], c["beta"], cot["dout"], c["r"], c["d0"], c["S0"], cot["dS_final"],
                     cot["dd_final"], eta=eta, anchor=anchor, alpha=alpha)
    u = lambda x: None if x is None else x[0, :, 0]
    got = chunk_backward(u(c["q"]), u(c["k"]), u(c["v"]), u(c["beta"]), u(c["r"]), c["d0"][0, 0], c["S0"][0, 0],
                         u(cot["dout"]), cot["dS_final"][0, 0], cot["dd_final"][0, 0], eta, anchor, C,
                         alpha=u(alpha))
    for name in ("dq", "dk", "dv", "dbeta", "dr", "dalpha"):
        want = u(ref[name])
        np.testing.assert_allclose(got[name], want, rtol=1e-8, atol=1e-9 * max(1.0, np.abs(want).max()),
                                   err_msg=name)
    for name in ("dd0", "dS0"):
        want = ref[name][0, 0]
        np.testing.assert_allclose(got[name], want, rtol=1e-8, atol=1e-9 * max(1.0, np.abs(want).max()),
                                   err_msg=name)
    got_c = chunk_backward(u(c["q"]), u(c["k"]), u(c["v"]), u(c["beta"]), u(c["r"]), c["d0"][0, 0], c["S0"][0, 0],
                           u(cot["dout"]), cot["dS_final"][0, 0], cot["dd_final"][0, 0], eta, anchor, C,
                           alpha=u(alpha), dalpha_form="cumsum")
    want = u(ref["dalpha"])
    np.testing.assert_allclose(got_c["dalpha"], want, rtol=1e-7, atol=1e-8 * max(1.0, np.abs(want).max()))


@pytest.mark.parametrize("T,C", [(150, 64), (97, 16)])
def test_gated_chunk_adjoint_with_zero_gates(T, C):
    """alpha = 0 at a chunk start, inside a chunk, twice in one chunk, and gates of 1e-6 and
    1e-30: the direct form of dalpha (no division by alpha) equals the oracle's gradients,
    every element at rtol 1e-7, where the reverse cumulative sum over 1 / alpha is undefined
    or cancels."""
    c, cot = _case(T + 2 * C, T)
    rng = np.random.default_rng(T + 5 * C)
    alpha = rng.uniform(0.3, 1.0, (1, T, 1))
    for t, val in ((0, 0.0), (C, 0.0), (C + 5, 0.0), (C + 9, 0.0), (3, 1e-6), (2 * C + 7, 1e-30), (T - 1, 0.0)):
        if t < T:
            alpha[0, t, 0] = val
    eta = 0.3
    ref = oracle.bwd(c["q"], c["k"], c["v"], c["beta"], cot["dout"], c["r"], c["d0"], c["S0"], cot["dS_final"],
                     cot["dd_final"], eta=eta, anchor=False, alpha=alpha)
    u = lambda x: None if x is None else x[0, :, 0]
    got = chunk_backward(u(c["q"]), u(c["k"]), u(c["v"]), u(c["beta"]), u(c["r"]), c["d0"][0, 0], c["S0"][0, 0],
                         u(cot["dout"]), cot["dS_final"][0, 0], cot["dd_final"][0, 0], eta, False, C,
                         alpha=u(alpha))
    for name in ("dq", "dk", "dv", "dbeta", "dr", "dalpha"):
        want = u(ref[name])
        np.testing.assert_allclose(got[name], want, rtol=1e-7, atol=1e-9 * max(1.0, np.abs(want).max()),
                                   err_msg=name)
    assert np.all(np.isfinite(got["dalpha"]))
    got_f = chunk_backward(u(c["q"]), u(c["k"]), u(c["v"]), u(c["beta"]), u(c["r"]), c["d0"][0, 0], c["S0"][0, 0],
                           u(cot["dout"]), cot["dS_final"][0, 0], cot["dd_final"][0, 0], eta, False, C,
                           alpha=u(alpha), dalpha_form="factorized")
    want = u(ref["dalpha"])
    np.testing.assert_allclose(got_f["dalpha"], want, rtol=1e-7, atol=1e-9 * max(1.0, np.abs(want).max()))


def chunk_dchain(k, beta, r, dD, dd_final, eta, L):
    """Ld_{t+1} for every token (the adjoint of d entering token t from later tokens)
    and Ld_0, by the chunk form above. k, dD: [T, dk]."""
    T, dk = k.shape
    a_all = k * k
    nrm = a_all.sum(1)
    c2 = np.where(nrm > 0, -eta * beta ** 2 / np.where(nrm > 0, nrm, 1.0), 0.0)
    Ld = dd_final.copy()
    L_next = np.zeros((T, dk))                     # Ld_{t+1} for token t
    for c0 in reversed(range(0, T, L)):
        n = min(L, T - c0)
        a, rr, cc, dDc = a_all[c0:c0 + n], r[c0:c0 + n], c2[c0:c0 + n], dD[c0:c0 + n]
        rho = np.ones((n + 1, n + 1))              # rho[i, j] = prod_{m=i}^{j-1} r_m (i <= j)
        for i in range(n + 1):
            for j in range(i + 1, n + 1):
                rho[i, j] = rho[i, j - 1] * rr[j - 1]
        G, E = a @ a.T, a @ dDc.T                  # <a_j, a_i>, <a_j, dD_i>
        U = np.zeros((n, n))
        bvec = np.zeros(n)
        for j in range(n):
            bvec[j] = rho[j + 1, n] * (a[j] @ Ld)
            for i in range(j + 1, n):
                U[j, i] = rho[j + 1, i] * cc[i] * G[j, i]
                bvec[j] += rho[j + 1, i] * E[j, i]
        y = np.linalg.solve(np.eye(n) - U, bvec)
        w = dDc + (cc * y)[:, None] * a            # dD_i + c2_i y_i a_i
        for j in range(n):                         # Ld_{j+1} for every token of the block
            L_next[c0 + j] = rho[j + 1, n] * Ld + sum(rho[j + 1, i] * w[i] for i in range(j + 1, n))
        Ld = rho[0, n] * Ld + sum(rho[0, i] * w[i] for i in range(n))
    return L_next, Ld


@pytest.mark.parametrize("T,L", [(150, 64), (97, 16), (64, 64), (5, 8)])
def test_chunk_form_of_the_reverse_preconditioner_recurrence(T, L):
    # the token-serial reverse, written out, against the chunk form above
    rng = np.random.default_rng(T * 7 + L)
    dk = 8
    k = rng.standard_normal((T, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    if T > 3:
        k[3] = 0.0
    beta, r = rng.uniform(0.1, 0.9, T), rng.uniform(0.8, 1.0, T)
    dD, dd_final, eta = rng.standard_normal((T, dk)), rng.standard_normal(dk), 0.3
    Ld = dd_final.copy()
    want = np.zeros((T, dk))
    for t in range(T - 1, -1, -1):
        want[t] = Ld
        a, n = k[t] ** 2, (k[t] ** 2).sum()
        ds = -(a @ Ld) * eta * beta[t] ** 2 / n if n > 0 else 0.0
        Ld = r[t] * Ld + dD[t] + ds * a
    got, got0 = chunk_dchain(k, beta, r, dD, dd_final, eta, L)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(got0, Ld, rtol=1e-10, atol=1e-12)
