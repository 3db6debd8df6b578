"""Pins for the oracle's backward (reverse-mode gradients of the OSDN recurrence).

The pages give no backward pass; the oracle's backward is the plain derivative of
the token recurrence of "OSDN: Improving Delta Rule with Provable Online
Preconditioning in Linear Attention" (gist.science technical summary, sections
2.1 write with the scaled key, 2.3 APF step), plus the gated and anchored options.
It is pinned here against things that do not share its adjoint formulas:
  * central finite differences of the (separately pinned) oracle forward;
  * exact linearity: (o, S_T) are jointly linear in (v, S0), and o is linear in q,
    so sum(v dv) + <S0, dS0> and sum(q dq) equal the loss they differentiate;
  * reverse-mode autograd of a token loop built from the definitions in torch.
"""
import numpy as np
import pytest
import torch

import oracle


def _case(seed, B=1, T=9, H=2, dk=3, dv=2, apf=True, gated=False, zero_key=True):
    rng = np.random.default_rng(seed)
    c = dict(q=rng.standard_normal((B, T, H, dk)), k=rng.standard_normal((B, T, H, dk)),
             v=rng.standard_normal((B, T, H, dv)), beta=rng.uniform(0.1, 0.9, (B, T, H)),
             r=rng.uniform(0.8, 1.0, (B, T, H)) if apf else None,
             alpha=rng.uniform(0.7, 1.0, (B, T, H)) if gated else None,
             d0=rng.uniform(0.5, 1.5, (B, H, dk)), S0=rng.standard_normal((B, H, dv, dk)))
    if zero_key and T > 3:
        c["k"][0, 3, H - 1] = 0.0          # ||k|| = 0: the d step is skipped there
    seeds = np.random.default_rng(seed + 1)
    cot = dict(dout=seeds.standard_normal((B, T, H, dv)), dS_final=seeds.standard_normal((B, H, dv, dk)),
               dd_final=seeds.standard_normal((B, H, dk)))
    return c, cot


def _loss(c, cot, eta, anchor):
    out, S, d = oracle.fwd(c["q"], c["k"], c["v"], c["beta"], c["r"], c["d0"], c["S0"], eta=eta,
                           anchor=anchor, alpha=c["alpha"], nthreads=1)
    return float((out * cot["dout"]).sum() + (S * cot["dS_final"]).sum() + (d * cot["dd_final"]).sum())


_GRAD = {"q": "dq", "k": "dk", "v": "dv", "beta": "dbeta", "r": "dr", "alpha": "dalpha", "d0": "dd0", "S0": "dS0"}


def _fd_check(c, cot, eta, anchor, n_samples=None, seed=0, tol=1e-6):
    g = oracle.bwd(c["q"], c["k"], c["v"], c["beta"], cot["dout"], c["r"], c["d0"], c["S0"],
                   cot["dS_final"], cot["dd_final"], eta=eta, anchor=anchor, alpha=c["alpha"], nthreads=1)
    rng = np.random.default_rng(seed)
    H = c["k"].shape[2]
    for name, gname in _GRAD.items():
        arr = c[name]
        if arr is None:
            assert g[gname] is None
            continue
        idxs = list(np.ndindex(arr.shape))
        if n_samples is not None and len(idxs) > n_samples:
            idxs = [idxs[i] for i in rng.choice(len(idxs), n_samples, replace=False)]
        for idx in idxs:
            if name == "k" and c["k"].shape[1] > 3 and idx[1] == 3 and idx[2] == H - 1:
                continue                    # ||k|| = 0 is a kink of the skip rule
            h = 1e-6 * max(1.0, abs(arr[idx]))
            cp = dict(c); cp[name] = arr.copy(); cp[name][idx] += h
            cm = dict(c); cm[name] = arr.copy(); cm[name][idx] -= h
            fd = (_loss(cp, cot, eta, anchor) - _loss(cm, cot, eta, anchor)) / (2 * h)
            assert abs(fd - g[gname][idx]) <= tol * max(1.0, abs(fd)), (name, idx, fd, g[gname][idx])


@pytest.mark.parametrize("apf,gated,anchor", [(True, False, False), (False, False, False),
                                              (True, True, False), (True, False, True), (True, True, True)])
def test_backward_matches_finite_differences(apf, gated, anchor):
    c, cot = _case(3, apf=apf, gated=gated)
    _fd_check(c, cot, eta=0.3, anchor=anchor)


def test_backward_finite_differences_across_checkpoint_segments():
    # 150 tokens: the oracle replays three 64-token segments from their checkpoints
    c, cot = _case(11, T=150, H=1, dk=4, dv=3, gated=True)
    c["k"] /= np.linalg.norm(c["k"], axis=-1, keepdims=True).clip(1e-12)   # keep the state bounded
    _fd_check(c, cot, eta=0.2, anchor=True, n_samples=12, seed=5, tol=1e-5)


def test_backward_linearity_identities():
    # (o, S_T) are jointly linear in (v, S0) and d_T does not depend on them, so with
    # dd_final = 0 the loss L = <dout, o> + <dS_final, S_T> satisfies
    # L = sum(v * dv) + <S0, dS0> exactly (Euler); o is linear in q: <dout, o> = sum(q * dq).
    c, cot = _case(7, B=2, T=200, H=2, dk=16, dv=8, zero_key=False)
    c["k"] /= np.linalg.norm(c["k"], axis=-1, keepdims=True)
    cot["dd_final"] = np.zeros_like(cot["dd_final"])
    out, S, _ = oracle.fwd(c["q"], c["k"], c["v"], c["beta"], c["r"], c["d0"], c["S0"], eta=0.05)
    g = oracle.bwd(c["q"], c["k"], c["v"], c["beta"], cot["dout"], c["r"], c["d0"], c["S0"],
                   cot["dS_final"], None, eta=0.05)
    lo = float((out * cot["dout"]).sum())
    L = lo + float((S * cot["dS_final"]).sum())
    assert abs(float((c["v"] * g["dv"]).sum() + (c["S0"] * g["dS0"]).sum()) - L) <= 1e-9 * max(1.0, abs(L))
    assert abs(float((c["q"] * g["dq"]).sum()) - lo) <= 1e-9 * max(1.0, abs(lo))
    # the d chain alone: with dout = dS_final = 0 nothing flows into q, v or S0
    z = oracle.bwd(c["q"], c["k"], c["v"], c["beta"], np.zeros_like(cot["dout"]), c["r"], c["d0"], c["S0"],
                   None, cot["dd_final"] + 1.0, eta=0.05)
    assert not z["dq"].any() and not z["dv"].any() and not z["dS0"].any()


def test_backward_matches_autograd_of_definitions():
    # A token loop from the definitions, differentiated by torch autograd in float64:
    # f_t(S) = 1/2 ||S k - v||^2, S_t = alpha S_{t-1} - beta grad f_t(alpha S_{t-1}) diag(d_t),
    # o_t = S_t q_t, d_{t+1} = r d_t + (1 - r) d0 - eta grad_d h_t(d_t) with
    # h_t(d) = ((1 - beta <d, k^2>)^2 - 1) / (2 ||k||^2).
    c, cot = _case(21, B=1, T=130, H=1, dk=6, dv=5, gated=True, zero_key=False)
    c["k"] /= np.linalg.norm(c["k"], axis=-1, keepdims=True)
    eta = 0.1
    tt = {n: torch.tensor(a, requires_grad=True) for n, a in c.items() if a is not None}
    S = tt["S0"][0, 0].clone()
    d = tt["d0"][0, 0].clone()
    d_anchor = tt["d0"][0, 0]
    outs = []
    for t in range(c["k"].shape[1]):
        k, q, v = tt["k"][0, t, 0], tt["q"][0, t, 0], tt["v"][0, t, 0]
        b, r, a = tt["beta"][0, t, 0], tt["r"][0, t, 0], tt["alpha"][0, t, 0]
        Sh = a * S
        grad_f = torch.outer(Sh @ k - v, k)                     # d/dS of 1/2 ||S k - v||^2
        S = Sh - b * grad_f @ torch.diag(d)
        outs.append(S @ q)
        k2 = k * k
        grad_h = -b * (1 - b * (d @ k2)) * k2 / (k2.sum())      # d/dd of h_t
        d = r * d + (1 - r) * d_anchor - eta * grad_h
    out = torch.stack(outs)
    L = (out * torch.tensor(cot["dout"][0, :, 0])).sum() + (S * torch.tensor(cot["dS_final"][0, 0])).sum() \
        + (d * torch.tensor(cot["dd_final"][0, 0])).sum()
    L.backward()
    g = oracle.bwd(c["q"], c["k"], c["v"], c["beta"], cot["dout"], c["r"], c["d0"], c["S0"],
                   cot["dS_final"], cot["dd_final"], eta=eta, anchor=True, alpha=c["alpha"])
    for name, gname in _GRAD.items():
        ref = tt[name].grad.numpy()
        np.testing.assert_allclose(g[gname], ref, rtol=1e-9, atol=1e-9 * np.abs(ref).max(), err_msg=name)
