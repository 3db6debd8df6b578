"""GPU parity of the backward (osdn_bwd) against the oracle's reverse-mode gradients.

The gradients are those of L = <dout, o> + <dS_final, S_T> + <dd_final, d_T> for the
OSDN forward ("OSDN: Improving Delta Rule with Provable Online Preconditioning in
Linear Attention", technical summary sections 2.1-2.3; the pages give no backward,
the oracle's is the plain derivative of its recurrence, pinned in
test_backward_oracle.py). Every comparison is element by element per (b, h) unit:
max |gpu - oracle| / max |oracle| within the unit, at the forward's tolerances
(1e-4 in fp32 mode, where every product runs as three tf32 passes; 2e-2 for bf16
inputs, where outputs are rounded to bf16 and the products run in one tf32 pass).
"""
import numpy as np
import pytest
import torch

import oracle
from preconditioned_delta_rule_token_b200 import workloads as W
from tests._util import BF16_TOL, FP32_TOL, slice_rel_err

pytestmark = pytest.mark.gpu

# unit axes of each gradient: [B, T, H, *] tensors -> (0, 2); [B, H, *] -> (0, 1)
_AXES = {"dq": (0, 2), "dk": (0, 2), "dv": (0, 2), "dbeta": (0, 2), "dr": (0, 2), "dd0": (0, 1), "dS0": (0, 1),
         "dalpha": (0, 2)}


def _gpu(x):
    return None if x is None else x.cuda()


def _run(w, anchor=False, dS=True, dd=True, units=None, alpha=None):
    import preconditioned_delta_rule_token_b200 as P
    inp = W.make_forward_inputs(w)
    cot = W.make_backward_cotangents(w, dS_final=dS, dd_final=dd)
    if alpha is not None:
        alpha = torch.as_tensor(alpha).to(inp["k"].dtype)
    g = P.backward(*(_gpu(inp[n]) for n in ("q", "k", "v", "beta")), _gpu(cot["dout"]), r=_gpu(inp["r"]),
                   d0=_gpu(inp["d0"]), S0=_gpu(inp["S0"]), dS_final=_gpu(cot["dS_final"]),
                   dd_final=_gpu(cot["dd_final"]), eta=w.eta, apf_anchor=anchor, alpha=_gpu(alpha))
    torch.cuda.synchronize()
    assert P.osdn_sync_status() == 0
    got = {n: (None if t is None else t.float().cpu().numpy()) for n, t in g.items()}
    f = {n: W.to_f64(inp[n]) for n in ("q", "k", "v", "beta", "r", "d0", "S0")}
    c = {n: W.to_f64(cot[n]) for n in ("dout", "dS_final", "dd_final")}
    fa = None if alpha is None else W.to_f64(alpha)
    if units is None:
        ref = oracle.bwd(f["q"], f["k"], f["v"], f["beta"], c["dout"], f["r"], f["d0"], f["S0"], c["dS_final"],
                         c["dd_final"], eta=w.eta, anchor=anchor, alpha=fa)
        return got, ref
    # sampled units of a large problem: the oracle runs on each (b, h) slice alone
    out = []
    for b, h in units:
        tok = lambda x: None if x is None else np.ascontiguousarray(x[b:b + 1, :, h:h + 1])
        st = lambda x: None if x is None else np.ascontiguousarray(x[b:b + 1, h:h + 1])
        ref = oracle.bwd(tok(f["q"]), tok(f["k"]), tok(f["v"]), tok(f["beta"]), tok(c["dout"]), tok(f["r"]),
                         st(f["d0"]), st(f["S0"]), st(c["dS_final"]), st(c["dd_final"]), eta=w.eta, anchor=anchor,
                         alpha=None if fa is None else np.ascontiguousarray(fa[b:b + 1, :, h:h + 1]))
        sl = {n: (None if got[n] is None else
                  (got[n][b:b + 1, :, h:h + 1] if _AXES[n] == (0, 2) else got[n][b:b + 1, h:h + 1]))
              for n in got}
        out.append((sl, ref))
    return out


def _compare(got, ref, tol, has_r):
    errs = {}
    for n, axes in _AXES.items():
        if (n == "dr" and not has_r) or (n == "dalpha" and ref.get(n) is None):
            assert got.get(n) is None and ref.get(n) is None
            continue
        errs[n] = slice_rel_err(got[n], ref[n], axes)
    bad = {n: e for n, e in errs.items() if not e <= tol}
    assert not bad, (bad, errs)
    return errs


def _small(name, B, H, T, dk, dv, dtype, apf=True, structure="gaussian", seed=11):
    return W.Workload(name, B, H, T, dk, dv, 64, dtype, apf, structure, eta=0.05, seed=seed, d0="uniform",
                      S0="normal")


@pytest.mark.parametrize("anchor", [False, True])
def test_backward_fp32_ragged(anchor):
    # 200 tokens: three full chunks and a ragged tail of 8
    w = _small("bwd fp32 ragged", 1, 2, 200, 64, 64, W.FP32)
    got, ref = _run(w, anchor=anchor)
    _compare(got, ref, FP32_TOL, True)


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64), (128, 128)])
def test_backward_fp32_widths(dk, dv):
    w = _small("bwd fp32 widths", 1, 1, 64 + 37, dk, dv, W.FP32, seed=5)
    got, ref = _run(w)
    _compare(got, ref, FP32_TOL, True)


def test_backward_bf16_shifted_keys_anchored():
    w = _small("bwd bf16 shifted", 2, 2, 130, 128, 128, W.BF16, structure="shifted", seed=2)
    got, ref = _run(w, anchor=True)
    _compare(got, ref, BF16_TOL, True)


def test_backward_bf16_apf_off_no_final_gradients():
    # r = None (no APF): dr is not produced; dS_final = dd_final = None (zero upstream)
    w = _small("bwd bf16 apf off", 1, 3, 70, 128, 64, W.BF16, apf=False, seed=3)
    got, ref = _run(w, dS=False, dd=False)
    _compare(got, ref, BF16_TOL, False)


def test_backward_single_token_and_empty():
    w = _small("bwd one token", 2, 2, 1, 64, 64, W.FP32, seed=9)
    got, ref = _run(w)
    _compare(got, ref, FP32_TOL, True)
    import preconditioned_delta_rule_token_b200 as P
    w0 = _small("bwd empty", 2, 2, 0, 64, 64, W.FP32)
    inp = W.make_forward_inputs(w0)
    cot = W.make_backward_cotangents(w0)
    g = P.backward(*(_gpu(inp[n]) for n in ("q", "k", "v", "beta")), _gpu(cot["dout"]), r=_gpu(inp["r"]),
                   d0=_gpu(inp["d0"]), S0=_gpu(inp["S0"]), dS_final=_gpu(cot["dS_final"]),
                   dd_final=_gpu(cot["dd_final"]))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(g["dS0"].cpu().numpy(), cot["dS_final"].numpy())
    np.testing.assert_array_equal(g["dd0"].cpu().numpy(), cot["dd_final"].numpy())


def test_backward_full_size_every_unit():
    # the 1.3B-shaped layer (B8 H16 T4096 d128 bf16, APF, shifted keys): every (b, h) unit
    # of every gradient against the oracle
    w = W.LAYER_1P3B
    got, ref = _run(w)
    _compare(got, ref, BF16_TOL, True)


@pytest.mark.parametrize("B,H,dtype,tol", [(4, 10, W.BF16, BF16_TOL), (8, 10, W.FP32, FP32_TOL)])
def test_backward_state_tile_widths(B, H, dtype, tol):
    # 40 and 80 (b, h) units: on 148 SMs the state passes take dv tiles of 64 and 128 rows
    # (the small cases above take 32), so every tile width runs against the oracle
    w = _small("bwd tiles", B, H, 70, 128, 128, dtype, seed=13)
    got, ref = _run(w)
    _compare(got, ref, tol, True)


def test_backward_default_initial_state_and_preconditioner():
    # d0 = NULL means ones and S0 = NULL means zeros: identical to passing them explicitly;
    # with anchored APF the anchor is that default d0
    import preconditioned_delta_rule_token_b200 as P
    w = _small("bwd defaults", 1, 2, 90, 64, 64, W.FP32, seed=17)
    inp = W.make_forward_inputs(w)
    cot = W.make_backward_cotangents(w)
    args = [_gpu(inp[n]) for n in ("q", "k", "v", "beta")] + [_gpu(cot["dout"])]
    kw = dict(r=_gpu(inp["r"]), dS_final=_gpu(cot["dS_final"]), dd_final=_gpu(cot["dd_final"]), eta=w.eta,
              apf_anchor=True)
    ones = torch.ones((w.B, w.H, w.dk), device="cuda")
    zeros = torch.zeros((w.B, w.H, w.dv, w.dk), device="cuda")
    g_def = P.backward(*args, **kw)
    g_exp = P.backward(*args, d0=ones, S0=zeros, **kw)
    torch.cuda.synchronize()
    for n in g_def:   # dbeta sums shared-memory atomic adds, whose order may differ between calls
        if g_def[n] is None:   # dalpha of the ungated call
            assert g_exp[n] is None
            continue
        a_, b_ = g_def[n].cpu().numpy(), g_exp[n].cpu().numpy()
        np.testing.assert_allclose(a_, b_, rtol=1e-5, atol=1e-6 * np.abs(b_).max(), err_msg=n)


@pytest.mark.parametrize("dv,anchor", [(64, False), (128, True)])
def test_backward_bf16_narrow_keys(dv, anchor):
    # bf16 inputs with dk = 64 (the tensor-core tile paths at the narrow key width)
    w = _small("bwd bf16 dk64", 2, 2, 130, 64, dv, W.BF16, seed=31)
    got, ref = _run(w, anchor=anchor)
    _compare(got, ref, BF16_TOL, True)


# ---------------------------------------------------------------------------
# Gated OSDN (osdn_bwd_gated): the gradients of the forward with the state decayed by
# alpha_t before token t's write, dalpha included, against oracle.bwd(alpha=...).

def _gates(B, T, H, lo, seed, zeros=True):
    """alpha ~ U(lo, 1); with zeros, alpha = 0 (a restart) at a chunk start, twice inside
    one chunk and at the last token, and a run of alpha = 0.2 over a whole chunk."""
    rng = np.random.default_rng(seed)
    a = rng.uniform(lo, 1.0, (B, T, H))
    if zeros:
        a[:, 64:128] = np.minimum(a[:, 64:128], 0.2)
        for t in (64, 70, 77, 3, T - 1):
            if 0 <= t < T:
                a[:, t] = 0.0
    return a


@pytest.mark.parametrize("anchor", [False, True])
def test_backward_gated_fp32_ragged_with_zero_gates(anchor):
    # 200 tokens (three full chunks and a ragged tail of 8), gates down to 0.05 and exact zeros
    w = _small("bwd gated fp32", 1, 2, 200, 64, 64, W.FP32, seed=41)
    got, ref = _run(w, anchor=anchor, alpha=_gates(1, 200, 2, 0.05, 41))
    assert np.all(np.isfinite(got["dalpha"]))
    _compare(got, ref, FP32_TOL, True)


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64), (128, 128)])
def test_backward_gated_fp32_widths(dk, dv):
    w = _small("bwd gated fp32 widths", 1, 2, 64 + 37, dk, dv, W.FP32, seed=43)
    got, ref = _run(w, alpha=_gates(1, 101, 2, 0.5, 43, zeros=False))
    _compare(got, ref, FP32_TOL, True)


@pytest.mark.parametrize("dk,dv,lo", [(128, 128, 0.05), (64, 128, 0.5), (128, 64, 0.9)])
def test_backward_gated_bf16(dk, dv, lo):
    w = _small("bwd gated bf16", 2, 2, 130, dk, dv, W.BF16, structure="shifted", seed=45)
    got, ref = _run(w, anchor=True, alpha=_gates(2, 130, 2, lo, 45, zeros=lo < 0.1))
    _compare(got, ref, BF16_TOL, True)


@pytest.mark.parametrize("B,H,dtype,tol", [(4, 10, W.BF16, BF16_TOL), (8, 10, W.FP32, FP32_TOL)])
def test_backward_gated_state_tile_widths(B, H, dtype, tol):
    # 40 and 80 units: the state passes take dv tiles of 64 and 128 rows under the gate
    w = _small("bwd gated tiles", B, H, 70, 128, 128, dtype, seed=47)
    got, ref = _run(w, alpha=_gates(B, 70, H, 0.3, 47))
    _compare(got, ref, tol, True)


def test_backward_gated_unit_gate_equals_ungated():
    # alpha = 1 everywhere: the gated kernels give the ungated gradients and dalpha matches
    import preconditioned_delta_rule_token_b200 as P
    w = _small("bwd gated ones", 2, 2, 150, 128, 128, W.BF16, seed=49)
    inp = W.make_forward_inputs(w)
    cot = W.make_backward_cotangents(w)
    args = [_gpu(inp[n]) for n in ("q", "k", "v", "beta")] + [_gpu(cot["dout"])]
    kw = dict(r=_gpu(inp["r"]), d0=_gpu(inp["d0"]), S0=_gpu(inp["S0"]), dS_final=_gpu(cot["dS_final"]),
              dd_final=_gpu(cot["dd_final"]), eta=w.eta)
    g1 = P.backward(*args, alpha=torch.ones((w.B, w.T, w.H), dtype=torch.bfloat16, device="cuda"), **kw)
    g0 = P.backward(*args, **kw)
    torch.cuda.synchronize()
    assert P.osdn_sync_status() == 0
    for n in g0:
        if g0[n] is None:
            continue
        a_, b_ = g1[n].float().cpu().numpy(), g0[n].float().cpu().numpy()
        # one bf16 ulp: dbeta sums shared-memory atomic adds, whose order may differ between calls
        np.testing.assert_allclose(a_, b_, rtol=8e-3, atol=1e-6 * np.abs(b_).max(), err_msg=n)
    f = {n: W.to_f64(inp[n]) for n in ("q", "k", "v", "beta", "r", "d0", "S0")}
    c = {n: W.to_f64(cot[n]) for n in ("dout", "dS_final", "dd_final")}
    ref = oracle.bwd(f["q"], f["k"], f["v"], f["beta"], c["dout"], f["r"], f["d0"], f["S0"], c["dS_final"],
                     c["dd_final"], eta=w.eta, alpha=np.ones((w.B, w.T, w.H)))
    assert slice_rel_err(g1["dalpha"].float().cpu().numpy(), ref["dalpha"], (0, 2)) <= BF16_TOL


def test_backward_gated_missing_gate_gradient_is_refused():
    import preconditioned_delta_rule_token_b200 as P
    w = _small("bwd gated refused", 1, 1, 70, 64, 64, W.FP32, seed=50)
    inp = W.make_forward_inputs(w)
    cot = W.make_backward_cotangents(w)
    p = P.make_params(w.B, w.T, w.H, w.dk, w.dv, inp["k"].dtype, w.eta, 64, False)
    ws = torch.empty(P.osdn_bwd_workspace_size(p), dtype=torch.uint8, device="cuda")
    g = {n: torch.empty_like(inp[m]).cuda() for n, m in (("dq", "q"), ("dk", "k"), ("dv", "v"), ("dbeta", "beta"))}
    alpha = torch.ones((w.B, w.T, w.H), device="cuda")
    with pytest.raises(P.OsdnError) as e:
        P.osdn_bwd_gated(p, *(_gpu(inp[n]) for n in ("q", "k", "v", "beta", "r")), alpha, None, None,
                         _gpu(cot["dout"]), None, None, g["dq"], g["dk"], g["dv"], g["dbeta"], None, None, None, None,
                         ws)
    assert e.value.code == P.OSDN_ERR_INVALID_ARG


def test_backward_gated_full_size_every_unit():
    # the 1.3B-shaped layer (B8 H16 T4096 d128 bf16, APF, shifted keys) with alpha ~ U(0.9, 1):
    # every (b, h) unit of every gradient, dalpha included, against the oracle
    w = W.LAYER_1P3B
    got, ref = _run(w, alpha=_gates(w.B, w.T, w.H, 0.9, 57, zeros=False))
    _compare(got, ref, BF16_TOL, True)
