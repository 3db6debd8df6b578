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
_AXES = {"dq": (0, 2), "dk": (0, 2), "dv": (0, 2), "dbeta": (0, 2), "dr": (0, 2), "dd0": (0, 1), "dS0": (0, 1)}


def _gpu(x):
    return None if x is None else x.cuda()


def _run(w, anchor=False, dS=True, dd=True, units=None):
    import preconditioned_delta_rule_token_b200 as P
    inp = W.make_forward_inputs(w)
    cot = W.make_backward_cotangents(w, dS_final=dS, dd_final=dd)
    g = P.backward(*(_gpu(inp[n]) for n in ("q", "k", "v", "beta")), _gpu(cot["dout"]), r=_gpu(inp["r"]),
                   d0=_gpu(inp["d0"]), S0=_gpu(inp["S0"]), dS_final=_gpu(cot["dS_final"]),
                   dd_final=_gpu(cot["dd_final"]), eta=w.eta, apf_anchor=anchor)
    torch.cuda.synchronize()
    assert P.osdn_sync_status() == 0
    got = {n: (None if t is None else t.float().cpu().numpy()) for n, t in g.items()}
    f = {n: W.to_f64(inp[n]) for n in ("q", "k", "v", "beta", "r", "d0", "S0")}
    c = {n: W.to_f64(cot[n]) for n in ("dout", "dS_final", "dd_final")}
    if units is None:
        ref = oracle.bwd(f["q"], f["k"], f["v"], f["beta"], c["dout"], f["r"], f["d0"], f["S0"], c["dS_final"],
                         c["dd_final"], eta=w.eta, anchor=anchor)
        return got, ref
    # sampled units of a large problem: the oracle runs on each (b, h) slice alone
    out = []
    for b, h in units:
        tok = lambda x: None if x is None else np.ascontiguousarray(x[b:b + 1, :, h:h + 1])
        st = lambda x: None if x is None else np.ascontiguousarray(x[b:b + 1, h:h + 1])
        ref = oracle.bwd(tok(f["q"]), tok(f["k"]), tok(f["v"]), tok(f["beta"]), tok(c["dout"]), tok(f["r"]),
                         st(f["d0"]), st(f["S0"]), st(c["dS_final"]), st(c["dd_final"]), eta=w.eta, anchor=anchor)
        sl = {n: (None if got[n] is None else
                  (got[n][b:b + 1, :, h:h + 1] if _AXES[n] == (0, 2) else got[n][b:b + 1, h:h + 1]))
              for n in got}
        out.append((sl, ref))
    return out


def _compare(got, ref, tol, has_r):
    errs = {}
    for n, axes in _AXES.items():
        if n == "dr" and not has_r:
            assert got[n] is None and ref[n] is None
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
        a_, b_ = g_def[n].cpu().numpy(), g_exp[n].cpu().numpy()
        np.testing.assert_allclose(a_, b_, rtol=1e-5, atol=1e-6 * np.abs(b_).max(), err_msg=n)


@pytest.mark.parametrize("dv,anchor", [(64, False), (128, True)])
def test_backward_bf16_narrow_keys(dv, anchor):
    # bf16 inputs with dk = 64 (the tensor-core tile paths at the narrow key width)
    w = _small("bwd bf16 dk64", 2, 2, 130, 64, dv, W.BF16, seed=31)
    got, ref = _run(w, anchor=anchor)
    _compare(got, ref, BF16_TOL, True)
