"""GPU parity: the CUDA path (through the C ABI) against the float64 CPU oracle
on the same seeded inputs.

Metric: max over (b, h) slices of max|gpu - oracle| / max|oracle|, separately
for out, final S and final d. Bar: 2e-2 for bf16 inputs with fp32
accumulation, 1e-4 in fp32 mode. Full-size workloads are checked on every
(b, h) unit.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from preconditioned_delta_rule_token_b200 import workloads as W
from tests._util import BF16_TOL, FP32_TOL, slice_rel_err

pytestmark = pytest.mark.gpu


def _dev(x):
    return None if x is None else x.cuda()


def _run_gpu(inp, eta, chunk=64):
    import preconditioned_delta_rule_token_b200 as pk
    out, S, d = pk.forward(_dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"]), _dev(inp["beta"]), _dev(inp["r"]),
                           _dev(inp["d0"]), _dev(inp["S0"]), eta=eta, chunk=chunk)
    assert pk.osdn_sync_status() == 0
    return out.float().cpu().numpy(), S.cpu().numpy(), d.cpu().numpy()


def _oracle(inp, eta):
    f = W.to_f64
    return oracle.fwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["beta"]), f(inp["r"]), f(inp["d0"]),
                      f(inp["S0"]), eta=eta)


def _errs(gpu, ref):
    return (slice_rel_err(gpu[0], ref[0], (0, 2)), slice_rel_err(gpu[1], ref[1], (0, 1)),
            slice_rel_err(gpu[2], ref[2], (0, 1)))


SMALL = [
    # dtype, B, H, T, dk, dv, apf, eta, d0, S0
    (W.FP32, 1, 1, 256, 64, 64, True, 1e-2, "ones", "zeros"),
    (W.FP32, 2, 3, 65, 128, 128, True, 1.0, "uniform", "normal"),
    (W.FP32, 2, 2, 130, 128, 64, False, 0.0, "uniform", "normal"),
    (W.FP32, 1, 3, 1, 64, 128, True, 1e-2, "ones", "normal"),
    (W.BF16, 2, 3, 200, 128, 128, True, 1e-2, "uniform", "normal"),
    (W.BF16, 2, 3, 63, 128, 128, False, 1.0, "uniform", "zeros"),
    (W.BF16, 1, 2, 129, 64, 64, True, 0.0, "ones", "normal"),
    (W.BF16, 3, 1, 192, 128, 64, True, 1e-2, "uniform", "normal"),
    (W.BF16, 1, 2, 64, 64, 128, False, 1e-2, "ones", "zeros"),
    (W.BF16, 2, 2, 1, 128, 128, True, 1.0, "uniform", "normal"),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "%s-B%dH%dT%d-dk%ddv%d-apf%d-eta%g-%s-%s" % c)
def test_small_cases_full_oracle(case):
    dtype, B, H, T, dk, dv, apf, eta, d0, S0 = case
    w = W.Workload("small", B, H, T, dk, dv, 64, dtype, apf, "gaussian", eta=eta, seed=100 + T + dk, d0=d0, S0=S0)
    inp = W.make_forward_inputs(w)
    errs = _errs(_run_gpu(inp, eta), _oracle(inp, eta))
    tol = FP32_TOL if dtype == W.FP32 else BF16_TOL
    assert max(errs) <= tol, errs


def test_tiny_fp32_workload():
    w = W.TINY_FP32
    inp = W.make_forward_inputs(w)
    errs = _errs(_run_gpu(inp, w.eta), _oracle(inp, w.eta))
    assert max(errs) <= FP32_TOL, errs


@pytest.mark.parametrize("w", [W.LAYER_340M, W.LAYER_1P3B, W.LONG_RECALL], ids=["340M", "1.3B", "long"])
def test_full_size_workloads_every_unit(w):
    """The full-size workloads in the launch configuration the bench times, every (b, h)
    unit compared element by element with the oracle (which runs all units on the host
    cores in a few seconds)."""
    inp = W.make_forward_inputs(w)
    gpu = _run_gpu(inp, w.eta)
    assert all(np.all(np.isfinite(x)) for x in gpu)
    errs = _errs(gpu, _oracle(inp, w.eta))
    assert max(errs) <= BF16_TOL, errs


def _with_silent_tokens(inp, seed):
    """Zero keys and zero write strengths inside chunks: in every (b, h) unit, a run of
    tokens with k_t = 0, scattered tokens with beta_t = 0, and one token with both."""
    g = torch.Generator().manual_seed(seed)
    k, beta = inp["k"].clone(), inp["beta"].clone()
    B, T, H, _ = k.shape
    for b in range(B):
        for h in range(H):
            t0 = int(torch.randint(0, max(1, T - 8), (1,), generator=g))
            k[b, t0:t0 + 5, h] = 0
            for t in torch.randint(0, T, (6,), generator=g).tolist():
                beta[b, t, h] = 0
            t1 = int(torch.randint(0, T, (1,), generator=g))
            k[b, t1, h] = 0
            beta[b, t1, h] = 0
    k[:, 0] = 0                       # the first token of every sequence writes nothing
    beta[:, 63] = 0                   # the last token of the first chunk
    out = dict(inp)
    out["k"], out["beta"] = k, beta
    return out


@pytest.mark.parametrize("apf,eta,T", [(True, 1e-2, 200), (True, 1.0, 130), (False, 0.5, 64)])
def test_bf16_zero_keys_and_zero_beta_inside_chunks(apf, eta, T):
    """bf16, dk = dv = 128 (the tensor-core scan and chunk kernels): tokens with k = 0
    (the preconditioner step is skipped, nothing is written) and tokens with beta = 0
    inside chunks; out, final S and final d compared element by element per unit."""
    w = W.Workload("silent tokens", 2, 3, T, 128, 128, 64, W.BF16, apf, "gaussian", eta=eta, seed=41 + T,
                   d0="uniform", S0="normal")
    inp = _with_silent_tokens(W.make_forward_inputs(w), seed=T)
    errs = _errs(_run_gpu(inp, w.eta), _oracle(inp, w.eta))
    assert max(errs) <= BF16_TOL, errs


def test_more_units_than_sms_every_unit():
    """320 (b, h) units (B5 H64) run the tensor-core scan and chunk kernels in more than
    one wave of CTAs (one CTA per unit, 148 SMs); ragged T = 130 spans three 64-token
    chunks and two 128-token scan blocks. Every unit is checked against the oracle."""
    w = W.Workload("multi-wave B5 H64 T130 d128 bf16", 5, 64, 130, 128, 128, 64, W.BF16, True, "gaussian",
                   d0="uniform", S0="normal", seed=21)
    inp = W.make_forward_inputs(w)
    gpu = _run_gpu(inp, w.eta)
    errs = _errs(gpu, _oracle(inp, w.eta))
    assert max(errs) <= BF16_TOL, errs


@pytest.mark.parametrize("dtype,dk,dv", [(W.BF16, 128, 128), (W.FP32, 128, 128), (W.BF16, 64, 128)])
def test_qkv_read_in_place_from_a_fused_projection(dtype, dk, dv):
    """q, k and v as column slices of one fused projection [B, T, H, 2 dk + dv]
    (strided views, last dimension contiguous), and out written into a column
    slice of a wider buffer: the library reads and writes them in place through
    the strides of osdn_params, with the result of dense inputs and the oracle."""
    import preconditioned_delta_rule_token_b200 as pk
    w = W.Workload("fused qkv", 2, 3, 150, dk, dv, 64, dtype, True, "gaussian", eta=0.1, seed=61, d0="uniform",
                   S0="normal")
    inp = W.make_forward_inputs(w)
    g = {k_: _dev(v_) for k_, v_ in inp.items()}
    fused = torch.cat([g["q"], g["k"], g["v"]], dim=-1)                    # [B, T, H, 2 dk + dv]
    q, k, v = fused[..., :dk], fused[..., dk:2 * dk], fused[..., 2 * dk:]
    assert not q.is_contiguous() and q.stride(-1) == 1
    wide = torch.full((w.B, w.T, w.H, dv + 64), 7.0, dtype=g["q"].dtype, device=q.device)
    out = wide[..., 32:32 + dv]
    p = pk.make_params(w.B, w.T, w.H, dk, dv, g["k"].dtype, w.eta, w.chunk)
    S = torch.empty((w.B, w.H, dv, dk), dtype=torch.float32, device=q.device)
    d = torch.empty((w.B, w.H, dk), dtype=torch.float32, device=q.device)
    ws = torch.empty(pk.osdn_fwd_workspace_size(p), dtype=torch.uint8, device=q.device)
    pk.osdn_fwd(p, q, k, v, g["beta"], g["r"], g["d0"], g["S0"], out, S, d, ws)
    assert pk.osdn_sync_status() == 0
    dense = pk.forward(g["q"], g["k"], g["v"], g["beta"], g["r"], g["d0"], g["S0"], eta=w.eta)
    torch.cuda.synchronize()
    assert torch.equal(out, dense[0]) and torch.equal(S, dense[1]) and torch.equal(d, dense[2])
    assert torch.all(wide[..., :32] == 7.0) and torch.all(wide[..., 32 + dv:] == 7.0)   # nothing outside out
    got = (out.float().cpu().numpy(), S.cpu().numpy(), d.cpu().numpy())
    tol = FP32_TOL if dtype == W.FP32 else BF16_TOL
    assert max(_errs(got, _oracle(inp, w.eta))) <= tol


def test_zero_tokens_returns_initial_state():
    import preconditioned_delta_rule_token_b200 as pk
    w = W.Workload("t0", 2, 2, 0, 128, 128, 64, W.BF16, True, d0="uniform", S0="normal", seed=5)
    inp = W.make_forward_inputs(w)
    out, S, d = pk.forward(_dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"]), _dev(inp["beta"]), _dev(inp["r"]),
                           _dev(inp["d0"]), _dev(inp["S0"]), eta=w.eta)
    torch.cuda.synchronize()
    assert out.numel() == 0
    assert torch.equal(S.cpu(), inp["S0"]) and torch.equal(d.cpu(), inp["d0"])
    out, S, d = pk.forward(_dev(inp["q"]), _dev(inp["k"]), _dev(inp["v"]), _dev(inp["beta"]), None, None, None)
    torch.cuda.synchronize()
    assert torch.all(S == 0) and torch.all(d == 1)


@pytest.mark.parametrize("dtype", [W.FP32, W.BF16])
def test_continuation_equals_one_forward(dtype):
    """Checkpoint/resume: forward over T1 then over T2 from the carried (S, d)
    equals one forward over T1 + T2 (T1 not a multiple of the chunk)."""
    import preconditioned_delta_rule_token_b200 as pk
    w = W.Workload("cont", 2, 2, 150, 128, 128, 64, dtype, True, d0="uniform", S0="normal", eta=0.5, seed=6)
    inp = W.make_forward_inputs(w)
    g = {k_: _dev(v_) for k_, v_ in inp.items()}
    o_full, S_full, d_full = pk.forward(g["q"], g["k"], g["v"], g["beta"], g["r"], g["d0"], g["S0"], eta=w.eta)
    T1 = 77
    part = lambda x, a, b: x[:, a:b].contiguous()
    o1, S1, d1 = pk.forward(part(g["q"], 0, T1), part(g["k"], 0, T1), part(g["v"], 0, T1), part(g["beta"], 0, T1),
                            part(g["r"], 0, T1), g["d0"], g["S0"], eta=w.eta)
    o2, S2, d2 = pk.forward(part(g["q"], T1, 150), part(g["k"], T1, 150), part(g["v"], T1, 150),
                            part(g["beta"], T1, 150), part(g["r"], T1, 150), d1, S1, eta=w.eta)
    torch.cuda.synchronize()
    tol = FP32_TOL if dtype == W.FP32 else BF16_TOL
    ref = _oracle(inp, w.eta)
    got = (torch.cat([o1, o2], 1).float().cpu().numpy(), S2.cpu().numpy(), d2.cpu().numpy())
    assert max(_errs(got, ref)) <= tol
    full = (o_full.float().cpu().numpy(), S_full.cpu().numpy(), d_full.cpu().numpy())
    assert max(_errs(got, full)) <= tol


@pytest.mark.parametrize("dtype", [W.FP32, W.BF16])
def test_decode_steps_equal_forward(dtype):
    """T calls of the single-token step equal one forward over the same tokens."""
    import preconditioned_delta_rule_token_b200 as pk
    w = W.Workload("dec", 2, 3, 40, 128, 128, 64, dtype, True, d0="uniform", S0="normal", eta=0.3, seed=7)
    inp = W.make_forward_inputs(w)
    g = {k_: _dev(v_) for k_, v_ in inp.items()}
    S = g["S0"].clone()
    d = g["d0"].clone()
    outs = []
    for t in range(w.T):
        outs.append(pk.step(g["q"][:, t].contiguous(), g["k"][:, t].contiguous(), g["v"][:, t].contiguous(),
                            g["beta"][:, t].contiguous(), S, d, r=g["r"][:, t].contiguous(), eta=w.eta))
    torch.cuda.synchronize()
    got = (torch.stack(outs, 1).float().cpu().numpy(), S.cpu().numpy(), d.cpu().numpy())
    ref = _oracle(inp, w.eta)
    tol = FP32_TOL if dtype == W.FP32 else BF16_TOL
    assert max(_errs(got, ref)) <= tol


def test_decode_workload_256_heads():
    """Decode workload: B = 256 sequences x H = 16 heads, 1024 single-token calls from
    S0 ~ N(0, 0.02^2). 256 heads (one per sequence, every head index 16 times) are
    followed by the oracle step by step; their outputs are compared every 64 calls and
    their S and d at the end."""
    import preconditioned_delta_rule_token_b200 as pk
    w = W.DECODE
    st = W.make_decode_state(w)
    S = st["S0"].cuda()
    d = st["d0"].cuda()
    bi = torch.arange(w.B)
    hi = bi % w.H
    pick = lambda x: None if x is None else np.ascontiguousarray(W.to_f64(x[bi, hi])[:, None])
    So = pick(st["S0"])
    do = pick(st["d0"])
    worst = 0.0
    for t in range(w.steps):
        tok = W.make_decode_token(w, t)
        o = pk.step(tok["q"].cuda(), tok["k"].cuda(), tok["v"].cuda(), tok["beta"].cuda(), S, d,
                    r=_dev(tok["r"]), eta=w.eta)
        ro = oracle.step(pick(tok["q"]), pick(tok["k"]), pick(tok["v"]), pick(tok["beta"]), So, do,
                         r=pick(tok["r"]), eta=w.eta)
        if t % 64 == 63:
            worst = max(worst, slice_rel_err(o[bi, hi].float().cpu().numpy()[:, None], ro, (0, 1)))
    torch.cuda.synchronize()
    worst = max(worst, slice_rel_err(S[bi, hi].cpu().numpy()[:, None], So, (0, 1)),
                slice_rel_err(d[bi, hi].cpu().numpy()[:, None], do, (0, 1)))
    assert worst <= BF16_TOL, worst


def test_gpu_preconditioner_is_decoupled_from_values_and_queries():
    """Section 2.2's decoupling on the GPU path: final d does not depend on v or q."""
    import preconditioned_delta_rule_token_b200 as pk
    w = W.Workload("dec2", 2, 2, 100, 128, 128, 64, W.BF16, True, d0="uniform", eta=0.5, seed=8)
    inp = W.make_forward_inputs(w)
    g = {k_: _dev(v_) for k_, v_ in inp.items()}
    _, _, d1 = pk.forward(g["q"], g["k"], g["v"], g["beta"], g["r"], g["d0"], None, eta=w.eta)
    _, _, d2 = pk.forward(torch.randn_like(g["q"]), g["k"], torch.randn_like(g["v"]), g["beta"], g["r"], g["d0"],
                          None, eta=w.eta)
    torch.cuda.synchronize()
    assert torch.equal(d1, d2)
