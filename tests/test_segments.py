"""Phase 2 split along the sequence for few (b, h) units (osdn_fwd_segments > 1).

"OSDN: Improving Delta Rule with Provable Online Preconditioning in Linear Attention",
technical summary section 2.1: the chunk update S <- S (I - W^T Kw) + U0^T Kw is affine in
S, so a segment's end state is S_start E + L, with L its end state from S = 0 and E its end
state from S = I with V = 0. The CPU tests pin that composition with the oracle (plain and
gated) and the segment plan through the library's host code; the GPU tests compare split
calls with the oracle on every unit.
"""
import numpy as np
import pytest
import torch

import oracle
from preconditioned_delta_rule_token_b200 import workloads as W
from tests._util import BF16_TOL, slice_rel_err


def _seg_case(seed, T, dk=16, dv=12, gated=False):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((1, T, 1, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q = rng.standard_normal((1, T, 1, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, 1, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal((1, T, 1))))
    r = 1 - 1e-2 / (1 + np.exp(-rng.standard_normal((1, T, 1))))
    d0 = rng.uniform(0.5, 1.5, (1, 1, dk))
    S0 = 0.3 * rng.standard_normal((1, 1, dv, dk))
    alpha = rng.uniform(0.3, 1.0, (1, T, 1)) if gated else None
    return q, k, v, beta, r, d0, S0, alpha


@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("P", [2, 4])
def test_segment_composition_equals_the_whole_sequence(gated, P):
    """Run each segment from S = 0 (L) and from S = I with V = 0 (E), each with the true d at
    its start; S_start(p + 1) = S_start(p) E_p + L_p, and each segment run again from its
    S_start gives the outputs and final state of the whole sequence."""
    T, eta = 48 * P, 0.3
    q, k, v, beta, r, d0, S0, alpha = _seg_case(7 + P, T, gated=gated)
    dk = S0.shape[3]
    o_ref, S_ref, d_ref = oracle.fwd(q, k, v, beta, r, d0, S0, eta=eta, alpha=alpha)
    Ls = T // P
    sl = [slice(p * Ls, (p + 1) * Ls) for p in range(P)]
    seg = lambda x, p: None if x is None else np.ascontiguousarray(x[:, sl[p]])
    # d at every segment start, from the scan of the prefix
    d_at = [d0] + [oracle.fwd(q[:, :p * Ls], k[:, :p * Ls], v[:, :p * Ls], beta[:, :p * Ls], r[:, :p * Ls], d0,
                              S0, eta=eta, alpha=None if alpha is None else alpha[:, :p * Ls])[2]
                   for p in range(1, P)]
    S = S0.copy()
    outs = []
    for p in range(P):
        args = (seg(q, p), seg(k, p), seg(v, p), seg(beta, p), seg(r, p), d_at[p])
        _, Lp, _ = oracle.fwd(*args, np.zeros_like(S0), eta=eta, alpha=seg(alpha, p))
        ident = np.zeros((1, 1, dk, dk))
        ident[0, 0] = np.eye(dk)
        # E is dk x dk: the state transfer applied from the right, S_end = S_start E + L
        _, Ep, _ = oracle.fwd(seg(q, p), seg(k, p), np.zeros((1, Ls, 1, dk)), seg(beta, p), seg(r, p), d_at[p],
                              ident, eta=eta, alpha=seg(alpha, p))
        o_p, S_check, _ = oracle.fwd(*args, S, eta=eta, alpha=seg(alpha, p))
        outs.append(o_p)
        S_next = S[0, 0] @ Ep[0, 0] + Lp[0, 0]
        np.testing.assert_allclose(S_next, S_check[0, 0], rtol=1e-10, atol=1e-12)
        S = S_next[None, None]
    np.testing.assert_allclose(np.concatenate(outs, axis=1), o_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], S_ref[0, 0], rtol=1e-10, atol=1e-12)


def _params(B, T, H, dk=128, dv=128, dtype=torch.bfloat16):
    import preconditioned_delta_rule_token_b200 as pk
    return pk.make_params(B, T, H, dk, dv, dtype, 1e-2)


@pytest.mark.parametrize("B,T,H,dtype,dk,want", [
    (1, 32768, 16, torch.bfloat16, 128, 16),   # long context, one sequence: overlapped, short segments
    (8, 4096, 16, torch.bfloat16, 128, 1),     # 128 units fill the SMs
    (8, 2048, 8, torch.bfloat16, 128, 1),      # 64 units: 2 segments would not pay (pipelined instead)
    (4, 1024, 16, torch.bfloat16, 128, 1),     # 64 units, pipelined in 2 segments of 512 tokens
    (2, 8192, 16, torch.bfloat16, 128, 4),     # 32 units: split (4 segments), not pipelined
    (2, 4096, 20, torch.bfloat16, 128, 1),     # 40 units, pipelined in 4 segments of 1024 tokens
    (2, 1536, 8, torch.bfloat16, 128, 1),      # 16 units, 2 pipelined segments (4 would be 384 tokens)
    (8, 2048, 10, torch.bfloat16, 128, 1),     # 80 units: more than half the SMs, not pipelined
    (1, 4096, 1, torch.bfloat16, 128, 8),      # 16 capped by T / P >= 512
    (1, 4096, 2, torch.bfloat16, 128, 8),
    (1, 4000, 2, torch.bfloat16, 128, 1),      # T not a multiple of 64 P for any P >= 4
    (1, 32768, 16, torch.float32, 128, 1),     # the FFMA path never splits
    (1, 32768, 16, torch.bfloat16, 64, 1),
])
def test_segment_plan(B, T, H, dtype, dk, want):
    """The plan through the library's host code (no GPU needed; without a device the SM
    count is the B200's 148) and the workspace it implies."""
    import preconditioned_delta_rule_token_b200 as pk
    p = _params(B, T, H, dk=dk, dtype=dtype)
    P = pk.osdn_fwd_segments(p)
    assert P == want
    kw = B * T * H * dk * (2 if dtype == torch.bfloat16 else 4)
    ws = pk.osdn_fwd_workspace_size(p)
    up = lambda x: -(-x // 256) * 256
    if P == 1:
        pipe = _pipe_count(B, T, H, dtype, dk)
        want_ws = max(256, up(kw))
        if pipe > 1:   # beta, r, alpha segment-major; two states and two d handed between segments
            units = B * H
            want_ws = up(up(kw) + 3 * up(B * T * H * 2) + 2 * units * 128 * 128 * 4 + 2 * units * 128 * 4)
        assert ws == want_ws
        assert pk.osdn_fwd_launches(p) == (1 + 2 * pipe if pipe > 1 else 2)
    else:
        st = B * P * H * 128 * 128 * 4
        want_ws = up(kw) + 3 * st + 64 * 128 * 2          # start states, own end states, transfers, zeros
        if B == 1:   # one sequence: the scan overlaps phase 2 in osdn_fwd, batches of nb segments
            nb = min((148 - H) // (2 * H), P // 2)
            want_ws = up(up(want_ws) + nb * H * 128 * 128 * 4 + P * H * 128 * 4) + nb * (T // P) * H * 128 * 2
        assert ws == want_ws


def _pipe_count(B, T, H, dtype, dk, sms=148):
    """The pipelined forward's segment count: phase 2 not split, the units at most half the SMs,
    four segments of at least 1024 tokens, else two of at least 512, else none."""
    if dtype != torch.bfloat16 or dk != 128 or T <= 0 or 2 * B * H > sms:
        return 1
    for P, least in ((4, 1024), (2, 512)):
        if T % (64 * P) == 0 and T // P >= least:
            return P
    return 1


def test_segment_plan_needs_dense_tensors():
    import preconditioned_delta_rule_token_b200 as pk
    p = _params(1, 32768, 16)
    p.stride_q[0], p.stride_q[1], p.stride_q[2] = 32768 * 16 * 384, 16 * 384, 384   # q from a fused projection
    assert pk.osdn_fwd_segments(p) == 1


# ---------------------------------------------------------------------------- GPU

def _dev(x):
    return None if x is None else x.cuda()


def _check_against_oracle(w, alpha=None, split_phases=False):
    import preconditioned_delta_rule_token_b200 as pk
    inp = W.make_forward_inputs(w)
    p = pk.make_params(w.B, w.T, w.H, w.dk, w.dv, inp["k"].dtype, w.eta)
    assert pk.osdn_fwd_segments(p) >= 4
    g = {n: _dev(x) for n, x in inp.items()}
    a = _dev(alpha)
    if split_phases:   # the bench's calls: phase 1, then phase 2 alone
        out = torch.empty_like(g["v"])
        S = torch.empty((w.B, w.H, w.dv, w.dk), dtype=torch.float32, device="cuda")
        d = torch.empty((w.B, w.H, w.dk), dtype=torch.float32, device="cuda")
        ws = torch.empty(pk.osdn_fwd_workspace_size(p), dtype=torch.uint8, device="cuda")
        pk.osdn_fwd_scan(p, g["k"], g["beta"], g["r"], g["d0"], d, ws)
        if a is None:
            pk.osdn_fwd_chunk(p, g["q"], g["k"], g["v"], g["beta"], g["S0"], out, S, ws)
        else:
            pk.osdn_fwd_chunk_gated(p, g["q"], g["k"], g["v"], g["beta"], a, g["S0"], out, S, ws)
    else:
        out, S, d = pk.forward(g["q"], g["k"], g["v"], g["beta"], g["r"], g["d0"], g["S0"], eta=w.eta, alpha=a)
    assert pk.osdn_sync_status() == 0
    f = W.to_f64
    ro, rS, rd = oracle.fwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["beta"]), f(inp["r"]), f(inp["d0"]),
                            f(inp["S0"]), eta=w.eta, alpha=None if alpha is None else f(alpha))
    errs = (slice_rel_err(out.float().cpu().numpy(), ro, (0, 2)), slice_rel_err(S.cpu().numpy(), rS, (0, 1)),
            slice_rel_err(d.cpu().numpy(), rd, (0, 1)))
    assert max(errs) <= BF16_TOL, errs
    return errs


def _few_units(B, H, T, seed, S0="normal"):
    return W.Workload("few units", B, H, T, 128, 128, 64, W.BF16, True, "gaussian", eta=1e-2, seed=seed,
                      d0="uniform", S0=S0)


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,T", [(1, 2, 4096), (2, 3, 2048), (1, 1, 8192)])
def test_gpu_split_forward_matches_oracle(B, H, T):
    # 2, 6 and 1 units: 8, 4 and 16 segments, from a nonzero initial state
    _check_against_oracle(_few_units(B, H, T, seed=60 + H))


@pytest.mark.gpu
def test_gpu_split_phase2_alone_matches_oracle():
    _check_against_oracle(_few_units(1, 4, 4096, seed=64, S0="zeros"), split_phases=True)


@pytest.mark.gpu
@pytest.mark.parametrize("lo", [0.9, 0.05])
def test_gpu_split_gated_forward_matches_oracle(lo):
    w = _few_units(1, 3, 4096, seed=65)
    alpha = (lo + (1 - lo) * torch.rand((w.B, w.T, w.H), generator=torch.Generator().manual_seed(66))).to(
        torch.bfloat16)
    _check_against_oracle(w, alpha=alpha)
    _check_against_oracle(w, alpha=alpha, split_phases=True)


@pytest.mark.gpu
def test_gpu_overlapped_forward_joins_the_callers_stream():
    """One sequence: osdn_fwd overlaps the scan with phase 2 on two library streams. Called
    twice on a non-default stream, each result read after synchronizing that stream alone:
    both bit-identical (every launch is joined back to the caller's stream), and equal to the
    oracle."""
    import preconditioned_delta_rule_token_b200 as pk
    w = _few_units(1, 2, 4096, seed=67)
    inp = W.make_forward_inputs(w)
    p = pk.make_params(w.B, w.T, w.H, w.dk, w.dv, inp["k"].dtype, w.eta)
    assert pk.osdn_fwd_segments(p) == 8 and pk.osdn_fwd_launches(p) == 12   # batches [0, 4), [4, 7)
    g = {n: _dev(x) for n, x in inp.items()}
    s = torch.cuda.Stream()
    res = []
    for _ in range(2):
        with torch.cuda.stream(s):
            out, S, d = pk.forward(g["q"], g["k"], g["v"], g["beta"], g["r"], g["d0"], g["S0"], eta=w.eta,
                                   stream=s)
        s.synchronize()
        res.append((out.cpu(), S.cpu(), d.cpu()))
    assert pk.osdn_sync_status() == 0
    for a, b in zip(*res):
        assert torch.equal(a, b)
    f = W.to_f64
    ro, rS, rd = oracle.fwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["beta"]), f(inp["r"]), f(inp["d0"]),
                            f(inp["S0"]), eta=w.eta)
    out, S, d = res[0]
    errs = (slice_rel_err(out.float().numpy(), ro, (0, 2)), slice_rel_err(S.numpy(), rS, (0, 1)),
            slice_rel_err(d.numpy(), rd, (0, 1)))
    assert max(errs) <= BF16_TOL, errs


@pytest.mark.gpu
def test_gpu_split_anchored_single_sequence():
    # anchored APF: one sequence splits phase 2 but does not overlap the scan (its segments would
    # each need the anchor d0 separately)
    import preconditioned_delta_rule_token_b200 as pk
    w = _few_units(1, 2, 4096, seed=68)
    inp = W.make_forward_inputs(w)
    p = pk.make_params(w.B, w.T, w.H, w.dk, w.dv, inp["k"].dtype, w.eta, 64, True)
    assert pk.osdn_fwd_segments(p) == 8 and pk.osdn_fwd_launches(p) == 6
    g = {n: _dev(x) for n, x in inp.items()}
    out, S, d = pk.forward(g["q"], g["k"], g["v"], g["beta"], g["r"], g["d0"], g["S0"], eta=w.eta, apf_anchor=True)
    assert pk.osdn_sync_status() == 0
    f = W.to_f64
    ro, rS, rd = oracle.fwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["beta"]), f(inp["r"]), f(inp["d0"]),
                            f(inp["S0"]), eta=w.eta, anchor=True)
    errs = (slice_rel_err(out.float().cpu().numpy(), ro, (0, 2)), slice_rel_err(S.cpu().numpy(), rS, (0, 1)),
            slice_rel_err(d.cpu().numpy(), rd, (0, 1)))
    assert max(errs) <= BF16_TOL, errs


@pytest.mark.gpu
def test_gpu_split_gated_several_sequences():
    # B = 2: phase 2 split into segments without the overlap (gated, alpha down to 0.05)
    import preconditioned_delta_rule_token_b200 as pk
    w = _few_units(2, 3, 2048, seed=69)
    p = pk.make_params(w.B, w.T, w.H, w.dk, w.dv, torch.bfloat16, w.eta)
    assert pk.osdn_fwd_segments(p) == 4 and pk.osdn_fwd_launches(p) == 6
    alpha = (0.05 + 0.95 * torch.rand((w.B, w.T, w.H), generator=torch.Generator().manual_seed(70))).to(
        torch.bfloat16)
    _check_against_oracle(w, alpha=alpha)


def _pipelined_case(w, alpha=None):
    """osdn_fwd (or osdn_fwd_gated) on a pipelined shape against the oracle, and bit for bit
    against the two phases called one after the other (osdn_fwd_scan, then osdn_fwd_chunk: the
    same kernels over whole sequences). Segments end on scan blocks and chunk boundaries and
    hand over d and S in fp32, so the two orders do the same arithmetic."""
    import preconditioned_delta_rule_token_b200 as pk
    inp = W.make_forward_inputs(w)
    p = pk.make_params(w.B, w.T, w.H, w.dk, w.dv, inp["k"].dtype, w.eta)
    P = _pipe_count(w.B, w.T, w.H, torch.bfloat16, 128)
    assert P > 1 and pk.osdn_fwd_segments(p) == 1 and pk.osdn_fwd_launches(p) == 1 + 2 * P
    g = {n: _dev(x) for n, x in inp.items()}
    a = _dev(alpha)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out, S, d = pk.forward(g["q"], g["k"], g["v"], g["beta"], g["r"], g["d0"], g["S0"], eta=w.eta, alpha=a,
                               stream=s)
    s.synchronize()
    out2 = torch.empty_like(g["v"])
    S2 = torch.empty((w.B, w.H, w.dv, w.dk), dtype=torch.float32, device="cuda")
    d2 = torch.empty((w.B, w.H, w.dk), dtype=torch.float32, device="cuda")
    ws = torch.empty(pk.osdn_fwd_workspace_size(p), dtype=torch.uint8, device="cuda")
    pk.osdn_fwd_scan(p, g["k"], g["beta"], g["r"], g["d0"], d2, ws)
    if a is None:
        pk.osdn_fwd_chunk(p, g["q"], g["k"], g["v"], g["beta"], g["S0"], out2, S2, ws)
    else:
        pk.osdn_fwd_chunk_gated(p, g["q"], g["k"], g["v"], g["beta"], a, g["S0"], out2, S2, ws)
    torch.cuda.synchronize()
    assert pk.osdn_sync_status() == 0
    f = W.to_f64
    ro, rS, rd = oracle.fwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["beta"]), f(inp["r"]), f(inp["d0"]),
                            f(inp["S0"]), eta=w.eta, alpha=None if alpha is None else f(alpha))
    errs = (slice_rel_err(out.float().cpu().numpy(), ro, (0, 2)), slice_rel_err(S.cpu().numpy(), rS, (0, 1)),
            slice_rel_err(d.cpu().numpy(), rd, (0, 1)))
    assert max(errs) <= BF16_TOL, errs
    assert torch.equal(out, out2) and torch.equal(S, S2) and torch.equal(d, d2)


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,T,apf", [(2, 2, 1024, True), (4, 10, 2048, True), (2, 20, 4096, False)])
def test_gpu_pipelined_forward_matches_oracle(B, H, T, apf):
    # 4 units with segments too short to split, and 40 units (more than 148 / 4, so not split
    # either): 2, 2 and 4 pipelined segments; from a nonzero initial state
    w = W.Workload("few units", B, H, T, 128, 128, 64, W.BF16, apf, "gaussian", eta=1e-2, seed=71 + T // 512,
                   d0="uniform", S0="normal")
    _pipelined_case(w)


@pytest.mark.gpu
def test_gpu_pipelined_gated_forward_matches_oracle():
    # alpha down to 0.05 with exact zeros (restarts) on both sides of segment boundaries
    w = _few_units(4, 10, 2048, seed=75)
    alpha = 0.05 + 0.95 * torch.rand((w.B, w.T, w.H), generator=torch.Generator().manual_seed(76))
    alpha[:, 510:514] = 0.0
    alpha[1, 1024] = 0.0
    _pipelined_case(w, alpha=alpha.to(torch.bfloat16))
