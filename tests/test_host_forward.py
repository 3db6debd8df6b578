"""The forward on host buffers (osdn_fwd_host): the batch goes through in groups of sequences,
each uploaded, run and read back on its own, the copies of one group overlapping the compute of
the others. Sequences are independent, so every group must equal the device-resident forward on
the same sequences bit for bit, and the whole batch must equal the oracle."""
import pytest
import torch

import oracle
from preconditioned_delta_rule_token_b200 import workloads as W
from tests._util import BF16_TOL, FP32_TOL, slice_rel_err


def _groups_of(B, groups):
    """The library's grouping: `groups` (0: 8) groups at most, one sequence each at least, up to 16."""
    g = min(groups if groups > 0 else 8, B, 16)
    per = -(-B // g)
    return [(b0, min(b0 + per, B)) for b0 in range(0, B, per)]


def _check(w, groups, pinned, tol):
    import preconditioned_delta_rule_token_b200 as pk
    inp = W.make_forward_inputs(w)
    host = {n: None if x is None else (x.pin_memory() if pinned else x.contiguous()) for n, x in inp.items()}
    s = torch.cuda.Stream()
    out, S, d = pk.forward_host(host["q"], host["k"], host["v"], host["beta"], host["r"], host["d0"], host["S0"],
                                eta=w.eta, groups=groups, stream=s)
    s.synchronize()
    assert not out.is_cuda and pk.osdn_sync_status() == 0
    for b0, b1 in _groups_of(w.B, groups):
        dev = {n: None if x is None else x[b0:b1].cuda() for n, x in inp.items()}
        o2, S2, d2 = pk.forward(dev["q"], dev["k"], dev["v"], dev["beta"], dev["r"], dev["d0"], dev["S0"], eta=w.eta)
        torch.cuda.synchronize()
        assert torch.equal(out[b0:b1], o2.cpu()) and torch.equal(S[b0:b1], S2.cpu()) and torch.equal(d[b0:b1], d2.cpu())
    f = W.to_f64
    ro, rS, rd = oracle.fwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["beta"]), f(inp["r"]), f(inp["d0"]),
                            f(inp["S0"]), eta=w.eta)
    errs = (slice_rel_err(out.float().numpy(), ro, (0, 2)), slice_rel_err(S.numpy(), rS, (0, 1)),
            slice_rel_err(d.numpy(), rd, (0, 1)))
    assert max(errs) <= tol, errs


@pytest.mark.gpu
@pytest.mark.parametrize("groups,pinned", [(2, True), (3, False), (0, True)])
def test_gpu_fwd_host_equals_the_device_forward_per_group(groups, pinned):
    # 4 sequences of 4 heads, 1088 tokens (a ragged last chunk): 2, 2 and 4 groups; pageable once
    w = W.Workload("host buffers", 4, 4, 1088, 128, 128, 64, W.BF16, True, "gaussian", eta=1e-2, seed=80,
                   d0="uniform", S0="normal")
    _check(w, groups, pinned, BF16_TOL)


@pytest.mark.gpu
def test_gpu_fwd_host_fp32_without_apf():
    w = W.Workload("host buffers fp32", 3, 2, 200, 64, 64, 64, W.FP32, False, "gaussian", eta=1e-2, seed=81)
    _check(w, 2, True, FP32_TOL)


@pytest.mark.gpu
@pytest.mark.parametrize("with_init", [True, False])
def test_gpu_fwd_host_empty_sequences(with_init):
    """T = 0: no tokens; the final state is the initial one (zeros and ones when none is given)."""
    import preconditioned_delta_rule_token_b200 as pk
    B, H, dk, dv = 3, 2, 128, 128
    q = torch.empty((B, 0, H, dk), dtype=torch.bfloat16).pin_memory()
    v = torch.empty((B, 0, H, dv), dtype=torch.bfloat16).pin_memory()
    beta = torch.empty((B, 0, H), dtype=torch.bfloat16).pin_memory()
    g = torch.Generator().manual_seed(82)
    d0 = (0.5 + torch.rand((B, H, dk), generator=g)).pin_memory() if with_init else None
    S0 = torch.randn((B, H, dv, dk), generator=g).pin_memory() if with_init else None
    s = torch.cuda.Stream()
    out, S, d = pk.forward_host(q, q, v, beta, None, d0, S0, groups=2, stream=s)
    s.synchronize()
    assert out.shape == (B, 0, H, dv) and pk.osdn_sync_status() == 0
    assert torch.equal(S, S0 if with_init else torch.zeros_like(S))
    assert torch.equal(d, d0 if with_init else torch.ones_like(d))
