"""Failure path of the tensor-core kernels, without a GPU fault.

Every device-side wait of the bf16 tensor-core kernels (mbarrier hand-offs
between TMA, MMA and the warp groups) is bounded. With the bound set to 1 ns
the first wait that is not already satisfied gives up: the CTA sets the
library's status word, lets its own copies and MMAs in flight finish and
returns, so the context stays usable. The host sees OSDN_ERR_TIMEOUT from
osdn_sync_status; results of that call are undefined. With the default bound
restored, the same call matches the oracle again.
"""
import numpy as np
import pytest

import oracle
from preconditioned_delta_rule_token_b200 import workloads as W
from tests._util import BF16_TOL, slice_rel_err

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_recovers():
    import preconditioned_delta_rule_token_b200 as pk
    w = W.Workload("failure path B2 H2 T300 d128 bf16", 2, 2, 300, 128, 128, 64, W.BF16, True, "gaussian",
                   d0="uniform", S0="normal", seed=11)
    inp = W.make_forward_inputs(w)
    g = {k: None if v is None else v.cuda() for k, v in inp.items()}
    assert pk.osdn_sync_status() == pk.OSDN_OK
    pk.osdn_set_wait_limit_ns(1)
    try:
        pk.forward(g["q"], g["k"], g["v"], g["beta"], g["r"], g["d0"], g["S0"], eta=w.eta)
        status = pk.osdn_sync_status()
    finally:
        pk.osdn_set_wait_limit_ns(0)
    assert status == pk.OSDN_ERR_TIMEOUT
    assert pk.osdn_sync_status() == pk.OSDN_OK      # the flag was cleared by the read

    out, S, d = pk.forward(g["q"], g["k"], g["v"], g["beta"], g["r"], g["d0"], g["S0"], eta=w.eta)
    assert pk.osdn_sync_status() == pk.OSDN_OK
    f = W.to_f64
    ro, rS, rd = oracle.fwd(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["beta"]), f(inp["r"]), f(inp["d0"]),
                            f(inp["S0"]), eta=w.eta)
    assert slice_rel_err(out.float().cpu().numpy(), ro, (0, 2)) < BF16_TOL
    assert slice_rel_err(S.cpu().numpy(), rS, (0, 1)) < BF16_TOL
    assert slice_rel_err(d.cpu().numpy(), rd, (0, 1)) < BF16_TOL
