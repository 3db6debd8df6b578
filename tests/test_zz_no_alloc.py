"""The forward entry point that allocates nothing (osdn_fwd_noalloc).

Some callers cannot allocate device memory when they call the forward: a
plugin whose device memory is owned and budgeted by a host framework, or a
latency-critical loop that must not enter the CUDA allocator (which can
synchronise the device). For them the library offers osdn_fwd_noalloc, which
keeps its scratch in one fixed device array of OSDN_NOALLOC_SCRATCH_BYTES.

This file is collected last on purpose, so a run that stops at the first
failure has run every other test before it. It passes alone in a fresh process
and after the rest of the suite.
"""
import ctypes

import pytest
import torch

from preconditioned_delta_rule_token_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _both(w):
    """Run osdn_fwd (caller workspace) and osdn_fwd_noalloc on the same inputs."""
    import preconditioned_delta_rule_token_b200 as pk
    from preconditioned_delta_rule_token_b200 import _binding as bd
    inp = W.make_forward_inputs(w)
    g = {k: None if v is None else v.cuda() for k, v in inp.items()}
    ref = pk.forward(g["q"], g["k"], g["v"], g["beta"], g["r"], g["d0"], g["S0"], eta=w.eta)
    p = bd.make_params(w.B, w.T, w.H, w.dk, w.dv, g["k"].dtype, w.eta, w.chunk)
    out = torch.empty_like(ref[0])
    S = torch.empty_like(ref[1])
    d = torch.empty_like(ref[2])
    bd.osdn_fwd_noalloc(p, g["q"], g["k"], g["v"], g["beta"], g["r"], g["d0"], g["S0"], out, S, d)
    assert bd.osdn_sync_status() == 0
    return ref, (out, S, d)


def test_noalloc_matches_workspace_forward_on_two_calls_in_a_row():
    # The two entry points launch the same kernels on the same inputs, so their results are
    # bit-identical. The second (smaller) case runs after a larger one, so the shared array
    # still holds stale data beyond its range: equality shows none of it is read.
    cases = [
        W.Workload("na1", 2, 3, 200, 128, 128, 64, W.BF16, True, d0="uniform", S0="normal", eta=0.1, seed=31),
        W.Workload("na2", 1, 2, 130, 64, 128, 64, W.FP32, False, S0="normal", eta=1e-2, seed=32),
        W.Workload("na3", 1, 2, 70, 128, 128, 64, W.BF16, True, d0="uniform", S0="normal", eta=0.1, seed=33),
    ]
    for w in cases:
        ref, got = _both(w)
        for name, a, b in zip(("out", "final_S", "final_d"), got, ref):
            assert torch.equal(a, b), (w.name, name)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from preconditioned_delta_rule_token_b200 import _binding as bd
    L = bd.lib()
    # 8 x 4096 x 16 x 128 bf16 scaled keys = 128 MiB > 32 MiB: rejected before any device work
    p = bd.make_params(8, 4096, 16, 128, 128, torch.bfloat16, 1e-2)
    fake = ctypes.c_void_p(1 << 20)
    rc = L.osdn_fwd_noalloc(ctypes.byref(p), fake, fake, fake, fake, None, None, None, fake, None, None, None)
    assert rc == bd.OSDN_ERR_INVALID_ARG
    assert "OSDN_NOALLOC_SCRATCH_BYTES" in bd.get_last_error()
