"""The C-ABI library: it builds, loads without a GPU, exports every entry
point declared in include/osdn.h, and rejects bad arguments on the host
before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(osdn_\w+)\s*\(", text))
    return names


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("osdn_fwd", "osdn_step", "osdn_fwd_workspace_size", "osdn_get_last_error"):
        assert required in names


def test_library_exports_every_declared_symbol(osdn_lib):
    lib = ctypes.CDLL(osdn_lib.LIB_PATH)
    for name in sorted(_declared_functions()):
        assert hasattr(lib, name), name
    assert lib.osdn_abi_version() == 3


def test_earlier_params_versions_are_accepted(osdn_lib):
    """osdn_params of ABI version 1 ended after eta (36 bytes) and version 2 after
    apf_anchor (40 bytes); such callers are accepted (plain APF for version 1, the
    dense layout for both). Version 3 appends the (b, t, h) element strides of q,
    k, v and out (136 bytes); any other size is refused."""
    L = osdn_lib.lib()
    n = ctypes.c_size_t(0)
    assert ctypes.sizeof(osdn_lib.osdn_params) == 136
    assert osdn_lib.osdn_params.stride_q.offset == 40
    p = _params(osdn_lib)
    for size in (36, 40, 136):
        p.struct_size = size
        p.apf_anchor = 1
        assert L.osdn_fwd_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 0, size
    p.struct_size = 44
    assert L.osdn_fwd_workspace_size(ctypes.byref(p), ctypes.byref(n)) == osdn_lib.OSDN_ERR_INVALID_ARG


def test_strides_are_checked_on_the_host(osdn_lib):
    """Strides are non-negative multiples of 8 elements; the decode step and the
    backward take dense tensors only."""
    L = osdn_lib.lib()
    n = ctypes.c_size_t(0)
    fake = ctypes.c_void_p(1 << 20)             # never dereferenced: checks fail first
    for bad in ((4, 0, 0), (-8, 0, 0), (0, 0, 1 << 40)):
        p = _params(osdn_lib)
        p.stride_k[:] = bad
        assert L.osdn_fwd_workspace_size(ctypes.byref(p), ctypes.byref(n)) == osdn_lib.OSDN_ERR_INVALID_ARG, bad
        assert "stride" in osdn_lib.get_last_error()
    p = _params(osdn_lib)
    p.stride_q[:] = (100 * 3 * 384, 3 * 384, 384)   # q as a column slice of a fused [B, T, H, 384] projection
    assert L.osdn_fwd_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 0
    assert L.osdn_step(ctypes.byref(p), fake, fake, fake, fake, None, fake, fake, fake, None) == \
        osdn_lib.OSDN_ERR_UNSUPPORTED
    assert L.osdn_bwd(ctypes.byref(p), *([fake] * 4), None, None, None, fake, None, None, *([fake] * 4), None, None,
                      None, fake, ctypes.c_size_t(1 << 40), None) == osdn_lib.OSDN_ERR_UNSUPPORTED


def _params(osdn_lib, **kw):
    import torch
    a = dict(B=2, T=100, H=3, dk=128, dv=64, dtype=torch.bfloat16, eta=1e-2, chunk=64)
    a.update(kw)
    return osdn_lib.make_params(**a)


def test_workspace_size_and_argument_checks(osdn_lib):
    L = osdn_lib.lib()
    n = ctypes.c_size_t(0)
    p = _params(osdn_lib)
    assert L.osdn_fwd_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 0
    assert n.value >= 2 * 100 * 3 * 128 * 2 and n.value % 256 == 0
    bad = _params(osdn_lib)
    bad.struct_size = 8
    assert L.osdn_fwd_workspace_size(ctypes.byref(bad), ctypes.byref(n)) == osdn_lib.OSDN_ERR_INVALID_ARG
    assert "struct_size" in osdn_lib.get_last_error()
    for kw, code in ((dict(dk=96), osdn_lib.OSDN_ERR_UNSUPPORTED), (dict(chunk=32), osdn_lib.OSDN_ERR_UNSUPPORTED),
                     (dict(B=0), osdn_lib.OSDN_ERR_INVALID_ARG), (dict(T=-1), osdn_lib.OSDN_ERR_INVALID_ARG),
                     (dict(eta=float("nan")), osdn_lib.OSDN_ERR_INVALID_ARG)):
        p = _params(osdn_lib, **kw)
        assert L.osdn_fwd_workspace_size(ctypes.byref(p), ctypes.byref(n)) == code, kw
        assert osdn_lib.get_last_error() != ""


def test_null_and_misaligned_pointers_are_rejected_on_the_host(osdn_lib):
    L = osdn_lib.lib()
    p = _params(osdn_lib)
    fake = ctypes.c_void_p(1 << 20)             # never dereferenced: checks fail first
    rc = L.osdn_fwd(ctypes.byref(p), None, fake, fake, fake, None, None, None, fake, None, None, fake,
                    ctypes.c_size_t(1 << 30), None)
    assert rc == osdn_lib.OSDN_ERR_INVALID_ARG and "NULL" in osdn_lib.get_last_error()
    odd = ctypes.c_void_p((1 << 20) + 4)
    rc = L.osdn_fwd(ctypes.byref(p), fake, odd, fake, fake, None, None, None, fake, None, None, fake,
                    ctypes.c_size_t(1 << 30), None)
    assert rc == osdn_lib.OSDN_ERR_INVALID_ARG and "aligned" in osdn_lib.get_last_error()
    rc = L.osdn_fwd(ctypes.byref(p), fake, fake, fake, fake, None, None, None, fake, None, None, fake,
                    ctypes.c_size_t(16), None)
    assert rc == osdn_lib.OSDN_ERR_INVALID_ARG and "workspace" in osdn_lib.get_last_error()
    rc = L.osdn_step(ctypes.byref(p), fake, fake, fake, fake, None, None, fake, fake, None)
    assert rc == osdn_lib.OSDN_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors(osdn_lib):
    import torch
    import preconditioned_delta_rule_token_b200 as pk
    x = torch.zeros((1, 4, 1, 64), dtype=torch.bfloat16)
    with pytest.raises(pk.OsdnError):
        pk.forward(x, x, x, torch.zeros((1, 4, 1), dtype=torch.bfloat16))


def test_binding_copies_the_strides_of_views(osdn_lib):
    """A column slice of a fused projection passes its (b, t, h) strides in the
    parameter block; a contiguous tensor passes zeros (dense)."""
    import torch
    fused = torch.zeros((2, 5, 3, 3 * 64))
    q, k = fused[..., :64], fused[..., 64:128]
    p = _params(osdn_lib, T=5, dk=64, dv=64)
    osdn_lib._set_strides(p, q=q, k=k.contiguous())
    assert tuple(p.stride_q) == (5 * 3 * 192, 3 * 192, 192) and tuple(p.stride_k) == (0, 0, 0)


def test_backward_workspace_and_argument_checks(osdn_lib):
    L = osdn_lib.lib()
    p = _params(osdn_lib)
    n = ctypes.c_size_t(0)
    assert L.osdn_bwd_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 0
    # fp32 chunk intermediates: at least d_t, Kw, W, dD and dK per token and head (5 * dk floats)
    assert n.value >= 5 * p.B * p.T * p.H * p.dk * 4 and n.value % 256 == 0
    fake = ctypes.c_void_p(1 << 20)             # never dereferenced: checks fail first
    args = [fake] * 4 + [None] * 3 + [fake, None, None] + [fake] * 4 + [None] * 3
    rc = L.osdn_bwd(ctypes.byref(p), *args, fake, ctypes.c_size_t(n.value - 256), None)
    assert rc == osdn_lib.OSDN_ERR_INVALID_ARG and "workspace" in osdn_lib.get_last_error()
    rc = L.osdn_bwd(ctypes.byref(p), *args[:7], None, *args[8:], fake, n, None)     # dout NULL
    assert rc == osdn_lib.OSDN_ERR_INVALID_ARG and "NULL" in osdn_lib.get_last_error()
    odd = ctypes.c_void_p((1 << 20) + 8)
    rc = L.osdn_bwd(ctypes.byref(p), *args[:-4], odd, *args[-3:], fake, n, None)       # dbeta misaligned
    assert rc == osdn_lib.OSDN_ERR_INVALID_ARG and "aligned" in osdn_lib.get_last_error()
    bad = _params(osdn_lib, dk=96)
    assert L.osdn_bwd_workspace_size(ctypes.byref(bad), ctypes.byref(n)) == osdn_lib.OSDN_ERR_UNSUPPORTED


def test_new_entry_points_check_their_arguments_on_the_host(osdn_lib):
    """osdn_bwd_gated refuses a NULL alpha or dalpha (T > 0) before touching the device;
    osdn_fwd_segments and osdn_fwd_launches refuse NULL outputs and report the plan."""
    L = osdn_lib.lib()
    fake = ctypes.c_void_p(1 << 20)             # never dereferenced: checks fail first
    p = _params(osdn_lib)
    args = [ctypes.byref(p)] + [fake] * 5        # q, k, v, beta, r
    tail = [None, None, fake, None, None, fake, fake, fake, fake, None]   # d0, S0, dout, dS_f, dd_f, dq..dbeta, dr
    for alpha, dalpha in ((None, fake), (fake, None)):
        rc = L.osdn_bwd_gated(*args, alpha, *tail, dalpha, None, None, fake, ctypes.c_size_t(1 << 40), None)
        assert rc == osdn_lib.OSDN_ERR_INVALID_ARG
        assert b"alpha" in L.osdn_get_last_error()
    n = ctypes.c_int(0)
    assert L.osdn_fwd_segments(ctypes.byref(p), None) == osdn_lib.OSDN_ERR_INVALID_ARG
    assert L.osdn_fwd_launches(ctypes.byref(p), None) == osdn_lib.OSDN_ERR_INVALID_ARG
    assert L.osdn_fwd_launches(ctypes.byref(p), ctypes.byref(n)) == 0 and n.value >= 1
    one_seq = osdn_lib.make_params(1, 32768, 16, 128, 128, __import__("torch").bfloat16, 1e-2)
    assert osdn_lib.osdn_fwd_segments(one_seq) == 16
    assert osdn_lib.osdn_fwd_launches(one_seq) == 2 + 5 * 4      # batches of 4 segments over 0 .. 14
    anchored = osdn_lib.make_params(1, 32768, 16, 128, 128, __import__("torch").bfloat16, 1e-2, 64, True)
    assert osdn_lib.osdn_fwd_launches(anchored) == 6              # split, not overlapped
    layer = osdn_lib.make_params(8, 4096, 16, 128, 128, __import__("torch").bfloat16, 1e-2)
    assert osdn_lib.osdn_fwd_segments(layer) == 1 and osdn_lib.osdn_fwd_launches(layer) == 2


def test_fwd_host_checks_on_the_host():
    """osdn_fwd_host and its buffer size: argument checks that finish before any device call."""
    import ctypes
    import torch
    import preconditioned_delta_rule_token_b200 as pk
    from preconditioned_delta_rule_token_b200 import _binding as b
    L = b.lib()
    p = pk.make_params(8, 4096, 16, 128, 128, torch.bfloat16, 1e-2)
    sizes = {g: pk.osdn_fwd_host_buffer_size(p, g) for g in (0, 1, 2, 4, 8, 64)}
    tok = 8 * 4096 * 16
    inputs = tok * 128 * 2 * 4 + tok * 2 * 2          # q, k, v, out; beta, r
    for g, n in sizes.items():
        assert n >= inputs and n % 256 == 0, (g, n)
    assert sizes[0] == sizes[8]                         # the default is min(B, 8) groups
    assert sizes[64] == sizes[8]                        # at most one group per sequence
    dummy = ctypes.c_void_p(1 << 20)
    args = [ctypes.byref(p)] + [dummy] * 5 + [None, None] + [dummy, None, None]
    rc = L.osdn_fwd_host(*args, None, ctypes.c_size_t(sizes[0]), 0, None)
    assert rc == pk.OSDN_ERR_INVALID_ARG and "device_buffer" in pk.get_last_error()
    rc = L.osdn_fwd_host(*args, ctypes.c_void_p(1 << 21), ctypes.c_size_t(sizes[0] - 256), 0, None)
    assert rc == pk.OSDN_ERR_INVALID_ARG and "too small" in pk.get_last_error()
    ps = pk.make_params(8, 4096, 16, 128, 128, torch.bfloat16, 1e-2)
    ps.stride_q[0], ps.stride_q[1], ps.stride_q[2] = 4096 * 16 * 384, 16 * 384, 384
    rc = L.osdn_fwd_host(ctypes.byref(ps), *args[1:], ctypes.c_void_p(1 << 21), ctypes.c_size_t(sizes[0]), 0, None)
    assert rc == pk.OSDN_ERR_UNSUPPORTED
