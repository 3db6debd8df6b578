"""ctypes binding of libosdn.so (argument marshalling only).

Every arithmetic step runs in the library's CUDA kernels; this module checks
tensors, builds the ``osdn_params`` block and passes raw device pointers and
the current CUDA stream. It raises if the library is missing or the tensors
are not on a CUDA device: there is no CPU path.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
_ROOT = os.path.dirname(_PKG)
_CSRC = os.path.join(_PKG, "csrc")
_INCLUDE = os.path.join(_ROOT, "include")
LIB_PATH = os.path.join(_PKG, "libosdn.so")

OSDN_OK, OSDN_ERR_INVALID_ARG, OSDN_ERR_UNSUPPORTED, OSDN_ERR_CUDA, OSDN_ERR_TIMEOUT = range(5)
OSDN_BF16, OSDN_FP32 = 0, 1
OSDN_NOALLOC_SCRATCH_BYTES = 32 << 20

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared", "-cudart", "static", "--expt-relaxed-constexpr"]


class osdn_params(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("B", ctypes.c_int32), ("T", ctypes.c_int32),
                ("H", ctypes.c_int32), ("dk", ctypes.c_int32), ("dv", ctypes.c_int32),
                ("chunk", ctypes.c_int32), ("dtype", ctypes.c_int32), ("eta", ctypes.c_float),
                ("apf_anchor", ctypes.c_int32), ("stride_q", ctypes.c_int64 * 3), ("stride_k", ctypes.c_int64 * 3),
                ("stride_v", ctypes.c_int64 * 3), ("stride_o", ctypes.c_int64 * 3)]


class OsdnError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__("osdn error %d: %s" % (code, msg))
        self.code = code


def _sources():
    return sorted(os.path.join(_CSRC, f) for f in os.listdir(_CSRC) if f.endswith((".cu", ".cuh")))


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libosdn.so in-tree for sm_100a with nvcc."""
    deps = _sources() + [os.path.join(_INCLUDE, "osdn.h")]
    if not force and os.path.exists(LIB_PATH):
        if os.path.getmtime(LIB_PATH) >= max(os.path.getmtime(p) for p in deps):
            return LIB_PATH
    tmp = LIB_PATH + ".tmp%d" % os.getpid()
    cmd = ["nvcc"] + NVCC_FLAGS + ["-I", _INCLUDE, "-I", _CSRC, "-o", tmp, os.path.join(_CSRC, "osdn_api.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


def build_if_missing() -> str:
    return build(force=False)


_lib = None


def lib():
    """The loaded library (raises if it was never built)."""
    global _lib
    if _lib is None:
        try:
            build(force=False)          # rebuild in-tree when a source is newer than the library
        except (OSError, subprocess.CalledProcessError) as exc:
            if not os.path.exists(LIB_PATH):
                raise OsdnError(OSDN_ERR_UNSUPPORTED, "libosdn.so is not built and nvcc failed: %s" % exc)
        L = ctypes.CDLL(LIB_PATH)
        vp, sz = ctypes.c_void_p, ctypes.c_size_t
        P = ctypes.POINTER(osdn_params)
        L.osdn_fwd_workspace_size.argtypes = [P, ctypes.POINTER(sz)]
        L.osdn_fwd_workspace_size.restype = ctypes.c_int
        L.osdn_fwd_segments.argtypes = [P, ctypes.POINTER(ctypes.c_int)]
        L.osdn_fwd_segments.restype = ctypes.c_int
        L.osdn_fwd_launches.argtypes = [P, ctypes.POINTER(ctypes.c_int)]
        L.osdn_fwd_launches.restype = ctypes.c_int
        L.osdn_fwd.argtypes = [P] + [vp] * 10 + [vp, sz, vp]
        L.osdn_fwd.restype = ctypes.c_int
        L.osdn_fwd_scan.argtypes = [P] + [vp] * 5 + [vp, sz, vp]
        L.osdn_fwd_scan.restype = ctypes.c_int
        L.osdn_fwd_scan_diag.argtypes = [P] + [vp] * 7 + [vp, sz, vp]
        L.osdn_fwd_scan_diag.restype = ctypes.c_int
        L.osdn_fwd_chunk.argtypes = [P] + [vp] * 7 + [vp, sz, vp]
        L.osdn_fwd_chunk.restype = ctypes.c_int
        L.osdn_fwd_noalloc.argtypes = [P] + [vp] * 10 + [vp]
        L.osdn_fwd_noalloc.restype = ctypes.c_int
        L.osdn_step.argtypes = [P] + [vp] * 8 + [vp]
        L.osdn_step.restype = ctypes.c_int
        L.osdn_step_ex.argtypes = [P] + [vp] * 9 + [vp]
        L.osdn_step_ex.restype = ctypes.c_int
        L.osdn_step_gated.argtypes = [P] + [vp] * 10 + [vp]
        L.osdn_step_gated.restype = ctypes.c_int
        L.osdn_fwd_gated.argtypes = [P] + [vp] * 11 + [vp, sz, vp]
        L.osdn_fwd_gated.restype = ctypes.c_int
        L.osdn_fwd_chunk_gated.argtypes = [P] + [vp] * 8 + [vp, sz, vp]
        L.osdn_fwd_chunk_gated.restype = ctypes.c_int
        L.osdn_fwd_host_buffer_size.argtypes = [P, ctypes.c_int, ctypes.POINTER(sz)]
        L.osdn_fwd_host_buffer_size.restype = ctypes.c_int
        L.osdn_fwd_host.argtypes = [P] + [vp] * 10 + [vp, sz, ctypes.c_int, vp]
        L.osdn_fwd_host.restype = ctypes.c_int
        L.osdn_bwd_workspace_size.argtypes = [P, ctypes.POINTER(sz)]
        L.osdn_bwd_workspace_size.restype = ctypes.c_int
        L.osdn_bwd.argtypes = [P] + [vp] * 17 + [vp, sz, vp]
        L.osdn_bwd.restype = ctypes.c_int
        L.osdn_bwd_gated.argtypes = [P] + [vp] * 20 + [sz, vp]
        L.osdn_bwd_gated.restype = ctypes.c_int
        L.osdn_sync_status.argtypes = [vp]
        L.osdn_sync_status.restype = ctypes.c_int
        L.osdn_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
        L.osdn_set_wait_limit_ns.restype = None
        L.osdn_get_last_error.argtypes = []
        L.osdn_get_last_error.restype = ctypes.c_char_p
        L.osdn_abi_version.argtypes = []
        L.osdn_abi_version.restype = ctypes.c_int
        _lib = L
    return _lib


def get_last_error() -> str:
    return lib().osdn_get_last_error().decode()


def _check(rc):
    if rc != OSDN_OK:
        raise OsdnError(rc, get_last_error())


def make_params(B, T, H, dk, dv, dtype, eta, chunk=64, apf_anchor=False) -> osdn_params:
    p = osdn_params()
    p.struct_size = ctypes.sizeof(osdn_params)
    p.B, p.T, p.H, p.dk, p.dv, p.chunk = int(B), int(T), int(H), int(dk), int(dv), int(chunk)
    p.dtype = OSDN_BF16 if dtype == torch.bfloat16 else OSDN_FP32
    p.eta = float(eta)
    p.apf_anchor = 1 if apf_anchor else 0
    return p


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise OsdnError(OSDN_ERR_INVALID_ARG, "tensor is not on a CUDA device (the library has no CPU path)")
    if not t.is_contiguous():
        raise OsdnError(OSDN_ERR_INVALID_ARG, "tensor is not contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _ptr_tok(t):
    """Pointer of a token tensor [B, T, H, width] that may be a strided view (last dimension contiguous);
    its other strides go into the parameter block (_set_strides)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise OsdnError(OSDN_ERR_INVALID_ARG, "tensor is not on a CUDA device (the library has no CPU path)")
    if t.dim() != 4 or (t.numel() > 0 and t.stride(-1) != 1):
        raise OsdnError(OSDN_ERR_INVALID_ARG, "token tensors are [B, T, H, width] with the last dimension contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _host_ptr(t):
    """Pointer of a dense host tensor (page-locked memory lets its copies overlap; pageable works too)."""
    if t is None:
        return None
    if t.is_cuda:
        raise OsdnError(OSDN_ERR_INVALID_ARG, "osdn_fwd_host takes host tensors (the device data lives in device_buffer)")
    if not t.is_contiguous():
        raise OsdnError(OSDN_ERR_INVALID_ARG, "tensor is not contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _set_strides(params, q=None, k=None, v=None, out=None):
    """Copy the (b, t, h) element strides of q, k, v, out into params (zeros: dense)."""
    for name, t in (("stride_q", q), ("stride_k", k), ("stride_v", v), ("stride_o", out)):
        dense = t is None or t.is_contiguous()
        getattr(params, name)[:] = (0, 0, 0) if dense else (t.stride(0), t.stride(1), t.stride(2))
    return params


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def osdn_fwd_workspace_size(params: osdn_params) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().osdn_fwd_workspace_size(ctypes.byref(params), ctypes.byref(n)))
    return n.value


def osdn_fwd_launches(params: osdn_params) -> int:
    """Kernel launches of one osdn_fwd call with these parameters."""
    n = ctypes.c_int(0)
    _check(lib().osdn_fwd_launches(ctypes.byref(params), ctypes.byref(n)))
    return n.value


def osdn_fwd_segments(params: osdn_params) -> int:
    """Segments per sequence that phase 2 splits into (1: none)."""
    n = ctypes.c_int(0)
    _check(lib().osdn_fwd_segments(ctypes.byref(params), ctypes.byref(n)))
    return n.value


def osdn_fwd(params, q, k, v, beta, r, d0, S0, out, final_S, final_d, workspace, stream=None):
    """Raw C-ABI call: every tensor preallocated by the caller (device memory)."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _set_strides(params, q, k, v, out)
    _check(lib().osdn_fwd(ctypes.byref(params), _ptr_tok(q), _ptr_tok(k), _ptr_tok(v), _ptr(beta), _ptr(r), _ptr(d0),
                          _ptr(S0), _ptr_tok(out), _ptr(final_S), _ptr(final_d), _ptr(workspace), ctypes.c_size_t(ws_bytes),
                          _stream(stream)))


def _ws_bytes(workspace):
    return 0 if workspace is None else workspace.numel() * workspace.element_size()


def osdn_fwd_host_buffer_size(params: osdn_params, groups: int = 0) -> int:
    """Bytes of the device buffer osdn_fwd_host needs for these parameters and group count."""
    n = ctypes.c_size_t(0)
    _check(lib().osdn_fwd_host_buffer_size(ctypes.byref(params), ctypes.c_int(int(groups)), ctypes.byref(n)))
    return n.value


def osdn_fwd_host(params, q, k, v, beta, r, d0, S0, out, final_S, final_d, device_buffer, groups=0, stream=None):
    """Raw C-ABI call: inputs and outputs are dense HOST tensors, device_buffer a CUDA tensor of at
    least osdn_fwd_host_buffer_size bytes."""
    _check(lib().osdn_fwd_host(ctypes.byref(params), _host_ptr(q), _host_ptr(k), _host_ptr(v), _host_ptr(beta),
                               _host_ptr(r), _host_ptr(d0), _host_ptr(S0), _host_ptr(out), _host_ptr(final_S),
                               _host_ptr(final_d), _ptr(device_buffer), ctypes.c_size_t(_ws_bytes(device_buffer)),
                               ctypes.c_int(int(groups)), _stream(stream)))


def osdn_fwd_scan(params, k, beta, r, d0, final_d, workspace, stream=None):
    """Raw C-ABI call of phase 1 (preconditioner scan into the workspace)."""
    _set_strides(params, k=k)
    _check(lib().osdn_fwd_scan(ctypes.byref(params), _ptr_tok(k), _ptr(beta), _ptr(r), _ptr(d0), _ptr(final_d),
                               _ptr(workspace), ctypes.c_size_t(_ws_bytes(workspace)), _stream(stream)))


def osdn_fwd_scan_diag(params, k, beta, r, d0, final_d, rho, q_geo, workspace, stream=None):
    """Raw C-ABI call of phase 1 with the residual-ratio diagnostic (rho, q_geo nullable)."""
    _set_strides(params, k=k)
    _check(lib().osdn_fwd_scan_diag(ctypes.byref(params), _ptr_tok(k), _ptr(beta), _ptr(r), _ptr(d0), _ptr(final_d),
                                    _ptr(rho), _ptr(q_geo), _ptr(workspace), ctypes.c_size_t(_ws_bytes(workspace)),
                                    _stream(stream)))


def osdn_fwd_chunk(params, q, k, v, beta, S0, out, final_S, workspace, stream=None):
    """Raw C-ABI call of phase 2 (chunked delta rule reading the workspace)."""
    _set_strides(params, q, k, v, out)
    _check(lib().osdn_fwd_chunk(ctypes.byref(params), _ptr_tok(q), _ptr_tok(k), _ptr_tok(v), _ptr(beta), _ptr(S0),
                                _ptr_tok(out),
                                _ptr(final_S), _ptr(workspace), ctypes.c_size_t(_ws_bytes(workspace)),
                                _stream(stream)))


def osdn_fwd_noalloc(params, q, k, v, beta, r, d0, S0, out, final_S, final_d, stream=None):
    """Raw C-ABI call of the forward that takes no workspace: the library uses
    its own fixed scratch array (see OSDN_NOALLOC_SCRATCH_BYTES in osdn.h)."""
    _set_strides(params, q, k, v, out)
    _check(lib().osdn_fwd_noalloc(ctypes.byref(params), _ptr_tok(q), _ptr_tok(k), _ptr_tok(v), _ptr(beta), _ptr(r),
                                  _ptr(d0), _ptr(S0), _ptr_tok(out), _ptr(final_S), _ptr(final_d), _stream(stream)))


def osdn_step(params, q, k, v, beta, r, S, d, out, stream=None):
    """Raw C-ABI call: one decode token for every (b, h); S and d updated in place."""
    _check(lib().osdn_step(ctypes.byref(params), _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(r), _ptr(S), _ptr(d),
                           _ptr(out), _stream(stream)))


def osdn_step_ex(params, q, k, v, beta, r, d_anchor, S, d, out, stream=None):
    """Raw C-ABI call: osdn_step with anchored APF toward d_anchor when params.apf_anchor is set."""
    _check(lib().osdn_step_ex(ctypes.byref(params), _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(r), _ptr(d_anchor),
                              _ptr(S), _ptr(d), _ptr(out), _stream(stream)))


def osdn_fwd_gated(params, q, k, v, beta, r, alpha, d0, S0, out, final_S, final_d, workspace, stream=None):
    """Raw C-ABI call of the gated forward (alpha decay of the state)."""
    _set_strides(params, q, k, v, out)
    _check(lib().osdn_fwd_gated(ctypes.byref(params), _ptr_tok(q), _ptr_tok(k), _ptr_tok(v), _ptr(beta), _ptr(r),
                                _ptr(alpha), _ptr(d0), _ptr(S0), _ptr_tok(out), _ptr(final_S), _ptr(final_d),
                                _ptr(workspace),
                                ctypes.c_size_t(_ws_bytes(workspace)), _stream(stream)))


def osdn_fwd_chunk_gated(params, q, k, v, beta, alpha, S0, out, final_S, workspace, stream=None):
    """Raw C-ABI call of phase 2 of the gated forward."""
    _set_strides(params, q, k, v, out)
    _check(lib().osdn_fwd_chunk_gated(ctypes.byref(params), _ptr_tok(q), _ptr_tok(k), _ptr_tok(v), _ptr(beta),
                                      _ptr(alpha), _ptr(S0), _ptr_tok(out), _ptr(final_S), _ptr(workspace),
                                      ctypes.c_size_t(_ws_bytes(workspace)), _stream(stream)))


def osdn_step_gated(params, q, k, v, beta, r, alpha, d_anchor, S, d, out, stream=None):
    """Raw C-ABI call: one gated decode token for every (b, h)."""
    _check(lib().osdn_step_gated(ctypes.byref(params), _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(r), _ptr(alpha),
                                 _ptr(d_anchor), _ptr(S), _ptr(d), _ptr(out), _stream(stream)))


def osdn_bwd_workspace_size(params: osdn_params) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().osdn_bwd_workspace_size(ctypes.byref(params), ctypes.byref(n)))
    return n.value


def osdn_bwd(params, q, k, v, beta, r, d0, S0, dout, dS_final, dd_final, dq, dk, dv, dbeta, dr, dd0, dS0, workspace,
             stream=None):
    """Raw C-ABI call of the backward: every tensor preallocated by the caller (device memory)."""
    _check(lib().osdn_bwd(ctypes.byref(params), _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(r), _ptr(d0), _ptr(S0),
                          _ptr(dout), _ptr(dS_final), _ptr(dd_final), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dbeta),
                          _ptr(dr), _ptr(dd0), _ptr(dS0), _ptr(workspace), ctypes.c_size_t(_ws_bytes(workspace)),
                          _stream(stream)))


def osdn_bwd_gated(params, q, k, v, beta, r, alpha, d0, S0, dout, dS_final, dd_final, dq, dk, dv, dbeta, dr, dalpha,
                   dd0, dS0, workspace, stream=None):
    """Raw C-ABI call of the gated backward: as osdn_bwd plus alpha [B,T,H] and dalpha [B,T,H]."""
    _check(lib().osdn_bwd_gated(ctypes.byref(params), _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(r), _ptr(alpha),
                                _ptr(d0), _ptr(S0), _ptr(dout), _ptr(dS_final), _ptr(dd_final), _ptr(dq), _ptr(dk),
                                _ptr(dv), _ptr(dbeta), _ptr(dr), _ptr(dalpha), _ptr(dd0), _ptr(dS0), _ptr(workspace),
                                ctypes.c_size_t(_ws_bytes(workspace)), _stream(stream)))


def osdn_sync_status(stream=None) -> int:
    return lib().osdn_sync_status(_stream(stream))


def osdn_set_wait_limit_ns(ns: int) -> None:
    """Upper bound on any device-side wait of kernels launched afterwards (0 = the 4 s default)."""
    lib().osdn_set_wait_limit_ns(int(ns))
