"""CPU oracle for the OSDN forward, its backward and the decode step (test
infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library and
its binding in ``preconditioned_delta_rule_token_b200``) never touches it, and
the two share no code.

The arithmetic lives in ``osdn_oracle.c`` (plain float64 C, one host thread per
group of independent (sequence, head) units). This module only compiles it
with gcc and marshals numpy float64 arrays.

Source of the method: "OSDN: Improving Delta Rule with Provable Online
Preconditioning in Linear Attention" (gist.science technical summary,
sections 1, 2.1, 2.2 and 2.3). The readings of the points the pages leave open
are listed at the top of ``osdn_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "osdn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library with gcc (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        lib.osdn_oracle_fwd.argtypes = [ctypes.c_int] * 5 + [ctypes.c_double] + [dp] * 10 + [ctypes.c_int]
        lib.osdn_oracle_fwd.restype = ctypes.c_int
        lib.osdn_oracle_fwd_rho.argtypes = [ctypes.c_int] * 5 + [ctypes.c_double] + [dp] * 11 + [ctypes.c_int]
        lib.osdn_oracle_fwd_rho.restype = ctypes.c_int
        lib.osdn_oracle_fwd_ex.argtypes = ([ctypes.c_int] * 5 + [ctypes.c_double, ctypes.c_int] + [dp] * 12 +
                                           [ctypes.c_int])
        lib.osdn_oracle_fwd_ex.restype = ctypes.c_int
        lib.osdn_oracle_step_ex.argtypes = [ctypes.c_int] * 4 + [ctypes.c_double] + [dp] * 10
        lib.osdn_oracle_step_ex.restype = ctypes.c_int
        lib.osdn_oracle_step.argtypes = [ctypes.c_int] * 4 + [ctypes.c_double] + [dp] * 8
        lib.osdn_oracle_step.restype = ctypes.c_int
        lib.osdn_oracle_bwd_ex.argtypes = ([ctypes.c_int] * 5 + [ctypes.c_double, ctypes.c_int] + [dp] * 19 +
                                           [ctypes.c_int])
        lib.osdn_oracle_bwd_ex.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def fwd(q, k, v, beta, r=None, d0=None, S0=None, eta=1e-2, nthreads=None, anchor=False, alpha=None):
    """Token-by-token OSDN forward in float64 (anchor: anchored APF, retention toward d0;
    alpha [B, T, H]: gated OSDN, S_t = alpha_t S_{t-1} (I - beta k kw^T) + beta v kw^T).

    q, k: [B, T, H, dk]; v: [B, T, H, dv]; beta, r: [B, T, H] (r None = APF off);
    d0: [B, H, dk] (None = ones); S0: [B, H, dv, dk] (None = zeros).
    Returns (out [B, T, H, dv], S_final [B, H, dv, dk], d_final [B, H, dk]).
    """
    q, k, v, beta, r, d0, S0, alpha = map(_f64, (q, k, v, beta, r, d0, S0, alpha))
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    assert q.shape == k.shape and v.shape == (B, T, H, dv) and beta.shape == (B, T, H)
    assert r is None or r.shape == (B, T, H)
    assert alpha is None or alpha.shape == (B, T, H)
    assert d0 is None or d0.shape == (B, H, dk)
    assert S0 is None or S0.shape == (B, H, dv, dk)
    out = np.zeros((B, T, H, dv), np.float64)
    S = np.zeros((B, H, dv, dk), np.float64)
    d = np.zeros((B, H, dk), np.float64)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = _load().osdn_oracle_fwd_ex(B, T, H, dk, dv, float(eta), int(bool(anchor)), _ptr(q), _ptr(k), _ptr(v),
                                    _ptr(beta), _ptr(r), _ptr(alpha), _ptr(d0), _ptr(S0),
                                    _ptr(out), _ptr(S), _ptr(d), None, int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the sizes")
    return out, S, d


def residual_ratio(q, k, v, beta, r=None, d0=None, S0=None, eta=1e-2, nthreads=None, anchor=False):
    """The forward of fwd() plus the per-token residual ratio
    rho_t = (1 - beta_t <d_t, k_t^2>)^2 = f_t(S_t) / f_t(S_{t-1}) [B, T, H] and its
    geometric mean over each sequence, q_geo = exp(mean_t log rho_t) [B, H]
    (1 for an empty sequence). Returns (out, S_final, d_final, rho, q_geo)."""
    q, k, v, beta, r, d0, S0 = map(_f64, (q, k, v, beta, r, d0, S0))
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    assert q.shape == k.shape and v.shape == (B, T, H, dv) and beta.shape == (B, T, H)
    out = np.zeros((B, T, H, dv), np.float64)
    S = np.zeros((B, H, dv, dk), np.float64)
    d = np.zeros((B, H, dk), np.float64)
    rho = np.zeros((B, T, H), np.float64)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = _load().osdn_oracle_fwd_ex(B, T, H, dk, dv, float(eta), int(bool(anchor)), _ptr(q), _ptr(k), _ptr(v),
                                    _ptr(beta), _ptr(r), None, _ptr(d0), _ptr(S0),
                                    _ptr(out), _ptr(S), _ptr(d), _ptr(rho), int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the sizes")
    with np.errstate(divide="ignore"):
        q_geo = np.exp(np.log(rho).mean(axis=1)) if T > 0 else np.ones((B, H))
    return out, S, d, rho, q_geo


def step(q, k, v, beta, S, d, r=None, eta=1e-2, d_anchor=None, alpha=None):
    """One decode token for every (b, h), float64, S [B,H,dv,dk] and d [B,H,dk]
    updated in place (they must be contiguous float64 arrays); d_anchor [B,H,dk]
    selects anchored APF toward it. Returns out [B,H,dv]."""
    q, k, v, beta, r, d_anchor, alpha = map(_f64, (q, k, v, beta, r, d_anchor, alpha))
    assert S.dtype == np.float64 and S.flags.c_contiguous
    assert d.dtype == np.float64 and d.flags.c_contiguous
    B, H, dk = k.shape
    dv = v.shape[-1]
    assert S.shape == (B, H, dv, dk) and d.shape == (B, H, dk)
    out = np.zeros((B, H, dv), np.float64)
    rc = _load().osdn_oracle_step_ex(B, H, dk, dv, float(eta), _ptr(q), _ptr(k), _ptr(v),
                                     _ptr(beta), _ptr(r), _ptr(alpha), _ptr(d_anchor), _ptr(S), _ptr(d), _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected the sizes")
    return out


def bwd(q, k, v, beta, dout, r=None, d0=None, S0=None, dS_final=None, dd_final=None, eta=1e-2,
        nthreads=None, anchor=False, alpha=None):
    """Reverse-mode gradients of fwd() in float64, token by token.

    The loss is L = sum(dout * out) + sum(dS_final * S_final) + sum(dd_final * d_final)
    (dS_final, dd_final None = 0). Returns a dict with dq, dk [B,T,H,dk], dv [B,T,H,dv],
    dbeta [B,T,H], dr [B,T,H] (None without r), dalpha [B,T,H] (None without alpha),
    dd0 [B,H,dk] and dS0 [B,H,dv,dk]. The adjoint formulas are written out at the top of
    osdn_oracle.c.
    """
    q, k, v, beta, r, d0, S0, alpha, dout, dS_final, dd_final = map(
        _f64, (q, k, v, beta, r, d0, S0, alpha, dout, dS_final, dd_final))
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    assert q.shape == k.shape and v.shape == (B, T, H, dv) and beta.shape == (B, T, H)
    assert dout.shape == (B, T, H, dv)
    assert r is None or r.shape == (B, T, H)
    assert alpha is None or alpha.shape == (B, T, H)
    assert d0 is None or d0.shape == (B, H, dk)
    assert S0 is None or S0.shape == (B, H, dv, dk)
    assert dS_final is None or dS_final.shape == (B, H, dv, dk)
    assert dd_final is None or dd_final.shape == (B, H, dk)
    g = {"dq": np.zeros((B, T, H, dk)), "dk": np.zeros((B, T, H, dk)), "dv": np.zeros((B, T, H, dv)),
         "dbeta": np.zeros((B, T, H)), "dr": None if r is None else np.zeros((B, T, H)),
         "dalpha": None if alpha is None else np.zeros((B, T, H)),
         "dd0": np.zeros((B, H, dk)), "dS0": np.zeros((B, H, dv, dk))}
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = _load().osdn_oracle_bwd_ex(B, T, H, dk, dv, float(eta), int(bool(anchor)), _ptr(q), _ptr(k), _ptr(v),
                                    _ptr(beta), _ptr(r), _ptr(alpha), _ptr(d0), _ptr(S0),
                                    _ptr(dout), _ptr(dS_final), _ptr(dd_final),
                                    _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dbeta"]),
                                    _ptr(g["dr"]), _ptr(g["dalpha"]), _ptr(g["dd0"]), _ptr(g["dS0"]),
                                    int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the sizes")
    return g
