"""OSDN (Online Scaled DeltaNet) forward, backward and decode on B200 (sm_100a).

The compute lives in ``libosdn.so`` (CUDA kernels behind the C ABI of
``include/osdn.h``); this package is its ctypes binding plus two convenience
wrappers that allocate outputs and workspace with PyTorch:

    out, S, d = forward(q, k, v, beta, r=None, d0=None, S0=None, eta=1e-2)
    grads = backward(q, k, v, beta, dout, r=None, d0=None, S0=None, eta=1e-2)
    o = step(q, k, v, beta, S, d, r=None, eta=1e-2)      # S, d updated in place

All tensors must be CUDA tensors; there is no CPU path.
"""
from __future__ import annotations

import torch

from ._binding import (OSDN_BF16, OSDN_ERR_CUDA, OSDN_ERR_INVALID_ARG, OSDN_ERR_TIMEOUT, OSDN_ERR_UNSUPPORTED,
                       OSDN_FP32, OSDN_OK, LIB_PATH, OsdnError, build, get_last_error, make_params, osdn_fwd,
                       osdn_fwd_chunk, osdn_fwd_scan, osdn_fwd_scan_diag,
                       osdn_fwd_workspace_size, osdn_fwd_segments, osdn_fwd_launches, osdn_params, osdn_set_wait_limit_ns, osdn_step, osdn_step_ex,
                       osdn_fwd_gated, osdn_fwd_chunk_gated, osdn_step_gated,
                       osdn_bwd, osdn_bwd_gated, osdn_bwd_workspace_size, osdn_sync_status,
                       osdn_fwd_host, osdn_fwd_host_buffer_size)

__all__ = ["forward", "backward", "step", "osdn_bwd", "osdn_bwd_gated", "osdn_bwd_workspace_size", "residual_ratio", "osdn_fwd_scan_diag", "osdn_fwd", "osdn_fwd_scan", "osdn_fwd_chunk", "osdn_step", "osdn_fwd_workspace_size", "osdn_fwd_segments", "osdn_fwd_launches", "osdn_sync_status",
           "osdn_set_wait_limit_ns", "osdn_step_ex",
           "osdn_fwd_gated", "osdn_fwd_chunk_gated", "osdn_step_gated", "osdn_fwd_host", "osdn_fwd_host_buffer_size",
           "forward_host", "osdn_params", "make_params", "get_last_error", "OsdnError", "build", "LIB_PATH",
           "OSDN_OK", "OSDN_ERR_INVALID_ARG", "OSDN_ERR_UNSUPPORTED", "OSDN_ERR_CUDA", "OSDN_ERR_TIMEOUT",
           "OSDN_BF16", "OSDN_FP32"]


def forward(q, k, v, beta, r=None, d0=None, S0=None, eta=1e-2, chunk=64, workspace=None, stream=None,
            apf_anchor=False, alpha=None):
    """OSDN forward. q, k [B,T,H,dk]; v [B,T,H,dv]; beta, r [B,T,H] (bf16 or fp32,
    one dtype); d0 [B,H,dk] and S0 [B,H,dv,dk] fp32 or None. apf_anchor: anchored
    APF, the retention pulls d toward d0 instead of 0. alpha [B,T,H] (same dtype): gated OSDN,
    S_t = alpha_t S_{t-1} (I - beta k kw^T) + beta v kw^T (bf16, dk = dv = 128).
    Returns (out [B,T,H,dv], final_S [B,H,dv,dk] fp32, final_d [B,H,dk] fp32)."""
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    p = make_params(B, T, H, dk, dv, k.dtype, eta, chunk, apf_anchor)
    dev = k.device
    out = torch.empty((B, T, H, dv), dtype=k.dtype, device=dev)
    final_S = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    final_d = torch.empty((B, H, dk), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(osdn_fwd_workspace_size(p), dtype=torch.uint8, device=dev)
    if alpha is None:
        osdn_fwd(p, q, k, v, beta, r, d0, S0, out, final_S, final_d, workspace, stream)
    else:
        osdn_fwd_gated(p, q, k, v, beta, r, alpha, d0, S0, out, final_S, final_d, workspace, stream)
    return out, final_S, final_d


def forward_host(q, k, v, beta, r=None, d0=None, S0=None, eta=1e-2, chunk=64, groups=0, device_buffer=None,
                 stream=None, apf_anchor=False):
    """forward() on HOST tensors (page-locked for overlapped copies): the library copies each group of
    sequences in, runs the forward on it and copies its results back, with the copies of one group
    overlapping the compute of its neighbours (osdn_fwd_host). groups = 0: the library's default.
    Returns host tensors (out, final_S, final_d); the call is asynchronous on `stream`."""
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    p = make_params(B, T, H, dk, dv, k.dtype, eta, chunk, apf_anchor)
    pin = q.is_pinned()
    out = torch.empty((B, T, H, dv), dtype=k.dtype, pin_memory=pin)
    final_S = torch.empty((B, H, dv, dk), dtype=torch.float32, pin_memory=pin)
    final_d = torch.empty((B, H, dk), dtype=torch.float32, pin_memory=pin)
    if device_buffer is None:
        device_buffer = torch.empty(osdn_fwd_host_buffer_size(p, groups), dtype=torch.uint8, device="cuda")
    osdn_fwd_host(p, q, k, v, beta, r, d0, S0, out, final_S, final_d, device_buffer, groups, stream)
    return out, final_S, final_d


def backward(q, k, v, beta, dout, r=None, d0=None, S0=None, dS_final=None, dd_final=None, eta=1e-2, chunk=64,
             workspace=None, stream=None, apf_anchor=False, alpha=None):
    """Gradients of L = sum(dout * out) + sum(dS_final * final_S) + sum(dd_final * final_d) for the
    forward() with the same inputs (plain or anchored APF; gated OSDN when alpha [B,T,H] is given).
    dout [B,T,H,dv] in the input dtype; dS_final [B,H,dv,dk], dd_final [B,H,dk] fp32 or None (= 0).
    Returns a dict with dq, dk, dv, dbeta, dr (None without r), dalpha (None without alpha) in the
    input dtype and dd0 [B,H,dk], dS0 [B,H,dv,dk] fp32."""
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    p = make_params(B, T, H, dk, dv, k.dtype, eta, chunk, apf_anchor)
    dev, dt = k.device, k.dtype
    g = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
         "dbeta": torch.empty_like(beta), "dr": None if r is None else torch.empty_like(r),
         "dd0": torch.empty((B, H, dk), dtype=torch.float32, device=dev),
         "dS0": torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)}
    if workspace is None:
        workspace = torch.empty(osdn_bwd_workspace_size(p), dtype=torch.uint8, device=dev)
    if alpha is None:
        osdn_bwd(p, q, k, v, beta, r, d0, S0, dout, dS_final, dd_final, g["dq"], g["dk"], g["dv"], g["dbeta"],
                 g["dr"], g["dd0"], g["dS0"], workspace, stream)
        g["dalpha"] = None
    else:
        g["dalpha"] = torch.empty_like(alpha)
        osdn_bwd_gated(p, q, k, v, beta, r, alpha, d0, S0, dout, dS_final, dd_final, g["dq"], g["dk"], g["dv"],
                       g["dbeta"], g["dr"], g["dalpha"], g["dd0"], g["dS0"], workspace, stream)
    return g


def residual_ratio(k, beta, r=None, d0=None, eta=1e-2, stream=None, apf_anchor=False):
    """Preconditioner scan with its residual-ratio diagnostic: k [B,T,H,dk]; beta, r [B,T,H];
    d0 [B,H,dk] fp32 (None = ones). Returns rho [B,T,H] fp32 (rho_t = (1 - beta_t <d_t, k_t^2>)^2,
    the factor by which token t's write shrinks its own loss), q_geo [B,H] fp32 (exp of the mean
    log rho over each sequence) and d after the last token [B,H,dk] fp32."""
    B, T, H, dk = k.shape
    p = make_params(B, T, H, dk, dk, k.dtype, eta, apf_anchor=apf_anchor)
    rho = torch.empty((B, T, H), dtype=torch.float32, device=k.device)
    q_geo = torch.empty((B, H), dtype=torch.float32, device=k.device)
    d = torch.empty((B, H, dk), dtype=torch.float32, device=k.device)
    ws = torch.empty(max(osdn_fwd_workspace_size(p), 256), dtype=torch.uint8, device=k.device)
    osdn_fwd_scan_diag(p, k, beta, r, d0, d, rho, q_geo, ws, stream)
    return rho, q_geo, d


def step(q, k, v, beta, S, d, r=None, eta=1e-2, stream=None, d_anchor=None, apf_anchor=False, alpha=None):
    """One decode token for every (b, h): q, k [B,H,dk]; v [B,H,dv]; beta, r [B,H];
    S [B,H,dv,dk] and d [B,H,dk] fp32, updated in place. Anchored APF (apf_anchor, or a
    d_anchor [B,H,dk] fp32 given) pulls d toward d_anchor (ones when None); alpha [B,H] decays S
    first (gated OSDN). Returns out [B,H,dv]."""
    B, H, dk = k.shape
    dv = v.shape[-1]
    p = make_params(B, 1, H, dk, dv, k.dtype, eta, apf_anchor=apf_anchor or d_anchor is not None)
    out = torch.empty((B, H, dv), dtype=k.dtype, device=k.device)
    if alpha is None:
        osdn_step_ex(p, q, k, v, beta, r, d_anchor, S, d, out, stream)
    else:
        osdn_step_gated(p, q, k, v, beta, r, alpha, d_anchor, S, d, out, stream)
    return out
