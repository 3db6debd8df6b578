"""Seeded synthetic inputs for the OSDN forward and decode step.

This module only draws random inputs; it holds none of the method's
arithmetic. Both the CUDA path and the CPU oracle are fed from it, so both
see bit-identical values: everything is drawn in float32 on the CPU with
``torch.Generator`` and then cast to the storage dtype (bf16 with
round-to-nearest-even, or left in fp32).

Distributions (the same for every workload unless stated):
  q, k  ~ N(0, I) then L2-normalised per token (before the cast);
  v     ~ N(0, I);
  beta  = sigmoid(N(0, 1));
  r     = 1 - 1e-3 * sigmoid(N(0, 1))   (APF retention, only when APF is on);
  d0    = ones.
Draw order: q, k, v, beta, r, then the structure-specific extras.

Structures:
  "gaussian" : as above.
  "shifted"  : k_t = normalise(mu_{b,h,seg} + eps_t), mu ~ N(0, I) redrawn
               every ``segment`` tokens (non-stationary key statistics, the
               setting adaptive preconditioner forgetting is meant for);
               q is not shifted.
  "recall"   : associative-recall layout per (b, h): the first ``npairs``
               tokens write pairs (kappa_j, nu_j) with q = k = kappa_j; every
               later round of ``npairs`` tokens re-presents the pairs in a
               random order with k = normalise(kappa_j + 0.1 eps),
               q = normalise(kappa_j + 0.1 eps'), v = nu_j.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

BF16 = "bf16"
FP32 = "fp32"


@dataclass(frozen=True)
class Workload:
    """One forward workload: shapes, storage dtype and input structure."""
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    chunk: int = 64
    dtype: str = BF16
    apf: bool = True
    structure: str = "gaussian"
    eta: float = 1e-2
    seed: int = 0
    segment: int = 512
    npairs: int = 256
    d0: str = "ones"          # "ones" or "uniform" (U[0.5, 1.5])
    S0: str = "zeros"         # "zeros" or "normal" (N(0, 0.02^2))

    @property
    def tokens(self) -> int:
        return self.B * self.T


@dataclass(frozen=True)
class DecodeWorkload:
    """Recurrent decode: ``steps`` single-token calls on B x H heads."""
    name: str
    B: int
    H: int
    dk: int
    dv: int
    steps: int
    dtype: str = BF16
    apf: bool = True
    eta: float = 1e-2
    seed: int = 4
    s0_std: float = 0.02


# The five workloads of the benchmark specification (index = seed).
TINY_FP32 = Workload("B1 H1 T256 dk=dv=64 C64 fp32", 1, 1, 256, 64, 64, 64, FP32, True, "gaussian", seed=0)
LAYER_340M = Workload("340M-shaped layer B8 H8 T2048 d128 bf16", 8, 8, 2048, 128, 128, 64, BF16, False,
                      "gaussian", seed=1)
LAYER_1P3B = Workload("1.3B-shaped layer B8 H16 T4096 d128 bf16 APF shifted keys", 8, 16, 4096, 128, 128, 64,
                      BF16, True, "shifted", seed=2)
LONG_RECALL = Workload("long-context recall B1 H16 T32768 d128 bf16", 1, 16, 32768, 128, 128, 64, BF16, False,
                       "recall", seed=3)
DECODE = DecodeWorkload("decode B256 H16 d128 bf16 x1024 steps", 256, 16, 128, 128, 1024, BF16, True, seed=4)

FORWARD_WORKLOADS = (TINY_FP32, LAYER_340M, LAYER_1P3B, LONG_RECALL)


def _torch_dtype(dtype: str):
    return torch.bfloat16 if dtype == BF16 else torch.float32


def _normalise(x: torch.Tensor) -> torch.Tensor:
    n = x.norm(dim=-1, keepdim=True)
    return x / torch.where(n > 0, n, torch.ones_like(n))


def make_forward_inputs(w: Workload) -> dict:
    """Draw the inputs of workload ``w`` (CPU tensors in the storage dtype;
    d0 and S0 always fp32). Keys: q, k, v, beta, r (None when APF is off),
    d0, S0 (None = zeros)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(w.seed))
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
    q = torch.randn((B, T, H, dk), generator=g)
    k = torch.randn((B, T, H, dk), generator=g)
    v = torch.randn((B, T, H, dv), generator=g)
    beta = torch.sigmoid(torch.randn((B, T, H), generator=g))
    r = 1.0 - 1e-3 * torch.sigmoid(torch.randn((B, T, H), generator=g)) if w.apf else None
    if w.structure == "gaussian":
        q, k = _normalise(q), _normalise(k)
    elif w.structure == "shifted":
        nseg = (T + w.segment - 1) // w.segment
        mu = torch.randn((B, nseg, H, dk), generator=g)
        seg_of_t = torch.arange(T) // w.segment
        k = _normalise(mu[:, seg_of_t] + k)
        q = _normalise(q)
    elif w.structure == "recall":
        P = w.npairs
        kappa = _normalise(torch.randn((B, H, P, dk), generator=g))
        nu = torch.randn((B, H, P, dv), generator=g)
        rounds = (T + P - 1) // P
        # order[b, h, t]: which pair token t presents; round 0 is the write pass
        order = torch.empty((B, H, rounds * P), dtype=torch.long)
        order[:, :, :P] = torch.arange(P)
        for rd in range(1, rounds):
            order[:, :, rd * P:(rd + 1) * P] = torch.argsort(torch.rand((B, H, P), generator=g), dim=-1)
        order = order[:, :, :T]
        ek = torch.randn((B, H, T, dk), generator=g)
        eq = torch.randn((B, H, T, dk), generator=g)
        kk = torch.gather(kappa, 2, order[..., None].expand(B, H, T, dk))
        vv = torch.gather(nu, 2, order[..., None].expand(B, H, T, dv))
        noisy = torch.ones((T,), dtype=torch.float32)
        noisy[:P] = 0.0
        noisy = noisy[None, None, :, None]
        k = _normalise(kk + 0.1 * noisy * ek).permute(0, 2, 1, 3).contiguous()
        q = _normalise(kk + 0.1 * noisy * eq).permute(0, 2, 1, 3).contiguous()
        v = vv.permute(0, 2, 1, 3).contiguous()
    else:
        raise ValueError("unknown structure %r" % (w.structure,))
    if w.d0 == "ones":
        d0 = torch.ones((B, H, dk))
    else:
        d0 = 0.5 + torch.rand((B, H, dk), generator=g)
    S0 = None
    if w.S0 == "normal":
        S0 = 0.02 * torch.randn((B, H, dv, dk), generator=g)
    td = _torch_dtype(w.dtype)
    return dict(q=q.to(td).contiguous(), k=k.to(td).contiguous(), v=v.to(td).contiguous(),
                beta=beta.to(td).contiguous(), r=None if r is None else r.to(td).contiguous(),
                d0=d0.contiguous(), S0=None if S0 is None else S0.contiguous())


def make_backward_cotangents(w: Workload, dS_final: bool = True, dd_final: bool = True) -> dict:
    """Upstream gradients for a backward call on workload ``w``: dout [B, T, H, dv] in the
    storage dtype, dS_final [B, H, dv, dk] and dd_final [B, H, dk] fp32 (None when not
    requested), all N(0, 1), from a generator seeded apart from the forward inputs."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(w.seed) * 7919 + 17)
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
    dout = torch.randn((B, T, H, dv), generator=g)
    dS = torch.randn((B, H, dv, dk), generator=g)
    dd = torch.randn((B, H, dk), generator=g)
    return dict(dout=dout.to(_torch_dtype(w.dtype)).contiguous(),
                dS_final=dS.contiguous() if dS_final else None,
                dd_final=dd.contiguous() if dd_final else None)


def make_decode_state(w: DecodeWorkload) -> dict:
    """Initial decode state: S0 ~ N(0, s0_std^2) fp32 [B, H, dv, dk], d0 = ones."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(w.seed))
    S0 = w.s0_std * torch.randn((w.B, w.H, w.dv, w.dk), generator=g)
    d0 = torch.ones((w.B, w.H, w.dk))
    return dict(S0=S0.contiguous(), d0=d0.contiguous())


def make_decode_token(w: DecodeWorkload, step: int) -> dict:
    """Inputs of decode call number ``step`` for every (b, h): q, k [B, H, dk],
    v [B, H, dv], beta, r [B, H] in the storage dtype."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(w.seed) * 1000003 + 1 + int(step))
    B, H, dk, dv = w.B, w.H, w.dk, w.dv
    q = _normalise(torch.randn((B, H, dk), generator=g))
    k = _normalise(torch.randn((B, H, dk), generator=g))
    v = torch.randn((B, H, dv), generator=g)
    beta = torch.sigmoid(torch.randn((B, H), generator=g))
    r = 1.0 - 1e-3 * torch.sigmoid(torch.randn((B, H), generator=g)) if w.apf else None
    td = _torch_dtype(w.dtype)
    return dict(q=q.to(td).contiguous(), k=k.to(td).contiguous(), v=v.to(td).contiguous(),
                beta=beta.to(td).contiguous(), r=None if r is None else r.to(td).contiguous())


def to_f64(t):
    """Exact upcast of a CPU tensor to a float64 numpy array (None passes)."""
    if t is None:
        return None
    return t.detach().to("cpu").to(torch.float64).numpy()
