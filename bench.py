#!/usr/bin/env python
"""Throughput of the OSDN chunkwise forward on B200: tokens/s, TFLOP/s and the
fraction of the HBM / bf16 roofline.

One step = one osdn_fwd over the whole workload (phase 1 preconditioner scan +
phase 2 chunked delta rule) with inputs resident in HBM. Default workload: the
1.3B-shaped layer (B=8, H=16, T=4096, dk=dv=128, C=64, bf16, APF on, shifted key
statistics). Inputs (q, k, v: 403 MB) are larger than the 126 MB L2, so no
flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own full workload (independent sequences;
no collective on the data path), so scaling is weak; the step time is the max
over ranks. ``--impl reference`` times the float64 CPU oracle on a bounded
sample of the same workload on the host cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from preconditioned_delta_rule_token_b200 import workloads as W  # noqa: E402

FLOPS_PER_TOKEN_HEAD = None   # set from the workload (6 dk dv + C (3 dk + 2 dv))
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOADS = {"340m": W.LAYER_340M, "1p3b": W.LAYER_1P3B, "long": W.LONG_RECALL}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="1p3b")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-groups", type=int, default=0,
                    help="groups of sequences the end-to-end call pipelines (0: the library's default)")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-decode", action="store_true", help="skip the osdn_step (decode) measurement")
    ap.add_argument("--no-gated", action="store_true", help="skip the gated-variant chunk measurement")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward (osdn_bwd) measurement")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def flops_per_token_head(w):
    return 6 * w.dk * w.dv + w.chunk * (3 * w.dk + 2 * w.dv)


def elem(w):
    return 2 if w.dtype == W.BF16 else 4


def path_bytes(w, with_S0=False, with_d0=False):
    """Algorithmic bytes of the whole forward: read q, k, v, beta (+ r), write out;
    per (b, h) write final S and d (read S0, d0 when given)."""
    e = elem(w)
    per_tok = (2 * w.dk + 2 * w.dv) * e + e + (e if w.apf else 0)
    per_unit = 4 * (w.dv * w.dk + w.dk) + (4 * w.dv * w.dk if with_S0 else 0) + (4 * w.dk if with_d0 else 0)
    return w.B * w.T * w.H * per_tok + w.B * w.H * per_unit


def scan_bytes(w):
    """Phase 1: read k, beta (+ r), write the scaled keys; write final d (d0 read: ones here)."""
    e = elem(w)
    return w.B * w.T * w.H * (2 * w.dk * e + e + (e if w.apf else 0)) + w.B * w.H * 4 * w.dk


def chunk_bytes(w):
    """Phase 2: read q, k, scaled keys, v, beta, write out; write final S."""
    e = elem(w)
    return w.B * w.T * w.H * ((3 * w.dk + 2 * w.dv) * e + e) + w.B * w.H * 4 * w.dv * w.dk


def source_sha(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


_CSRC = "preconditioned_delta_rule_token_b200/csrc/"
KERNEL_SOURCES = {   # the sources each timed kernel is built from (bf16, dk = dv = 128 path)
    "chunk": [_CSRC + f for f in ("chunk_wy.cuh", "tc_ptx.cuh", "tril_inv.cuh", "common.cuh")],
    "scan": [_CSRC + f for f in ("scan_ws.cuh", "tc_ptx.cuh", "tril_inv.cuh", "common.cuh")],
}


def ncu_traffic(kernel, workload_name):
    """DRAM bytes per launch from a committed ncu capture (profiles/traffic.txt),
    only if the kernel source is unchanged since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    sha = source_sha(KERNEL_SOURCES[kernel])
    with open(path) as fh:
        for line in fh:
            parts = line.split("\t")
            if len(parts) >= 4 and not line.startswith("#"):
                if parts[0] == kernel and parts[1] == sha and parts[2] == workload_name:
                    return float(parts[3])
    return None


class ClockSampler:
    """SM clock and throttle-reason samples taken during the timed region, from a
    host thread polling NVML every few milliseconds (so short regions still
    get samples)."""
    REASONS = (("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20), ("hw_thermal_slowdown", 0x40),
               ("sw_power_cap", 0x4))

    def __init__(self, device, enabled=True, period_s=0.005):
        import threading
        self.samples = []
        self._stop = threading.Event()
        self._thread = None
        self.handle = None
        if not enabled:
            return
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.smax = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            self.nvml = pynvml
        except Exception:
            self.handle = None
            return

        def run():
            while not self._stop.is_set():
                try:
                    sm = self.nvml.nvmlDeviceGetClockInfo(self.handle, self.nvml.NVML_CLOCK_SM)
                    rs = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                    self.samples.append((sm, rs))
                except Exception:
                    pass
                self._stop.wait(period_s)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": "nvml"}
        reasons = sorted({name for _, rs in self.samples for name, bit in self.REASONS if rs & bit})
        return {"sm_mhz": statistics.median(s for s, _ in self.samples), "sm_max_mhz": self.smax,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml"}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def rank_workload(w, rank):
    """Rank r runs the same workload shape on its own inputs (seed + 1000 r): weak
    scaling over independent sequences, no data shared between ranks."""
    if rank == 0:
        return w
    import dataclasses
    return dataclasses.replace(w, seed=w.seed + 1000 * rank)


def max_over_ranks(values, world, device):
    """Element-wise max of per-rank timings (an all-reduce MAX over the process
    group, device tensors under NCCL, host tensors under gloo)."""
    if world <= 1:
        return list(values)
    t = torch.tensor(list(values), device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def aggregate_tokens_per_s(w, world, ms):
    """Whole-job throughput: every rank processes B*T tokens (of H heads each) in
    the slowest rank's step time ms."""
    return world * w.B * w.T / (ms / 1e3)


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(w, seconds=12.0, max_units=None):
    """Time the float64 oracle on a bounded sample of workload w: the first n
    (b, h) units over the full sequence, n sized from a short calibration run
    so the sample takes about `seconds`. Returns (tokens/s, description, cores)."""
    import oracle
    cores = cpu_cores()
    inp = W.make_forward_inputs(w)
    f = W.to_f64
    units = [(b, h) for b in range(w.B) for h in range(w.H)]

    def run(n, T):
        sel = units[:n]
        q = f(inp["q"])[:, :T]
        k = f(inp["k"])[:, :T]
        v = f(inp["v"])[:, :T]
        be = f(inp["beta"])[:, :T]
        r = None if inp["r"] is None else f(inp["r"])[:, :T]
        # gather the sampled units as B = n sequences of one head

        def pick4(x):
            return None if x is None else np.ascontiguousarray(np.stack([x[b, :, h] for (b, h) in sel])[:, :, None])
        t0 = time.perf_counter()
        oracle.fwd(pick4(q), pick4(k), pick4(v), pick4(be), pick4(r), None, None, eta=w.eta, nthreads=cores)
        return time.perf_counter() - t0

    Tc = min(w.T, 256)
    nc = min(len(units), cores)
    tcal = run(nc, Tc)
    per_unit_token = tcal * min(nc, cores) / (nc * Tc)         # core-seconds per unit-token
    n = int(seconds * cores / (per_unit_token * w.T))
    n = max(1, min(len(units) if max_units is None else max_units, n))
    el = run(n, w.T)
    tokens = n * w.T / w.H                                       # layer tokens (all H heads) equivalent
    desc = "%d of %d (b,h) units x full T=%d (%.1f s); tokens counted as units*T/H" % (n, len(units), w.T, el)
    return tokens / el, desc, cores


def run_reference(args, world, rank):
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    cores = cpu_cores()
    budget = 150.0 / max(1, args.steps + args.warmup)
    times, toks = [], []
    desc = ""
    for i in range(args.warmup + args.steps):
        tps, desc, cores = oracle_sample(w, seconds=budget)
        if i >= args.warmup:
            toks.append(tps)
    value = statistics.median(toks)
    line = {"impl": "reference", "metric": "OSDN chunkwise fwd tokens/s", "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": w.B * w.T / value * 1e3,
            "ms_per_step_note": "one step over the whole workload at the sample's rate (extrapolated)",
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": config_of(w, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def decode_bytes(w):
    """HBM bytes of one decode call over all B*H heads: S read + written (fp32), d read +
    written (fp32), q, k, v read and out written (storage dtype), beta and r."""
    e = elem(w)
    return w.B * w.H * (2 * w.dv * w.dk * 4 + 2 * w.dk * 4 + (2 * w.dk + w.dv) * e + w.dv * e + 2 * e)


def run_decode(dev, stream, hbm, n_calls=200, warmup=5):
    """osdn_step on the decode workload (B256 H16 d128 bf16): S, d and eight distinct
    tokens resident in HBM (S alone is 268 MB > L2); per-call time by CUDA events."""
    import preconditioned_delta_rule_token_b200 as pk
    w = W.DECODE
    st0 = W.make_decode_state(w)
    S, d = st0["S0"].to(dev), st0["d0"].to(dev)
    toks = [{k_: None if v_ is None else v_.to(dev) for k_, v_ in W.make_decode_token(w, i).items()}
            for i in range(8)]
    p = pk.make_params(w.B, 1, w.H, w.dk, w.dv, toks[0]["k"].dtype, w.eta)
    out = torch.empty((w.B, w.H, w.dv), dtype=toks[0]["k"].dtype, device=dev)

    def call(i):
        t = toks[i % len(toks)]
        pk.osdn_step(p, t["q"], t["k"], t["v"], t["beta"], t["r"], S, d, out, stream)

    for i in range(warmup):
        call(i)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n_calls):
        call(i)
    e1.record(stream)
    torch.cuda.synchronize()
    assert pk.osdn_sync_status(stream) == 0
    us = e0.elapsed_time(e1) * 1e3 / n_calls
    gbs = decode_bytes(w) / (us * 1e-6) / 1e9
    return {"workload": w.name, "calls": n_calls, "us_per_call": us, "tokens_per_s": w.B / (us * 1e-6),
            "bytes_per_call": decode_bytes(w), "achieved_gbs": gbs, "peak_gbs": hbm, "frac": gbs / hbm,
            "bound": "hbm"}


def run_gated(w, g, p, ws, out, Sf, stream, hbm, steps=20, warmup=3):
    """Phase 2 of the gated variant (osdn_fwd_chunk_gated) on the same layer with
    alpha ~ U(0.9, 1) (bf16, resident), after the scan has filled the workspace."""
    import preconditioned_delta_rule_token_b200 as pk
    alpha = (0.9 + 0.1 * torch.rand((w.B, w.T, w.H), generator=torch.Generator().manual_seed(w.seed + 5))).to(
        g["k"].dtype).to(g["k"].device)
    for _ in range(warmup):
        pk.osdn_fwd_chunk_gated(p, g["q"], g["k"], g["v"], g["beta"], alpha, None, out, Sf, ws, stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        pk.osdn_fwd_chunk_gated(p, g["q"], g["k"], g["v"], g["beta"], alpha, None, out, Sf, ws, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    assert pk.osdn_sync_status(stream) == 0
    ms = e0.elapsed_time(e1) / steps
    nbytes = chunk_bytes(w) + w.B * w.T * w.H * elem(w)            # + alpha
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"kernel": "osdn gated chunk kernel (phase 2)", "alpha": "U(0.9, 1)", "launch_ms": ms,
            "algorithmic_bytes": nbytes, "achieved_gbs": gbs, "peak_gbs": hbm, "frac": gbs / hbm, "bound": "hbm"}


def backward_bytes(w):
    """Algorithmic HBM bytes of one osdn_bwd call: reads q, k, v, dout, beta (and r),
    writes dq, dk, dv, dbeta (and dr), all in the input dtype; per (b, h) reads dS_final,
    dd_final and writes dS0, dd0 in fp32 (S0 and d0 are the defaults, not read)."""
    e, apf = elem(w), 1 if w.apf else 0
    per_tok = e * ((2 * w.dk + 2 * w.dv + 1 + apf) + (2 * w.dk + w.dv + 1 + apf))
    per_unit = 4 * 2 * (w.dv * w.dk + w.dk)
    return w.B * w.T * w.H * per_tok + w.B * w.H * per_unit


def backward_flops(w):
    """Algorithmic FLOPs of one osdn_bwd call: the chunk form's dense products (the
    forward recomputed and the adjoint), triangular ones counted at half. Per chunk of C
    tokens, multiply-adds = 8 C dk dv + C^2 (5.5 dk + 3 dv) + (7/6) C^3."""
    C, nch = w.chunk, w.B * w.H * ((w.T + w.chunk - 1) // w.chunk)
    mac = 8 * C * w.dk * w.dv + C * C * (5.5 * w.dk + 3 * w.dv) + (7.0 / 6.0) * C ** 3
    return 2.0 * mac * nch


def run_backward(w, g, stream, hbm, tf_peak, steps=5, warmup=2, gated=False):
    """osdn_bwd (gated: osdn_bwd_gated with alpha ~ U(0.9, 1)) on the same layer with inputs
    and upstream gradients resident in HBM and the workspace preallocated; CUDA events on the
    launching stream."""
    import preconditioned_delta_rule_token_b200 as pk
    dev = g["k"].device
    cot = {k_: (None if v_ is None else v_.to(dev)) for k_, v_ in W.make_backward_cotangents(w).items()}
    p = pk.make_params(w.B, w.T, w.H, w.dk, w.dv, g["k"].dtype, w.eta, w.chunk)
    ws = torch.empty(pk.osdn_bwd_workspace_size(p), dtype=torch.uint8, device=dev)
    grads = {n: torch.empty_like(g[m]) for n, m in (("dq", "q"), ("dk", "k"), ("dv", "v"), ("dbeta", "beta"))}
    grads["dr"] = None if g["r"] is None else torch.empty_like(g["r"])
    dd0 = torch.empty((w.B, w.H, w.dk), dtype=torch.float32, device=dev)
    dS0 = torch.empty((w.B, w.H, w.dv, w.dk), dtype=torch.float32, device=dev)
    alpha = dalpha = None
    if gated:
        alpha = (0.9 + 0.1 * torch.rand((w.B, w.T, w.H), generator=torch.Generator().manual_seed(w.seed + 77))).to(
            g["k"].dtype).to(dev)
        dalpha = torch.empty_like(alpha)

    def call():
        if gated:
            pk.osdn_bwd_gated(p, g["q"], g["k"], g["v"], g["beta"], g["r"], alpha, None, None, cot["dout"],
                              cot["dS_final"], cot["dd_final"], grads["dq"], grads["dk"], grads["dv"], grads["dbeta"],
                              grads["dr"], dalpha, dd0, dS0, ws, stream)
        else:
            pk.osdn_bwd(p, g["q"], g["k"], g["v"], g["beta"], g["r"], None, None, cot["dout"], cot["dS_final"],
                        cot["dd_final"], grads["dq"], grads["dk"], grads["dv"], grads["dbeta"], grads["dr"], dd0,
                        dS0, ws, stream)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    assert pk.osdn_sync_status(stream) == 0
    ms = e0.elapsed_time(e1) / steps
    nbytes, F = backward_bytes(w) + (2 * w.B * w.T * w.H * elem(w) if gated else 0), backward_flops(w)
    t_hbm, t_tc = nbytes / (hbm * 1e9), F / (tf_peak * 1e12)
    t_roof = max(t_hbm, t_tc)
    del ws
    return {"call": "osdn_bwd_gated (6 kernel launches), alpha ~ U(0.9, 1)" if gated else
            "osdn_bwd (6 kernel launches)", "ms": ms, "tokens_per_s": w.B * w.T / (ms / 1e3),
            "algorithmic_bytes": nbytes, "flops": F, "t_roofline_us": t_roof * 1e6,
            "bound": "tensor" if t_tc >= t_hbm else "hbm", "frac": t_roof / (ms / 1e3),
            "tflops": F / (ms / 1e3) / 1e12, "gbs": nbytes / (ms / 1e3) / 1e9,
            "dtype": "bf16 in and out; fp32 state and intermediates, tf32 tensor-core products"}


def config_of(w, world):
    return {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "dk": w.dk, "dv": w.dv, "chunk": w.chunk,
            "apf": w.apf, "eta": w.eta, "structure": w.structure, "global_batch": w.B * world, "seq_len": w.T,
            "parallelism": "dp%d (independent sequences per rank)" % world,
            "l2": "inputs larger than L2 (q,k,v %.0f MB > 126 MB); no flush" % (
                w.B * w.T * w.H * (2 * w.dk + w.dv) * elem(w) / 1e6)}


def run_ours(args, world, rank, local):
    import preconditioned_delta_rule_token_b200 as pk
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = rank_workload(WORKLOADS[args.workload], rank)
    inp = W.make_forward_inputs(w)
    g = {k: None if v is None else v.to(dev) for k, v in inp.items()}
    g["d0"] = None            # d0 = ones (the library's default), as in the workload
    p = pk.make_params(w.B, w.T, w.H, w.dk, w.dv, g["k"].dtype, w.eta, w.chunk)
    out = torch.empty((w.B, w.T, w.H, w.dv), dtype=g["k"].dtype, device=dev)
    Sf = torch.empty((w.B, w.H, w.dv, w.dk), dtype=torch.float32, device=dev)
    df = torch.empty((w.B, w.H, w.dk), dtype=torch.float32, device=dev)
    ws = torch.empty(pk.osdn_fwd_workspace_size(p), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():   # one forward through the public entry point (both phases)
        pk.osdn_fwd(p, g["q"], g["k"], g["v"], g["beta"], g["r"], None, None, out, Sf, df, ws, stream)

    def phases(ev):   # the two phases as separate calls, for the per-kernel figures
        ev[0].record(stream)
        pk.osdn_fwd_scan(p, g["k"], g["beta"], g["r"], None, df, ws, stream)
        ev[1].record(stream)
        pk.osdn_fwd_chunk(p, g["q"], g["k"], g["v"], g["beta"], None, out, Sf, ws, stream)
        ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev, enabled=not args.no_clocks)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall = time.perf_counter()
    e_start.record(stream)
    for i in range(args.steps):
        step()
    e_end.record(stream)
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    clocks.stop()
    assert pk.osdn_sync_status(stream) == 0
    ms = e_start.elapsed_time(e_end) / args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for i in range(args.steps):
        phases(ev[i])
    torch.cuda.synchronize()
    assert pk.osdn_sync_status(stream) == 0
    scan_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    chunk_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    ms, scan_ms, chunk_ms = max_over_ranks([ms, scan_ms, chunk_ms], world, dev)

    # end-to-end through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e:
        host = {k: None if v is None else v.pin_memory() for k, v in inp.items() if k in ("q", "k", "v", "beta", "r")}
        h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h_S = torch.empty(Sf.shape, dtype=Sf.dtype).pin_memory()
        h_d = torch.empty(df.shape, dtype=df.dtype).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
        d2h = sum(t.numel() * t.element_size() for t in (h_out, h_S, h_d))

        # osdn_fwd_host: the library uploads a group of sequences, runs the forward on it and reads it
        # back, the copies of one group overlapping the compute of the others (one device buffer,
        # allocated here, outside the timed region)
        dev_buf = torch.empty(pk.osdn_fwd_host_buffer_size(p, args.e2e_groups), dtype=torch.uint8, device=dev)

        def e2e_step():
            pk.osdn_fwd_host(p, host["q"], host["k"], host["v"], host["beta"], host["r"], None, None, h_out, h_S, h_d,
                             dev_buf, args.e2e_groups, stream)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(3, min(args.steps, 10))
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks([e0.elapsed_time(e1) / n_e2e], world, dev)[0]
        e2e = {"value": aggregate_tokens_per_s(w, world, e2e_ms), "unit": "tokens/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "call": "osdn_fwd_host (pinned host buffers, %s groups of sequences)" % (args.e2e_groups or "default")}

    if rank != 0:
        return
    peaks, peak_kind = load_peaks()
    hbm = peaks["hbm_gbs"]
    tf_peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    F = flops_per_token_head(w) * w.B * w.T * w.H
    t_roof = max(F / (tf_peak * 1e12), path_bytes(w) / (hbm * 1e9))
    kernels = {
        "chunk": dict(ms=chunk_ms, bytes=chunk_bytes(w), name="osdn chunk kernel (phase 2)"),
        "scan": dict(ms=scan_ms, bytes=scan_bytes(w), name="osdn scan kernel (phase 1)"),
    }
    dom = max(kernels, key=lambda k_: kernels[k_]["ms"])
    kd = kernels[dom]
    achieved = kd["bytes"] / (kd["ms"] / 1e3) / 1e9
    traffic = ncu_traffic(dom, args.workload)
    # the method's own bytes (q, k, v, beta, r, out + state: 1,028 B per token-head) over the
    # dominant kernel's time, and the DRAM traffic of the whole step over those bytes
    method_gbs = path_bytes(w) / (kd["ms"] / 1e3) / 1e9
    step_traffic = [ncu_traffic(k_, args.workload) for k_ in kernels]
    step_traffic = None if any(t_ is None for t_ in step_traffic) else sum(step_traffic)
    line = {
        "metric": "OSDN chunkwise fwd tokens/s", "value": aggregate_tokens_per_s(w, world, ms), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == W.BF16
        else "f32", "data": "synthetic", "config": config_of(w, world),
        "tflops": world * F / (ms / 1e3) / 1e12,
        "path_roofline": {"t_roofline_us": t_roof * 1e6, "frac": t_roof / (ms / 1e3), "bound": "hbm" if
                          path_bytes(w) / (hbm * 1e9) >= F / (tf_peak * 1e12) else "tensor",
                          "bytes": path_bytes(w), "flops": F, "peak_kind": peak_kind},
        "roofline": {"kernel": kd["name"], "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": traffic, "algorithmic_bytes": kd["bytes"],
                     "launch_ms": kd["ms"], "peak_kind": peak_kind + " hbm_gbs",
                     "method_bytes": path_bytes(w), "frac_method_bytes": method_gbs / hbm,
                     "step_traffic": step_traffic,
                     "step_traffic_over_method_bytes": None if step_traffic is None else step_traffic / path_bytes(w)},
        "kernels_ms": {k_: v_["ms"] for k_, v_ in kernels.items()},
        "gpu_launches": pk.osdn_fwd_launches(p) * args.steps,
        "segments": pk.osdn_fwd_segments(p),
        "clocks": clocks.summary(),
        "wall_s_timed_region": t_wall,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if world == 1 and not args.no_decode:
        line["decode"] = run_decode(dev, stream, hbm)
    if world == 1 and not args.no_gated and w.dtype == W.BF16 and w.dk == 128 and w.dv == 128:
        step()                                                      # the workspace holds this layer's scaled keys
        line["gated"] = run_gated(w, g, p, ws, out, Sf, stream, hbm)
    if world == 1 and not args.no_backward:
        line["backward"] = run_backward(w, g, stream, hbm, tf_peak)
        line["backward_gated"] = run_backward(w, g, stream, hbm, tf_peak, gated=True)
    if world == 1 and not args.no_cpu_baseline:
        v_, desc, cores = oracle_sample(w, seconds=12.0)
        line["cpu_baseline"] = {"value": v_, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup(args)
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
