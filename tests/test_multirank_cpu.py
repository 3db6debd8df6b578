"""Multi-rank host logic of bench.py on CPU: two gloo ranks (world size 2).

Every (b, h) sequence is independent, so N ranks run N copies of the workload
on their own inputs with no data-path collective (weak scaling). What the ranks
share is host logic, checked here without a GPU:
  * each rank draws its own inputs (seed + 1000 * rank);
  * timings reduce to the element-wise max over ranks;
  * the whole-job value counts every rank's tokens against that max.
"""
import datetime
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, queue):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from preconditioned_delta_rule_token_b200 import workloads as W
        w = bench.rank_workload(W.TINY_FP32, rank)
        inp = W.make_forward_inputs(w)
        # rank r reports step times (1 + r, 5 - r) ms: the max over ranks is (2, 5) on both
        ms = bench.max_over_ranks([1.0 + rank, 5.0 - rank], world, torch.device("cpu"))
        value = bench.aggregate_tokens_per_s(w, world, ms[0])
        queue.put((rank, w.seed, float(inp["k"].double().sum()), ms, value, w.B * w.T))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), queue), nprocs=world, join=True, start_method="spawn")
    res = sorted(queue.get(timeout=30) for _ in range(world))
    (r0, seed0, ksum0, ms0, val0, tok), (r1, seed1, ksum1, ms1, val1, _) = res
    assert (r0, r1) == (0, 1)
    assert seed1 == seed0 + 1000
    assert ksum0 != ksum1                       # independent inputs per rank
    assert ms0 == ms1 == [2.0, 5.0]             # element-wise max over ranks
    assert val0 == val1 == pytest.approx(world * tok / 2.0e-3)
