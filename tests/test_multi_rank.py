"""The N > 1 path of bench.py with two gloo ranks on CPU: each rank runs its
own batch (different seeds, same shapes), timings combine as the max over
ranks on every rank, and the whole-job throughput counts all ranks' tokens
over the slowest rank's time. The path has no data-path collective."""

import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from kernelized_linear_attention_phi_b200 import workloads as W
        wl = W.WORKLOADS["multi_head"]
        seed = bench.rank_seed(wl, rank)
        q_, k_, v_ = W.qkv(1, 2, 64, 16, 1.0, seed, "f32", "cpu")
        times = bench.max_over_ranks([0.25 + rank, 1.0 + 0.5 * rank], torch.device("cpu"))
        value = bench.aggregate_tokens_per_s(100, 10, world, times[0])
        q.put((rank, seed, float(q_.sum()), tuple(q_.shape), times, value))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_weak_scaling_logic():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=90) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, sum0, shape0, t0, v0), (r1, s1, sum1, shape1, t1, v1) = res
    assert (r0, r1) == (0, 1)
    assert s0 != s1 and sum0 != sum1 and shape0 == shape1   # own batch per rank
    assert t0 == t1 == [1.25, 1.5]                           # max over ranks, on both
    assert v0 == v1 == pytest.approx(100 * 10 * 2 / 1.25)    # all ranks' tokens / slowest time
