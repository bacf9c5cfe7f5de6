"""N > 1 plumbing of bench.py on CPU: two gloo ranks, no GPU.

Heads and videos are independent, so N GPUs run N independent replicas of the
workload with no data-path collective; the only cross-rank steps are the
barrier and the max-over-ranks of the step time.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [3.0, 5.0][rank]
        bench.barrier(world)
        ms = bench.max_over_ranks(local_ms, world, device="cpu")
        w = bench.replica_workload(workloads.CONFIGS["tiny"], rank)
        q, _, _ = workloads.call_tensors(w)
        out.put((rank, ms, w.seed, float(q.sum())))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_slowest_time_and_distinct_replicas():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    world, port = 2, _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=100) for _ in range(world))
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [5.0, 5.0]           # both ranks see the max
    assert res[0][2] != res[1][2]                       # distinct replica seeds
    assert res[0][3] != res[1][3]                       # hence distinct inputs


def test_job_throughput_counts_every_rank():
    assert bench.job_throughput(1000, 1, 1.0) == pytest.approx(1e6)
    assert bench.job_throughput(1000, 4, 2.0) == pytest.approx(2e6)
