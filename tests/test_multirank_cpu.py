"""CPU-only, world size 2 over gloo: the benchmark's rank aggregation.

Replicas run with no data-path collective; the only collective is the max over
ranks of the per-step time. Also: the reference arm runs on rank 0 only.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 1.0 + rank * 0.75          # rank 1 is the slower one
        ms = bench.max_over_ranks(local_ms, world)
        flops = 1e12
        value = world * flops / (ms * 1e-3) / 1e12
        q.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [1.75, 1.75]      # every rank sees the max
    assert res[0][2] == pytest.approx(2 * 1e12 / 1.75e-3 / 1e12)


def test_reference_arm_non_zero_rank_does_no_work(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    w = bench.workloads.get(1)

    class A:
        steps, warmup, gpus = 2, 3, 2
    assert bench.reference_arm(A, w) == 0


def test_max_over_ranks_single_process_is_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5
