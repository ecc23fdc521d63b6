"""Multi-rank host logic of bench.py on the CPU (gloo, world size 2).

Each rank runs its own batch (weak scaling, no collective on the data path);
the only cross-rank steps are a barrier and the max over ranks of the timed
durations, from which rank 0 computes whole-job throughput.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        times = [1.0 + rank, 5.0 - rank, 2.5]
        got = bench.reduce_max(times)
        env = bench.dist_env()
        thr = bench.aggregate_throughput(100.0, world, got[0])
        dist.barrier()
        q.put((rank, got, env, thr))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, env, thr in res:
        assert got == [2.0, 5.0, 2.5]           # element-wise max over the two ranks
        assert env == (2, rank, rank)
        # 100 units on each of 2 ranks in 2 ms (slowest rank) -> 100000 units/s
        assert thr == pytest.approx(100.0 * 2 / 2e-3)


def test_single_rank_reduce_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert not (dist.is_available() and dist.is_initialized())
    assert bench.reduce_max([3.0, 1.0]) == [3.0, 1.0]
    assert bench.aggregate_throughput(10.0, 1, 5.0) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench

    class A:
        steps, warmup, gpus = 1, 3, 2

    called = []
    monkeypatch.setattr(bench, "headline_head_inputs", lambda: called.append(1))
    assert bench.run_reference(A, 2, 1) == 0   # rank 1: exits without work
    assert called == []


def test_flop_and_byte_accounting():
    sys.path.insert(0, ROOT)
    import bench
    import workloads

    # causal N x N: N(N+1)/2 visible pairs; 4*d FLOPs each
    w = workloads.PREFILL_MHA_2K
    assert bench.visible_pairs(2048, 2048, True) == 2048 * 2049 // 2
    assert bench.prefill_flops(w) == 4.0 * 128 * 4 * 16 * 2048 * 2049 // 2
    # bottom-right alignment: Nq < Nk sees Nk - Nq extra keys per row
    assert bench.visible_pairs(2, 5, True) == 4 + 5
    assert bench.visible_pairs(5, 2, True) == 1 + 2
    assert bench.decode_kv_bytes([3, 0, -1, 5], 2, 128) == 2 * 8 * 2 * 128 * 2
