"""The benchmark's multi-rank host logic on CPU with two gloo ranks: the
max-over-ranks timing, the whole-job aggregate and the reference arm's
rank-0-only rule.  (Every GPU call in this environment has one GPU; the
kernels themselves have no cross-rank step.)"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w, r, lr = bench.dist_env()
        ms = bench.max_over_ranks([10.0 + rank, 5.0 - rank])
        q.put((r, w, lr, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
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
    assert [r[0] for r in res] == [0, 1]
    for rank, world, local, ms in res:
        assert world == 2 and local == rank
        assert ms == [11.0, 5.0]  # max over ranks, element-wise


def test_whole_job_value_and_single_rank_identity():
    assert bench.max_over_ranks([1.5, 2.0]) == [1.5, 2.0]
    # 2 ranks, 1e12 flops each in 1000 ms -> 2 TFLOP/s aggregate
    assert bench.whole_job_value(2, 1e12, 1000.0) == pytest.approx(2.0)
    assert bench.whole_job_value(1, 4e12, 500.0) == pytest.approx(8.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        steps, warmup = 1, 1
    bench.run_reference(Args(), bench.WORKLOADS["tiny_1k"])  # returns before any work
    assert capsys.readouterr().out == ""
