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


def _shard_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        shard = bench.head_shard(32, 8, 32, world, rank)
        # each rank's flops differ (different heads): the job sums them
        total = bench.sum_over_ranks([1e12 * (rank + 1)])
        q.put((rank, shard, total))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_head_sharding_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    shards = [r[1] for r in res]
    assert shards == [(0, 16, 0, 4, 0, 16), (16, 32, 4, 8, 16, 32)]
    assert all(r[2] == [3e12] for r in res)


@pytest.mark.parametrize("Hq,Hkv,H_sel,world", [(32, 8, 32, 4), (32, 8, 8, 8), (8, 8, 8, 2),
                                                (1, 1, 1, 1)])
def test_head_shards_partition_the_layer(Hq, Hkv, H_sel, world):
    G = Hq // Hkv
    seen_q, seen_kv, seen_s = [], [], []
    for r in range(world):
        q0, q1, kv0, kv1, s0, s1 = bench.head_shard(Hq, Hkv, H_sel, world, r)
        seen_q += range(q0, q1)
        seen_kv += range(kv0, kv1)
        seen_s += range(s0, s1)
        # a query head's KV head and index set stay on its rank
        for h in range(q0, q1):
            assert kv0 <= h // G < kv1 and s0 <= h * H_sel // Hq < s1
    assert seen_q == list(range(Hq)) and seen_kv == list(range(Hkv))
    assert seen_s == list(range(H_sel))
    with pytest.raises(ValueError):
        bench.head_shard(32, 8, 32, 3, 0)
