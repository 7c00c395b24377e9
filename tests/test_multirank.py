"""The benchmark's multi-rank host logic on CPU: gloo process group, world size 2.

Every rank runs an independent problem (weak scaling, no data-path
collective); the only collective is the max over ranks of the measured time.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        r, w, local = bench.dist_env()
        local_ms = 10.0 + 5.0 * rank
        mx = bench.reduce_max(local_ms)
        seeds = bench.rank_seed(r)
        value = bench.whole_job_tokens_per_s(32768, w, 100, mx)
        q.put((r, w, mx, seeds, value))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_weak_scaling_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, mx0, s0, v0), (r1, w1, mx1, s1, v1) = res
    assert (r0, r1, w0, w1) == (0, 1, 2, 2)
    assert mx0 == mx1 == 15.0           # both ranks see the slowest rank's time
    assert s0 != s1                     # independent problems per rank
    # units of all ranks over the max time: 2 ranks x 100 steps x 32768 tokens / 15 ms
    assert v0 == v1 == pytest.approx(2 * 100 * 32768 / 0.015)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
    assert capsys.readouterr().out == ""


def test_single_rank_reduce_is_identity():
    assert bench.reduce_max(3.5) == 3.5
    assert bench.kept_flops(10, 64, 128) == 4 * 64 * 64 * 128 * 10
