"""Multi-process (gloo, world size 2, CPU) tests of the replica bookkeeping: the N > 1 path of
the benchmark exchanges nothing on the hot path, only the slowest rank's time and the job's
unit count.  Failures are made on the host (a rank that raises, a rank that never joins)."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from cross_model_attention_mf_b200 import replicas


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port, timeout_s=30):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=timeout_s))


def _worker_aggregate(rank, world, port, q):
    _init(rank, world, port)
    try:
        mine = replicas.owned(10, world, rank)
        # pretend each rank ran its units in (rank + 1) seconds
        slowest = replicas.max_over_ranks(float(rank + 1))
        total = replicas.sum_over_ranks(len(mine))
        q.put((rank, list(mine), slowest, total, replicas.job_throughput(total, slowest)))
    finally:
        dist.destroy_process_group()


def _worker_one_fails(rank, world, port, q):
    _init(rank, world, port, timeout_s=5)
    try:
        if rank == 1:
            raise RuntimeError("rank 1 fails before the collective")
        try:
            replicas.max_over_ranks(1.0)
            q.put((rank, "no error"))
        except Exception as e:  # the survivor learns of the failure through the timeout
            q.put((rank, type(e).__name__))
    finally:
        dist.destroy_process_group()


def _run(fn, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=fn, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = []
    for p in procs:
        p.join(timeout=120)
    while not q.empty():
        out.append(q.get())
    for p in procs:
        if p.is_alive():
            p.kill()
    return sorted(out), [p.exitcode for p in procs]


def test_owned_partitions_units():
    for n in (0, 1, 7, 10, 128):
        for world in (1, 2, 3, 8):
            parts = replicas.shares(n, world)
            assert sum(len(p) for p in parts) == n
            assert [u for p in parts for u in p] == list(range(n))
            assert max(map(len, parts)) - min(map(len, parts)) <= 1
    with pytest.raises(ValueError):
        replicas.owned(4, 2, 2)


def test_single_process_needs_no_group():
    assert replicas.max_over_ranks(3.5) == 3.5
    assert replicas.sum_over_ranks(4) == 4
    assert replicas.job_throughput(8, 2.0) == 4.0


def test_two_ranks_take_the_slowest_time_and_all_units():
    out, codes = _run(_worker_aggregate)
    assert codes == [0, 0]
    assert [r for r, *_ in out] == [0, 1]
    (_, u0, s0, t0, v0), (_, u1, s1, t1, v1) = out
    assert u0 == [0, 1, 2, 3, 4] and u1 == [5, 6, 7, 8, 9]
    assert s0 == s1 == 2.0 and t0 == t1 == 10 and v0 == v1 == 5.0


def test_a_failed_rank_ends_the_others_collective_with_an_error():
    out, codes = _run(_worker_one_fails)
    assert codes[1] != 0                      # the failing rank exits with its exception
    assert out and out[0][0] == 0 and out[0][1] != "no error"
