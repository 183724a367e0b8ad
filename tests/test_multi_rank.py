"""The bench's multi-GPU path on the CPU: world_size-2 gloo ranks.

Multi-GPU runs are data-parallel replicas (the layer has no exchange step): every
rank runs the same workload, the ranks meet at a barrier around the timed region,
and rank 0 reports the whole job's tokens over the slowest rank's time.  Here two
host processes take the places of the GPUs and run that logic -- process group,
barrier, max over ranks, the throughput formula and the teardown -- over gloo on
127.0.0.1.  The reference arm's other ranks leave at once without a process group.
"""
import multiprocessing as mp
import os
import socket
import sys

import pytest

import bench

WORLD = 2
STEPS, TOKENS = 4, 16


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_env(rank: int, port: int):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(WORLD), LOCAL_RANK=str(rank))


def _replica(rank: int, port: int, q):
    try:
        _rank_env(rank, port)
        world, r, local = bench.dist_setup(backend="gloo")
        bench.barrier(world)
        mine = 10.0 + 5.0 * r                      # rank 1 is the slower replica
        slowest = bench.max_over_ranks(mine, world)
        bench.barrier(world)
        q.put((r, local, world, slowest, bench.throughput(TOKENS, world, STEPS, slowest)))
        bench.dist_teardown(world)
    except Exception as e:  # reported to the parent, which fails the test
        q.put(("error", rank, repr(e)))


def _reference_rank(rank: int, q):
    try:
        _rank_env(rank, 1)  # no rendezvous may happen: the port is never opened
        sys.argv = ["bench.py", "--impl", "reference", "--gpus", str(WORLD), "--steps", "1", "--warmup", "0"]
        bench.main()
        q.put(("done", rank))
    except Exception as e:
        q.put(("error", rank, repr(e)))


def _run(target, args_of_rank, n):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=target, args=(*args_of_rank(r), q)) for r in range(n)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(n)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    errors = [o for o in out if o[0] == "error"]
    assert not errors, errors
    return out


def test_replicas_report_the_slowest_rank():
    port = _free_port()
    out = sorted(_run(_replica, lambda r: (r, port), WORLD))
    assert [o[0] for o in out] == list(range(WORLD))
    for r, local, world, slowest, value in out:
        assert local == r and world == WORLD
        assert slowest == 15.0                       # the max over ranks, seen by every rank
        assert value == pytest.approx(TOKENS * WORLD * STEPS / 15e-3)


def test_reference_arm_other_ranks_leave_without_work():
    # rank 0 alone times the oracle; rank 1 returns at once and opens no process group
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_reference_rank, args=(1, q))
    p.start()
    res = q.get(timeout=60)
    p.join(timeout=30)
    assert p.exitcode == 0 and res == ("done", 1)
