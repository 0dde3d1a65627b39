"""Rank plumbing of the replica runs, on CPU with two gloo ranks.

A chunk does not shard, so several GPUs run independent replicas; the only
collectives are the host barrier and the max-over-ranks reduction of the
measured time.  These run here as world-size-2 gloo process groups."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    from flow_matching_action_dm0_b200 import replicas as R
    info = R.init("gloo", timeout_s=30)
    try:
        R.barrier(info)
        mx = R.max_over_ranks(1.5 + rank, info)
        sm = R.sum_over_ranks(1.0, info)
        q.put((rank, info.world, info.is_main, mx, sm))
    finally:
        R.shutdown(info)


def test_two_gloo_ranks_reduce_max_and_sum():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == 2 for r in res)
    assert [r[2] for r in res] == [True, False]
    assert all(r[3] == 2.5 for r in res)     # max over ranks
    assert all(r[4] == 2.0 for r in res)     # sum over ranks


def test_single_process_needs_no_group():
    from flow_matching_action_dm0_b200 import replicas as R
    info = R.rank_info()
    assert info.world == 1 and info.is_main
    assert R.max_over_ranks(3.0, info) == 3.0
