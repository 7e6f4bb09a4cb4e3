"""The multi-GPU host logic of bench.py on CPU: two `gloo` ranks.

The path shards without any data-path collective (every rank runs its own
batch); the only collectives are the timing reductions, the maximum over ranks
of the step time, which every rank calls in the same order.  A rank that stops
taking part must make the others fail within the process group's timeout
instead of waiting for ever.
"""
import datetime
import os
import socket

import pytest

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port, timeout_s):
    import torch
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world, init_method=f"tcp://127.0.0.1:{port}",
                                         timeout=datetime.timedelta(seconds=timeout_s))


def _reduce_worker(rank, world, port, q):
    import torch
    _init(rank, world, port, 30)
    try:
        local = [3.0, 7.5][rank]
        first = bench.max_over_ranks(local, "cpu")          # step time: the slowest rank
        second = bench.max_over_ranks(10.0 - local, "cpu")  # a second reduction, same order on every rank
        q.put((rank, first, second))
    finally:
        torch.distributed.destroy_process_group()


def _dropout_worker(rank, world, port, q):
    import torch
    _init(rank, world, port, 5)
    try:
        bench.max_over_ranks(1.0, "cpu")
        if rank == 1:
            q.put((rank, "left"))
            return  # leaves between steps: takes no part in the next reduction
        try:
            bench.max_over_ranks(2.0, "cpu")
            q.put((rank, "no error"))
        except Exception as e:  # the process group's timeout ends the collective
            q.put((rank, "error: " + type(e).__name__))
    finally:
        try:
            torch.distributed.destroy_process_group()
        except Exception:
            pass


def _run(target, timeout_s):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=target, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(timeout_s)
    for p in ps:
        if p.is_alive():
            p.kill()
            p.join()
    out = []
    while not q.empty():
        out.append(q.get(timeout=5))
    return [p.exitcode for p in ps], sorted(out)


def test_step_time_is_the_maximum_over_two_gloo_ranks():
    codes, out = _run(_reduce_worker, 120)
    assert codes == [0, 0]
    assert out == [(0, 7.5, 7.0), (1, 7.5, 7.0)]


def test_a_rank_that_leaves_makes_the_next_reduction_fail():
    codes, out = _run(_dropout_worker, 120)
    assert (1, "left") in out
    r0 = [o for o in out if o[0] == 0]
    assert r0 and r0[0][1].startswith("error"), out


def test_single_rank_maximum_is_the_value():
    assert bench.max_over_ranks(4.25, "cpu") == 4.25


def test_weak_scaling_value_counts_every_rank():
    assert bench.weak_scaling_value(2, 1e12, 1000.0) == pytest.approx(2.0)
    assert bench.weak_scaling_value(1, 2.198e13, 22.5) == pytest.approx(976.9, rel=1e-3)
