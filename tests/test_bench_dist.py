"""bench.py's multi-rank host logic on CPU: two gloo ranks, each timing its
own replica, agree on the maximum duration and on the whole-job value."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench

    d = bench.Dist("gloo")
    d.init()
    d.barrier()
    secs = d.max(1.0 + rank)  # rank r "took" 1 + r seconds
    steps = 10
    out.put((rank, secs, d.world * steps / secs))
    d.barrier()
    d.close()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=100) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert [r for r, _, _ in res] == [0, 1]
    assert all(s == 2.0 for _, s, _ in res)          # both ranks see the slower rank
    assert all(v == 2 * 10 / 2.0 for _, _, v in res)  # all ranks' units / max time


def test_single_rank_needs_no_process_group():
    import bench

    d = bench.Dist("gloo")
    assert d.world == int(os.environ.get("WORLD_SIZE", "1"))
    if d.world == 1:
        d.init()
        assert d.pg is None and d.max(3.5) == 3.5
