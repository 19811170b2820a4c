"""The replica bench's multi-rank host logic on the CPU: two gloo ranks run the reductions
bench.py runs under torchrun (the max of the ranks' device times, the sum of their committed
tokens), and a check that fails on one rank makes every rank raise at the same collective
instead of leaving the others waiting in a later one."""
import datetime
import os
import socket

import pytest
import torch.multiprocessing as mp


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    res = {
        "ms": bench.rank_reduce(10.0 + rank, "max", world, "cpu"),
        "tokens": bench.rank_reduce(100 + 7 * rank, "sum", world, "cpu"),
        "min": bench.rank_reduce(5.0 - rank, "min", world, "cpu"),
    }
    try:
        bench.raise_on_any_rank(None, world, "cpu")
        res["clean"] = True
    except RuntimeError:
        res["clean"] = False
    try:
        bench.raise_on_any_rank("accept lengths differ" if rank == 1 else None, world, "cpu")
        res["raised"] = None
    except RuntimeError as e:
        res["raised"] = str(e)
    # both ranks still take the next collective together
    res["after"] = bench.rank_reduce(1, "sum", world, "cpu")
    dist.destroy_process_group()
    q.put((rank, res))


def test_two_gloo_ranks_reduce_and_fail_together():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(2):
        assert out[r]["ms"] == 11.0 and out[r]["tokens"] == 207 and out[r]["min"] == 4.0
        assert out[r]["clean"] is True and out[r]["after"] == 2
    assert out[1]["raised"] == "accept lengths differ"
    assert out[0]["raised"] == "another rank failed its checks"


def test_single_rank_is_the_identity():
    import bench
    assert bench.rank_reduce(3.5, "max", 1, "cpu") == 3.5
    assert bench.rank_reduce(12, "sum", 1, "cpu") == 12
    bench.raise_on_any_rank(None, 1, "cpu")
    with pytest.raises(RuntimeError, match="planted"):
        bench.raise_on_any_rank("planted", 1, "cpu")
