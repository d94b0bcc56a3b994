"""World-size-2 checks of bench.py's multi-rank plumbing on CPU with gloo:
the timing reduction is a max over ranks, the whole-job value sums every rank's
work, and a rank that fails ends its peers' collectives with an error instead
of a hang (short process-group timeout)."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, mode, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=10))
        r, lr, w = bench.dist_env()
        assert (r, lr, w) == (rank, rank, world)
        if mode == "max":
            bench.barrier(world)
            t = bench.max_over_ranks(10.0 * (rank + 1), world, torch.device("cpu"))
            q.put((rank, t))
        elif mode == "fail":
            if rank == 1:
                raise RuntimeError("rank 1 fails before the collective")
            try:
                bench.max_over_ranks(1.0, world, torch.device("cpu"))
                q.put((rank, "no error"))
            except Exception as e:  # the peer never joined: the collective must end with an error
                q.put((rank, "error: " + type(e).__name__))
        dist.destroy_process_group()
    except RuntimeError as e:
        q.put((rank, "raised: " + str(e)))


def _run(mode):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, mode, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(timeout=90)
        if p.is_alive():
            p.kill()
    out = {}
    while not q.empty():
        r, v = q.get()
        out[r] = v
    return out


def test_max_over_ranks_two_ranks():
    out = _run("max")
    assert out == {0: 20.0, 1: 20.0}


def test_failed_rank_ends_peer_collective_with_error():
    out = _run("fail")
    assert out[1].startswith("raised")
    assert out[0].startswith("error")
