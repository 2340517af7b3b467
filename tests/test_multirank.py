"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2): replicas get
distinct tokens, timings reduce as max, token counts as sum."""

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    import synth
    bench.dist_init(world, "gloo")
    dev = torch.device("cpu")
    w, r, l = bench.dist_env()
    assert (w, r) == (world, rank)
    mx = bench.dist_max(world, 10.0 + rank, dev)
    sm = bench.dist_sum(world, 5.0, dev)
    bench.dist_barrier(world)
    x = synth.tokens(2, 256, first_token=100000 * rank)
    q.put((rank, mx, sm, x.float().sum().item()))
    torch.distributed.destroy_process_group()


def test_two_rank_reductions():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert all(r[1] == 11.0 for r in res)
    assert all(r[2] == 10.0 for r in res)
    assert res[0][3] != res[1][3]  # each replica draws its own tokens
