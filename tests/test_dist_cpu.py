"""Multi-rank plumbing of the benchmark on CPU (gloo, world size 2)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from post_weight_quantization_10_b200 import dist as D


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        r, w, lr = D.world()
        D.barrier(w)
        mx = D.max_over_ranks(10.0 + r, w)
        sm = D.sum_over_ranks(1.0, w)
        units = D.my_units(7, r, w)
        q.put((r, w, lr, mx, sm, units))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, l0, mx0, sm0, u0), (r1, w1, l1, mx1, sm1, u1) = res
    assert (r0, r1) == (0, 1) and w0 == w1 == 2
    assert mx0 == mx1 == 11.0 and sm0 == sm1 == 2.0
    assert u0 == [0, 2, 4, 6] and u1 == [1, 3, 5]
    assert sorted(u0 + u1) == list(range(7))


def test_single_rank_is_identity():
    assert D.max_over_ranks(3.5, 1) == 3.5
    assert D.my_units(3, 0, 1) == [0, 1, 2]
