"""The sharded single-layer solve's host logic on CPU (gloo, world size 2):
token and row blocks, the all-reduce of the partial Grams, the per-rank solve
of a row block and the summed objective.  The compute backend here is a
float64 stand-in built on the oracle (the GPU path uses the C-ABI library);
the result must equal the unsharded oracle solve of the whole layer."""
import datetime
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import admmq_oracle as O
from post_weight_quantization_10_b200 import sharded, workloads


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class _OracleBackend:
    """Float64 stand-in for the library: same calls, oracle arithmetic."""

    @staticmethod
    def build_hessian(X):
        Xd = X.double()
        return Xd.T @ Xd

    class Solver:
        def __init__(self, d_in, d_out, params, device=None):
            self.p = params

        def prepare(self, G, W, stream=None):
            self.G, self.W = G.numpy(), W.double().numpy()

        def eigh(self, stream=None):
            pass

        def solve(self, stream=None):
            p = self.p
            H = O.damping(self.G, p.lambda_rel)[0]
            res = O.admm_q(H, self.W.T, p.bits, p.group, p.iters, rho0=p.rho0, gamma=p.gamma,
                           grid=p.grid)
            self.codes = torch.from_numpy(res["codes"].T.copy())
            self.scale = torch.from_numpy(res["scale"].T.copy())
            self.zero = torch.from_numpy(res["zero"].T.copy())
            self.objective = torch.tensor([res["objective"]], dtype=torch.float64)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from post_weight_quantization_10_b200.admmq import Params
        p = workloads.PRESETS["tiny"]
        Xn, Wn = workloads.tiny_layer(0)
        t0, t1 = sharded.block(Xn.shape[0], world, rank)
        r0, r1 = sharded.block(Wn.shape[0], world, rank)
        prm = Params(bits=p.bits, group=p.group, iters=p.iters, rho0=p.rho0, gamma=p.gamma,
                     lambda_rel=p.lambda_rel, grid="lsq")
        res = sharded.solve_layer_sharded(torch.from_numpy(Xn[t0:t1]), torch.from_numpy(Wn[r0:r1]),
                                          (r0, r1), prm, _OracleBackend, world)
        q.put((rank, res.rows, res.codes.numpy(), res.objective))
    finally:
        dist.destroy_process_group()


def test_block_partition():
    for n in (0, 1, 7, 32, 1000):
        for w in (1, 2, 3, 8):
            blocks = [sharded.block(n, w, r) for r in range(w)]
            assert blocks[0][0] == 0 and blocks[-1][1] == n
            assert all(blocks[i][1] == blocks[i + 1][0] for i in range(w - 1))
            sizes = [b - a for a, b in blocks]
            assert max(sizes) - min(sizes) <= 1


def test_two_rank_sharded_solve_equals_whole_layer():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for pr in procs:
        pr.start()
    res = sorted((q.get(timeout=300) for _ in range(2)), key=lambda t: t[0])
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    p = workloads.PRESETS["tiny"]
    Xn, Wn = workloads.tiny_layer(0)
    H = O.hessian(Xn, p.lambda_rel)
    whole = O.admm_q(H, Wn.T.astype(np.float64), p.bits, p.group, p.iters, rho0=p.rho0,
                     gamma=p.gamma, grid="lsq")
    (_, rows0, c0, obj0), (_, rows1, c1, obj1) = res
    assert rows0 == (0, 16) and rows1 == (16, 32)
    np.testing.assert_array_equal(np.concatenate([c0, c1]), whole["codes"].T)
    assert obj0 == obj1 == np.float64(obj0)
    assert abs(obj0 - whole["objective"]) <= 1e-9 * abs(whole["objective"])
