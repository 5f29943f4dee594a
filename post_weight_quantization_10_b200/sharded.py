"""One layer solved on several GPUs (one process per GPU, torch.distributed).

The layer objective is a sum over output rows and every step of the ADMM-Q
iteration acts row by row, so output rows are independent problems once H is
known.  The one real exchange is H itself when the calibration tokens are
split across GPUs: each rank forms the Gram of its tokens, the ranks sum the
d_in x d_in partial Grams (an all-reduce: NCCL over NVLink on GPUs, gloo in
CPU tests), then each rank eigendecomposes the same H~ and solves its own
block of output rows.  The objective and the residual history are sums over
rows: one more scalar all-reduce.

`backend` is the compute module (the C-ABI binding `admmq` on GPUs); the
collectives go through torch.distributed on whatever process group is given.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


def block(n: int, world: int, rank: int) -> tuple[int, int]:
    """Balanced contiguous block [lo, hi) of n items for `rank` of `world`."""
    base, extra = divmod(n, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


@dataclass
class ShardedResult:
    rows: tuple[int, int]       # this rank's output rows [r0, r1)
    codes: torch.Tensor         # u8 [r1 - r0][d_in]
    scale: torch.Tensor         # fp32 [r1 - r0][d_in / group]
    zero: torch.Tensor
    objective: float            # whole-layer objective (sum over all ranks)
    solver: object              # the backend's per-rank solver (buffers, timing)


def gram_allreduce(X_local: torch.Tensor, backend, world: int, group=None) -> torch.Tensor:
    """H = sum over ranks of X_r^T X_r (fp32, no damping), on every rank."""
    G = backend.build_hessian(X_local)
    if world > 1:
        dist.all_reduce(G, op=dist.ReduceOp.SUM, group=group)
    return G


def solve_layer_sharded(X_local: torch.Tensor, W_rows: torch.Tensor, rows: tuple[int, int], params,
                        backend, world: int, group=None, stream=None) -> ShardedResult:
    """X_local: this rank's calibration tokens [n_r][d_in]; W_rows: this
    rank's block rows = (r0, r1) of W_hat's output rows, [r1 - r0][d_in]
    (see `block`)."""
    G = gram_allreduce(X_local, backend, world, group)
    s = backend.Solver(X_local.shape[1], W_rows.shape[0], params, device=W_rows.device)
    s.prepare(G, W_rows, stream)
    s.eigh(stream)
    s.solve(stream)
    obj = s.objective.clone()
    if world > 1:
        dist.all_reduce(obj, op=dist.ReduceOp.SUM, group=group)
    return ShardedResult(rows=tuple(rows), codes=s.codes, scale=s.scale, zero=s.zero,
                         objective=float(obj.cpu()), solver=s)
