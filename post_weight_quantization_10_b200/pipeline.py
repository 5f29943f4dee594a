"""Host-to-device staging that overlaps the next layer's input copy with the
current layer's solve.

Quantizing a model solves its layers one after another from calibration
activations that live in host memory.  Only the Gram needs X (a few ms);
the iterations that follow (most of the solve) do not, so the copy of layer
i+1's activations and weights can run on a second stream while layer i is
solved.  `InputPipeline` keeps two device copies of the inputs: a copy into
one slot waits until the last kernel that read that slot has finished, and
the solve of a slot waits until its copy has landed (CUDA events, no host
synchronisation).  `solve_layers` runs whole layers through it.

`solve_overlapped` runs the solves of several Hessians (e.g. the four of a
decoder layer) with the most expensive eigendecomposition on a second stream,
while the other solves go ahead on the caller's stream.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


class InputPipeline:
    """Device slots (two by default) for a fixed set of input tensors (shapes,
    dtypes).  One slot is enough when something else runs between a slot's
    use and its next copy (e.g. one pipeline per solve of a decoder layer,
    the copy for solve i + 1 running during solve i)."""

    def __init__(self, like: list[torch.Tensor], device, slots: int = 2,
                 copy_stream: torch.cuda.Stream | None = None):
        self.slots = [[torch.empty(t.shape, dtype=t.dtype, device=device) for t in like]
                      for _ in range(slots)]
        self.copy_stream = copy_stream or torch.cuda.Stream(device=device)
        self.copied = [torch.cuda.Event() for _ in range(slots)]
        self.used = [torch.cuda.Event() for _ in range(slots)]
        self.next = 0

    def prefetch(self, host: list[torch.Tensor]) -> int:
        """Enqueue the copy of `host` (pinned tensors) into the next slot on the
        copy stream; returns the slot."""
        slot = self.next
        self.next = (self.next + 1) % len(self.slots)
        with torch.cuda.stream(self.copy_stream):
            self.copy_stream.wait_event(self.used[slot])  # its previous readers are done
            for dst, src in zip(self.slots[slot], host):
                dst.copy_(src, non_blocking=True)
            self.copied[slot].record(self.copy_stream)
        return slot

    def acquire(self, slot: int) -> list[torch.Tensor]:
        """The slot's device tensors, with the current stream ordered after
        their copy."""
        torch.cuda.current_stream().wait_event(self.copied[slot])
        return self.slots[slot]

    def release(self, slot: int):
        """Mark the slot free once the work enqueued so far on the current
        stream has run."""
        self.used[slot].record(torch.cuda.current_stream())


@dataclass
class LayerResult:
    codes: torch.Tensor      # pinned host u8 [d_out][d_in]
    scale: torch.Tensor      # pinned host fp32 [d_out][d_in / group]
    zero: torch.Tensor
    packed: torch.Tensor     # pinned host int32 [d_out][d_in * bits / 32]
    objective: torch.Tensor  # pinned host fp64 [1]


def solve_layers(layers, params, device="cuda"):
    """Solve a sequence of same-shaped layers given as (X, W_hat) pinned host
    tensors (bf16 [n][d_in], fp32 or bf16 [d_out][d_in]); yields a LayerResult
    per layer, read back on the compute stream (synchronise before reading the
    host tensors).  Each layer gets its own Gram, scaling, eigendecomposition
    and solve; the next layer's inputs are copied during the current solve."""
    from . import admmq as A
    it = iter(layers)
    first = next(it, None)
    if first is None:
        return
    X0, W0 = first
    n, d_in = X0.shape
    d_out = W0.shape[0]
    pipe = InputPipeline([X0, W0], device)
    solver = A.Solver(d_in, d_out, params, device=device)
    H = torch.empty((d_in, d_in), dtype=torch.float32, device=device)
    ws = torch.empty(A.gram_workspace_bytes(n, d_in), dtype=torch.uint8, device=device)
    packed = torch.empty((d_out, d_in * params.bits // 32), dtype=torch.int32, device=device)
    slot = pipe.prefetch([X0, W0])
    pending = next(it, None)
    while True:
        X, W = pipe.acquire(slot)
        nxt = pipe.prefetch(list(pending)) if pending is not None else None
        A.build_hessian(X, H, workspace=ws)
        solver.prepare(H, W)
        solver.eigh()
        solver.solve()
        A.pack(solver.codes, params.bits, out=packed)
        pipe.release(slot)
        res = LayerResult(*(torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                            for t in (solver.codes, solver.scale, solver.zero, packed,
                                      solver.objective)))
        for dst, src in zip((res.codes, res.scale, res.zero, res.packed, res.objective),
                            (solver.codes, solver.scale, solver.zero, packed, solver.objective)):
            dst.copy_(src, non_blocking=True)
        yield res
        if nxt is None:
            return
        slot = nxt
        pending = next(it, None)


def solve_overlapped(jobs, stream=None):
    """Prepare, eigendecompose and solve several layers, given as (Solver,
    G, W_hat) with G = X^T X already built, so that the largest
    eigendecomposition overlaps the other work.  The job with the largest
    d_in (its eigendecomposition costs O(d_in^3), e.g. 1.3 s at 12288
    against 0.09 s at 4096) is prepared and eigendecomposed on a second
    stream from a host thread (the library releases the GIL and the
    eigendecomposition synchronises only its own stream).  The other jobs
    run prepare, eigh and solve one after another on `stream`.  The largest
    job's solve runs last, on `stream`, after its eigendecomposition.  The
    results are those of solving each job alone; the call returns when all
    are enqueued and the side stream's work is done."""
    import threading
    if not jobs:
        return
    main = stream if stream is not None else torch.cuda.current_stream()
    big = max(range(len(jobs)), key=lambda i: jobs[i][0].d_in)
    side = torch.cuda.Stream(device=main.device)
    side.wait_stream(main)  # G and W_hat are ready on the side stream too
    errors = []

    def worker():
        try:
            torch.cuda.set_device(main.device)
            s, G, W = jobs[big]
            s.prepare(G, W, side)
            s.eigh(side)
        except Exception as e:  # re-raised by the caller after the join
            errors.append(e)

    th = threading.Thread(target=worker)
    th.start()
    try:
        for i, (s, G, W) in enumerate(jobs):
            if i != big:
                s.prepare(G, W, main)
                s.eigh(main)
                s.solve(main)
    finally:
        th.join()
    if errors:
        raise errors[0]
    done = torch.cuda.Event()
    done.record(side)
    main.wait_event(done)
    jobs[big][0].solve(main)
