"""The GPU side of the free-running parity bar (test infrastructure): the
GPU's per-step difference from the oracle, at which oracle.spread samples
the oracle's own spread."""
from __future__ import annotations

import numpy as np

from oracle import admmq_oracle as O
from oracle.spread import (AGREE_ADD, AGREE_BAR, EPS_FLOOR, REL_ADD, REL_BAR,  # noqa: F401
                           SPREAD_FACTOR, bars, noisy_runs)


def step0_error(A, p, X, W, H, Wm, grid, split="auto", scaling=True, rescale_dual=False,
                fit_on_w=False):
    """Relative difference between the GPU's W~ after iteration 0 (from the
    bit-exact RTN start) and the oracle's: the size of the GPU's per-step
    difference, at which the oracle's spread is sampled (needs a GPU)."""
    import torch
    prm = A.Params(bits=p.bits, group=p.group, iters=1, rho0=p.rho0, gamma=p.gamma,
                   lambda_rel=p.lambda_rel, grid=grid, split=split, scaling=scaling,
                   rescale_dual=rescale_dual, fit_on_w=fit_on_w)
    s = A.Solver(X.shape[1], W.shape[0], prm)
    s.prepare(A.build_hessian(X), W)
    s.eigh()
    s.init()
    wt = torch.empty((W.shape[0], X.shape[1]), dtype=torch.float32, device=X.device)
    s.dump_wtilde(wt)
    s.iterate(0, 1)
    s.dump_wtilde(None)
    torch.cuda.synchronize()
    trace = []
    O.admm_q(H, Wm, p.bits, p.group, 1, rho0=p.rho0, gamma=p.gamma, grid=grid, scaling=scaling,
             trace=trace, rescale_dual=rescale_dual, fit_on_w=fit_on_w)
    ref = trace[0]["W_tilde"].T
    return float(np.linalg.norm(wt.cpu().numpy().astype(np.float64) - ref) / np.linalg.norm(ref))
