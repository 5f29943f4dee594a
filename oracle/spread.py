"""How far the float64 oracle's own free-running solve moves on a layer when
its W-update carries relative noise of a given size.

TEST INFRASTRUCTURE ONLY, like the rest of oracle/: the tests and the smoke
check use it to set the bar a free-running GPU solve is held to.

The ADMM-Q iteration with a non-convex projection is path-sensitive: a
perturbation at the level of the last bits of float32 can send a row into
another basin of the iteration (ADMM-Q summary, Methodology section 2: the
D-update is a discrete projection; convergence holds under the growing
penalty, but the limit point depends on the path).  A GPU solve differs from
the oracle's by its float32 Gram and its split-precision W-update; its
per-step difference is measured (W~ after iteration 0 against the
oracle's) and the oracle is re-run
with random relative noise of that size on every W-update.  The GPU's
free-running result is then judged against the spread of those runs, and
against the fixed acceptance bar (codes >= 99.9% equal, objective within
1e-3) wherever that spread is tighter.
"""
from __future__ import annotations

import numpy as np

from . import admmq_oracle as O

# The acceptance bar: codes >= 99.9% equal, objective within 1e-3 relative.
AGREE_BAR, REL_BAR = 0.999, 1e-3
# Where the oracle's own spread is wider than the bar, the bar is widened to
# 2 x that spread (plus 1e-3 of the codes or 1e-4 of the objective): the
# spread is sampled with a handful of seeds, and the GPU's perturbation is a
# fixed one (its float32 Gram and split-precision roundings), not random.
SPREAD_FACTOR, AGREE_ADD, REL_ADD = 2.0, 1e-3, 1e-4
# Noise below this is not resolved by the float64 oracle's own roundings.
EPS_FLOOR = 1e-7


def noisy_runs(H, Wm, p, grid, eps, seeds=6, eig=None, **kw):
    """The exact oracle solve and `seeds` solves whose W-update result is
    multiplied by (1 + eps * N(0, 1)) elementwise (numpy PCG64, seed i).
    Returns (exact result, [noisy results])."""
    res = O.admm_q(H, Wm, p.bits, p.group, p.iters, rho0=p.rho0, gamma=p.gamma, grid=grid,
                   eig=eig, **kw)
    w_update = O.w_update
    runs = []
    try:
        for seed in range(seeds):
            rng = np.random.default_rng(seed)

            def noisy(*a, rng=rng):
                Wt = w_update(*a)
                return Wt * (1.0 + eps * rng.standard_normal(Wt.shape))

            O.w_update = noisy
            runs.append(O.admm_q(H, Wm, p.bits, p.group, p.iters, rho0=p.rho0, gamma=p.gamma,
                                 grid=grid, eig=eig, **kw))
    finally:
        O.w_update = w_update
    return res, runs


def bars(res, runs):
    """(lowest code agreement to accept, largest |objective change| to
    accept, lowest noisy agreement, largest noisy change) for a result
    compared with the exact run `res`: the acceptance bar, widened only as far
    as the oracle's own spread `runs` requires."""
    agrees = [float(np.mean(r["codes"] == res["codes"])) for r in runs]
    rels = [abs(r["objective"] / res["objective"] - 1.0) if res["objective"] > 0 else
            abs(r["objective"]) for r in runs]
    lo, hi = min(agrees), max(rels)
    agree_bar = min(AGREE_BAR, 1.0 - (SPREAD_FACTOR * (1.0 - lo) + AGREE_ADD))
    rel_bar = max(REL_BAR, SPREAD_FACTOR * hi + REL_ADD)
    return agree_bar, rel_bar, lo, hi
