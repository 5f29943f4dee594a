"""Degenerate layers through the whole solve (needs a B200).

A single output row, the smallest input width (32: less than one fp16-split
stage of 64 K-elements; 96: a last stage half past the K extent, read as
zeros), fewer calibration tokens than input channels (X is
rank deficient; H is positive definite only through the damping), all-zero
weight rows, weights with outliers over six orders of magnitude under the
fp16 split's power-of-two row scales, and T = 0 (the solve is the RTN start).
Each result must be a valid solution (codes in [0, L], positive scales,
integer zero points in [0, L], the reported objective equal to the objective
of the returned codes), within the acceptance bar of the float64 oracle's
free-running solve (widened only as far as the oracle's own spread under
noise of the GPU's per-step size requires, as in the free-running tests),
and exact where the method fixes it.
"""
import numpy as np
import pytest
import torch

import _spread as S
from oracle import admmq_oracle as O
from post_weight_quantization_10_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def A():
    from post_weight_quantization_10_b200 import admmq
    admmq.lib()
    return admmq


BASE = workloads.PRESETS["q_proj"]
CASES = {
    # name: (n, d_in, d_out, group, split, weight edit)
    "one_row": (2048, 128, 1, 128, "auto", None),
    "d32": (1024, 32, 40, 32, "auto", None),
    "d32_f16": (1024, 32, 40, 32, "f16", None),      # K = 32 < one 64-element stage
    "d96_f16": (2048, 96, 40, 32, "f16", None),      # last stage half past the K extent
    "few_tokens": (16, 256, 64, 64, "auto", None),
    "zero_rows": (2048, 128, 48, 64, "auto", "zero_rows"),
    "outliers_f16": (2048, 256, 64, 64, "f16", "outliers"),
}


def _case(name, seed=0):
    n, d, m, g, split, edit = CASES[name]
    p = workloads.scaled(BASE, n, d, m, group=g, iters=40, rank=min(16, d // 2))
    X = workloads.make_activations(p, seed=seed, device="cuda")
    W = workloads.make_weights(p, seed=seed, device="cuda", dtype=torch.float32)
    if edit == "zero_rows":
        W[5] = 0.0
        W[17] = 0.0
    elif edit == "outliers":
        W[:, 7] *= 1000.0         # one input channel with huge weights in every row
        W[3] *= 1e-6              # one nearly-zero row
    return p, split, X, W


def _solve(A, p, split, X, W, iters=None):
    prm = A.Params(bits=p.bits, group=p.group, iters=p.iters if iters is None else iters,
                   rho0=p.rho0, gamma=p.gamma, lambda_rel=p.lambda_rel, grid="lsq", split=split)
    s = A.solve_layer(X, W, prm)
    s.check()
    return s


def _valid(p, s, H, Wm):
    L = (1 << p.bits) - 1
    codes = s.codes.cpu().numpy().astype(np.int64)
    sc, ze = s.scale.cpu().numpy(), s.zero.cpu().numpy()
    assert codes.min() >= 0 and codes.max() <= L
    assert np.all(sc > 0) and np.all(np.isfinite(sc))
    assert np.all((ze >= 0) & (ze <= L) & (ze == np.rint(ze)))
    D = (np.repeat(sc, p.group, axis=1) * (codes - np.repeat(ze, p.group, axis=1))).astype(np.float32)
    obj = float(s.objective.cpu())
    assert O.objective(H, D.T.astype(np.float64), Wm) == pytest.approx(obj, rel=1e-4)
    return codes, obj


@pytest.mark.parametrize("name", sorted(CASES))
def test_degenerate_layer_solves(A, name):
    p, split, X, W = _case(name)
    s = _solve(A, p, split, X, W)
    H = O.hessian(X.float().cpu().numpy(), p.lambda_rel)
    Wm = W.float().cpu().numpy().T.astype(np.float64)
    eps = max(S.step0_error(A, p, X, W, H, Wm, "lsq", split=split), S.EPS_FLOOR)
    res, runs = S.noisy_runs(H, Wm, p, "lsq", eps, seeds=16)
    codes, obj = _valid(p, s, H, Wm)
    agree = float(np.mean(codes == res["codes"].T))
    rel = obj / res["objective"] - 1.0 if res["objective"] > 0 else obj
    agree_bar, rel_bar, lo, hi = S.bars(res, runs)
    print(f"{name}: split {s.split}, codes agree {agree:.5f}, objective rel {rel:+.3e}; "
          f"oracle at noise {eps:.1e}: agree >= {lo:.5f}, |rel| <= {hi:.2e}")
    assert agree >= agree_bar and abs(rel) <= rel_bar
    if name == "zero_rows":
        # a zero row stays on its RTN grid (s = 1, z = 0) with every code 0
        for r in (5, 17):
            assert np.all(codes[r] == 0)
            assert np.all(s.scale[r].cpu().numpy() == 1.0) and np.all(s.zero[r].cpu().numpy() == 0.0)


@pytest.mark.parametrize("split", ["auto", "f16"])
def test_zero_iterations_is_the_rtn_start(A, split):
    """T = 0: the solve returns the RTN start bit for bit, and its objective."""
    p = workloads.scaled(BASE, 2048, 256, 72, group=64, rank=16)
    X = workloads.make_activations(p, seed=4, device="cuda")
    W = workloads.make_weights(p, seed=4, device="cuda", dtype=torch.float32)
    s = _solve(A, p, split, X, W, iters=0)
    Wm = W.float().cpu().numpy().T.astype(np.float64)
    codes, scale, zero, D = O.rtn(Wm, p.bits, p.group)
    np.testing.assert_array_equal(s.codes.cpu().numpy(), codes.T)
    np.testing.assert_array_equal(s.scale.cpu().numpy(), scale.T.astype(np.float32))
    np.testing.assert_array_equal(s.zero.cpu().numpy(), zero.T.astype(np.float32))
    H = O.hessian(X.float().cpu().numpy(), p.lambda_rel)
    assert float(s.objective.cpu()) == pytest.approx(O.objective(H, D, Wm), rel=1e-4)


@pytest.mark.parametrize("bits", [1, 8])
@pytest.mark.parametrize("split", ["auto", "f16"])
def test_extreme_bit_widths(A, bits, split):
    """b = 1 (two levels per group) and b = 8 (256 levels): valid solutions
    within the bar of the free-running tests, with codes spanning the whole
    range [0, 2^b - 1]."""
    p = workloads.scaled(BASE, 2048, 256, 64, group=64, bits=bits, iters=40, rank=16)
    X = workloads.make_activations(p, seed=6, device="cuda")
    W = workloads.make_weights(p, seed=6, device="cuda", dtype=torch.float32)
    s = _solve(A, p, split, X, W)
    H = O.hessian(X.float().cpu().numpy(), p.lambda_rel)
    Wm = W.float().cpu().numpy().T.astype(np.float64)
    eps = max(S.step0_error(A, p, X, W, H, Wm, "lsq", split=split), S.EPS_FLOOR)
    res, runs = S.noisy_runs(H, Wm, p, "lsq", eps, seeds=16)
    codes, obj = _valid(p, s, H, Wm)
    assert codes.min() == 0 and codes.max() == (1 << bits) - 1
    agree = float(np.mean(codes == res["codes"].T))
    rel = obj / res["objective"] - 1.0
    agree_bar, rel_bar, lo, hi = S.bars(res, runs)
    print(f"bits {bits} / {s.split}: codes agree {agree:.5f}, objective rel {rel:+.3e}; "
          f"oracle at noise {eps:.1e}: agree >= {lo:.5f}, |rel| <= {hi:.2e}")
    assert agree >= agree_bar and abs(rel) <= rel_bar
