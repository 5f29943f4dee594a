"""The free-running parity bar (oracle.spread) on the CPU: without noise the
re-runs are the exact run; the bar is the acceptance bar (>= 99.9% of codes,
objective within 1e-3) when the runs agree and widens to twice the observed
spread otherwise; the oracle's W-update is restored after the noisy runs."""
import numpy as np
import pytest

from oracle import admmq_oracle as O
from oracle import spread as S
from post_weight_quantization_10_b200 import workloads


def _layer():
    p = workloads.PRESETS["tiny"]
    Xn, W = workloads.tiny_layer(0)
    H = O.hessian(Xn, p.lambda_rel)
    return workloads.scaled(p, p.n, p.d_in, p.d_out, iters=20), H, W.T.astype(np.float64)


def test_zero_noise_reproduces_the_exact_run():
    p, H, Wm = _layer()
    res, runs = S.noisy_runs(H, Wm, p, "lsq", 0.0, seeds=2)
    for r in runs:
        assert np.array_equal(r["codes"], res["codes"])
        assert r["objective"] == res["objective"]
    assert S.bars(res, runs) == (S.AGREE_BAR, S.REL_BAR, 1.0, 0.0)


def test_noise_moves_the_run_and_w_update_is_restored():
    p, H, Wm = _layer()
    w_update = O.w_update
    res, runs = S.noisy_runs(H, Wm, p, "lsq", 1e-2, seeds=3)
    assert O.w_update is w_update
    assert any(not np.array_equal(r["W_tilde"], res["W_tilde"]) for r in runs)


def test_bar_widens_to_twice_the_spread():
    codes = np.zeros((10, 10), np.uint8)
    res = {"codes": codes, "objective": 2.0}
    moved = codes.copy()
    moved[:1] = 1                      # 90% of the codes agree
    runs = [{"codes": codes, "objective": 2.0}, {"codes": moved, "objective": 2.1}]
    agree_bar, rel_bar, lo, hi = S.bars(res, runs)
    assert lo == pytest.approx(0.9) and hi == pytest.approx(0.05)
    assert agree_bar == pytest.approx(1.0 - (2.0 * 0.1 + 1e-3))
    assert rel_bar == pytest.approx(2.0 * 0.05 + 1e-4)
    # a spread inside the acceptance bar leaves the bar as it is
    runs = [{"codes": codes, "objective": 2.0 * (1 + 1e-5)}]
    assert S.bars(res, runs)[:2] == (S.AGREE_BAR, S.REL_BAR)
