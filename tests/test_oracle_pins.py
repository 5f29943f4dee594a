"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test ties an oracle function to something other than itself: values the
pages print (tests/golden/), closed forms, brute force, or an independent
route to the same number.
"""
import os

import numpy as np
import pytest

from oracle import admmq_oracle as O
from oracle import projection_fp32 as P
from post_weight_quantization_10_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = (x.strip() for x in line.split("=", 1))
            vals[k] = v
    return vals


def _vec(s):
    return np.array([float(x) for x in s.split()])


def _spd(d, rng, cond=50.0):
    A = rng.standard_normal((d, d))
    Qm, _ = np.linalg.qr(A)
    ev = np.exp(np.linspace(0, np.log(cond), d))
    return (Qm * ev) @ Qm.T


# ---------------------------------------------------------------- GPTQ pins


def test_worked_example_compensation_values():
    """GPTQ tutorial section 2: delta = (0.2, -0.1), cost 0.04 -> 0.03."""
    g = _read_golden("gptq_worked_example.txt")
    H = np.array([_vec(r) for r in g["H"].split(";")])
    q = int(g["forced_index"])
    d = float(g["forced_change"])
    delta = O.compensation(H, q, d)
    np.testing.assert_allclose(delta, _vec(g["expected_delta"]), atol=1e-15)
    e = np.zeros(2)
    e[q] = d
    assert 0.5 * e @ H @ e == pytest.approx(float(g["cost_uncompensated"]), abs=1e-15)
    assert 0.5 * delta @ H @ delta == pytest.approx(float(g["cost_compensated"]), abs=1e-15)


def test_worked_example_through_gptq_algorithm():
    """The same example run through Algorithm 1: the first column is forced
    up by 0.2 on a coarse grid, the second sits on a very fine grid, so its
    quantized value is the compensated weight."""
    g = _read_golden("gptq_worked_example.txt")
    H = np.array([_vec(r) for r in g["H"].split(";")])
    W = np.array([[0.3, 0.0]])                       # 0.3 -> 0.5 on step 0.5
    scale = np.array([[0.5, 1e-9]], dtype=np.float32)
    zero = np.zeros((1, 2), dtype=np.float32)
    codes, Qw = O.gptq(H, W, scale, zero, bits=8, group=1, block=2, clamp=False)
    delta = Qw[0] - W[0]
    np.testing.assert_allclose(delta, _vec(g["expected_delta"]), atol=1e-8)
    assert 0.5 * delta @ H @ delta == pytest.approx(float(g["cost_compensated"]), abs=1e-8)


def test_collinear_example_gptq_and_admm():
    """GPTQ tutorial section 2: x1 = x2, weights 0.49/0.51 on the grid {0, 1}:
    GPTQ gives (0, 1) and the output is preserved; the objective equals the
    brute-force optimum lambda * 0.49^2, and ADMM-Q on the same fixed grid
    reaches it too."""
    g = _read_golden("gptq_collinear_example.txt")
    w = _vec(g["weights"])
    rng = np.random.default_rng(0)
    x = rng.standard_normal(64)
    X = np.stack([x, x], axis=1)
    G = O.gram(X)
    assert np.linalg.matrix_rank(G) == 1              # singular without damping
    H, lam = O.damping(G, 0.01)
    scale = np.ones((1, 1), np.float32)
    zero = np.zeros((1, 1), np.float32)
    codes, Qw = O.gptq(H, w[None, :], scale, zero, bits=1, group=2)
    np.testing.assert_array_equal(codes[0], _vec(g["expected_codes"]).astype(int))
    np.testing.assert_allclose(X @ Qw[0], X @ w, rtol=0, atol=1e-12)
    best, _ = O.brute_force_column(H, w, np.ones(1), np.zeros(1), bits=1, group=2)
    assert best == pytest.approx(lam * 0.49 ** 2, rel=1e-12)
    assert O.objective(H, Qw[0][:, None], w[:, None]) == pytest.approx(best, rel=1e-12)
    res = O.admm_q(H, w[:, None], bits=1, group=2, iters=200, grid="frozen",
                   grid0=(np.ones((1, 1)), np.zeros((1, 1))))
    assert res["objective"] == pytest.approx(best, rel=1e-9)


def test_gptq_first_step_is_closed_form_compensation():
    rng = np.random.default_rng(1)
    d = 8
    H = _spd(d, rng)
    w = rng.standard_normal(d)
    scale = np.full((1, d), 1e-9, np.float32)
    scale[0, 0] = 0.7
    zero = np.zeros((1, d), np.float32)
    _, Qw = O.gptq(H, w[None, :], scale, zero, bits=8, group=1, clamp=False)
    q0 = 0.7 * np.rint(w[0] / 0.7)
    delta = O.compensation(H, 0, q0 - w[0])
    np.testing.assert_allclose(Qw[0], w + delta, atol=1e-6)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_gptq_block_size_invariance(seed):
    """Algorithm 1's lazy block update changes the order of the arithmetic only."""
    rng = np.random.default_rng(seed)
    d, m, g, bits = 24, 5, 8, 3
    X = rng.standard_normal((200, d)) @ rng.standard_normal((d, d))
    H = O.hessian(X)
    W = rng.standard_normal((m, d)) * 0.1
    s, z = O.minmax_grid_rows(W, bits, g)
    ref, _ = O.gptq(H, W, s, z, bits, g, block=1)
    for B in (3, 8, 128):
        c, _ = O.gptq(H, W, s, z, bits, g, block=B)
        np.testing.assert_array_equal(c, ref)


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_back_to_front_gptq_equals_babai(seed):
    """Theorem 4 of the Babai page: GPTQ run from the last input channel to the
    first returns Babai's nearest-plane point (no clipping, no LLL)."""
    rng = np.random.default_rng(seed)
    d, g = 12, 4
    X = rng.standard_normal((100, d)) @ rng.standard_normal((d, d))
    H = O.hessian(X)
    w = rng.standard_normal(d)
    s_grp = np.abs(rng.standard_normal(d // g)) * 0.3 + 0.05
    s = np.repeat(s_grp, g)
    scale = s_grp[None, :].astype(np.float64)
    zero = np.zeros_like(scale)
    codes, _ = O.gptq(H, w[None, :], scale, zero, bits=8, group=g,
                      order=np.arange(d)[::-1], clamp=False)
    c_babai = O.babai_nearest_plane(H, w, s)
    np.testing.assert_array_equal(codes[0], c_babai.astype(int))


@pytest.mark.parametrize("seed", range(6))
def test_babai_error_bound_theorem5(seed):
    rng = np.random.default_rng(seed)
    d = 10
    H = O.hessian(rng.standard_normal((60, d)) @ rng.standard_normal((d, d)))
    w = rng.standard_normal(d)
    s = np.abs(rng.standard_normal(d)) + 0.1
    c = O.babai_nearest_plane(H, w, s)
    e = w - s * c
    assert e @ H @ e <= O.babai_error_bound(H, s) * (1 + 1e-12)
    # the mechanism of the bound: each nearest-plane residual is at most half
    # a step of its Gram-Schmidt length
    R = np.linalg.cholesky(H).T
    assert np.all(np.abs(R @ e) <= 0.5 * np.diag(R) * s * (1 + 1e-9))


# ------------------------------------------------------- ADMM-Q building blocks


def test_gram_and_damping():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((20000, 7)).astype(np.float32)
    G = O.gram(X, chunk=4096)
    Xd = X.astype(np.float64)
    np.testing.assert_allclose(G, np.einsum("ni,nj->ij", Xd, Xd), rtol=1e-12)
    H, lam = O.damping(G, 0.01)
    assert lam == pytest.approx(0.01 * np.trace(G) / 7, rel=1e-14)
    np.testing.assert_allclose(np.diag(H) - np.diag(G), lam, rtol=1e-12)


def test_objective_equals_output_error():
    """1/2 Tr(D^T H D) = 1/2 (||X D||^2 + lambda ||D||^2) for H = X^T X + lambda I."""
    rng = np.random.default_rng(4)
    X = rng.standard_normal((300, 9))
    H, lam = O.damping(O.gram(X), 0.01)
    W_hat = rng.standard_normal((9, 4))
    W = W_hat + rng.standard_normal((9, 4)) * 0.1
    Dl = W - W_hat
    direct = 0.5 * (np.sum((X @ Dl) ** 2) + lam * np.sum(Dl ** 2))
    assert O.objective(H, W, W_hat) == pytest.approx(direct, rel=1e-12)


def test_scaling_unit_diagonal_and_invariance():
    rng = np.random.default_rng(5)
    X = rng.standard_normal((400, 12)) * np.exp(rng.standard_normal(12) * 2)
    H = O.hessian(X)
    sigma, Ht = O.diagonal_scaling(H)
    np.testing.assert_allclose(np.diag(Ht), 1.0, rtol=1e-14)
    W_hat = rng.standard_normal((12, 3))
    W = W_hat + rng.standard_normal((12, 3))
    a = O.objective(H, W, W_hat)
    b = O.objective(Ht, W / sigma[:, None], W_hat / sigma[:, None])
    assert a == pytest.approx(b, rel=1e-12)


def test_w_update_matches_linear_solve():
    """Eigenbasis W-update = the solution of (H~ + rho I) W = H~ W^~ + rho (D~ - V~)."""
    rng = np.random.default_rng(6)
    d, m = 32, 5
    H = O.hessian(rng.standard_normal((200, d)) @ rng.standard_normal((d, d)))
    _, Ht = O.diagonal_scaling(H)
    lam, Q = np.linalg.eigh(Ht)
    Wt_hat = rng.standard_normal((d, m))
    Dt = rng.standard_normal((d, m))
    Vt = rng.standard_normal((d, m)) * 0.1
    for rho in (0.1, 3.7, 250.0):
        a = O.w_update(Q, lam, Ht @ Wt_hat, rho, Dt, Vt)
        b = np.linalg.solve(Ht + rho * np.eye(d), Ht @ Wt_hat + rho * (Dt - Vt))
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-10 * np.abs(b).max())
        # it minimises the augmented objective: gradient vanishes
        grad = Ht @ (a - Wt_hat) + rho * (a - Dt + Vt)
        assert np.abs(grad).max() < 1e-9 * (1 + rho) * np.abs(a).max()


# ------------------------------------------------------------ grid and projection


def test_minmax_grid_hand_example():
    """y = (-1, 0.5, 2), 2 bits: mn=-1, mx=2, s=1, z=1; codes (0, 1, 3) with
    rint(0.5) = 0 (ties to even)."""
    y = np.array([[-1.0, 0.5, 2.0]], np.float32)
    s, z = P.fit_minmax(y, 3)
    assert (s[0], z[0]) == (1.0, 1.0)
    q = P.round_to_grid(y, s, z, 3)
    np.testing.assert_array_equal(q[0], [0, 1, 3])
    np.testing.assert_array_equal(P.dequantize(q, s, z)[0], [-1, 0, 2])


def test_minmax_grid_one_signed_groups():
    """The range always includes 0, so a one-signed group still gets a grid
    with 0 on it and an integer zero point in [0, L]: y = (0.5, 1, 2), 2 bits:
    mn = 0, mx = 2, s = 2/3, z = 0, codes (1, 2, 3); y = (-2, -1, -0.5): mn =
    -2, mx = 0, s = 2/3, z = rint(2 / fl(2/3)) = 3, codes (0, 1, 2) with
    rint(-1.5) = -2 (ties to even)."""
    f = np.float32
    y = np.array([[0.5, 1.0, 2.0], [-2.0, -1.0, -0.5]], f)
    s, z = P.fit_minmax(y, 3)
    np.testing.assert_array_equal(s, [f(2) / f(3), f(2) / f(3)])
    np.testing.assert_array_equal(z, [0.0, 3.0])
    np.testing.assert_array_equal(P.round_to_grid(y, s, z, 3), [[1, 2, 3], [0, 1, 2]])


def test_minmax_grid_all_zero_group():
    y = np.zeros((1, 8), np.float32)
    s, z = P.fit_minmax(y, 7)
    assert (s[0], z[0]) == (1.0, 0.0)
    np.testing.assert_array_equal(P.round_to_grid(y, s, z, 7), 0)


def test_mse_clip_hand_example():
    """2 bits, one group of 128: a zero, 126 ones and one outlier 3.2.  The
    min/max grid (s = 3.2/3) misses every 1 by 1/15: error 126/225 = 0.56.  The
    ratio 30/32 clips the range to [0, 3]: s = 1 puts every 1 on the grid
    and costs only (3.2 - 3)^2 = 0.04 at the outlier, less than any other
    ratio (31/32 leaves 126 * (1/30)^2 = 0.14 on the ones).  Mirrored, the
    zero point moves to 3."""
    y = np.ones((1, 128), np.float32)
    y[0, 0], y[0, -1] = 0.0, 3.2
    s, z, e = P.fit_mse(y, 3, return_error=True)
    assert (s[0], z[0]) == (1.0, 0.0)
    assert abs(e[0] - 0.04) < 1e-6
    s_mm, _ = P.fit_minmax(y, 3)
    assert abs(s_mm[0] - 3.2 / 3) < 1e-6
    s, z = P.fit_mse(-y, 3)
    assert (s[0], z[0]) == (1.0, 3.0)


def test_mse_clip_all_zero_group():
    y = np.zeros((2, 16), np.float32)
    s, z = P.fit_mse(y, 7)
    np.testing.assert_array_equal(s, 1.0)
    np.testing.assert_array_equal(z, 0.0)


def test_mse_clip_exact_grid_keeps_minmax():
    """Points that fill a grid from level 0 to level L are reproduced exactly
    by the min/max grid, so the search keeps it (later ratios tie or lose)."""
    rng = np.random.default_rng(11)
    L = 7
    G, g = 30, 32
    s_true = (2.0 ** -rng.integers(3, 9, G)).astype(np.float32)
    z_true = rng.integers(1, L, G).astype(np.float32)
    q = rng.integers(0, L + 1, (G, g)).astype(np.float32)
    q[:, 0], q[:, 1] = 0, L
    y = P.dequantize(q, s_true, z_true)
    s, z, e = P.fit_mse(y, L, return_error=True)
    np.testing.assert_array_equal(s, s_true)
    np.testing.assert_array_equal(z, z_true)
    np.testing.assert_array_equal(e, 0.0)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_mse_clip_search_against_float64(bits):
    """Heavy-tailed groups: the chosen grid is never worse than min/max and
    is, within float32 rounding of the error sums, the best of the clipped
    grids, each evaluated here in float64 by brute force over its levels."""
    rng = np.random.default_rng(100 + bits)
    L = (1 << bits) - 1
    G, g = 300, 64
    y = (rng.standard_t(3, (G, g)) * 0.02).astype(np.float32)
    s, z = P.fit_mse(y, L)
    y64 = y.astype(np.float64)

    def err64(sg, zg):
        lev = sg[:, None] * (np.arange(L + 1)[None, :] - zg[:, None])
        return (np.abs(y64[:, :, None] - lev[:, None, :]).min(axis=2) ** 2).sum(axis=1)

    e_pick = err64(s.astype(np.float64), z.astype(np.float64))
    mn = np.minimum(y64.min(axis=1), 0.0)
    mx = np.maximum(y64.max(axis=1), 0.0)
    e_all = []
    for k in range(16):
        a = 1.0 - k / 32.0
        sk = (a * mx - a * mn) / L
        zk = np.rint(-a * mn / sk)
        e_all.append(err64(sk, zk))
    e_all = np.array(e_all)
    assert np.all(e_pick <= e_all[0] * (1 + 1e-5) + 1e-12)
    assert np.all(e_pick <= e_all.min(axis=0) * (1 + 1e-4) + 1e-12)
    assert np.mean(e_pick < e_all[0] * (1 - 1e-3)) > 0.5   # clipping pays on t(3) tails


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_projection_is_nearest_grid_point(bits):
    """On a fixed grid the D-update rounds each entry to its nearest level
    (brute force over all 2^b levels); codes lie in [0, L]; D is on the grid,
    which contains 0."""
    rng = np.random.default_rng(bits)
    L = (1 << bits) - 1
    y = (rng.standard_normal((50, 16)) * 0.05).astype(np.float32)
    s, z = P.fit_minmax(y, L)
    q = P.round_to_grid(y, s, z, L)
    D = P.dequantize(q, s, z)
    assert q.min() >= 0 and q.max() <= L
    levels = s[:, None] * (np.arange(L + 1)[None, :] - z[:, None])        # (G, L+1)
    assert np.all(np.any(levels == 0, axis=1))
    dist = np.abs(y[:, :, None].astype(np.float64) - levels[:, None, :])
    best = levels[np.arange(50)[:, None], dist.argmin(axis=2)]
    np.testing.assert_allclose(D, best, rtol=0, atol=1e-7)
    # perturbing y off the grid still returns the nearest level
    y2 = (y * 3).astype(np.float32)
    q2 = P.round_to_grid(y2, s, z, L)
    D2 = P.dequantize(q2, s, z)
    dist2 = np.abs(y2[:, :, None].astype(np.float64) - levels[:, None, :])
    np.testing.assert_allclose(D2, levels[np.arange(50)[:, None], dist2.argmin(axis=2)], atol=1e-7)


def test_lsq_refit_recovers_exact_grid():
    """Points exactly on a grid s (q - z) are fitted back to (s, z) by the
    weighted least-squares refresh, whatever the (positive) weights."""
    rng = np.random.default_rng(7)
    L = 7
    G, g = 40, 32
    s_true = (rng.random(G) * 0.1 + 0.01).astype(np.float32)
    z_true = rng.integers(1, L, G).astype(np.float32)
    q = rng.integers(0, L + 1, (G, g)).astype(np.float32)
    q[:, 0], q[:, 1] = 0, L
    y = P.dequantize(q, s_true, z_true)
    w = (rng.random((G, g)) * 10 + 0.1).astype(np.float32)
    s, z = P.fit_lsq(y, w, (s_true * 1.01).astype(np.float32), z_true, L)
    np.testing.assert_array_equal(z, z_true)
    np.testing.assert_allclose(s, s_true, rtol=1e-5)


def test_lsq_refit_does_not_increase_weighted_error():
    rng = np.random.default_rng(8)
    L = 7
    y = (rng.standard_normal((200, 64)) * 0.05).astype(np.float32)
    w = (np.exp(rng.standard_normal((200, 64)))).astype(np.float32)
    s0, z0 = P.fit_minmax(y, L)
    s1, z1 = P.fit_lsq(y, w, s0, z0, L)

    def err(s, z):
        D = P.dequantize(P.round_to_grid(y, s, z, L), s, z)
        return np.sum(w.astype(np.float64) * (y - D) ** 2, axis=1)
    e0, e1 = err(s0, z0), err(s1, z1)
    assert np.mean(e1 <= e0 * (1 + 1e-6)) > 0.95
    assert e1.sum() < e0.sum()


def test_lsq_refit_stages_against_lstsq():
    """Each stage of the least-squares refresh against numpy's least-squares
    solver in float64 on the same data (an independent route; the refit
    itself sums in float32, by 32-column blocks):
    1. with the codes q of the previous grid, the weighted straight-line fit
       y ~ s1 q + b gives the slope s1 and the zero point z = -b / s1, which
       is rounded and clamped to an integer zc;
    2. with zc fixed, the scale minimises sum w (y - s (q - zc))^2.
    Groups whose fit falls back (a non-positive slope) keep the previous
    grid."""
    rng = np.random.default_rng(31)
    L = 7
    G, g = 300, 128
    y = (rng.standard_normal((G, g)) * 0.05 + rng.standard_normal((G, 1)) * 0.02).astype(np.float32)
    w = np.exp(rng.standard_normal((G, g))).astype(np.float32)
    s0, z0 = P.fit_minmax((y * 1.2).astype(np.float32), L)
    s, z = P.fit_lsq(y, w, s0, z0, L)
    q = P.round_to_grid(y, s0, z0, L).astype(np.float64)
    yd, wd = y.astype(np.float64), w.astype(np.float64)
    checked = 0
    for i in range(G):
        rw = np.sqrt(wd[i])
        A = np.stack([q[i], np.ones(g)], axis=1) * rw[:, None]
        slope, icpt = np.linalg.lstsq(A, yd[i] * rw, rcond=None)[0]
        if slope <= 0:
            assert s[i] == s0[i] and z[i] == z0[i]
            continue
        zc = float(np.clip(np.rint(-icpt / slope), 0, L))
        if abs(-icpt / slope - np.rint(-icpt / slope)) < 1e-3:
            continue  # a zero point within float32 reach of a rounding tie
        assert z[i] == zc, (i, z[i], zc)
        a = (q[i] - zc) * rw
        s_ref = np.linalg.lstsq(a[:, None], yd[i] * rw, rcond=None)[0][0]
        if s_ref > 0:
            assert s[i] == pytest.approx(s_ref, rel=2e-5), i
        checked += 1
    assert checked > 0.8 * G


def test_lsq_refit_scale_is_a_weighted_minimum():
    """The refitted scale minimises the weighted squared error of the codes
    it was fitted from, at the refitted zero point: moving it by 1e-3
    either way increases sum w (y - s (q - z))^2."""
    rng = np.random.default_rng(32)
    L = 3
    y = (rng.standard_normal((100, 64)) * 0.05).astype(np.float32)
    w = np.exp(rng.standard_normal((100, 64))).astype(np.float32)
    s0, z0 = P.fit_minmax(y, L)
    s, z = P.fit_lsq(y, w, s0, z0, L)
    q = P.round_to_grid(y, s0, z0, L).astype(np.float64)
    yd, wd = y.astype(np.float64), w.astype(np.float64)

    def e(sc):
        return np.sum(wd * (yd - sc[:, None] * (q - z.astype(np.float64)[:, None])) ** 2, axis=1)
    sd = s.astype(np.float64)
    moved = (s != s0) | (z != z0)
    assert moved.mean() > 0.5
    assert np.all((e(sd) <= e(sd * (1 + 1e-3)))[moved])
    assert np.all((e(sd) <= e(sd * (1 - 1e-3)))[moved])


def _epilogue_inputs(m, d, g, bits, seed):
    """A [d_out][d_in] tile of W~ and V~ with a scaling vector, its inverse,
    diag(H) = 1/sigma^2, and a previous grid and codes (the min/max RTN grid
    of a perturbed W~)."""
    rng = np.random.default_rng(seed)
    L = (1 << bits) - 1
    W = (rng.standard_normal((m, d)) * 0.05).astype(np.float32)
    V = (rng.standard_normal((m, d)) * 0.005).astype(np.float32)
    sig = (rng.random(d) + 0.5).astype(np.float32)
    rsig = (1.0 / sig.astype(np.float64)).astype(np.float32)
    hd = (rsig.astype(np.float64) ** 2).astype(np.float32)
    prev = (W * 1.1).reshape(m * (d // g), g)
    s0, z0 = P.fit_minmax(prev, L)
    c0 = P.round_to_grid(prev, s0, z0, L).reshape(m, d).astype(np.uint8)
    return W, V, sig, rsig, hd, s0.reshape(m, d // g), z0.reshape(m, d // g), c0


@pytest.mark.parametrize("mode", ["minmax", "lsq", "mse", "frozen"])
@pytest.mark.parametrize("bits,g,m,d", [(3, 32, 5, 96), (2, 64, 3, 128), (4, 32, 4, 64)])
def test_epilogue_step_follows_the_d_and_dual_updates(mode, bits, g, m, d):
    """The memory-layout ([d_out][d_in]) statement of one fused step against
    the D-update of the float64 route (oracle.admmq_oracle.project, the
    [d_in][d_out] layout) on the same float32 iterate y = sigma (W~ + V~),
    and against the dual and residual definitions taken in float64:
    V~' = (W~ + V~) - D~, P = D~ - V~' (so P = 2 D~ - (W~ + V~) up to
    rounding), D~ = D / sigma, r2 = ||W~ - D~||^2, s2 = ||D~ - D~_prev||^2."""
    W, V, sig, rsig, hd, s0, z0, c0 = _epilogue_inputs(m, d, g, bits, seed=bits + g + m)
    out = P.epilogue_step(W, V, sig, rsig, hd, s0, z0, c0, bits, g, mode)
    t = (W + V).astype(np.float32)
    y = (sig[None, :] * t).astype(np.float32)
    codes, sc, ze, D = O.project(y.T, bits, g, mode, hd, s0.T, z0.T)
    np.testing.assert_array_equal(out["codes"], codes.T)
    np.testing.assert_array_equal(out["scale"], sc.T)
    np.testing.assert_array_equal(out["zero"], ze.T)
    Dt = D.T / sig.astype(np.float64)[None, :]
    f = np.float64
    assert np.allclose(out["P"].astype(f) + out["V"].astype(f) - Dt, 0, atol=4e-7 * np.abs(Dt).max())
    assert np.allclose(out["V"].astype(f), t.astype(f) - Dt, atol=4e-7 * np.abs(t).max())
    assert np.allclose(out["P"].astype(f), 2 * Dt - t.astype(f), atol=8e-7 * np.abs(t).max())
    L = (1 << bits) - 1
    lev_prev = s0.astype(f).repeat(g, axis=1) * (c0.astype(f) - z0.astype(f).repeat(g, axis=1))
    Dt_prev = lev_prev / sig.astype(f)[None, :]
    assert out["r2"] == pytest.approx(np.sum((W.astype(f) - Dt) ** 2), rel=1e-5)
    assert out["s2"] == pytest.approx(np.sum((Dt - Dt_prev) ** 2), rel=1e-5, abs=1e-12)
    assert out["codes"].max() <= L


@pytest.mark.parametrize("bits,g,m,d", [(3, 32, 6, 96), (2, 64, 2, 128), (8, 32, 3, 64)])
def test_init_step_is_rtn_in_memory_layout(bits, g, m, d):
    """The RTN start in [d_out][d_in] layout equals oracle.admmq_oracle.rtn on
    the [d_in][d_out] matrix, with P = D~ = D / sigma and V~ = 0."""
    rng = np.random.default_rng(bits * 7 + g)
    Wr = (rng.standard_normal((m, d)) * 0.05).astype(np.float32)
    sig = (rng.random(d) + 0.5).astype(np.float32)
    rsig = (1.0 / sig.astype(np.float64)).astype(np.float32)
    out = P.init_step(Wr, rsig, bits, g)
    codes, sc, ze, D = O.rtn(Wr.T, bits, g)
    np.testing.assert_array_equal(out["codes"], codes.T)
    np.testing.assert_array_equal(out["scale"], sc.T)
    np.testing.assert_array_equal(out["zero"], ze.T)
    np.testing.assert_allclose(out["P"], D.T / sig.astype(np.float64)[None, :], rtol=2e-7, atol=0)


def test_tf32_split_reconstructs_float32():
    """3xTF32 operand planes: hi and lo carry 11 significant bits each, so
    hi + lo holds x to about 2^-22 relative, and hi is the nearest tf32."""
    rng = np.random.default_rng(10)
    x = (rng.standard_normal(10000) * np.exp(rng.standard_normal(10000) * 3)).astype(np.float32)
    hi, lo = P.split_tf32(x)
    assert np.all((hi.view(np.uint32) & 0x1FFF) == 0) and np.all((lo.view(np.uint32) & 0x1FFF) == 0)
    rec = hi.astype(np.float64) + lo
    assert np.max(np.abs(rec - x) / np.abs(x)) < 2.0 ** -21
    assert np.all(np.abs(x - hi.astype(np.float64)) <= np.abs(x) * 2.0 ** -11)
    # hand example: 1 + 2^-11 is a tie between 1 and 1 + 2^-10 -> even (1.0)
    t = np.array([1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11], np.float32)
    np.testing.assert_array_equal(P.tf32_round(t), np.array([1.0, 1 + 2.0 ** -9], np.float32))


def test_f16_split_encoding():
    """fp16 split of the eigenbasis GEMMs' operands: hi = fp16(x s), lo =
    fp16(x s - hi) with a power-of-two scale s.  Hand examples: 3 + 2^-9 + 2^-20
    splits exactly into hi = 3 + 2^-9 (fp16 spacing 2^-9 on [2, 4)) and lo =
    2^-20 (an fp16 subnormal, 16 * 2^-24); an eigenvector entry 1 scaled by 2^14
    is 16384; 4 * 2^14 = 65536 is past fp16's largest value and raises the
    flag.  On random data hi + lo keeps 22 bits and the three fp16 products
    hi.hi + hi.lo + lo.hi give the dot product to ~2^-20."""
    t = np.zeros((1, 8), np.float32)
    t[0, 0] = np.float32(3 + 2.0 ** -9 + 2.0 ** -20)
    t[0, 1] = 1.0
    hi, lo, bad = P.split_f16(t, np.float32(1.0))
    assert not bad
    assert hi.view(np.float16)[0, 0] == np.float16(3 + 2.0 ** -9)
    assert lo.view(np.float16)[0, 0].astype(np.float64) == 2.0 ** -20
    h2, l2, bad2 = P.split_f16(t, P.F16_B_SCALE)
    assert not bad2 and h2.view(np.float16)[0, 1] == 16384.0 and l2.view(np.float16)[0, 1] == 0.0
    t[0, 2] = 4.0
    assert P.split_f16(t, P.F16_B_SCALE)[2]
    rng = np.random.default_rng(13)
    x = (rng.standard_normal((6, 256)) * np.exp(rng.standard_normal((6, 256)))).astype(np.float32)
    s = P.row_scales_f16(x)
    h, l, bad = P.split_f16(x, s)
    assert not bad
    xs = x.astype(np.float64) * s[:, None]
    rec = h.view(np.float16).astype(np.float64) + l.view(np.float16).astype(np.float64)
    # 22 bits relative to the value, or the fp16 subnormal step 2^-24 absolute
    assert np.all(np.abs(rec - xs) <= np.maximum(2.0 ** -22 * np.abs(xs), 2.0 ** -25))
    b = rng.uniform(-1, 1, (7, 256)).astype(np.float32)       # eigenvector-like entries
    hb, lb, _ = P.split_f16(b, P.F16_B_SCALE)
    ha, la = h.view(np.float16).astype(np.float64), l.view(np.float16).astype(np.float64)
    hbf, lbf = hb.view(np.float16).astype(np.float64), lb.view(np.float16).astype(np.float64)
    prod = (ha @ hbf.T + ha @ lbf.T + la @ hbf.T) / (s[:, None].astype(np.float64) * 2.0 ** 14)
    exact = x.astype(np.float64) @ b.astype(np.float64).T
    scale = np.abs(x.astype(np.float64)) @ np.abs(b.astype(np.float64)).T
    assert np.max(np.abs(prod - exact) / scale) < 2.0 ** -20


def test_f16_row_scales():
    """The A operands' row scale 2^e puts the row norm of W^~ in [2^9, 2^10)
    (64x headroom below fp16's 65504 for entries up to the norm), and a zero
    row gets 1."""
    rng = np.random.default_rng(14)
    W = rng.standard_normal((20, 300)) * np.exp(3 * rng.standard_normal((20, 1)))
    W[3] = 0.0
    s = P.row_scales_f16(W)
    n = np.linalg.norm(W, axis=1) * s
    ok = np.arange(20) != 3
    assert np.all((n[ok] >= 2.0 ** 9) & (n[ok] < 2.0 ** 10))
    assert s[3] == 1.0
    assert np.all(np.log2(s) == np.round(np.log2(s)))      # powers of two


def test_mixed_split_encoding():
    """Operand encoding of the eigenbasis GEMMs: hi = tf32(x) is the plane-0
    value, lo = x - hi is exact in float32, and the correction rows hold
    bf16(hi) / bf16(lo) in blocks of 32 columns, swapped on the B side, so
    that one tf32 product plus one bf16 product over a row pair gives
    hi.hi + hi.lo + lo.hi to ~2^-19 relative."""
    rng = np.random.default_rng(12)
    x = (rng.standard_normal((3, 64)) * np.exp(rng.standard_normal((3, 64)))).astype(np.float32)
    hi, ca = P.split_mix(x, "A")
    _, cb = P.split_mix(x, "B")
    np.testing.assert_array_equal(hi, P.tf32_round(x))
    lo = (x.astype(np.float64) - hi).astype(np.float32)
    assert np.array_equal(hi.astype(np.float64) + lo, x.astype(np.float64))   # exact split
    assert ca.shape == (3, 128) and ca.dtype == np.uint16
    for b in range(2):                       # blocks of 32 columns
        blk = slice(32 * b, 32 * b + 32)
        np.testing.assert_array_equal(ca[:, 64 * b:64 * b + 32], P.bf16_bits(hi[:, blk]))
        np.testing.assert_array_equal(ca[:, 64 * b + 32:64 * b + 64], P.bf16_bits(lo[:, blk]))
        np.testing.assert_array_equal(cb[:, 64 * b:64 * b + 32], ca[:, 64 * b + 32:64 * b + 64])
        np.testing.assert_array_equal(cb[:, 64 * b + 32:64 * b + 64], ca[:, 64 * b:64 * b + 32])
    # hand example: x = 1 + 2^-11 + 2^-20 -> hi = 1 + 2^-10 (round up past the
    # tie), lo = -2^-11 + 2^-20, bf16(lo) = -2^-11 (2^-20 is below bf16's 8 bits)
    t = np.zeros((1, 32), np.float32)
    t[0, 0] = np.float32(1 + 2.0 ** -11 + 2.0 ** -20)
    th, tc = P.split_mix(t, "A")
    assert th[0, 0] == np.float32(1 + 2.0 ** -10)
    assert P.bf16_value(tc[0, 32]) == np.float32(-(2.0 ** -11))
    # the two products reproduce x_a . x_b to the bf16 level of the corrections
    a = (rng.standard_normal((4, 256))).astype(np.float32)
    bm = (rng.standard_normal((5, 256))).astype(np.float32)
    ha, cA = P.split_mix(a, "A")
    hb, cB = P.split_mix(bm, "B")
    prod = ha.astype(np.float64) @ hb.T.astype(np.float64) + \
        P.bf16_value(cA).astype(np.float64) @ P.bf16_value(cB).T.astype(np.float64)
    exact = a.astype(np.float64) @ bm.T.astype(np.float64)
    scale = np.abs(a).astype(np.float64) @ np.abs(bm).T.astype(np.float64)
    assert np.max(np.abs(prod - exact) / scale) < 2.0 ** -18


def test_bf16_split_reconstructs_float32():
    rng = np.random.default_rng(9)
    x = (rng.standard_normal(10000) * np.exp(rng.standard_normal(10000) * 3)).astype(np.float32)
    hi, lo = P.split_bf16(x)
    rec = P.bf16_value(hi).astype(np.float64) + P.bf16_value(lo)
    assert np.max(np.abs(rec - x) / np.abs(x)) < 2.0 ** -16
    # hi is the nearest bf16: |x - hi| <= half an ulp of bf16
    assert np.all(np.abs(x - P.bf16_value(hi)) <= np.abs(x) * 2.0 ** -8)


# --------------------------------------------------------------- ADMM-Q pins


def _tiny():
    X, W_rows = workloads.tiny_layer(0)
    return O.hessian(X), W_rows.T.astype(np.float64)


def test_diagonal_hessian_frozen_grid_gives_rtn():
    """With H diagonal the objective separates per weight, RTN is the optimum
    on the fixed grid, and ADMM-Q returns exactly the RTN codes."""
    H, W = _tiny()
    Hd = np.diag(np.diag(H))
    c_rtn = O.rtn(W, 3, 64)[0]
    for T in (50, 200):
        res = O.admm_q(Hd, W, 3, 64, T, grid="frozen")
        np.testing.assert_array_equal(res["codes"], c_rtn)


@pytest.mark.parametrize("grid", ["minmax", "lsq", "mse", "frozen"])
def test_admm_converges_to_common_limit(grid):
    """Under rho_t = rho0 gamma^t the continuous and discrete iterates reach
    the same limit: once rho >> lambda_max(H~) the primal residual vanishes
    and the codes stop changing."""
    H, W = _tiny()
    _, Ht = O.diagonal_scaling(H)
    lmax = np.linalg.eigvalsh(Ht)[-1]
    T = int(np.ceil(np.log(1e3 * lmax / 0.1) / np.log(1.05))) + 1
    res = O.admm_q(H, W, 3, 64, T, grid=grid)
    rel = res["r"][-1] / np.linalg.norm(res["D"] / res["sigma"][:, None])
    assert rel <= 1e-3
    assert np.all(res["code_changes"][-10:] == 0)
    assert res["codes"].min() >= 0 and res["codes"].max() <= 7
    # the returned D is exactly the dequantised codes
    L = 7
    D = np.repeat(res["scale"], 64, axis=0) * (res["codes"] - np.repeat(res["zero"], 64, axis=0))
    np.testing.assert_array_equal(D.astype(np.float32), res["D"].astype(np.float32))
    assert L == 7


@pytest.mark.parametrize("seed", [0, 1])
def test_tiny_layers_against_brute_force(seed):
    """d_in = 4: exhaustive enumeration of every assignment on a fixed grid
    lower-bounds ADMM-Q, RTN and GPTQ on that grid, and ADMM-Q with the frozen
    grid reaches the optimum on most columns."""
    rng = np.random.default_rng(seed)
    d, m, bits, g = 4, 6, 2, 4
    X = rng.standard_normal((64, d)) @ rng.standard_normal((d, d))
    H = O.hessian(X)
    W = rng.standard_normal((d, m)) * 0.1
    codes0, s, z, D0 = O.rtn(W, bits, g)
    res = O.admm_q(H, W, bits, g, 300, grid="frozen")
    _, Qg = O.gptq(H, W.T, s.T, z.T, bits, g)
    hits = 0
    for j in range(m):
        best, _ = O.brute_force_column(H, W[:, j], s[:, j], z[:, j], bits, g)
        a = O.objective(H, res["D"][:, [j]], W[:, [j]])
        r = O.objective(H, D0[:, [j]], W[:, [j]])
        q = O.objective(H, Qg.T[:, [j]], W[:, [j]])
        # D is float32 on both sides of the comparison up to rounding of s (q - z)
        tol = 1e-6 * best
        assert a >= best - tol and r >= best - tol and q >= best - tol
        hits += a <= best + tol
    assert hits >= m // 2


def test_admm_beats_rtn_and_gptq_with_lsq_refresh():
    """Quality report on a correlated synthetic layer (not a pin of a page
    value): with the scaled-metric least-squares refresh ADMM-Q's objective is
    below GPTQ's, which is below RTN's."""
    rng = np.random.default_rng(11)
    n, d, m, g = 2048, 128, 48, 64
    X = rng.standard_t(4, (n, d)) + rng.standard_normal((n, 8)) @ rng.standard_normal((8, d))
    X[:, :2] *= 30
    H = O.hessian(X)
    W = rng.standard_normal((d, m)) * 0.02
    _, s, z, D0 = O.rtn(W, 3, g)
    _, Qg = O.gptq(H, W.T, s.T, z.T, 3, g)
    res = O.admm_q(H, W, 3, g, 100, grid="lsq")
    f_rtn, f_gptq = O.objective(H, D0, W), O.objective(H, Qg.T, W)
    assert res["objective"] < f_gptq < f_rtn


# ------------------------------------------------------------------------ pack


def test_dual_rescaling_keeps_the_unscaled_dual():
    """With rescale_dual the scaled dual is multiplied by rho_t / rho_{t+1}
    after its update: rho_{t+1} V~_{t+1} = rho_t (V~_t + W~_t - D~_{t+1}), the
    unscaled dual's ADMM update.  With gamma = 1 it changes nothing; with
    gamma > 1 it changes the iterates."""
    rng = np.random.default_rng(11)
    X = rng.standard_normal((400, 16)) @ rng.standard_normal((16, 16))
    H = O.hessian(X)
    W_hat = rng.standard_normal((16, 3)) * 0.05
    rho0, gamma = 0.1, 1.3
    trace = []
    res = O.admm_q(H, W_hat, 3, 8, 12, rho0=rho0, gamma=gamma, grid="minmax", trace=trace,
                   rescale_dual=True)
    sigma = res["sigma"][:, None]
    for t in range(len(trace) - 1):
        e, nxt = trace[t], trace[t + 1]
        lhs = nxt["rho"] * e["Vt_out"]
        rhs = e["rho"] * (e["Vt"] + e["W_tilde"] - nxt["Dt"])
        np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-14 * np.abs(rhs).max())
        assert nxt["Dt"] == pytest.approx(O.project(e["Y"], 3, 8, "minmax", np.diag(H), e["scale"],
                                                    e["zero"])[3] / sigma, rel=1e-15)
    a = O.admm_q(H, W_hat, 3, 8, 12, rho0=rho0, gamma=1.0, grid="minmax", rescale_dual=True)
    b = O.admm_q(H, W_hat, 3, 8, 12, rho0=rho0, gamma=1.0, grid="minmax")
    np.testing.assert_array_equal(a["V_tilde"], b["V_tilde"])
    c = O.admm_q(H, W_hat, 3, 8, 12, rho0=rho0, gamma=gamma, grid="minmax")
    assert not np.array_equal(res["V_tilde"], c["V_tilde"])


def test_epilogue_step_dual_scale():
    """The float32 statement with a dual scale r: V~' = fl(fl(t - D~) r) and
    P = fl(D~ - V~'); r = 1 gives the unscaled step bit for bit."""
    W, V, sig, rsig, hd, s0, z0, c0 = _epilogue_inputs(4, 64, 32, 3, seed=5)
    base = P.epilogue_step(W, V, sig, rsig, hd, s0, z0, c0, 3, 32, "lsq")
    one = P.epilogue_step(W, V, sig, rsig, hd, s0, z0, c0, 3, 32, "lsq", dual_scale=1.0)
    for k in ("codes", "scale", "zero", "V", "P"):
        np.testing.assert_array_equal(base[k], one[k])
    r = np.float32(1 / 1.05)
    out = P.epilogue_step(W, V, sig, rsig, hd, s0, z0, c0, 3, 32, "lsq", dual_scale=r)
    np.testing.assert_array_equal(out["codes"], base["codes"])
    f = np.float64
    np.testing.assert_allclose(out["V"].astype(f), base["V"].astype(f) * f(r), rtol=1e-7, atol=0)
    # P + V~' = D~ in both (the same D~: same codes and grid)
    Dt = base["P"].astype(f) + base["V"].astype(f)
    np.testing.assert_allclose(out["P"].astype(f) + out["V"].astype(f), Dt, rtol=0,
                               atol=2e-7 * np.abs(Dt).max())


@pytest.mark.parametrize("mode", ["minmax", "lsq", "mse"])
def test_grid_fitted_on_w(mode):
    """fit_on_w refreshes the grid from sigma W~ and rounds sigma (W~ + V~)
    onto it: the memory-layout statement equals the float64 route's D-update
    given the fit target separately; with V~ = 0 (the first iteration) it is
    the default step; later iterates differ from the default solve's."""
    W, V, sig, rsig, hd, s0, z0, c0 = _epilogue_inputs(5, 96, 32, 3, seed=9)
    out = P.epilogue_step(W, V, sig, rsig, hd, s0, z0, c0, 3, 32, mode, fit_on_w=True)
    y = (sig[None, :] * (W + V).astype(np.float32)).astype(np.float32)
    yw = (sig[None, :] * W).astype(np.float32)
    codes, sc, ze, _ = O.project(y.T, 3, 32, mode, hd, s0.T, z0.T, Y_fit=yw.T)
    np.testing.assert_array_equal(out["codes"], codes.T)
    np.testing.assert_array_equal(out["scale"], sc.T)
    np.testing.assert_array_equal(out["zero"], ze.T)
    default = P.epilogue_step(W, V, sig, rsig, hd, s0, z0, c0, 3, 32, mode)
    assert not np.array_equal(out["scale"], default["scale"])
    Z = np.zeros_like(V)
    a = P.epilogue_step(W, Z, sig, rsig, hd, s0, z0, c0, 3, 32, mode, fit_on_w=True)
    b = P.epilogue_step(W, Z, sig, rsig, hd, s0, z0, c0, 3, 32, mode)
    for k in ("codes", "scale", "zero", "V", "P"):
        np.testing.assert_array_equal(a[k], b[k])
    rng = np.random.default_rng(12)
    X = rng.standard_normal((300, 16)) @ rng.standard_normal((16, 16))
    H = O.hessian(X)
    W_hat = rng.standard_normal((16, 3)) * 0.05
    one = O.admm_q(H, W_hat, 3, 8, 1, grid=mode, fit_on_w=True)
    ref = O.admm_q(H, W_hat, 3, 8, 1, grid=mode)
    np.testing.assert_array_equal(one["codes"], ref["codes"])
    many = O.admm_q(H, W_hat, 3, 8, 30, grid=mode, fit_on_w=True)
    assert not np.array_equal(many["V_tilde"], O.admm_q(H, W_hat, 3, 8, 30, grid=mode)["V_tilde"])


def test_pack_hand_examples():
    c4 = np.array([[1, 2, 3, 4, 5, 6, 7, 8]])
    assert O.pack(c4, 4)[0, 0] == 0x87654321
    c2 = np.array([[1, 2, 3, 0] * 4])
    assert O.pack(c2, 2)[0, 0] == 0x39393939
    c3 = np.full((1, 32), 7)
    np.testing.assert_array_equal(O.pack(c3, 3), [[0xFFFFFFFF] * 3])


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_pack_matches_big_integer_route(bits):
    """Independent route: the row's codes as one base-2^b integer."""
    rng = np.random.default_rng(bits)
    d = 64
    codes = rng.integers(0, 1 << bits, (3, d))
    words = O.pack(codes, bits)
    for r in range(3):
        big = sum(int(c) << (bits * k) for k, c in enumerate(codes[r]))
        ref = [(big >> (32 * i)) & 0xFFFFFFFF for i in range(d * bits // 32)]
        np.testing.assert_array_equal(words[r], ref)
    np.testing.assert_array_equal(O.unpack(words, bits, d), codes)
