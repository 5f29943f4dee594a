"""Float64 CPU oracle for the ADMM-Q layer solve, RTN and GPTQ.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
baseline leg of the benchmark may import this module.  It shares no code with
the CUDA path: it is plain numpy, written from the pages, slow and readable.

Orientation follows the ADMM-Q pages: W and W_hat are d_in x d_out, the
calibration activations X are n x d_in and H = X^T X + lambda I is d_in x d_in.
A quantization group is `group` consecutive input rows of one output column.
GPTQ uses the GPTQ tutorial's orientation (weights d_o x d_i, one row per
output channel), which is the transpose.

Sources (by page and section):
  [ADMM-Q]  "ADMM-Q: An Improved Hessian-based Weight Quantizer for Post-Training
            Quantization of Large Language Models", technical summary pages
            (gist.science 2605.11222; zh/it/ja), "Methodology" section 1
            (problem formulation) and section 2 (key algorithmic components:
            diagonal scaling, ADMM split, W-/D-/dual updates, grid refresh,
            convergence under rho_t = rho0 * gamma^t).
  [GPTQ]    "061 . GPTQ" tutorial (wq-win.github.io), section 2 (Lagrange
            compensation, worked example, collinear example, damping) and
            section 3 (Algorithm 1, blocked lazy updates).
  [BABAI]   "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane
            Algorithm" summary (gist.science 2507.18553), sections 2.1-2.3
            (CVP form, Theorem 1, Theorem 4, Theorem 5).

Decisions that turn floats into integers (the grid fit and the rounding) are
taken in float32, the precision of the CUDA kernels, by oracle.projection_fp32.
Everything continuous is float64.

Pins: every function here is checked in tests/test_oracle_pins.py against
values the pages print, closed forms, brute force or an independent route.
Parity unpinned: the exact semantics of the grid refresh, the initial iterate
and the dual handling when rho changes are not fixed by the pages; the oracle
and the kernels follow the same documented reading, and those parts are pinned
only by their invariants (codes in range, D on its grid, convergence).
"""
from __future__ import annotations

import numpy as np

from . import projection_fp32 as p32

# ---------------------------------------------------------------------------
# Hessian, damping, diagonal scaling  ([ADMM-Q] Methodology 1 and 2)
# ---------------------------------------------------------------------------


def gram(X: np.ndarray, chunk: int = 8192) -> np.ndarray:
    """G = X^T X in float64, accumulated over row chunks of X ([ADMM-Q] section 1)."""
    X = np.asarray(X)
    d = X.shape[1]
    G = np.zeros((d, d), dtype=np.float64)
    for r0 in range(0, X.shape[0], chunk):
        Xc = X[r0:r0 + chunk].astype(np.float64)
        G += Xc.T @ Xc
    return G


def damping(G: np.ndarray, lambda_rel: float = 0.01) -> tuple[np.ndarray, float]:
    """H = G + lambda I with lambda = lambda_rel * mean(diag G).

    [ADMM-Q] section 1 defines H = X^T X + lambda I; the GPTQ tutorial
    (section 2, "why damping") explains why lambda > 0 is needed when channels
    are collinear.  The relative size of lambda is our reading (1% of the mean
    diagonal, the usual GPTQ choice).
    """
    lam = float(lambda_rel) * float(np.mean(np.diag(G)))
    return G + lam * np.eye(G.shape[0]), lam


def hessian(X: np.ndarray, lambda_rel: float = 0.01) -> np.ndarray:
    return damping(gram(X), lambda_rel)[0]


def diagonal_scaling(H: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Sigma = Diag(H)^(-1/2) as a vector, and H~ = Sigma H Sigma ([ADMM-Q] section 2)."""
    sigma = 1.0 / np.sqrt(np.diag(H))
    return sigma, sigma[:, None] * H * sigma[None, :]


def objective(H: np.ndarray, W: np.ndarray, W_hat: np.ndarray) -> float:
    """1/2 Tr((W - W_hat)^T H (W - W_hat))  ([ADMM-Q] section 1)."""
    Dl = np.asarray(W, dtype=np.float64) - np.asarray(W_hat, dtype=np.float64)
    return 0.5 * float(np.sum(Dl * (H @ Dl)))


# ---------------------------------------------------------------------------
# Grids: RTN and the D-update projection
# ---------------------------------------------------------------------------


def _groups(A: np.ndarray, group: int) -> np.ndarray:
    """d_in x d_out -> (d_out * d_in/group) x group, one group per row."""
    d, m = A.shape
    return np.ascontiguousarray(A.T).reshape(m * (d // group), group)


def _ungroup(Ag: np.ndarray, d: int, m: int) -> np.ndarray:
    return Ag.reshape(m, d).T


def rtn(W_hat: np.ndarray, bits: int, group: int):
    """Round-to-nearest on a per-group asymmetric grid fitted on W_hat.

    RTN rounds each weight independently ([ADMM-Q] problem statement).  The
    grid is the min/max grid of oracle.projection_fp32.fit_minmax.
    Returns (codes, scale, zero, D) with codes/D d_in x d_out and scale/zero
    (d_in/group) x d_out.
    """
    d, m = W_hat.shape
    L = (1 << bits) - 1
    yg = _groups(np.asarray(W_hat, dtype=np.float32), group)
    s, z = p32.fit_minmax(yg, L)
    q = p32.round_to_grid(yg, s, z, L)
    D = p32.dequantize(q, s, z)
    return (_ungroup(q, d, m).astype(np.uint8), s.reshape(m, d // group).T.copy(),
            z.reshape(m, d // group).T.copy(), _ungroup(D, d, m).astype(np.float64))


def project(Y: np.ndarray, bits: int, group: int, mode: str, hdiag: np.ndarray,
            s_prev: np.ndarray, z_prev: np.ndarray, Y_fit=None):
    """D-update: project Y = Sigma (W~ + V~) onto a per-group grid ([ADMM-Q] section 2).

    The decision is taken in float32 (the kernels' precision).  `mode` selects
    how the grid is refreshed from the current iterate:
      "minmax": scale/zero refitted from the group's min/max (with 0 included);
      "lsq":    one weighted least-squares refit in the scaled metric
                (weights diag H), warm-started from the previous grid;
      "mse":    the clipped min/max grid with the smallest squared error over
                the ratios of oracle.projection_fp32.CLIP_RATIOS (a clipping
                heuristic by MSE grid search, [ADMM-Q] Methodology section 3,
                modularity);
      "frozen": the previous grid is kept (GPTQ-style fixed grid).
    `Y_fit` (optional): the grid is refreshed from Y_fit instead of Y, and Y
    is rounded onto it.
    Returns (codes, scale, zero, D) like rtn().
    """
    d, m = Y.shape
    L = (1 << bits) - 1
    yg = _groups(np.asarray(Y, dtype=np.float32), group)
    fg = yg if Y_fit is None else _groups(np.asarray(Y_fit, dtype=np.float32), group)
    sp = np.ascontiguousarray(np.asarray(s_prev, np.float32).T).reshape(-1)
    zp = np.ascontiguousarray(np.asarray(z_prev, np.float32).T).reshape(-1)
    if mode == "minmax":
        s, z = p32.fit_minmax(fg, L)
    elif mode == "lsq":
        wg = np.broadcast_to(np.asarray(hdiag, np.float32).reshape(d // group, group)[None],
                             (m, d // group, group)).reshape(-1, group)
        s, z = p32.fit_lsq(fg, wg, sp, zp, L)
    elif mode == "mse":
        s, z = p32.fit_mse(fg, L)
    elif mode == "frozen":
        s, z = sp, zp
    else:
        raise ValueError(mode)
    q = p32.round_to_grid(yg, s, z, L)
    D = p32.dequantize(q, s, z)
    return (_ungroup(q, d, m).astype(np.uint8), s.reshape(m, d // group).T.copy(),
            z.reshape(m, d // group).T.copy(), _ungroup(D, d, m).astype(np.float64))


# ---------------------------------------------------------------------------
# ADMM-Q  ([ADMM-Q] section 2)
# ---------------------------------------------------------------------------


def w_update(Q: np.ndarray, lam: np.ndarray, B: np.ndarray, rho: float,
             Dt: np.ndarray, Vt: np.ndarray) -> np.ndarray:
    """W~ = Q diag(1/(Lambda + rho)) Q^T (B + rho (D~ - V~)), with B = H~ W_hat~.

    This is the minimiser of 1/2 Tr((W~-W^~)^T H~ (W~-W^~)) + rho/2 ||W~ - D~ + V~||^2,
    solved with the eigendecomposition H~ = Q Lambda Q^T that is computed once
    per layer ([ADMM-Q] section 2, W-update).
    """
    return Q @ ((Q.T @ (B + rho * (Dt - Vt))) / (lam + rho)[:, None])


def admm_q(H: np.ndarray, W_hat: np.ndarray, bits: int, group: int, iters: int,
           rho0: float = 0.1, gamma: float = 1.05, grid: str = "minmax",
           scaling: bool = True, eig=None, grid0=None, trace=None,
           rescale_dual: bool = False, fit_on_w: bool = False) -> dict:
    """The ADMM-Q layer solve, step by step in the pages' order.

    1. Sigma = Diag(H)^(-1/2); H~ = Sigma H Sigma; W^~ = Sigma^-1 W_hat.
    2. H~ = Q Lambda Q^T once.
    3. Start: D = RTN(W_hat) (grid fitted on W_hat), V~ = 0.
    4. For t = 0..iters-1 with rho_t = rho0 * gamma^t:
         W~ = argmin (W-update, eigenbasis closed form)
         D  = grid projection of Sigma (W~ + V~) with the grid refreshed
         V~ = V~ + W~ - D~
    5. Return the last D as codes + per-group scale/zero, and its objective.

    `scaling=False` replaces Sigma by the identity (the pages' ablation).
    `rescale_dual=True` multiplies V~ by rho_t / rho_{t+1} after its update, so
    that the unscaled dual rho V~ carries over unchanged when the penalty
    grows (the pages say nothing on this; without the flag V~ is literally
    V~ + W~ - D~, the reading the default follows).
    `fit_on_w=True` refreshes the grid from Sigma W~ instead of the point
    being projected, Sigma (W~ + V~) (the pages' "current continuous
    iterate" read as W~; the default reads it as the projected point).
    `eig` optionally passes a precomputed (Lambda, Q) of H~; `grid0` an
    initial (scale, zero) pair ((d_in/group) x d_out each) replacing the RTN
    grid of W_hat (the start D is then W_hat rounded on that grid).
    """
    H = np.asarray(H, dtype=np.float64)
    W_hat = np.asarray(W_hat, dtype=np.float64)
    d, m = W_hat.shape
    if scaling:
        sigma, Ht = diagonal_scaling(H)
    else:
        sigma, Ht = np.ones(d), H.copy()
    hdiag = np.diag(H).astype(np.float32)
    Wt_hat = W_hat / sigma[:, None]
    lam, Q = np.linalg.eigh(Ht) if eig is None else eig
    B = Ht @ Wt_hat
    if grid0 is None:
        codes, s, z, D = rtn(W_hat, bits, group)
    else:
        s0, z0 = (np.asarray(a, np.float32) for a in grid0)
        codes, s, z, D = project(W_hat, bits, group, "frozen", hdiag, s0, z0)
    Dt = D / sigma[:, None]
    Vt = np.zeros_like(Dt)
    r_hist, s_hist, code_changes = [], [], []
    Wt = Wt_hat
    for t in range(iters):
        rho = rho0 * gamma ** t
        entry = None
        if trace is not None:
            entry = dict(t=t, rho=rho, Dt=Dt.copy(), Vt=Vt.copy(), codes=codes.copy(),
                         scale=s.copy(), zero=z.copy())
        Wt = w_update(Q, lam, B, rho, Dt, Vt)
        Y = sigma[:, None] * (Wt + Vt)
        Y_fit = sigma[:, None] * Wt if fit_on_w else None
        codes_new, s, z, D = project(Y, bits, group, grid, hdiag, s, z, Y_fit=Y_fit)
        Dt_new = D / sigma[:, None]
        Vt = Vt + Wt - Dt_new
        if rescale_dual:
            Vt = Vt * (rho / (rho0 * gamma ** (t + 1)))
        if entry is not None:
            entry.update(W_tilde=Wt.copy(), Y=Y.copy(), codes_out=codes_new.copy(),
                         scale_out=s.copy(), zero_out=z.copy(), Vt_out=Vt.copy())
            trace.append(entry)
        r_hist.append(float(np.linalg.norm(Wt - Dt_new)))
        s_hist.append(float(rho * np.linalg.norm(Dt_new - Dt)))
        code_changes.append(int(np.count_nonzero(codes_new != codes)))
        Dt, codes = Dt_new, codes_new
    out = dict(codes=codes, scale=s, zero=z, D=D, objective=objective(H, D, W_hat),
               r=np.array(r_hist), s=np.array(s_hist), code_changes=np.array(code_changes),
               W_tilde=Wt, V_tilde=Vt, sigma=sigma, lam=lam, Q=Q)
    return out


# ---------------------------------------------------------------------------
# GPTQ ([GPTQ] sections 2-3) and its geometric reading ([BABAI])
# ---------------------------------------------------------------------------


def compensation(H: np.ndarray, q: int, d: float) -> np.ndarray:
    """delta = d H^-1 e_q / (H^-1)_qq: the change of all weights that fixes
    delta_q = d and minimises 1/2 delta^T H delta ([GPTQ] section 2, Lagrange box)."""
    Hinv = np.linalg.inv(H)
    return d * Hinv[:, q] / Hinv[q, q]


def minmax_grid_rows(W: np.ndarray, bits: int, group: int):
    """Per-(row, group) min/max grid of a d_o x d_i matrix (GPTQ orientation)."""
    L = (1 << bits) - 1
    do, di = W.shape
    s, z = p32.fit_minmax(np.asarray(W, np.float32).reshape(do * (di // group), group), L)
    return s.reshape(do, di // group), z.reshape(do, di // group)


def gptq(H: np.ndarray, W: np.ndarray, scale: np.ndarray, zero: np.ndarray, bits: int,
         group: int, block: int = 128, order=None, clamp: bool = True):
    """GPTQ Algorithm 1 ([GPTQ] section 3) on a d_o x d_i weight matrix.

    H is the (already damped) d_i x d_i Hessian; R is the upper Cholesky factor
    of H^-1 (R^T R = H^-1).  Columns are visited in `order` (natural order by
    default) in blocks of `block`; inside a block each column is quantized on
    the fixed input grid (scale/zero per row and group of the ORIGINAL column
    index), its scaled error is pushed onto the rest of the block, and the
    block's errors update the later columns in one product.  `clamp=False`
    drops the [0, L] bound (the no-clipping setting of [BABAI] section 2.3).
    Returns (codes, Qw) in the original column order.
    """
    W = np.array(W, dtype=np.float64)
    do, di = W.shape
    L = (1 << bits) - 1
    perm = np.arange(di) if order is None else np.asarray(order)
    Hp = np.asarray(H, np.float64)[np.ix_(perm, perm)]
    R = np.linalg.cholesky(np.linalg.inv(Hp)).T
    Wp = W[:, perm].copy()
    Qp = np.zeros_like(Wp)
    Cp = np.zeros(Wp.shape, dtype=np.int64)
    for a in range(0, di, block):
        b = min(a + block, di)
        E = np.zeros((do, b - a))
        for j in range(a, b):
            col = perm[j]
            s = scale[:, col // group].astype(np.float64)
            z = zero[:, col // group].astype(np.float64)
            c = np.rint(Wp[:, j] / s) + z
            if clamp:
                c = np.clip(c, 0, L)
            Cp[:, j] = c
            Qp[:, j] = s * (c - z)
            E[:, j - a] = (Wp[:, j] - Qp[:, j]) / R[j, j]
            Wp[:, j:b] -= np.outer(E[:, j - a], R[j, j:b])
        Wp[:, b:] -= E @ R[a:b, b:]
    codes = np.zeros_like(Cp)
    Qw = np.zeros_like(Qp)
    codes[:, perm] = Cp
    Qw[:, perm] = Qp
    return codes, Qw


def babai_nearest_plane(H: np.ndarray, w: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Babai's nearest-plane rounding of w onto the lattice diag(s) Z^d in the
    metric of H, without basis reduction ([BABAI] sections 2.1-2.2).

    By Theorem 1 any factor of H gives an equivalent CVP; we use H = R^T R with
    R upper triangular (Cholesky), basis columns s_k R[:, k] and target R w.
    The Gram-Schmidt vectors of an upper-triangular basis are axis-aligned, so
    the nearest plane for coordinate k (taken from the last to the first) is a
    plain rounding of the residual's k-th component.  Returns integer codes c
    (the lattice point is s * c).
    """
    R = np.linalg.cholesky(np.asarray(H, np.float64)).T
    t = R @ np.asarray(w, np.float64)
    d = len(t)
    c = np.zeros(d)
    for k in range(d - 1, -1, -1):
        c[k] = np.rint(t[k] / (R[k, k] * s[k]))
        t = t - c[k] * s[k] * R[:, k]
    return c


def babai_error_bound(H: np.ndarray, s: np.ndarray) -> float:
    """Theorem 5 of [BABAI], no clipping, natural order: the error
    (w - s c)^T H (w - s c) is at most 1/4 sum_k D_k s_k^2 with D the diagonal
    of the LDL^T factorisation of H (D_k = R_kk^2 for the Cholesky factor R)."""
    R = np.linalg.cholesky(np.asarray(H, np.float64)).T
    return 0.25 * float(np.sum((np.diag(R) * s) ** 2))


# ---------------------------------------------------------------------------
# Packing and brute force
# ---------------------------------------------------------------------------


def pack(codes_rows: np.ndarray, bits: int) -> np.ndarray:
    """Pack codes [d_out][d_in] into little-endian b-bit streams per row.

    Our reading of "the same format as GPTQ" ([ADMM-Q] experimental results,
    inference): code k of a row occupies bits [b k, b k + b) of that row's
    bit stream, stored in uint32 words; a row holds d_in * b / 32 words.
    Written bit by bit.
    """
    codes_rows = np.asarray(codes_rows, dtype=np.int64)
    m, d = codes_rows.shape
    assert (d * bits) % 32 == 0
    words = np.zeros((m, d * bits // 32), dtype=np.uint64)
    for k in range(d):
        for b in range(bits):
            pos = k * bits + b
            bit = (codes_rows[:, k] >> b) & 1
            words[:, pos // 32] |= bit.astype(np.uint64) << np.uint64(pos % 32)
    return words.astype(np.uint32)


def unpack(words: np.ndarray, bits: int, d: int) -> np.ndarray:
    words = np.asarray(words, dtype=np.uint64)
    m = words.shape[0]
    codes = np.zeros((m, d), dtype=np.int64)
    for k in range(d):
        for b in range(bits):
            pos = k * bits + b
            codes[:, k] |= ((words[:, pos // 32] >> np.uint64(pos % 32)) & 1).astype(np.int64) << b
    return codes


def brute_force_column(H: np.ndarray, w_hat: np.ndarray, s: np.ndarray, z: np.ndarray,
                       bits: int, group: int):
    """Exhaustive minimum of 1/2 (D - w_hat)^T H (D - w_hat) over every code
    assignment of one output column on a fixed grid (tiny d_in only)."""
    d = len(w_hat)
    L = (1 << bits) - 1
    idx = np.indices((L + 1,) * d).reshape(d, -1).T
    D = np.empty(idx.shape, dtype=np.float64)
    for i in range(d):
        D[:, i] = s[i // group] * (idx[:, i] - z[i // group])
    e = D - np.asarray(w_hat, np.float64)[None, :]
    v = 0.5 * np.sum((e @ H) * e, axis=1)
    k = int(np.argmin(v))
    return float(v[k]), idx[k].copy()
