"""Float32 op-by-op reference of the grid fit, the projection and the fused
ADMM-Q epilogue (TEST INFRASTRUCTURE ONLY; see oracle/__init__.py).

The D-update of ADMM-Q is a projection onto a per-group asymmetric integer
grid whose scale and zero-point are refreshed from the current iterate
(ADMM-Q technical summary, Methodology section 2: D-update and grid refresh).
Where a float decides an integer, the CUDA kernels and the oracle must take
that decision in the same precision, so the decision is spelled out here as a
sequence of IEEE float32 operations, each rounded to nearest-even on its own
(no fused multiply-add), with rint = round half to even.  Given the same
float32 inputs the kernels must reproduce these outputs bit for bit.

Signed zeros: every clamp and every zero point is followed by "+ 0", which
turns -0 into +0, so results never depend on which zero a min/max returns.

Grid semantics (our reading; the pages do not define the fit):
  minmax  mn = min(0, min y), mx = max(0, max y), s = (mx - mn) / L,
          z = rint(-mn / s); an all-zero group gets s = 1, z = 0.
  lsq     codes on the previous grid, then one weighted least-squares refit of
          y ~ s (q - z) with weights w = diag(H) (the metric of the scaled
          problem): first slope and offset, then the integer zero point, then
          the slope again for that zero point.  Groups whose fit is degenerate
          keep the previous grid.  Each of the fit's five sums is taken over
          consecutive blocks of 32 columns, each block in element order, and
          the block sums are then added pairwise ((B0 + B1) + (B2 + B3) for a
          group of 128, B0 + B1 for 64, B0 alone for 32): the pages state the
          fit in exact arithmetic, so the float32 summation order is ours to
          fix, and blocks let one thread per block share a group.
  mse     clipping search: for each ratio a in CLIP_RATIOS (1, 31/32, ..., 17/32,
          exact in float32) the min/max grid of the clipped range
          (a * mn, a * mx); each candidate's squared error sum (y - D)^2 is
          summed in element order, and the first smallest one wins.  The
          ratio 1 candidate is the min/max grid itself.
  rounding q = clamp(rint(y / s) + z, 0, L);  D = s (q - z).
"""
from __future__ import annotations

import numpy as np

f32 = np.float32


def _f(x):
    return np.asarray(x, dtype=np.float32)


CLIP_RATIOS = tuple((32 - k) / 32 for k in range(16))


def _range_grid(mn: np.ndarray, mx: np.ndarray, L: int):
    """Grid spanning [mn, mx] (mn <= 0 <= mx): s = (mx - mn) / L, z = rint(-mn / s)."""
    s = _f(np.subtract(mx, mn, dtype=f32) / f32(L))
    zero_range = s == f32(0)
    s_safe = np.where(zero_range, f32(1), s).astype(f32)
    z = _f(np.rint(_f(np.negative(mn) / s_safe)) + f32(0))
    z = np.where(zero_range, f32(0), z).astype(f32)
    return s_safe, z


def _group_range(yg: np.ndarray):
    yg = _f(yg)
    return np.minimum(yg.min(axis=1), f32(0)), np.maximum(yg.max(axis=1), f32(0))


def fit_minmax(yg: np.ndarray, L: int):
    """(scale, zero) per group; yg has one group per row."""
    return _range_grid(*_group_range(yg), L)


def fit_mse(yg: np.ndarray, L: int, return_error: bool = False):
    """Clipping search: the candidate grid with the smallest squared error.

    Candidate a spans (a * mn, a * mx); its error is sum_i (y_i - D_i)^2 with
    each square and each partial sum rounded to float32 in element order.  A
    later candidate replaces the best one only when strictly smaller."""
    yg = _f(yg)
    mn, mx = _group_range(yg)
    best = None
    for a in CLIP_RATIOS:
        a = f32(a)
        s, z = _range_grid(_f(a * mn), _f(a * mx), L)
        d = _f(yg - dequantize(round_to_grid(yg, s, z, L), s, z))
        d2 = _f(d * d)
        e = np.zeros(yg.shape[0], f32)
        for i in range(yg.shape[1]):
            e = _f(e + d2[:, i])
        if best is None:
            best = [s, z, e]
        else:
            take = e < best[2]
            best = [np.where(take, s, best[0]).astype(f32), np.where(take, z, best[1]).astype(f32),
                    np.where(take, e, best[2]).astype(f32)]
    return tuple(best) if return_error else (best[0], best[1])


LSQ_BLOCK = 32  # columns per element-ordered block of the least-squares sums


def _pairwise(parts):
    """Adjacent block sums added pairwise, level by level (an odd last one
    moves up a level unchanged)."""
    while len(parts) > 1:
        nxt = [tuple(_f(a + b) for a, b in zip(parts[i], parts[i + 1]))
               for i in range(0, len(parts) - 1, 2)]
        if len(parts) % 2:
            nxt.append(parts[-1])
        parts = nxt
    return parts[0]


def fit_lsq(yg: np.ndarray, wg: np.ndarray, s_prev: np.ndarray, z_prev: np.ndarray, L: int):
    """Weighted least-squares grid refit; each sum is the pairwise float32 sum
    of its 32-column block sums, each block taken in element order."""
    yg, wg = _f(yg), _f(wg)
    s0, z0 = _f(s_prev), _f(z_prev)
    q = round_to_grid(yg, s0, z0, L)
    G, g = yg.shape
    blocks = []
    for lo in range(0, g, LSQ_BLOCK):
        hi = min(lo + LSQ_BLOCK, g)
        Sw = np.zeros(G, f32); Sq = np.zeros(G, f32); Sqq = np.zeros(G, f32)
        Sy = np.zeros(G, f32); Sqy = np.zeros(G, f32)
        for i in range(lo, hi):
            w, qi, yi = wg[:, i], q[:, i], yg[:, i]
            wq = _f(w * qi)
            Sw = _f(Sw + w)
            Sq = _f(Sq + wq)
            Sqq = _f(Sqq + _f(wq * qi))
            Sy = _f(Sy + _f(w * yi))
            Sqy = _f(Sqy + _f(wq * yi))
        blocks.append((Sw, Sq, Sqq, Sy, Sqy))
    Sw, Sq, Sqq, Sy, Sqy = _pairwise(blocks)
    qm = _f(Sq / Sw)
    ym = _f(Sy / Sw)
    var = _f(Sqq - _f(Sq * qm))
    cov = _f(Sqy - _f(Sq * ym))
    ok = (var > 0) & (cov > 0)
    s1 = _f(cov / np.where(ok, var, f32(1)))
    zc = _f(np.clip(np.rint(_f(qm - _f(ym / np.where(ok, s1, f32(1))))), f32(0), f32(L)) + f32(0))
    num = _f(Sqy - _f(zc * Sy))
    den = _f(_f(Sqq - _f(_f(f32(2) * zc) * Sq)) + _f(_f(zc * zc) * Sw))
    ok2 = (den > 0) & (num > 0)
    s2 = np.where(ok2, _f(num / np.where(ok2, den, f32(1))), s1).astype(f32)
    s = np.where(ok, s2, s0).astype(f32)
    z = np.where(ok, zc, z0).astype(f32)
    return s, z


def round_to_grid(yg: np.ndarray, s: np.ndarray, z: np.ndarray, L: int) -> np.ndarray:
    """q = clamp(rint(y / s) + z, 0, L), as float32 integers."""
    r = np.rint(_f(_f(yg) / _f(s)[:, None]))
    return _f(np.clip(_f(r + _f(z)[:, None]), f32(0), f32(L)) + f32(0))


def dequantize(q: np.ndarray, s: np.ndarray, z: np.ndarray) -> np.ndarray:
    """D = s (q - z) in float32 (q - z is an exact small integer)."""
    return _f(_f(s)[:, None] * _f(_f(q) - _f(z)[:, None]))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16, nearest-even; returns the 16-bit patterns."""
    b = _f(x).view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    return (((b + 0x7FFF + lsb) >> 16) & 0xFFFF).astype(np.uint16)


def bf16_value(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint32) << 16).view(np.float32)


def split_bf16(x: np.ndarray):
    """x ~= hi + lo with hi = bf16(x), lo = bf16(x - hi); returns bit patterns."""
    hi = bf16_bits(x)
    lo = bf16_bits(_f(_f(x) - bf16_value(hi)))
    return hi, lo


def tf32_round(x: np.ndarray) -> np.ndarray:
    """Round float32 to tf32 (10 explicit mantissa bits), nearest-even; the
    result is a float32 whose 13 low mantissa bits are zero."""
    b = _f(x).view(np.uint32).astype(np.uint64)
    lsb = (b >> 13) & 1
    r = (((b + 0xFFF + lsb) >> 13) << 13) & 0xFFFFFFFF
    return r.astype(np.uint32).view(np.float32)


def split_tf32(x: np.ndarray):
    """x ~= hi + lo with hi = tf32(x), lo = tf32(x - hi): the operand planes of
    the 3xTF32 eigenbasis GEMMs (float32 arrays)."""
    hi = tf32_round(x)
    lo = tf32_round(_f(_f(x) - hi))
    return hi, lo


def split_mix(x: np.ndarray, side: str = "A"):
    """The eigenbasis GEMMs' operand encoding of a float32 matrix x [rows][K]
    (K % 32 == 0): plane 0 = hi = tf32(x) (float32); plane 1 = uint16 bf16
    bit patterns [rows][2K], per 32 columns the 32 values bf16(hi) then the
    32 values bf16(lo) with lo = x - hi (exact in float32) for side "A", the
    two halves swapped for side "B".  One tf32 product of the hi planes plus
    one bf16 product of the correction rows gives hi.hi + hi.lo + lo.hi."""
    x = _f(x)
    rows, K = x.shape
    hi = tf32_round(x)
    lo = _f(x - hi)
    hb = bf16_bits(hi).reshape(rows, K // 32, 32)
    lb = bf16_bits(lo).reshape(rows, K // 32, 32)
    first, second = (hb, lb) if side == "A" else (lb, hb)
    return hi, np.concatenate([first, second], axis=2).reshape(rows, 2 * K)


def _rows_to_groups(A: np.ndarray, g: int) -> np.ndarray:
    m, d = A.shape
    return A.reshape(m * (d // g), g)


F16_B_SCALE = np.float32(2.0 ** 14)
F16_LIMIT = np.float32(65504.0)


def split_f16(x: np.ndarray, s):
    """fp16 pair of x scaled by s (a power of two, per row or scalar): hi =
    fp16(x s), lo = fp16(x s - hi), nearest-even, as uint16 bit patterns, and
    whether any |x s| reached fp16's largest finite value (the range flag).
    hi + lo carries 22 significant bits; each product of two fp16 values is
    exact in float32, so hi.hi + hi.lo + lo.hi gives the fp32-accurate
    product as three fp16 tensor-core products."""
    x = _f(x)
    s = _f(s)
    xs = _f(x * (s[:, None] if s.ndim == 1 else s))
    with np.errstate(over="ignore"):
        hi = xs.astype(np.float16)
        lo = _f(xs - hi.astype(np.float32)).astype(np.float16)
    bad = bool(np.any(~(np.abs(xs) < F16_LIMIT)))
    return hi.view(np.uint16), lo.view(np.uint16), bad


def row_scales_f16(W_tilde_rows: np.ndarray):
    """Per-row power-of-two scale of the A operands under the fp16 split: 2^e
    with 2^e ||row|| in [2^9, 2^10) (row norms of W^~ = Sigma^-1 W_hat,
    rows = output channels, computed in float64), e clamped to [-60, 60];
    1 for a zero row."""
    n = np.sqrt(np.sum(np.asarray(W_tilde_rows, np.float64) ** 2, axis=1))
    e = np.zeros(n.shape, np.int64)
    ok = (n > 0) & np.isfinite(n)
    _, k = np.frexp(n[ok])
    e[ok] = np.clip(10 - k, -60, 60)
    return np.ldexp(np.float32(1), e).astype(np.float32)


def encode_operand(x: np.ndarray, split: str, side: str = "A", row_scale=None):
    """The eigenbasis GEMMs' operand planes of x in the given split precision:
    "3xtf32" -> (tf32(x), tf32(x - tf32(x))) as float32; "mixed" -> split_mix;
    "f16" -> split_f16 with the rows' scales (side "A", row_scale) or 2^14
    (side "B")."""
    if split == "3xtf32":
        return split_tf32(x)
    if split == "mixed":
        return split_mix(x, side)
    if split == "f16":
        s = F16_B_SCALE if side == "B" else np.asarray(row_scale, np.float32)
        hi, lo, _ = split_f16(x, s)
        return hi, lo
    raise ValueError(split)


def init_step(W_rows: np.ndarray, rsig: np.ndarray, bits: int, group: int, split: str = "mixed",
              row_scale=None):
    """RTN start of the iteration in memory layout ([d_out][d_in]).

    y = W_hat; minmax grid; D = s (q - z); D~ = D * rsig (rsig = sqrt(diag H)),
    V~ = 0 and P = D~ - V~ = D~.
    """
    L = (1 << bits) - 1
    m, d = W_rows.shape
    yg = _rows_to_groups(_f(W_rows), group)
    s, z = fit_minmax(yg, L)
    q = round_to_grid(yg, s, z, L)
    D = dequantize(q, s, z).reshape(m, d)
    Dt = _f(D * _f(rsig)[None, :])
    hi, pc = encode_operand(Dt, split, "A", row_scale)
    return dict(codes=q.reshape(m, d).astype(np.uint8), scale=s.reshape(m, d // group),
                zero=z.reshape(m, d // group), P=Dt, P_hi=hi, P_lo=pc)


def epilogue_step(W_acc: np.ndarray, V: np.ndarray, sigma: np.ndarray, rsig: np.ndarray,
                  hdiag: np.ndarray, s_prev: np.ndarray, z_prev: np.ndarray,
                  codes_prev: np.ndarray, bits: int, group: int, mode: str,
                  split: str = "mixed", row_scale=None, dual_scale=None, fit_on_w=False):
    """One fused projection + dual update in memory layout ([d_out][d_in]).

    Per element (i = input channel):
      t  = W~ + V~          y  = sigma_i t
      grid (minmax | lsq | mse | frozen) per group of `group` columns of one row
      q  = clamp(rint(y/s) + z, 0, L),  D = s (q - z),  D~ = D * rsig_i
      V~' = t - D~          P  = D~ - V~'   (in the operand encoding of `split`)
    With `dual_scale` r (the dual rescaling rho_t / rho_{t+1}, a float32):
      V~' = (t - D~) r, rounded after the subtraction and after the product.
    With `fit_on_w` the grid is fitted on y_w = sigma_i W~ (the dual left
    out); y is still the point rounded onto it.
    Residual sums (float64 here; the kernels sum in float32, compared with a
    tolerance): r2 = sum (W~ - D~)^2 and s2 = sum (D~ - D~_prev)^2 where
    D~_prev = s_prev (q_prev - z_prev) * rsig.
    """
    L = (1 << bits) - 1
    m, d = W_acc.shape
    W_acc, V = _f(W_acc), _f(V)
    t = _f(W_acc + V)
    y = _f(_f(sigma)[None, :] * t)
    yg = _rows_to_groups(y, group)
    fg = _rows_to_groups(_f(_f(sigma)[None, :] * W_acc), group) if fit_on_w else yg
    sp = _f(s_prev).reshape(-1)
    zp = _f(z_prev).reshape(-1)
    if mode == "minmax":
        s, z = fit_minmax(fg, L)
    elif mode == "lsq":
        wg = np.broadcast_to(_f(hdiag).reshape(d // group, group)[None],
                             (m, d // group, group)).reshape(-1, group)
        s, z = fit_lsq(fg, wg, sp, zp, L)
    elif mode == "mse":
        s, z = fit_mse(fg, L)
    elif mode == "frozen":
        s, z = sp, zp
    else:
        raise ValueError(mode)
    q = round_to_grid(yg, s, z, L)
    D = dequantize(q, s, z).reshape(m, d)
    Dt = _f(D * _f(rsig)[None, :])
    V_new = _f(t - Dt)
    if dual_scale is not None:
        V_new = _f(V_new * f32(dual_scale))
    P = _f(Dt - V_new)
    hi, lo = encode_operand(P, split, "A", row_scale)
    qp = _rows_to_groups(_f(codes_prev), group)
    Dt_prev = _f(dequantize(qp, sp, zp).reshape(m, d) * _f(rsig)[None, :])
    r2 = float(np.sum((W_acc.astype(np.float64) - Dt) ** 2))
    s2 = float(np.sum((Dt.astype(np.float64) - Dt_prev) ** 2))
    return dict(codes=q.reshape(m, d).astype(np.uint8), scale=s.reshape(m, d // group),
                zero=z.reshape(m, d // group), V=V_new, P=P, P_hi=hi, P_lo=lo, r2=r2, s2=s2)
