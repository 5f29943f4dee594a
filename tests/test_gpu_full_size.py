"""Parity at the full q_proj sizes, in the launch configuration the benchmark
times (d_in = d_out = 4096, group 128, 3 bits, T = 100), on sampled outputs
that the float64 oracle computes one by one (needs a B200).

- Gram over the full n = 262144 tokens: sampled entries H_ij against float64
  dot products of the same bf16 columns.
- ADMM-Q iterations (least-squares and min/max grid refresh): every output
  row follows its own trajectory (the
  W-update, the grid projection and the dual update act row by row), so the
  oracle runs the solve for a few sampled rows on the same H~ and the GPU
  runs all 4096.  The Hessian here comes from n = 8192 tokens, which the
  oracle forms in full; the iteration kernels do not depend on n.
"""
import numpy as np
import pytest
import torch

import _spread as S
from oracle import admmq_oracle as O
from oracle import projection_fp32 as P
from post_weight_quantization_10_b200 import workloads

pytestmark = pytest.mark.gpu

D = 4096
ROWS = np.array([0, 1, 77, 128, 1000, 2047, 2048, 3001, 3500, 4000, 4094, 4095])
STEPS = (0, 1, 30, 60, 99)


@pytest.fixture(scope="module")
def A():
    from post_weight_quantization_10_b200 import admmq
    admmq.lib()
    return admmq


def test_full_gram_sampled(A):
    """H = X^T X over 262144 tokens x 4096 features: 24 x 24 sampled entries
    (the diagonal among them) within 1e-5 of sqrt(H_ii H_jj)."""
    p = workloads.PRESETS["q_proj"]
    X = workloads.make_activations(p, seed=0, device="cuda")
    H = A.build_hessian(X)
    torch.cuda.synchronize()
    rng = np.random.default_rng(11)
    I = np.sort(rng.choice(D, 20, replace=False))
    I = np.unique(np.concatenate([I, [0, 127, 128, D - 1]]))
    cols = torch.from_numpy(I).cuda()
    Xc = X[:, cols].float().cpu().numpy().astype(np.float64)
    del X
    ref = Xc.T @ Xc
    got = H[cols][:, cols].cpu().numpy().astype(np.float64)
    dg = np.sqrt(np.outer(np.diag(ref), np.diag(ref)))
    err = np.max(np.abs(got - ref) / dg)
    assert err <= 1e-5, err
    assert np.array_equal(got, got.T)


@pytest.fixture(scope="module")
def full_setup(A):
    p = workloads.scaled(workloads.PRESETS["q_proj"], 8192, D, D)
    X = workloads.make_activations(p, seed=0, device="cuda")
    W = workloads.make_weights(p, seed=0, device="cuda", dtype=torch.float32)
    H = O.hessian(X.float().cpu().numpy(), p.lambda_rel)
    Wm = W[torch.from_numpy(ROWS).cuda()].cpu().numpy().T.astype(np.float64)
    eig = np.linalg.eigh(O.diagonal_scaling(H)[1])
    return p, X, W, H, Wm, eig, {}


def _oracle_run(full_setup, grid):
    p, X, W, H, Wm, eig, cache = full_setup
    if grid not in cache:
        trace = []
        res = O.admm_q(H, Wm, p.bits, p.group, p.iters, rho0=p.rho0, gamma=p.gamma, grid=grid,
                       eig=eig, trace=trace)
        cache[grid] = (res, trace)
    return cache[grid]


def _solver(A, p, X, W, grid, split="auto"):
    prm = A.Params(bits=p.bits, group=p.group, iters=p.iters, rho0=p.rho0, gamma=p.gamma,
                   lambda_rel=p.lambda_rel, grid=grid, split=split)
    G = A.build_hessian(X)
    s = A.Solver(D, D, prm)
    s.prepare(G, W)
    s.eigh()
    return s


@pytest.mark.parametrize("grid,split", [("lsq", "auto"), ("minmax", "auto"), ("mse", "auto"),
                                        ("lsq", "3xtf32"), ("lsq", "mixed")])
def test_full_size_teacher_forced(A, full_setup, grid, split):
    """RTN start bit-exact on the sampled rows; then, at sampled iterations,
    the oracle's state of those rows is loaded into the GPU's state and one
    GPU iteration runs: W~ within 1e-4 relative, codes equal on >= 99.9%,
    mismatches one level apart where the grid agrees.  At this size the
    automatic split precision is the fp16 one; 3xTF32 and mixed are forced once each."""
    p, X, W, H, Wm, _, _ = full_setup
    res, trace = _oracle_run(full_setup, grid)
    s = _solver(A, p, X, W, grid, split)
    assert s.split == (split if split != "auto" else "f16")
    s.init()
    torch.cuda.synchronize()
    rows = torch.from_numpy(ROWS).cuda()
    np.testing.assert_array_equal(s.codes[rows].cpu().numpy(), trace[0]["codes"].T)
    np.testing.assert_array_equal(s.scale[rows].cpu().numpy(), trace[0]["scale"].T)
    wt = torch.empty((D, D), dtype=torch.float32, device="cuda")
    s.dump_wtilde(wt)
    cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    for t in STEPS:
        e = trace[t]
        if t > 0:
            hi, lo = P.encode_operand((e["Dt"] - e["Vt"]).T.astype(np.float32), s.split, "A",
                                      s.buffer("row_in")[rows].cpu().numpy())
            s.buffer("V")[rows] = cu(e["Vt"].T.astype(np.float32))
            s.buffer("P_hi")[rows] = cu(hi.view(np.int16) if s.split == "f16" else hi)
            s.buffer("P_lo")[rows] = cu(lo.view(np.int16) if s.split in ("mixed", "f16") else lo)
            s.codes[rows] = cu(e["codes"].T)
            s.scale[rows] = cu(e["scale"].T.astype(np.float32))
            s.zero[rows] = cu(e["zero"].T.astype(np.float32))
        s.iterate(t, 1)
        torch.cuda.synchronize()
        ref = e["W_tilde"].T
        got = wt[rows].cpu().numpy().astype(np.float64)
        err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert err <= 1e-4, (t, err)
        c = s.codes[rows].cpu().numpy().astype(int)
        co = e["codes_out"].T.astype(int)
        assert np.mean(c != co) <= 1e-3, (t, np.mean(c != co))
        same_grid = np.repeat(s.zero[rows].cpu().numpy() == e["zero_out"].T, p.group, axis=1)
        assert np.all(np.abs(c - co)[same_grid] <= 1), t
        print(f"full-size {grid}/{s.split} step {t}: W~ rel err {err:.2e}, code mismatches {np.mean(c != co):.2e}")
    s.dump_wtilde(None)


@pytest.mark.parametrize("grid", ["lsq", "minmax"])
def test_full_size_free_running(A, full_setup, grid):
    """The whole T = 100 solve at 4096 x 4096: valid codes and grids, and on
    the sampled rows codes and objective within the acceptance bar, widened
    only as far as the method's own spread at this size requires: the oracle
    re-run on the same rows with its W-update perturbed by relative noise of
    the GPU's measured per-step size (the W~ difference after iteration 0 on
    the sampled rows), three seeds.  The trajectory amplifies last-bit
    differences; step parity is the teacher-forced test above."""
    p, X, W, H, Wm, eig, _ = full_setup
    res, trace = _oracle_run(full_setup, grid)
    s = _solver(A, p, X, W, grid)
    rows = torch.from_numpy(ROWS).cuda()
    s.init()
    wt = torch.empty((D, D), dtype=torch.float32, device="cuda")
    s.dump_wtilde(wt)
    s.iterate(0, 1)
    s.dump_wtilde(None)
    torch.cuda.synchronize()
    ref0 = trace[0]["W_tilde"].T
    eps = float(np.linalg.norm(wt[rows].cpu().numpy().astype(np.float64) - ref0)
                / np.linalg.norm(ref0))
    del wt
    s.solve()
    torch.cuda.synchronize()
    codes = s.codes[rows].cpu().numpy()
    sc, ze = s.scale[rows].cpu().numpy(), s.zero[rows].cpu().numpy()
    L = (1 << p.bits) - 1
    assert codes.max() <= L and np.all(sc > 0)
    assert np.all((ze >= 0) & (ze <= L) & (ze == np.rint(ze)))
    Dg = np.repeat(sc, p.group, axis=1) * (codes - np.repeat(ze, p.group, axis=1))
    obj_gpu = O.objective(H, Dg.T.astype(np.float64), Wm)
    rel = obj_gpu / res["objective"] - 1.0
    agree = float(np.mean(codes == res["codes"].T))
    _, runs = S.noisy_runs(H, Wm, p, grid, max(eps, S.EPS_FLOOR), seeds=3, eig=eig)
    agree_bar, rel_bar, lo, hi = S.bars(res, runs)
    print(f"full-size free-running {grid}: codes agree {agree:.5f}, objective rel {rel:+.3e}; "
          f"oracle at noise {eps:.1e}: agree >= {lo:.5f}, |rel| <= {hi:.3e}; "
          f"bar: agree >= {agree_bar:.5f}, |rel| <= {rel_bar:.3e}")
    assert agree >= agree_bar
    assert abs(rel) <= rel_bar


FIRST_ITERATION_SHAPES = {
    # the eigenbasis GEMMs reduce over K = 12288
    "down_proj": ("down_proj", 12288, 4096,
                  [0, 1, 500, 1023, 1024, 2047, 2048, 2500, 3071, 3500, 4094, 4095]),
    # 25600 rows: 100 unit rows of 256, the largest tile grid of the workloads
    "up_proj_32b": ("up_proj_32b", 5120, 25600,
                    [0, 255, 256, 4095, 12799, 12800, 20000, 25343, 25344, 25598, 25599, 7777]),
}


@pytest.mark.parametrize("shape", sorted(FIRST_ITERATION_SHAPES))
def test_first_iteration_sampled(A, shape):
    """A deep and a tall layer at their real sizes (the fp16 split): the RTN
    start bit-exact on 12 sampled rows (across unit-row boundaries), then W~
    after iteration 0 within 1e-4 relative of the W-update's closed form
    W~* = (H~ + rho0 I)^-1 (H~ W^~ + rho0 D~_0) solved in float64 for those
    rows, and the codes of that step equal to the oracle's projection of W~*
    on >= 99.9% of entries.  H comes from n = 8192 tokens."""
    preset, d_in, d_out, rows = FIRST_ITERATION_SHAPES[shape]
    p = workloads.scaled(workloads.PRESETS[preset], 8192, d_in, d_out)
    rows = np.array(rows)
    X = workloads.make_activations(p, seed=0, device="cuda")
    W = workloads.make_weights(p, seed=0, device="cuda", dtype=torch.float32)
    prm = A.Params(bits=p.bits, group=p.group, iters=p.iters, rho0=p.rho0, gamma=p.gamma,
                   lambda_rel=p.lambda_rel, grid="lsq")
    s = A.Solver(p.d_in, p.d_out, prm)
    s.prepare(A.build_hessian(X), W)
    s.eigh()
    assert s.split == "f16"
    s.init()
    wt = torch.empty((p.d_out, p.d_in), dtype=torch.float32, device="cuda")
    s.dump_wtilde(wt)
    c_init = s.codes[torch.from_numpy(rows).cuda()].cpu().numpy()
    s.iterate(0, 1)
    s.check()
    s.dump_wtilde(None)
    r_idx = torch.from_numpy(rows).cuda()
    got_w, got_c = wt[r_idx].cpu().numpy().astype(np.float64), s.codes[r_idx].cpu().numpy()
    del wt

    H = O.hessian(X.float().cpu().numpy(), p.lambda_rel)
    del X
    Wm = W[r_idx].cpu().numpy().T.astype(np.float64)       # [d_in][12]
    sigma, Ht = O.diagonal_scaling(H)
    hdiag = np.diag(H).astype(np.float32)
    del H
    codes0, s0, z0, D0 = O.rtn(Wm, p.bits, p.group)
    np.testing.assert_array_equal(c_init, codes0.T)
    rhs = Ht @ (Wm / sigma[:, None]) + p.rho0 * (D0 / sigma[:, None])
    Ht[np.diag_indices_from(Ht)] += p.rho0
    w_ref = np.linalg.solve(Ht, rhs)                        # [d_in][12]
    err = np.linalg.norm(got_w - w_ref.T) / np.linalg.norm(w_ref)
    c_ref = O.project(sigma[:, None] * w_ref, p.bits, p.group, "lsq", hdiag, s0, z0)[0]
    mism = np.mean(got_c != c_ref.T)
    print(f"{shape} first iteration: W~ rel err {err:.2e}, code mismatches {mism:.2e}")
    assert err <= 1e-4
    assert mism <= 1e-3
