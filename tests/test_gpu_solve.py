"""Layer-solve parity of the CUDA path against the float64 oracle (needs a B200).

Both sides start from the same seeded X (bf16) and W_hat.  The oracle runs
the whole solve itself (Gram, damping, scaling, eigh, ADMM, objective); the
tolerances are the ones the method's acceptance bar fixes: codes agree on
>= 99.9% of entries, objective within 1e-3 relative, the W iterate of the
first iteration within 1e-4 relative, the RTN start bit-exact.
"""
import numpy as np
import pytest
import torch

from oracle import admmq_oracle as O
from oracle import projection_fp32 as P
from post_weight_quantization_10_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def A():
    from post_weight_quantization_10_b200 import admmq
    admmq.lib()
    return admmq


def _layer(name, seed=0):
    if name == "tiny":
        p = workloads.PRESETS["tiny"]
        Xn, W = workloads.tiny_layer(seed)
        return p, torch.from_numpy(Xn).to(torch.bfloat16).cuda(), torch.from_numpy(W).cuda()
    base, n, d, m, extra = {
        # the configs' own iteration counts (T = 100 for q_proj, 150 for
        # down_proj): by then the iterates have converged (no code changes at
        # the end), which is where the codes are a well-posed comparison
        "ragged": ("q_proj", 4096, 384, 200, dict(rank=16)),
        "down_small": ("down_proj", 4096, 256, 130, dict()),
    }[name]
    p = workloads.scaled(workloads.PRESETS[base], n, d, m, **extra)
    X = workloads.make_activations(p, seed=seed, device="cuda")
    W = workloads.make_weights(p, seed=seed, device="cuda", dtype=torch.float32)
    return p, X, W


def _oracle(p, X, W, grid, iters=None):
    Xn = X.float().cpu().numpy()
    H = O.hessian(Xn, p.lambda_rel)
    Wm = W.float().cpu().numpy().T.astype(np.float64)
    res = O.admm_q(H, Wm, p.bits, p.group, p.iters if iters is None else iters, rho0=p.rho0,
                   gamma=p.gamma, grid=grid)
    return H, Wm, res


def _solver(A, p, X, W, grid, iters=None):
    prm = A.Params(bits=p.bits, group=p.group, iters=p.iters if iters is None else iters,
                   rho0=p.rho0, gamma=p.gamma, lambda_rel=p.lambda_rel, grid=grid)
    G = A.build_hessian(X)
    s = A.Solver(X.shape[1], W.shape[0], prm)
    s.prepare(G, W)
    s.eigh()
    return s


@pytest.mark.parametrize("name", ["tiny", "ragged"])
def test_setup_matches_oracle(A, name):
    p, X, W = _layer(name)
    s = _solver(A, p, X, W, "minmax")
    torch.cuda.synchronize()
    H = O.hessian(X.float().cpu().numpy(), p.lambda_rel)
    sigma, Ht = O.diagonal_scaling(H)
    np.testing.assert_allclose(s.buffer("sigma").cpu().numpy(), sigma, rtol=2e-5)
    np.testing.assert_allclose(s.buffer("hdiag").cpu().numpy(), np.diag(H), rtol=2e-5)
    lam = np.linalg.eigvalsh(Ht)
    np.testing.assert_allclose(s.buffer("lambda").cpu().numpy(), lam, rtol=1e-4,
                               atol=1e-4 * lam.max())


@pytest.mark.parametrize("name", ["tiny", "ragged"])
def test_rtn_start_bitexact(A, name):
    p, X, W = _layer(name)
    s = _solver(A, p, X, W, "minmax")
    s.init()
    torch.cuda.synchronize()
    Wr = W.cpu().numpy()
    # codes / scale / zero of the start depend on W_hat alone
    ref = P.init_step(Wr, np.ones(Wr.shape[1], np.float32), p.bits, p.group)
    np.testing.assert_array_equal(s.codes.cpu().numpy(), ref["codes"])
    np.testing.assert_array_equal(s.scale.cpu().numpy(), ref["scale"])
    np.testing.assert_array_equal(s.zero.cpu().numpy(), ref["zero"])
    c_o, s_o, z_o, _ = O.rtn(Wr.T.astype(np.float64), p.bits, p.group)
    np.testing.assert_array_equal(s.codes.cpu().numpy(), c_o.T)
    np.testing.assert_array_equal(s.scale.cpu().numpy(), s_o.T)


@pytest.mark.parametrize("name", ["tiny", "ragged"])
@pytest.mark.parametrize("grid", ["minmax", "lsq"])
def test_first_iteration_w_update(A, name, grid):
    """W~ after iteration 0 (from the bit-exact RTN start) within 1e-4 relative
    of the oracle's float64 W-update; the fused epilogue then equals the
    standalone projection kernel applied to that W~."""
    p, X, W = _layer(name)
    s = _solver(A, p, X, W, grid, iters=1)
    s.init()
    V0 = s.buffer("V").clone()
    c0, s0, z0 = s.codes.clone(), s.scale.clone(), s.zero.clone()
    wt = torch.empty((W.shape[0], X.shape[1]), dtype=torch.float32, device="cuda")
    s.dump_wtilde(wt)
    s.iterate(0, 1)
    s.dump_wtilde(None)
    torch.cuda.synchronize()
    H, Wm, res = _oracle(p, X, W, grid, iters=1)
    Wt_ref = res["W_tilde"].T
    got = wt.cpu().numpy().astype(np.float64)
    err = np.linalg.norm(got - Wt_ref) / np.linalg.norm(Wt_ref)
    assert err <= 1e-4, err
    # fused epilogue == standalone projection kernel on the same W~
    V = V0.clone()
    codes, scale, zero = c0.clone(), s0.clone(), z0.clone()
    phi = torch.empty_like(s.buffer("P_hi"))
    plo = torch.empty_like(phi)
    A.project(wt, V, s.buffer("sigma"), s.buffer("rsig"), s.buffer("hdiag"), p.bits, p.group,
              grid, codes, scale, zero, phi, plo)
    torch.cuda.synchronize()
    assert torch.equal(codes, s.codes) and torch.equal(scale, s.scale) and torch.equal(zero, s.zero)
    assert torch.equal(V, s.buffer("V"))
    assert torch.equal(phi, s.buffer("P_hi")) and torch.equal(plo, s.buffer("P_lo"))


@pytest.mark.parametrize("name", ["tiny", "ragged", "down_small"])
@pytest.mark.parametrize("grid", ["minmax", "lsq", "frozen"])
def test_solve_matches_oracle(A, name, grid):
    p, X, W = _layer(name)
    s = _solver(A, p, X, W, grid)
    s.solve()
    torch.cuda.synchronize()
    H, Wm, res = _oracle(p, X, W, grid)
    codes = s.codes.cpu().numpy()
    agree = np.mean(codes == res["codes"].T)
    assert agree >= 0.999, agree
    obj = float(s.objective.cpu())
    assert obj == pytest.approx(res["objective"], rel=1e-3)
    # the objective the GPU reports is the one of the codes it returns
    L = (1 << p.bits) - 1
    Dg = (np.repeat(s.scale.cpu().numpy(), p.group, axis=1) *
          (codes - np.repeat(s.zero.cpu().numpy(), p.group, axis=1))).astype(np.float32)
    assert O.objective(H, Dg.T, Wm) == pytest.approx(obj, rel=1e-4)
    assert codes.max() <= L
    # residual history: the trajectories coincide at the start; later a flipped
    # code near a rounding tie may shift a single iterate's residual
    r = s.resid.cpu().numpy()[: p.iters]
    np.testing.assert_allclose(r[:5, 0], res["r"][:5], rtol=1e-3)
    assert np.median(np.abs(r[:, 0] - res["r"]) / res["r"]) <= 1e-2

