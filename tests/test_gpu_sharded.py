"""The sharded single-layer solve on one GPU (needs a B200): with world size
1 it is the plain solve; split by hand into two row blocks on the same H, the
row blocks reproduce the whole layer's codes bit for bit (rows are
independent through every step); split into two token blocks, the summed
partial Grams equal the whole Gram within fp32 rounding."""
import numpy as np
import pytest
import torch

from post_weight_quantization_10_b200 import sharded, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def A():
    from post_weight_quantization_10_b200 import admmq
    admmq.lib()
    return admmq


def _layer():
    p = workloads.scaled(workloads.PRESETS["q_proj"], 8192, 1024, 600)
    X = workloads.make_activations(p, seed=3, device="cuda")
    W = workloads.make_weights(p, seed=3, device="cuda", dtype=torch.float32)
    prm = dict(bits=p.bits, group=p.group, iters=40, rho0=p.rho0, gamma=p.gamma,
               lambda_rel=p.lambda_rel, grid="lsq")
    return p, X, W, prm


def test_world_one_is_the_plain_solve(A):
    p, X, W, prm = _layer()
    res = sharded.solve_layer_sharded(X, W, (0, W.shape[0]), A.Params(**prm), A, world=1)
    whole = A.solve_layer(X, W, A.Params(**prm))
    torch.cuda.synchronize()
    assert torch.equal(res.codes, whole.codes)
    assert res.objective == pytest.approx(float(whole.objective.cpu()), rel=1e-12)


def test_row_blocks_reproduce_the_whole_layer(A):
    p, X, W, prm = _layer()
    G = A.build_hessian(X)
    whole = A.Solver(p.d_in, W.shape[0], A.Params(**prm))
    whole.prepare(G, W)
    whole.eigh()
    whole.solve()
    parts, obj = [], 0.0
    for r in range(2):
        r0, r1 = sharded.block(W.shape[0], 2, r)
        s = A.Solver(p.d_in, r1 - r0, A.Params(**prm))
        s.prepare(G, W[r0:r1].contiguous())
        s.eigh()
        s.solve()
        parts.append(s.codes)
        obj += float(s.objective.cpu())
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts), whole.codes)
    # Same codes, hence the same D; the objective is summed from float32
    # partials per 32-row warp and 128-row tile, and the row blocks start a
    # tile at row 300 where the whole layer does not, so the two totals
    # group the rows differently: they agree to the rounding of float32
    # partial sums of ~160 terms (~1e-6 relative), not bit for bit.
    assert obj == pytest.approx(float(whole.objective.cpu()), rel=1e-6)


def test_token_blocks_sum_to_the_whole_gram(A):
    p, X, W, prm = _layer()
    G = A.build_hessian(X)
    Gs = sum(A.build_hessian(X[slice(*sharded.block(X.shape[0], 2, r))].contiguous())
             for r in range(2))
    torch.cuda.synchronize()
    err = float((Gs.double() - G.double()).norm() / G.double().norm())
    assert err <= 1e-6, err
