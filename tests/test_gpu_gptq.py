"""GPU GPTQ (the baseline of the objective report) against the float64 oracle's
GPTQ Algorithm 1 (needs a B200).

Both sides get the same inputs: the Gram of the seeded bf16 activations,
formed by the oracle in float64 and rounded to fp32 (the GPU takes fp32 G),
and W_hat.  Both run GPTQ in float64 on the same min/max grid, so the codes
agree except where the trailing products' summation order decides a tie;
the grid is bit-exact.
"""
import numpy as np
import pytest
import torch

from oracle import admmq_oracle as O
from post_weight_quantization_10_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def A():
    from post_weight_quantization_10_b200 import admmq
    admmq.lib()
    return admmq


def _layer(name):
    if name == "tiny":
        p = workloads.PRESETS["tiny"]
        Xn, W = workloads.tiny_layer(0)
        return p, Xn.astype(np.float32), W.astype(np.float32)
    base, n, d, m = {"ragged": ("q_proj", 4096, 384, 200),
                     "mid": ("q_proj", 8192, 1024, 256),
                     "down_small": ("down_proj", 4096, 256, 130)}[name]
    p = workloads.scaled(workloads.PRESETS[base], n, d, m)
    X = workloads.make_activations(p, seed=0, device="cuda").float().cpu().numpy()
    W = workloads.make_weights(p, seed=0, device="cuda", dtype=torch.float32).cpu().numpy()
    return p, X, W


def _inputs(p, X, W):
    G32 = O.gram(X).astype(np.float32)
    H = O.damping(G32.astype(np.float64), p.lambda_rel)[0]
    return G32, H


def _dequant(codes, scale, zero, g):
    return np.repeat(scale, g, axis=1) * (codes.astype(np.float64) - np.repeat(zero, g, axis=1))


@pytest.mark.parametrize("name", ["tiny", "ragged", "mid", "down_small"])
def test_gptq_matches_oracle(A, name):
    p, X, W = _layer(name)
    G32, H = _inputs(p, X, W)
    codes, scale, zero = A.gptq(torch.from_numpy(G32).cuda(), torch.from_numpy(W).cuda(), p.bits,
                                p.group, p.lambda_rel)
    torch.cuda.synchronize()
    s_o, z_o = O.minmax_grid_rows(W, p.bits, p.group)
    np.testing.assert_array_equal(scale.cpu().numpy(), s_o)
    np.testing.assert_array_equal(zero.cpu().numpy(), z_o)
    c_o, Q_o = O.gptq(H, W.astype(np.float64), s_o, z_o, p.bits, p.group)
    c = codes.cpu().numpy().astype(np.int64)
    mism = np.mean(c != c_o)
    print(f"gptq {name}: code mismatches {mism:.2e}")
    assert mism <= 1e-3
    Wm = W.T.astype(np.float64)
    obj_gpu = O.objective(H, _dequant(c, s_o, z_o, p.group).T, Wm)
    obj_o = O.objective(H, Q_o.T, Wm)
    assert obj_gpu == pytest.approx(obj_o, rel=1e-3)


def test_gptq_block_size_invariance_and_beats_rtn(A):
    """The block size only regroups the same updates (GPTQ section 3): codes
    of B = 32, 64, 128 agree; GPTQ's objective is below RTN's on the same
    grid."""
    p, X, W = _layer("ragged")
    G32, H = _inputs(p, X, W)
    Gd, Wd = torch.from_numpy(G32).cuda(), torch.from_numpy(W).cuda()
    outs = [A.gptq(Gd, Wd, p.bits, p.group, p.lambda_rel, block=b)[0].cpu().numpy()
            for b in (32, 64, 128)]
    torch.cuda.synchronize()
    assert np.mean(outs[0] != outs[2]) <= 1e-4 and np.mean(outs[1] != outs[2]) <= 1e-4
    s_o, z_o = O.minmax_grid_rows(W, p.bits, p.group)
    Wm = W.T.astype(np.float64)
    c_rtn, _, _, D_rtn = O.rtn(Wm, p.bits, p.group)
    obj_gptq = O.objective(H, _dequant(outs[2], s_o, z_o, p.group).T, Wm)
    assert obj_gptq < O.objective(H, D_rtn, Wm)


def test_gptq_full_size_sampled_rows(A):
    """4096 x 4096 (q_proj shape, n = 8192): the GPU quantizes every row; the
    oracle quantizes 12 sampled rows (GPTQ treats rows independently)."""
    rows = np.array([0, 1, 77, 128, 1000, 2047, 2048, 3001, 3500, 4000, 4094, 4095])
    p = workloads.scaled(workloads.PRESETS["q_proj"], 8192, 4096, 4096)
    X = workloads.make_activations(p, seed=0, device="cuda").float().cpu().numpy()
    W = workloads.make_weights(p, seed=0, device="cuda", dtype=torch.float32).cpu().numpy()
    G32, H = _inputs(p, X, W)
    codes, scale, zero = A.gptq(torch.from_numpy(G32).cuda(), torch.from_numpy(W).cuda(), p.bits,
                                p.group, p.lambda_rel)
    torch.cuda.synchronize()
    Ws = W[rows]
    s_o, z_o = O.minmax_grid_rows(Ws, p.bits, p.group)
    np.testing.assert_array_equal(scale.cpu().numpy()[rows], s_o)
    c_o, _ = O.gptq(H, Ws.astype(np.float64), s_o, z_o, p.bits, p.group)
    mism = np.mean(codes.cpu().numpy()[rows] != c_o)
    print(f"gptq full size: code mismatches on sampled rows {mism:.2e}")
    assert mism <= 1e-3
