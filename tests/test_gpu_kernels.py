"""Kernel-level parity of the CUDA path against the oracle (needs a B200).

Inputs come from seeded generators only; expected values come from oracle/.
Bit-exact where the work is integer or an explicitly specified float32
sequence (projection, RTN start, packing); Gram within 1e-4 relative
Frobenius (fp32 tensor-core sums of exact bf16 products).
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


# ------------------------------------------------------------------- Gram


@pytest.mark.parametrize("n,d", [(512, 64), (1000, 192), (4133, 384), (20000, 512)])
def test_gram_matches_oracle(A, n, d):
    p = workloads.scaled(workloads.PRESETS["q_proj"], n, d, 8, rank=8)
    X = workloads.make_activations(p, seed=3, device="cuda")
    H = A.build_hessian(X)
    torch.cuda.synchronize()
    G = O.gram(X.float().cpu().numpy())
    Hc = H.cpu().numpy().astype(np.float64)
    assert np.array_equal(Hc, Hc.T)
    err = np.linalg.norm(Hc - G) / np.linalg.norm(G)
    assert err <= 1e-4, err


def test_gram_accumulate_and_empty(A):
    p = workloads.scaled(workloads.PRESETS["q_proj"], 3000, 256, 8, rank=8)
    X = workloads.make_activations(p, seed=4, device="cuda")
    H = A.build_hessian(X[:1700])
    A.build_hessian(X[1700:], H=H, accumulate=True)
    A.build_hessian(X[:0], H=H, accumulate=True)
    torch.cuda.synchronize()
    G = O.gram(X.float().cpu().numpy())
    assert np.linalg.norm(H.cpu().numpy() - G) / np.linalg.norm(G) <= 1e-4
    Z = A.build_hessian(X[:0])
    torch.cuda.synchronize()
    assert float(Z.abs().max()) == 0.0


def test_gram_tiny_layer(A):
    Xn, _ = workloads.tiny_layer(0)
    X = torch.from_numpy(Xn).to(torch.bfloat16).cuda()
    H = A.build_hessian(X)
    torch.cuda.synchronize()
    G = O.gram(Xn)
    assert np.linalg.norm(H.cpu().numpy() - G) / np.linalg.norm(G) <= 1e-5


# ------------------------------------------------------ projection, bit-exact


def _proj_inputs(m, d, g, bits, seed):
    rng = np.random.default_rng(seed)
    L = (1 << bits) - 1
    sig = np.exp(rng.standard_normal(d)).astype(np.float32) * 0.05
    rsig = (1.0 / sig).astype(np.float32)
    hd = (rsig.astype(np.float64) ** 2).astype(np.float32)
    W = (rng.standard_normal((m, d)) * 2).astype(np.float32)
    V = (rng.standard_normal((m, d)) * 0.3).astype(np.float32)
    s0 = (rng.random((m, d // g)) * 0.05 + 0.01).astype(np.float32)
    z0 = rng.integers(0, L + 1, (m, d // g)).astype(np.float32)
    c0 = rng.integers(0, L + 1, (m, d)).astype(np.uint8)
    W[0, :g] = 0.0            # an all-zero group (zero range) when V is zero there
    V[0, :g] = 0.0
    return dict(W=W, V=V, sig=sig, rsig=rsig, hd=hd, s0=s0, z0=z0, c0=c0)


@pytest.mark.parametrize("split", ["mixed", "3xtf32", "f16"])
@pytest.mark.parametrize("grid", ["minmax", "lsq", "mse", "frozen"])
@pytest.mark.parametrize("bits,g,m,d", [(3, 128, 200, 384), (2, 64, 33, 128), (4, 32, 130, 96),
                                        (3, 64, 32, 64)])
# the study variants: dual rescaling factor, grid fitted on sigma W~ alone
@pytest.mark.parametrize("variant", ["plain", "dual", "fit_w"])
def test_projection_kernel_bitexact(A, grid, bits, g, m, d, split, variant):
    dual = np.float32(1 / 1.05) if variant == "dual" else None
    fit_w = variant == "fit_w"
    x = _proj_inputs(m, d, g, bits, seed=bits * 100 + g + m)
    rng = np.random.default_rng(m + d)
    # the fp16 split's per-row powers of two (1 for the other encodings)
    rs = (np.ldexp(np.float32(1), rng.integers(-4, 5, m)).astype(np.float32) if split == "f16"
          else None)
    ref = P.epilogue_step(x["W"], x["V"], x["sig"], x["rsig"], x["hd"], x["s0"], x["z0"], x["c0"],
                          bits, g, grid, split, row_scale=rs, dual_scale=dual, fit_on_w=fit_w)
    cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    V = cu(x["V"])
    codes, scale, zero = cu(x["c0"]), cu(x["s0"]), cu(x["z0"])
    if split == "f16":
        phi = torch.empty((m, d), dtype=torch.int16, device="cuda")
        plo = torch.empty((m, d), dtype=torch.int16, device="cuda")
    else:
        phi = torch.empty((m, d), dtype=torch.float32, device="cuda")
        plo = (torch.empty((m, 2 * d), dtype=torch.int16, device="cuda") if split == "mixed"
               else torch.empty((m, d), dtype=torch.float32, device="cuda"))
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    resid = A.project(cu(x["W"]), V, cu(x["sig"]), cu(x["rsig"]), cu(x["hd"]), bits, g, grid,
                      codes, scale, zero, phi, plo, split=split,
                      row_scale=cu(rs) if rs is not None else None, range_flag=flag,
                      dual_scale=1.0 if dual is None else float(dual), fit_on_w=fit_w)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(codes.cpu().numpy(), ref["codes"])
    np.testing.assert_array_equal(scale.cpu().numpy().view(np.uint32), ref["scale"].view(np.uint32))
    np.testing.assert_array_equal(zero.cpu().numpy().view(np.uint32), ref["zero"].view(np.uint32))
    np.testing.assert_array_equal(V.cpu().numpy().view(np.uint32), ref["V"].view(np.uint32))
    if split == "f16":
        np.testing.assert_array_equal(phi.cpu().numpy().view(np.uint16), ref["P_hi"])
    else:
        np.testing.assert_array_equal(phi.cpu().numpy().view(np.uint32), ref["P_hi"].view(np.uint32))
    np.testing.assert_array_equal(plo.cpu().numpy().view(np.uint16), ref["P_lo"].view(np.uint16))
    assert int(flag.item()) == 0
    r = resid.cpu().numpy()
    assert r[0] == pytest.approx(ref["r2"], rel=1e-4)
    assert r[1] == pytest.approx(ref["s2"], rel=1e-4, abs=1e-12)


def test_projection_f16_range_flag(A):
    """An fp16-split operand scaled past fp16's largest value raises the range
    flag (the kernel writes the rounded planes and carries on)."""
    m, d, g, bits = 40, 128, 64, 3
    x = _proj_inputs(m, d, g, bits, seed=5)
    cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    rs = np.ones(m, np.float32)
    rs[7] = np.float32(2.0 ** 40)           # row 7's P entries land far past 65504
    ref = P.epilogue_step(x["W"], x["V"], x["sig"], x["rsig"], x["hd"], x["s0"], x["z0"], x["c0"],
                          bits, g, "lsq", "f16", row_scale=rs)
    phi = torch.empty((m, d), dtype=torch.int16, device="cuda")
    plo = torch.empty((m, d), dtype=torch.int16, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    A.project(cu(x["W"]), cu(x["V"]), cu(x["sig"]), cu(x["rsig"]), cu(x["hd"]), bits, g, "lsq",
              cu(x["c0"]), cu(x["s0"]), cu(x["z0"]), phi, plo, split="f16", row_scale=cu(rs),
              range_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == 1
    np.testing.assert_array_equal(phi.cpu().numpy().view(np.uint16)[:7], ref["P_hi"][:7])


# ------------------------------------------------------------------ packing


@pytest.mark.parametrize("bits", range(1, 9))
@pytest.mark.parametrize("m,d", [(7, 32), (5, 96), (3, 128), (33, 384)])
def test_pack_bitexact(A, bits, m, d):
    rng = np.random.default_rng(bits * 1000 + d + m)
    codes = rng.integers(0, 1 << bits, (m, d)).astype(np.uint8)
    out = A.pack(torch.from_numpy(codes).cuda(), bits)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out.cpu().numpy().view(np.uint32), O.pack(codes, bits))


def test_pack_rejects_bad_shapes(A):
    c = torch.zeros((4, 48), dtype=torch.uint8, device="cuda")
    with pytest.raises(A.AdmmqError):
        A.pack(c, 3, out=torch.empty((4, 8), dtype=torch.int32, device="cuda"))


def test_quotient_rounding_matches_correct_division(A):
    """The projection rounds y / s through a reciprocal product and divides
    exactly only near a rounding tie; the integers must equal rint of the
    correctly rounded float32 quotient (numpy's IEEE division) everywhere:
    random data over wide magnitudes, exact half-integer quotients, their
    neighbours a few ulps away, zeros of both signs, tiny and huge values."""
    rng = np.random.default_rng(21)
    nb = 200_000
    s = (np.exp(rng.uniform(-12, 6, nb)) * rng.choice([1.0, 1.5, 1.25, 0.875], nb)).astype(np.float32)
    y = (rng.standard_normal((nb, 8)) * rng.choice([1.0, 10.0, 300.0], (nb, 1)) * s[:, None]).astype(np.float32)
    # exact ties (k + 1/2) s for s with short mantissas, and their neighbours
    t = nb // 4
    k = rng.integers(-300, 300, (t, 8)).astype(np.float32) + np.float32(0.5)
    s_short = np.ldexp(np.float32(1), rng.integers(-20, 10, t)).astype(np.float32) * np.float32(1.5)
    s[:t] = s_short
    y[:t] = (k * s_short[:, None]).astype(np.float32)
    for j, steps in enumerate((1, -1, 2, -2, 3, -3)):
        y[t // 8 * j:t // 8 * (j + 1), 7] = np.nextafter(
            y[t // 8 * j:t // 8 * (j + 1), 7], np.float32(np.inf) if steps > 0 else np.float32(-np.inf))
    y[t:t + 100, 0] = 0.0
    y[t + 100:t + 200, 0] = -0.0
    y[t + 200:t + 300, 1] = np.float32(1e-40)          # subnormal numerators
    y[t + 300:t + 400, 2] = np.float32(3e38)           # huge numerators
    s[t + 400:t + 500] = np.float32(1e-39)             # subnormal divisors
    out = A.debug_rint_div(torch.from_numpy(y.reshape(-1)).cuda(), torch.from_numpy(s).cuda())
    torch.cuda.synchronize()
    with np.errstate(over="ignore", invalid="ignore", divide="ignore"):
        ref = np.rint(y / s[:, None]).astype(np.float32).reshape(-1)
    got = out.cpu().numpy()
    np.testing.assert_array_equal(got.view(np.uint32), ref.view(np.uint32))
