"""Seeded synthetic layer inputs for the ADMM-Q layer solve.

This module only draws random numbers: it holds none of the quantizer's
arithmetic, so both the GPU path and the float64 oracle can be fed from it.

The pages' workload is Qwen3 linear layers calibrated on 128 x 2048 = 262144
WikiText-2 tokens (GPTQ tutorial, section 4 "evidence"; ADMM-Q summary,
"Experimental results").  Neither the weights nor the dataset are available,
so the layers below stand in for them with the same shapes and qualitative
statistics: heavy-tailed activations, a small fraction of outlier channels,
channel correlation from a shared low-rank component, and a SiLU-gated
(half near-zero) input for down_proj.

Layouts (memory):
  X      [n][d_in]      token-major, bf16 (the Gram kernel's input type)
  W_hat  [d_out][d_in]  torch nn.Linear layout (= the pages' d_in x d_out
                        matrix stored column-major)
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

# ---------------------------------------------------------------------------
# Layer presets (shapes, bits, group, iterations).
# ---------------------------------------------------------------------------


@dataclass(frozen=True)
class LayerPreset:
    name: str
    n: int            # calibration tokens
    d_in: int
    d_out: int
    bits: int
    group: int
    iters: int
    kind: str         # activation recipe
    nu: int = 4       # Student-t degrees of freedom
    outlier_frac: float = 0.01
    outlier_scale: float = 30.0
    rank: int = 64    # shared low-rank component (0 = none)
    w_std: float = 0.02
    rho0: float = 0.1
    gamma: float = 1.05
    lambda_rel: float = 0.01


PRESETS = {
    # 512 x 64 N(0,1) activations with channels 3 and 17 scaled x20,
    # W_hat 64 x 32 N(0, 0.02^2), 3-bit, one group per output column.
    "tiny": LayerPreset("tiny", 512, 64, 32, 3, 64, 50, "tiny"),
    "q_proj": LayerPreset("q_proj", 262144, 4096, 4096, 3, 128, 100,
                          "student_lowrank", nu=4, outlier_frac=0.01,
                          outlier_scale=30.0, rank=64, w_std=0.02),
    "down_proj": LayerPreset("down_proj", 262144, 12288, 4096, 2, 128, 150,
                             "silu_gated", nu=4, outlier_frac=0.005,
                             outlier_scale=50.0, rank=0, w_std=0.015),
    "up_proj_32b": LayerPreset("up_proj_32b", 262144, 5120, 25600, 3, 128, 100,
                               "student_lowrank", nu=3, outlier_frac=0.01,
                               outlier_scale=40.0, rank=128, w_std=0.02),
}


def decoder_layer(bits: int = 3, n: int = 262144):
    """A Qwen3-8B-shaped decoder layer as four solves, one per distinct input
    (and Hessian): q/k/v (4096 -> 4096 + 1024 + 1024) and gate/up (4096 ->
    12288 + 12288) share their input, so each pair of stacked output rows is
    one problem; o (4096 -> 4096) and down (12288 -> 4096) stand alone.  The
    attention-side inputs use the q_proj activation recipe, the MLP's down
    input the SiLU-gated one.  T = 100 iterations (150 for 2 bits).
    Returns [(label, preset, seed)]."""
    T = 150 if bits == 2 else 100
    q, dn = PRESETS["q_proj"], PRESETS["down_proj"]
    mk = lambda base, name, d_in, d_out: LayerPreset(
        **{**base.__dict__, "name": name, "n": n, "d_in": d_in, "d_out": d_out, "bits": bits,
           "iters": T})
    return [("qkv", mk(q, "qkv", 4096, 6144), 0),
            ("o", mk(q, "o", 4096, 4096), 10),
            ("gate_up", mk(q, "gate_up", 4096, 24576), 20),
            ("down", mk(dn, "down", 12288, 4096), 30)]


def scaled(preset: LayerPreset, n: int, d_in: int, d_out: int, **kw) -> LayerPreset:
    """The same recipe at other sizes (used for parity cases the oracle finishes)."""
    fields = dict(preset.__dict__)
    fields.update(dict(n=n, d_in=d_in, d_out=d_out, name=f"{preset.name}@{n}x{d_in}x{d_out}"))
    fields.update(kw)
    return LayerPreset(**fields)


# ---------------------------------------------------------------------------
# The tiny layer: numpy PCG64, X first, then W_hat.
# ---------------------------------------------------------------------------


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


def tiny_layer(seed: int = 0):
    """X [512][64] (bf16-representable float32) and W_hat [32][64] float32."""
    rng = np.random.Generator(np.random.PCG64(seed))
    X = rng.standard_normal((512, 64))
    X[:, 3] *= 20.0
    X[:, 17] *= 20.0
    W_math = rng.standard_normal((64, 32)) * 0.02       # d_in x d_out
    return bf16_round(X.astype(np.float32)), np.ascontiguousarray(W_math.T.astype(np.float32))


# ---------------------------------------------------------------------------
# Torch recipes (CPU or CUDA), drawn in 8192-row chunks from one generator.
# ---------------------------------------------------------------------------


def _student_t(shape, nu: int, gen, device):
    z = torch.randn(shape, generator=gen, device=device)
    chi2 = torch.zeros(shape, device=device)
    for _ in range(nu):
        chi2.add_(torch.randn(shape, generator=gen, device=device).square_())
    return z / torch.sqrt(chi2 / nu)


def make_activations(p: LayerPreset, seed: int = 0, device="cpu", chunk: int = 8192) -> torch.Tensor:
    """X [n][d_in] bf16 following the preset's recipe."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    cgen = torch.Generator(device="cpu")
    cgen.manual_seed(seed + 2)
    n_out = max(1, int(round(p.outlier_frac * p.d_in)))
    idx = torch.randperm(p.d_in, generator=cgen)[:n_out]
    c = torch.ones(p.d_in)
    c[idx] = p.outlier_scale
    c = c.to(device)
    B = None
    if p.rank > 0:
        B = torch.randn((p.d_in, p.rank), generator=gen, device=device) / np.sqrt(p.rank)
    X = torch.empty((p.n, p.d_in), dtype=torch.bfloat16, device=device)
    for r0 in range(0, p.n, chunk):
        r1 = min(p.n, r0 + chunk)
        rows = r1 - r0
        if p.kind == "student_lowrank":
            x = _student_t((rows, p.d_in), p.nu, gen, device) * c
            if B is not None:
                G = torch.randn((rows, p.rank), generator=gen, device=device)
                x = x + G @ B.T
        elif p.kind == "silu_gated":
            a = torch.randn((rows, p.d_in), generator=gen, device=device)
            x = torch.nn.functional.silu(a) * _student_t((rows, p.d_in), p.nu, gen, device) * c
        else:
            raise ValueError(f"unknown activation recipe {p.kind!r}")
        X[r0:r1] = x.to(torch.bfloat16)
    return X


def make_weights(p: LayerPreset, seed: int = 0, device="cpu", dtype=torch.bfloat16) -> torch.Tensor:
    """W_hat [d_out][d_in] ~ N(0, w_std^2)."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed + 1)
    return (torch.randn((p.d_out, p.d_in), generator=gen, device=device) * p.w_std).to(dtype)


def make_layer(p: LayerPreset, seed: int = 0, device="cpu", w_dtype=torch.bfloat16):
    """(X, W_hat) for a preset; the tiny preset uses its numpy recipe."""
    if p.kind == "tiny":
        X, W = tiny_layer(seed)
        return (torch.from_numpy(X).to(torch.bfloat16).to(device),
                torch.from_numpy(W).to(device=device, dtype=torch.float32))
    return make_activations(p, seed, device), make_weights(p, seed, device, w_dtype)
