"""Thin Python binding of libadmmq.so (C ABI in include/admmq.h).

Argument marshalling only: torch provides device memory and streams, every
step of the solve runs in the library's CUDA kernels (and cuSOLVER for the
one-time eigendecomposition).  A missing library raises; there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

from .build import LIB

OK = 0
GRID_MINMAX, GRID_LSQ, GRID_FROZEN, GRID_MSE = 0, 1, 2, 3
GRID_MODES = {"minmax": GRID_MINMAX, "lsq": GRID_LSQ, "frozen": GRID_FROZEN, "mse": GRID_MSE}
SPLIT_MODES = {"auto": 0, "3xtf32": 1, "mixed": 2, "f16": 3}
SCHEDULES = {"fused": 0, "per_gemm": 1}
DTYPE_F32, DTYPE_BF16 = 0, 1
BUFFERS = ["sigma", "rsig", "hdiag", "lambda", "V", "C0", "P_hi", "P_lo", "T_hi", "T_lo",
           "E_hi", "E_lo", "Ht", "status", "row_in", "row_out"]
ERR_TIMEOUT, ERR_RANGE = -6, -9


class AdmmqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class _Params(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int), ("group", ctypes.c_int), ("iters", ctypes.c_int),
                ("rho0", ctypes.c_float), ("gamma", ctypes.c_float),
                ("lambda_rel", ctypes.c_float), ("grid_mode", ctypes.c_int),
                ("split_mode", ctypes.c_int), ("no_scaling", ctypes.c_int),
                ("schedule", ctypes.c_int), ("rescale_dual", ctypes.c_int),
                ("fit_on_w", ctypes.c_int)]


@dataclass
class Params:
    bits: int = 3
    group: int = 128
    iters: int = 100
    rho0: float = 0.1
    gamma: float = 1.05
    lambda_rel: float = 0.01
    grid: str = "lsq"
    split: str = "auto"   # eigenbasis GEMM split precision: auto | 3xtf32 | mixed | f16
    scaling: bool = True  # False: Sigma = I (the unscaled ablation)
    schedule: str = "fused"  # fused: one launch per iterate call | per_gemm: two per iteration
    rescale_dual: bool = False  # V~ *= rho_t / rho_{t+1} after each iteration (a study variant)
    fit_on_w: bool = False  # refresh the grid from Sigma W~ instead of Sigma (W~ + V~) (a study variant)

    def c(self) -> _Params:
        return _Params(self.bits, self.group, self.iters, self.rho0, self.gamma, self.lambda_rel,
                       GRID_MODES[self.grid], SPLIT_MODES[self.split], int(not self.scaling),
                       SCHEDULES[self.schedule], int(self.rescale_dual), int(self.fit_on_w))


_lib = None
_vp, _i, _i64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t


def _preload_solver_runtime():
    """Use the cuSOLVER build that matches torch's cuBLAS when torch ships one,
    so one process never mixes two cuBLAS versions."""
    try:
        import nvidia.cusolver  # type: ignore
        for base in nvidia.cusolver.__path__:
            p = os.path.join(base, "lib", "libcusolver.so.11")
            if os.path.exists(p):
                ctypes.CDLL(p, mode=ctypes.RTLD_GLOBAL)
                return
    except Exception:
        pass


def lib():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB):
        raise RuntimeError(f"{LIB} is missing: build it with "
                           "`python -m post_weight_quantization_10_b200.build`")
    torch.cuda.init() if torch.cuda.is_available() else None
    _preload_solver_runtime()
    L = ctypes.CDLL(LIB)
    sig = {
        "admmq_status_string": (ctypes.c_char_p, [_i]),
        "admmq_version": (_i, []),
        "admmq_launch_count": (ctypes.c_int64, []),
        "admmq_gram_workspace_bytes": (_sz, [_i64, _i]),
        "admmq_build_hessian": (_i, [_vp, _i64, _i, _vp, _i, _vp, _sz, _vp]),
        "admmq_workspace_bytes": (_sz, [_i, _i, ctypes.POINTER(_Params)]),
        "admmq_create": (_i, [ctypes.POINTER(_vp), _i, _i, ctypes.POINTER(_Params), _vp, _sz]),
        "admmq_destroy": (None, [_vp]),
        "admmq_prepare": (_i, [_vp, _vp, _vp, _i, _vp]),
        "admmq_eigh": (_i, [_vp, _vp]),
        "admmq_setup": (_i, [ctypes.POINTER(_vp), _vp, _vp, _i, _i, _i, ctypes.POINTER(_Params),
                             _vp, _sz, _vp]),
        "admmq_init": (_i, [_vp, _vp, _vp, _vp, _vp]),
        "admmq_iterate": (_i, [_vp, _i, _i, _vp, _vp, _vp, _vp]),
        "admmq_finish": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp]),
        "admmq_solve": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp]),
        "admmq_pack": (_i, [_vp, _i, _i, _i, _vp, _vp]),
        "admmq_get_buffer": (_i, [_vp, _i, ctypes.POINTER(_vp), ctypes.POINTER(_sz)]),
        "admmq_debug_dump_wtilde": (_i, [_vp, _vp]),
        "admmq_set_timing": (_i, [_vp, _i]),
        "admmq_get_timing": (_i, [_vp, ctypes.POINTER(ctypes.c_double),
                                  ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]),
        "admmq_project": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp,
                               _vp, _vp, _vp, _vp, _vp, ctypes.c_float, _i, _vp]),
        "admmq_split_mode": (_i, [_vp]),
        "admmq_set_split": (_i, [_vp, _i, _vp]),
        "admmq_check": (_i, [_vp, _vp]),
        "admmq_debug_skew_ready": (_i, [_vp, _i]),
        "admmq_debug_rint_div": (_i, [_vp, _vp, _i64, _vp, _vp]),
        "admmq_gptq_workspace_bytes": (_sz, [_i, _i, _i]),
        "admmq_gptq": (_i, [_vp, _vp, _i, _i, _i, _i, _i, ctypes.c_float, _i, _vp, _vp, _vp, _vp,
                            _sz, _vp]),
    }
    for name, (res, args) in sig.items():
        if name.startswith("admmq_debug_") and not hasattr(L, name):
            continue  # test hooks of another build; calling one raises
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def launch_count() -> int:
    """Kernels launched by libadmmq.so in this process."""
    return int(lib().admmq_launch_count())


def status_string(s: int) -> str:
    return lib().admmq_status_string(s).decode()


def _check(rc: int, where: str):
    if rc != OK:
        raise AdmmqError(rc, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


# ------------------------------------------------------------------ Hessian


def gram_workspace_bytes(n: int, d_in: int) -> int:
    return int(lib().admmq_gram_workspace_bytes(n, d_in))


def build_hessian(X: torch.Tensor, H: torch.Tensor | None = None, accumulate: bool = False,
                  workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """H = X^T X (fp32, both triangles) from bf16 activations X [n][d_in]."""
    assert X.is_cuda and X.dtype == torch.bfloat16 and X.dim() == 2 and X.is_contiguous()
    n, d = X.shape
    if H is None:
        H = torch.empty((d, d), dtype=torch.float32, device=X.device)
    need = gram_workspace_bytes(n, d)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    _check(lib().admmq_build_hessian(_ptr(X), n, d, _ptr(H), int(accumulate), _ptr(workspace),
                                     workspace.numel(), _stream(stream)), "admmq_build_hessian")
    return H


# ------------------------------------------------------------------- solver


class Solver:
    """One layer solve: owns the workspace tensor and the C context."""

    def __init__(self, d_in: int, d_out: int, params: Params, device="cuda"):
        self.d_in, self.d_out, self.params = d_in, d_out, params
        self._cp = params.c()
        need = int(lib().admmq_workspace_bytes(d_in, d_out, ctypes.byref(self._cp)))
        if need == 0:
            raise AdmmqError(-1, "admmq_workspace_bytes")
        self.workspace = torch.empty(need, dtype=torch.uint8, device=device)
        self._ctx = ctypes.c_void_p()
        _check(lib().admmq_create(ctypes.byref(self._ctx), d_in, d_out, ctypes.byref(self._cp),
                                  _ptr(self.workspace), need), "admmq_create")
        self._W_hat = None
        ng = d_in // params.group
        self.codes = torch.empty((d_out, d_in), dtype=torch.uint8, device=device)
        self.scale = torch.empty((d_out, ng), dtype=torch.float32, device=device)
        self.zero = torch.empty((d_out, ng), dtype=torch.float32, device=device)
        self.resid = torch.zeros((max(params.iters, 1), 2), dtype=torch.float64, device=device)
        self.objective = torch.zeros(1, dtype=torch.float64, device=device)

    def close(self):
        if self._ctx:
            lib().admmq_destroy(self._ctx)
            self._ctx = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def prepare(self, G: torch.Tensor, W_hat: torch.Tensor, stream=None):
        assert G.dtype == torch.float32 and G.shape == (self.d_in, self.d_in) and G.is_contiguous()
        assert W_hat.shape == (self.d_out, self.d_in) and W_hat.is_contiguous()
        dt = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16}[W_hat.dtype]
        self._W_hat = W_hat  # the library reads it again in finish()
        _check(lib().admmq_prepare(self._ctx, _ptr(G), _ptr(W_hat), dt, _stream(stream)),
               "admmq_prepare")

    def eigh(self, stream=None):
        _check(lib().admmq_eigh(self._ctx, _stream(stream)), "admmq_eigh")

    def init(self, stream=None):
        _check(lib().admmq_init(self._ctx, _ptr(self.codes), _ptr(self.scale), _ptr(self.zero),
                                _stream(stream)), "admmq_init")

    def iterate(self, t0: int, count: int, stream=None):
        _check(lib().admmq_iterate(self._ctx, t0, count, _ptr(self.codes), _ptr(self.scale),
                                   _ptr(self.zero), _stream(stream)), "admmq_iterate")

    def finish(self, resid=True, objective=True, stream=None):
        _check(lib().admmq_finish(self._ctx, _ptr(self.codes), _ptr(self.scale), _ptr(self.zero),
                                  _ptr(self.resid) if resid else None,
                                  _ptr(self.objective) if objective else None, _stream(stream)),
               "admmq_finish")

    def objective_of(self, codes, scale, zero, stream=None) -> float:
        """1/2 Tr((D - W_hat)^T H (D - W_hat)) of any codes on any grid of this
        layer (e.g. a GPTQ result), through the same eigenbasis GEMM."""
        out = torch.zeros(1, dtype=torch.float64, device=codes.device)
        _check(lib().admmq_finish(self._ctx, _ptr(codes), _ptr(scale), _ptr(zero), None,
                                  _ptr(out), _stream(stream)), "admmq_finish")
        return float(out.cpu())

    def solve(self, stream=None):
        _check(lib().admmq_solve(self._ctx, _ptr(self.codes), _ptr(self.scale), _ptr(self.zero),
                                 _ptr(self.resid), _ptr(self.objective), _stream(stream)),
               "admmq_solve")

    def kernel_status(self) -> int:
        """The kernels' status word (0 = ok, 1 = a bounded wait gave up);
        synchronises with the device."""
        return int(self.buffer("status")[0].item())

    def check(self, stream=None):
        """Synchronise and raise AdmmqError if a kernel's bounded wait gave up
        (ERR_TIMEOUT) or an fp16-split operand left fp16's range (ERR_RANGE)."""
        _check(lib().admmq_check(self._ctx, _stream(stream)), "admmq_check")

    def debug_skew_ready(self, iterations: int):
        """Failure-path test hook (see include/admmq.h)."""
        _check(lib().admmq_debug_skew_ready(self._ctx, iterations), "admmq_debug_skew_ready")

    def buffer(self, name: str) -> torch.Tensor:
        """A torch view of a workspace buffer (see include/admmq.h for layouts)."""
        which = BUFFERS.index(name)
        p, nb = ctypes.c_void_p(), ctypes.c_size_t()
        _check(lib().admmq_get_buffer(self._ctx, which, ctypes.byref(p), ctypes.byref(nb)),
               "admmq_get_buffer")
        off = p.value - self.workspace.data_ptr()
        raw = self.workspace[off:off + nb.value]
        d, m = self.d_in, self.d_out
        if name in ("sigma", "rsig", "hdiag", "lambda", "row_in", "row_out"):
            return raw.view(torch.float32)
        if name in ("V", "C0"):
            return raw.view(torch.float32).view(m, d)
        mixed = self.split == "mixed"
        if self.split == "f16" and name in ("P_hi", "P_lo", "T_hi", "T_lo"):   # fp16 bit patterns
            return raw[:2 * m * d].view(torch.int16).view(m, d)
        if self.split == "f16" and name in ("E_hi", "E_lo"):
            return raw[:2 * d * d].view(torch.int16).view(d, d)
        if name in ("P_hi", "T_hi") or (name in ("P_lo", "T_lo") and not mixed):
            return raw.view(torch.float32).view(m, d)
        if name in ("P_lo", "T_lo"):   # bf16 correction rows (bit patterns)
            return raw.view(torch.int16).view(m, 2 * d)
        if name == "E_hi" or (name == "E_lo" and not mixed):
            return raw.view(torch.float32).view(d, d)
        if name == "E_lo":
            return raw.view(torch.int16).view(d, 2 * d)
        if name == "Ht":
            return raw.view(torch.float64).view(d, d)
        return raw.view(torch.int32)

    @property
    def split(self) -> str:
        """The eigenbasis GEMMs' split precision: "3xtf32", "mixed" or "f16"."""
        mode = int(lib().admmq_split_mode(self._ctx))
        return {1: "3xtf32", 2: "mixed", 3: "f16"}[mode]

    def set_split(self, split: str, stream=None):
        """Switch to another split precision after eigh(); init() or solve()
        must come next (see admmq_set_split in include/admmq.h)."""
        _check(lib().admmq_set_split(self._ctx, SPLIT_MODES[split], _stream(stream)),
               "admmq_set_split")

    def dump_wtilde(self, out: torch.Tensor | None):
        _check(lib().admmq_debug_dump_wtilde(self._ctx, _ptr(out)), "admmq_debug_dump_wtilde")

    def set_timing(self, enable: bool):
        _check(lib().admmq_set_timing(self._ctx, int(enable)), "admmq_set_timing")

    def get_timing(self):
        """([ms GEMM 1, ms GEMM 2], [launches, launches], iterations timed); with
        the fused schedule index 0 is the fused launches and index 1 is zero."""
        ms = (ctypes.c_double * 2)()
        n = (ctypes.c_int * 2)()
        iters = ctypes.c_int(0)
        _check(lib().admmq_get_timing(self._ctx, ms, n, ctypes.byref(iters)), "admmq_get_timing")
        return [ms[0], ms[1]], [n[0], n[1]], iters.value


# --------------------------------------------------------------- pack etc.


def pack(codes: torch.Tensor, bits: int, out: torch.Tensor | None = None, stream=None):
    m, d = codes.shape
    if out is None:
        out = torch.empty((m, d * bits // 32), dtype=torch.int32, device=codes.device)
    _check(lib().admmq_pack(_ptr(codes), d, m, bits, _ptr(out), _stream(stream)), "admmq_pack")
    return out


def project(wtilde, V, sigma, rsig, hdiag, bits, group, grid, codes, scale, zero, P_hi, P_lo,
            resid=None, split="mixed", row_scale=None, range_flag=None, dual_scale=1.0,
            fit_on_w=False, stream=None):
    """Stand-alone projection; P planes in the encoding of `split`: "3xtf32"
    fp32 [m][d] x2, "mixed" fp32 [m][d] + int16 (bf16 bit patterns) [m][2d],
    "f16" int16 (fp16 bit patterns) [m][d] x2 with the rows' scales
    `row_scale` (fp32 [m]; None = 1) and an optional int32 range flag;
    `dual_scale` multiplies the new V~ (the dual rescaling); `fit_on_w`
    refreshes the grid from sigma W~ alone."""
    m, d = wtilde.shape
    if resid is None:
        resid = torch.zeros(2, dtype=torch.float64, device=wtilde.device)
    _check(lib().admmq_project(_ptr(wtilde), _ptr(V), _ptr(sigma), _ptr(rsig), _ptr(hdiag), d, m,
                               bits, group, GRID_MODES[grid], SPLIT_MODES[split], _ptr(codes),
                               _ptr(scale), _ptr(zero), _ptr(P_hi), _ptr(P_lo), _ptr(row_scale),
                               _ptr(range_flag), _ptr(resid), ctypes.c_float(dual_scale),
                               int(fit_on_w), _stream(stream)),
           "admmq_project")
    return resid


def debug_rint_div(y: torch.Tensor, s: torch.Tensor, stream=None) -> torch.Tensor:
    """rint(y / s[i // 8]) as the projection computes it (tests)."""
    out = torch.empty_like(y)
    _check(lib().admmq_debug_rint_div(_ptr(y), _ptr(s), y.numel(), _ptr(out), _stream(stream)),
           "admmq_debug_rint_div")
    return out


def gptq(G: torch.Tensor, W_hat: torch.Tensor, bits: int, group: int, lambda_rel: float = 0.01,
         block: int = 128, stream=None):
    """GPTQ on the fixed min/max grid of W_hat: returns (codes, scale, zero)."""
    m, d = W_hat.shape
    assert G.dtype == torch.float32 and G.shape == (d, d) and G.is_contiguous()
    assert W_hat.is_contiguous()
    dt = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16}[W_hat.dtype]
    need = int(lib().admmq_gptq_workspace_bytes(d, m, block))
    if need == 0:
        raise AdmmqError(-1, "admmq_gptq_workspace_bytes")
    ws = torch.empty(need, dtype=torch.uint8, device=W_hat.device)
    codes = torch.empty((m, d), dtype=torch.uint8, device=W_hat.device)
    scale = torch.empty((m, d // group), dtype=torch.float32, device=W_hat.device)
    zero = torch.empty_like(scale)
    _check(lib().admmq_gptq(_ptr(G), _ptr(W_hat), dt, d, m, bits, group, lambda_rel, block,
                            _ptr(codes), _ptr(scale), _ptr(zero), _ptr(ws), need, _stream(stream)),
           "admmq_gptq")
    return codes, scale, zero


def solve_layer(X: torch.Tensor, W_hat: torch.Tensor, params: Params, stream=None) -> Solver:
    """Gram -> setup -> solve for one layer; the Solver holds codes/scale/zero,
    the residual history and the objective.  Synchronises once at the end to
    read the status words: when the fp16 split's range word is set, the layer
    is solved again with the mixed split (admmq_set_split); any other error
    raises AdmmqError."""
    H = build_hessian(X, stream=stream)
    s = Solver(X.shape[1], W_hat.shape[0], params, device=X.device)
    s.prepare(H, W_hat, stream)
    s.eigh(stream)
    s.solve(stream)
    try:
        s.check(stream)
    except AdmmqError as e:
        if e.status != ERR_RANGE:
            raise
        s.set_split("mixed", stream)
        s.solve(stream)
        s.check(stream)
    return s
