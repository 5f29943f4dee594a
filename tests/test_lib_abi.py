"""The C-ABI library loads and exports every entry point include/admmq.h
declares; argument checks that need no GPU reject bad input."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    src = open(os.path.join(ROOT, "include", "admmq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(admmq_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from post_weight_quantization_10_b200 import admmq, build
    build.build()
    return admmq.lib()


def test_exports_every_declared_function(lib):
    names = _header_functions()
    assert len(names) >= 10
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings(lib):
    from post_weight_quantization_10_b200 import admmq
    for code in range(0, -9, -1):
        s = admmq.status_string(code)
        assert s and s != "unknown status"
    assert admmq.status_string(-99) == "unknown status"
    assert lib.admmq_version() >= 100


def test_argument_checks_without_gpu(lib):
    from post_weight_quantization_10_b200 import admmq
    p = admmq.Params(bits=3, group=128, iters=10).c()
    # d_in not a multiple of the group / of 32, bad bits, bad group
    assert lib.admmq_workspace_bytes(100, 8, ctypes.byref(p)) == 0
    bad = admmq.Params(bits=9, group=128).c()
    assert lib.admmq_workspace_bytes(256, 8, ctypes.byref(bad)) == 0
    bad = admmq.Params(bits=3, group=48).c()
    assert lib.admmq_workspace_bytes(96, 8, ctypes.byref(bad)) == 0
    bad = admmq.Params(bits=3, group=128).c()
    bad.grid_mode = 4
    assert lib.admmq_workspace_bytes(256, 8, ctypes.byref(bad)) == 0
    bad = admmq.Params(bits=3, group=128).c()
    bad.rescale_dual = 2
    assert lib.admmq_workspace_bytes(256, 8, ctypes.byref(bad)) == 0
    bad = admmq.Params(bits=3, group=128).c()
    bad.fit_on_w = -1
    assert lib.admmq_workspace_bytes(256, 8, ctypes.byref(bad)) == 0
    assert lib.admmq_gram_workspace_bytes(100, 30) == 0
    assert lib.admmq_pack(None, 64, 4, 3, None, None) == -1
    assert lib.admmq_pack(ctypes.c_void_p(16), 48, 4, 3, ctypes.c_void_p(16), None) == -1
    assert lib.admmq_build_hessian(None, 10, 64, None, 0, None, 0, None) == -1
    ctx = ctypes.c_void_p()
    assert lib.admmq_create(ctypes.byref(ctx), 100, 8, ctypes.byref(p), None, 0) == -1
    assert lib.admmq_init(None, None, None, None, None) == -1
    assert lib.admmq_iterate(None, 0, 1, None, None, None, None) == -1
    lib.admmq_destroy(None)


def test_alignment_checks_without_gpu(lib):
    """The epilogues move eight words per access: the standalone projection
    rejects state buffers that are not 32-byte aligned before touching the
    device (the pointers below are never dereferenced)."""
    ok = [ctypes.c_void_p(0x10000 * (i + 1)) for i in range(12)]
    # wt V sig rsig hd | d m bits g mode split | codes scale zero p_hi p_lo | row_scale flag
    # | resid dual_scale fit_on_w stream
    def call(ptrs, split=2, mode=0, row_scale=None, flag=None, dual_scale=1.0, fit_on_w=0):
        return lib.admmq_project(*ptrs[:5], 256, 8, 3, 128, mode, split, *ptrs[5:10], row_scale,
                                 flag, ptrs[10], ctypes.c_float(dual_scale), fit_on_w, None)
    for k in (1, 5, 8, 9):  # V, codes, P_hi, P_lo off by 16 bytes
        bad = list(ok)
        bad[k] = ctypes.c_void_p(ok[k].value + 16)
        assert call(bad) == -1, k
    bad = list(ok)
    bad[0] = ctypes.c_void_p(ok[0].value + 8)  # W~ needs 16 bytes
    assert call(bad) == -1
    for split in (0, 4, -1):                   # the kernel needs a concrete split precision
        assert call(list(ok), split) == -1, split
    assert call(list(ok), 3, row_scale=ctypes.c_void_p(0x10002)) == -1   # fp32 scales, 4-byte aligned
    assert call(list(ok), 3, flag=ctypes.c_void_p(0x10001)) == -1
    for mode in (-1, 4):                       # grid modes are 0 (minmax) .. 3 (mse)
        assert call(list(ok), mode=mode) == -1, mode
    for r in (0.0, -1.0, float("nan"), float("inf")):  # the dual factor is positive and finite
        assert call(list(ok), dual_scale=r) == -1, r
    assert call(list(ok), fit_on_w=2) == -1
    assert lib.admmq_split_mode(None) == -1
    assert lib.admmq_set_split(None, 2, None) == -1
    assert lib.admmq_debug_dump_wtilde(None, None) == -1


def test_gptq_argument_checks_without_gpu(lib):
    """GPTQ entry points reject bad sizes and pointers before touching a device."""
    fake = ctypes.c_void_p(0x10000)
    assert lib.admmq_gptq_workspace_bytes(100, 8, 128) == 0      # d_in % 32
    assert lib.admmq_gptq_workspace_bytes(256, 8, 96) == 0       # block
    assert lib.admmq_gptq_workspace_bytes(256, 0, 128) == 0
    args = [fake, fake, 0, 256, 8, 3, 128, 0.01, 128, fake, fake, fake, fake, 1 << 30, None]
    for k, bad in ((0, None), (1, None), (9, None), (12, None),    # null pointers
                   (3, 200), (6, 96), (5, 9), (8, 16), (2, 5), (7, -1.0)):
        a = list(args)
        a[k] = bad
        assert lib.admmq_gptq(*a) == -1, k
    a = list(args)
    a[12] = ctypes.c_void_p(0x10000 + 64)                       # workspace alignment
    assert lib.admmq_gptq(*a) == -1
