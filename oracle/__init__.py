"""CPU oracle for the ADMM-Q layer solve (TEST INFRASTRUCTURE ONLY).

Only `tests/`, `__graft_entry__.smoke()` and the `cpu_baseline` / reference
leg of `bench.py` may import this package.  The product (the C-ABI library and
its Python binding) never calls it: there is no CPU fallback.

  admmq_oracle     float64 Hessian, scaling, ADMM-Q, RTN, GPTQ, Babai, pack
  projection_fp32  float32 op-by-op grid fit / projection / fused epilogue,
                   the bit-exact specification of the projection kernels
  spread           the oracle's own spread under W-update noise, which sets
                   the bar for free-running GPU solves

Pinned by tests/test_oracle_pins.py; "parity unpinned" parts are listed in the
admmq_oracle module docstring.
"""
from . import admmq_oracle, projection_fp32, spread  # noqa: F401
