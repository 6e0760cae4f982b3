"""fp64 CPU oracle for the W4A16 weight-only quantized matmul.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports, links or calls this
package; only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` use it, to check the CUDA path and to time a CPU baseline.

What it computes (plain definitions, no blocking, no fusion):

* ``formats``: decoders of the storage types named by the checkpoint
  contracts (BF16, OCP FP8-E4M3, FP4-E2M1) and round-to-nearest-even onto
  BF16 from an exact binary64 value.
* ``w4a16``: dequantisation of the checkpoint formats (int4, NVFP4, FP8) into BF16 weights
  (one rounding of the exact product), then y = x . W_deq^T accumulated in
  fp64, plus the per-element tolerance bound sum_k |W_deq[n][k] * x[m][k]|;
  and the fused gate/up layer h = SiLU(gate) * up with its tolerance.
* ``w4a4``: groundwork for W4A4 NVFP4 (activations quantised too): the
  activation quantiser and the exact GEMM of the quantised operands.

It works from the *logical* tensors (int8 q or uint8 codes, [N][K]; scales per
output column and K-group) and never from the library's packed layout, so it
shares no code, table or layout knowledge with the CUDA side.
"""

from .formats import (bf16_to_f64, e4m3_to_f64, e2m1_to_f64, f64_to_bf16_rne,  # noqa: F401
                      f64_to_e4m3_rne, f64_to_e2m1_rne)
from . import w4a4  # noqa: F401
from .w4a16 import (  # noqa: F401
    dequant_int4_g128,
    dequant_nvfp4,
    dequant_fp8_e4m3,
    gemm_ref,
    abs_bound,
    within_tolerance,
    silu,
    gate_up_silu_ref,
    gate_up_silu_allowed,
    TOL_REL,
    TOL_ABS,
)
