"""CPU oracle for the fused RMSNorm + quantization path (test infrastructure).

Only the tests, the smoke check and the benchmark's CPU baseline use this
package.  The product path (the CUDA library and its binding) never imports it.

Every function takes and returns numpy arrays: bf16 tensors travel as their
uint16 bit patterns, codes and E8M0 scales as uint8, FP8 scales as float32.

Parity status of each function (what pins it is in tests/test_oracle_pins.py):
  bf16_from_double, fp16_to_double/from_double, e4m3_encode/decode,
  e2m1_encode/decode, mx_scale_code, quant_rows, rstd, rmsnorm_quant (bf16 and
  binary16 I/O), qk_norm_gate, qk_norm_gate_fp8, place_scales, hc_mix: pinned.
"""
from .oracle import (  # noqa: F401
    FP8_PER_TOKEN, FP8_PER_GROUP128, MXFP4, OracleError, load, bf16_from_double,
    bf16_to_double, e4m3_encode, e4m3_decode, e2m1_encode, e2m1_decode,
    mx_scale_code, rstd, quant_rows, rmsnorm_quant, qk_norm_gate, scale_shape,
    code_shape, place_scales, qk_norm_gate_fp8, SCALE_SWIZZLE_32_4_4, SCALE_MN_MAJOR,
    IO_BF16, IO_FP16, fp16_to_double, fp16_from_double, hc_mix,
)
