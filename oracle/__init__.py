"""CPU oracle for the packed 4-bit weight path.

TEST INFRASTRUCTURE ONLY.  The test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only code that may import this package.
The product path (``packed_bit_weight_b200``) never imports it and shares no
code with it: the C file ``qmm_oracle.c`` has its own fp16 / E4M3FN / E2M1
codecs and its own copy of the IQ4_NL table, written from the format
definitions on the pages ("Mark-Experimental-V3-8B", section "Quantization";
"Mamb2_8B_FP4_Recall_SQ3.25", section "Representation").

Parity status of each function is stated in ``PINS`` below.
"""
from .oracle import (  # noqa: F401
    FMT_IQ4_NL, FMT_FP4G16_F16, FMT_FP4G16_E4M3, FMT_MXFP4, PINS, build, lib,
    f16_to_f64, f64_to_f16, e4m3_to_f64, e8m0_to_f64, e2m1_to_f64, iq4nl_value,
    data_bytes, scale_bytes, dequant, dequant_row, quantize, matmul, matmul_sampled,
    route, grouped_gemv, router_topk, silu, swiglu, combine,
)
