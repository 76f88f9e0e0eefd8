"""MXFP4 block quantizer for NVIDIA B200 (sm_100a).

The computation lives in libmxfp4.so (C ABI, include/mxfp4.h); this package
is its thin Python binding. See ``_binding`` for the functions.
"""
from ._binding import (  # noqa: F401
    BF16, COLS, F32, RNE, ROWS, SR, STATUS_WAIT_TIMEOUT, SYMBOLS, Mxfp4Error, dequantize,
    double_quantize, gemm, gemm_quantize_a, lib, mxfp4_dequantize, mxfp4_double_quantize,
    mxfp4_gemm, mxfp4_gemm_quantize_a,
    mxfp4_osc_step, mxfp4_osc_synthetic_update, mxfp4_qema_quantize, mxfp4_qramp_step,
    mxfp4_quantize, mxfp4_quantize_oas, mxfp4_rht_quantize, mxfp4_scales_to_blocked,
    mxfp4_status_string, osc_step, osc_synthetic_update, qema_quantize,
    qramp_step, quantize, rht_quantize, scales_to_blocked, status_string)
