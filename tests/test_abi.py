"""The C-ABI library on the host: it loads, exports every entry point that
include/*.h declares, and rejects bad arguments with the documented status
before any launch. No kernel runs here (CPU only)."""
import ctypes
import glob
import os
import re

import pytest

import mxfp4_block_quantization_quantizer_b200 as m
from mxfp4_block_quantization_quantizer_b200 import _binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, NULL, SHAPE, ALIGN, ENUM, CUDA = range(6)
P = ctypes.c_void_p(4096)       # a 16-byte aligned non-null pointer
PODD = ctypes.c_void_p(4096 + 8)  # misaligned by 8 bytes
NUL = ctypes.c_void_p(0)
P2 = ctypes.c_void_p(4096 + 2)  # not even 4-byte aligned


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(mxfp4_[a-z0-9_]+)\s*\(", text))
    return names


def test_library_exports_every_declared_entry_point():
    L = m.lib()
    decl = declared_symbols()
    assert decl == set(_binding.SYMBOLS)
    for name in decl:
        assert getattr(L, name) is not None


def test_library_is_the_in_tree_build():
    assert os.path.dirname(_binding.LIB_PATH) == os.path.join(
        ROOT, "mxfp4_block_quantization_quantizer_b200")
    assert os.path.exists(_binding.LIB_PATH)


def test_status_strings():
    for s in range(6):
        assert m.status_string(s)
    assert m.status_string(99) == "unknown status"


@pytest.mark.parametrize("args,want", [
    ((P, 2, 64, 64, 0, 0, 0, P, P, NUL), ENUM),      # bad dtype
    ((P, 1, 64, 64, 2, 0, 0, P, P, NUL), ENUM),      # bad axis
    ((P, 1, 64, 64, 0, 5, 0, P, P, NUL), ENUM),      # bad rounding
    ((NUL, 1, 64, 64, 0, 0, 0, P, P, NUL), NULL),
    ((P, 1, 64, 64, 0, 0, 0, NUL, P, NUL), NULL),
    ((P, 1, 64, 64, 0, 0, 0, P, NUL, NUL), NULL),
    ((P, 1, 0, 64, 0, 0, 0, P, P, NUL), SHAPE),      # empty
    ((P, 1, 64, -32, 0, 0, 0, P, P, NUL), SHAPE),
    ((P, 1, 64, 48, 0, 0, 0, P, P, NUL), SHAPE),     # ROWS needs cols % 32
    ((P, 1, 48, 64, 1, 0, 0, P, P, NUL), SHAPE),     # COLS needs rows % 32
    ((P, 1, 1 << 32, 32, 0, 0, 0, P, P, NUL), SHAPE),  # past the size limit
    ((P, 1, 1 << 30, 1 << 20, 0, 0, 0, P, P, NUL), SHAPE),
    ((PODD, 1, 64, 64, 0, 0, 0, P, P, NUL), ALIGN),
    ((P, 1, 64, 64, 0, 0, 0, PODD, P, NUL), ALIGN),
])
def test_quantize_rejects_bad_arguments(args, want):
    assert m.lib().mxfp4_quantize(*args) == want


def test_quantize_oas_rejects_bad_arguments():
    L = m.lib()
    assert L.mxfp4_quantize_oas(P, 2, 64, 64, 0, 0, 0, P, P, NUL) == ENUM
    assert L.mxfp4_quantize_oas(NUL, 1, 64, 64, 0, 0, 0, P, P, NUL) == NULL
    assert L.mxfp4_quantize_oas(P, 1, 64, 48, 0, 0, 0, P, P, NUL) == SHAPE
    assert L.mxfp4_quantize_oas(PODD, 1, 64, 64, 0, 0, 0, P, P, NUL) == ALIGN


def test_overflow_aware_double_and_rotation_reject_bad_arguments():
    L = m.lib()
    assert L.mxfp4_double_quantize_oas(P, 2, 64, 64, 0, P, P, P, P, NUL) == ENUM
    assert L.mxfp4_double_quantize_oas(P, 1, 64, 48, 0, P, P, P, P, NUL) == SHAPE
    assert L.mxfp4_double_quantize_oas(P, 1, 48, 64, 0, P, P, P, P, NUL) == SHAPE
    assert L.mxfp4_double_quantize_oas(P, 1, 64, 64, 0, P, NUL, P, P, NUL) == NULL
    assert L.mxfp4_double_quantize_oas(PODD, 1, 64, 64, 0, P, P, P, P, NUL) == ALIGN
    assert L.mxfp4_rht_quantize_oas(P, 1, 64, 40, 0, 0, 0, P, P, NUL, NUL, NUL) == SHAPE
    assert L.mxfp4_rht_quantize_oas(P, 1, 64, 64, 0, 3, 0, P, P, NUL, NUL, NUL) == ENUM
    assert L.mxfp4_rht_quantize_oas(NUL, 1, 64, 64, 0, 0, 0, P, P, NUL, NUL, NUL) == NULL
    assert L.mxfp4_rht_quantize_oas(P, 1, 64, 64, 0, 0, 0, P, P, PODD, NUL, NUL) == ALIGN


def test_other_entry_points_reject_bad_arguments():
    L = m.lib()
    assert L.mxfp4_dequantize(P, P, 64, 64, 0, P, 3, NUL) == ENUM
    assert L.mxfp4_dequantize(NUL, P, 64, 64, 0, P, 1, NUL) == NULL
    assert L.mxfp4_dequantize(P, P, 64, 40, 0, P, 1, NUL) == SHAPE
    assert L.mxfp4_dequantize(P, P, 64, 64, 0, PODD, 1, NUL) == ALIGN
    assert L.mxfp4_double_quantize(P, 1, 64, 48, 0, P, P, P, P, NUL) == SHAPE
    assert L.mxfp4_double_quantize(P, 1, 48, 64, 0, P, P, P, P, NUL) == SHAPE
    assert L.mxfp4_double_quantize(P, 1, 64, 64, 0, P, P, NUL, P, NUL) == NULL
    assert L.mxfp4_double_quantize(P, 1, 64, 64, 0, P, P, PODD, P, NUL) == ALIGN
    assert L.mxfp4_rht_quantize(P, 1, 64, 40, 0, 0, 0, P, P, NUL, NUL, NUL) == SHAPE
    assert L.mxfp4_rht_quantize(P, 1, 64, 64, 0, 3, 0, P, P, NUL, NUL, NUL) == ENUM
    assert L.mxfp4_rht_quantize(P, 1, 64, 64, 0, 0, 0, P, P, PODD, NUL, NUL) == ALIGN
    assert L.mxfp4_osc_step(P, P, NUL, P, 64, 64, 0, 4.0, NUL, NUL) == NULL
    assert L.mxfp4_osc_step(P, P, P, P, 64, 40, 0, 4.0, NUL, NUL) == SHAPE
    assert L.mxfp4_osc_step(P, PODD, P, P, 64, 64, 0, 4.0, NUL, NUL) == ALIGN
    assert L.mxfp4_osc_synthetic_update(NUL, 4, 4, 0, 0, 1e-4, NUL) == NULL
    assert L.mxfp4_osc_synthetic_update(P, 0, 4, 0, 0, 1e-4, NUL) == SHAPE
    q = (P, P, P, P, P, P, P)
    assert L.mxfp4_qramp_step(P, P, P, P, P, P, NUL, 64, 64, 0, 30, 16.0, 5, NUL, NUL) == NULL
    assert L.mxfp4_qramp_step(*q, 64, 48, 0, 30, 16.0, 5, NUL, NUL) == SHAPE
    assert L.mxfp4_qramp_step(*q, 64, 64, -1, 30, 16.0, 5, NUL, NUL) == SHAPE
    assert L.mxfp4_qramp_step(*q, 64, 64, 0, -1, 16.0, 5, NUL, NUL) == SHAPE
    assert L.mxfp4_qramp_step(*q, 64, 64, 0, 30, 16.0, 0, NUL, NUL) == SHAPE
    assert L.mxfp4_qramp_step(P, P, P, P, P, P, PODD, 64, 64, 0, 30, 16.0, 5, NUL, NUL) == ALIGN
    assert L.mxfp4_qema_quantize(P, NUL, 64, 64, 0.998, P, P, NUL) == NULL
    assert L.mxfp4_qema_quantize(P, P, 64, 48, 0.998, P, P, NUL) == SHAPE
    assert L.mxfp4_qema_quantize(P, PODD, 64, 64, 0.998, P, P, NUL) == ALIGN
    assert L.mxfp4_scales_to_blocked(NUL, 128, 4, P, NUL) == NULL
    assert L.mxfp4_scales_to_blocked(P, 128, 4, NUL, NUL) == NULL
    assert L.mxfp4_scales_to_blocked(P, 0, 4, P, NUL) == SHAPE
    assert L.mxfp4_scales_to_blocked(P, 128, -4, P, NUL) == SHAPE
    assert L.mxfp4_scales_to_blocked(P, 1 << 32, 4, P, NUL) == SHAPE
    assert L.mxfp4_scales_to_blocked(PODD, 128, 4, PODD, NUL) == ALIGN
    assert L.mxfp4_gemm(P, P, P, NUL, 128, 128, 256, P, NUL, NUL) == NULL
    assert L.mxfp4_gemm(P, P, P, P, 128, 128, 48, P, NUL, NUL) == SHAPE
    assert L.mxfp4_gemm(P, P, P, P, 0, 128, 256, P, NUL, NUL) == SHAPE
    assert L.mxfp4_gemm(P, P, P, P, 128, 128, 256, PODD, NUL, NUL) == ALIGN
    assert L.mxfp4_gemm(P, PODD, P, P, 128, 128, 256, P, NUL, NUL) == ALIGN
    g = L.mxfp4_gemm_quantize_a
    assert g(P, 128, 256, 256, 2, 0, P, P, P, NUL, NUL, NUL, NUL) == ENUM
    assert g(NUL, 128, 256, 256, 0, 0, P, P, P, NUL, NUL, NUL, NUL) == NULL
    assert g(P, 128, 256, 256, 1, 0, P, P, P, P, NUL, NUL, NUL) == NULL  # codes, no scales
    assert g(P, 128, 256, 128, 0, 0, P, P, P, NUL, NUL, NUL, NUL) == SHAPE  # k % 256
    assert g(P, 0, 256, 256, 0, 0, P, P, P, NUL, NUL, NUL, NUL) == SHAPE
    assert g(PODD, 128, 256, 256, 0, 0, P, P, P, NUL, NUL, NUL, NUL) == ALIGN
    assert g(P, 128, 256, 256, 0, 0, P, P, P, PODD, P, NUL, NUL) == ALIGN
    assert g(P, 128, 256, 256, 0, 0, P, P, P, NUL, NUL, P2, NUL) == ALIGN
    # the status word needs 4-byte alignment only
    assert L.mxfp4_gemm(P, P, P, P, 128, 128, 256, P, P2, NUL) == ALIGN
    assert L.mxfp4_rht_quantize(P, 1, 64, 64, 0, 0, 0, P, P, NUL, P2, NUL) == ALIGN
    assert L.mxfp4_rht_quantize_oas(P, 1, 64, 64, 0, 0, 0, P, P, NUL, P2, NUL) == ALIGN


def test_binding_refuses_host_tensors():
    import torch
    x = torch.zeros(32, 32, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        m.quantize(x)
    with pytest.raises(TypeError):
        m.double_quantize(x)
