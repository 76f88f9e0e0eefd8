"""Regression test of the E2M1 decode: every one of the 256 code bytes goes
through each place a kernel decodes codes (the dequantizer's word decode in
both layouts and both output types; the double quantizer's decode of its
staged Q_D(X) codes, bf16 and fp32 inputs, both scale rules), against the
oracle. The decodes read 32-bit code words loaded from memory; a form that
fed freshly encoded codes to the conversion in registers once decoded
wrong values, and this test would show such a regression.
"""
import numpy as np
import pytest
import torch

import mxfp4_block_quantization_quantizer_b200 as m
import oracle as O
from gpu_util import BF16, assert_bits_equal, to_dev, to_np

pytestmark = pytest.mark.gpu

# E2M1 code -> value (sign in bit 3), the grid {0, .5, 1, 1.5, 2, 3, 4, 6}
GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def code_value(c):
    v = GRID[c & 7]
    return -v if c & 8 else v


@pytest.mark.parametrize("axis", [O.ROWS, O.COLS])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_dequantize_every_byte(axis, out):
    # a [64, 512] tensor: 16384 codes = every byte 64 times, in both layouts
    R, C = 64, 512
    g = np.random.Generator(np.random.PCG64(31))
    codes = np.tile(np.arange(256, dtype=np.uint8), R * C // 2 // 256)
    g.shuffle(codes)
    codes = codes.reshape((R, C // 2) if axis == O.ROWS else (C, R // 2))
    n_scales = R * C // 32
    scales = np.array([1, 2, 100, 127, 128, 200, 252, 254], np.uint8)[
        g.integers(0, 8, n_scales)].reshape((R, C // 32) if axis == O.ROWS else (C, R // 32))
    got = m.dequantize(to_dev(codes), to_dev(scales), R, C, axis,
                       out_dtype=torch.bfloat16 if out == "bf16" else torch.float32)
    want = O.dequantize(codes, scales, R, C, axis, out)
    assert_bits_equal(to_np(got), want, "decode of every byte")


def byte_tensor(rows, dtype):
    """[rows, 512] whose 1x32 row groups hold exact grid values arranged so
    that each row's RNE codes are the 256 bytes in order (group j: bytes
    16j .. 16j+15; every group holds a 6, so its scale is 2^0 times the
    row's power of two). Row r is scaled by 2^(r % 7 - 3)."""
    b = np.arange(256)
    row = np.empty(512)
    row[0::2] = [code_value(v & 15) for v in b]
    row[1::2] = [code_value(v >> 4) for v in b]
    x = np.stack([row * 2.0 ** (r % 7 - 3) for r in range(rows)])
    return x.astype(BF16 if dtype == "bf16" else np.float32)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("oas", [False, True])
def test_double_quantize_decodes_every_byte(dtype, oas):
    x = byte_tensor(64, dtype)
    got = m.double_quantize(to_dev(x), seed=9, oas=oas)
    want = O.double_quantize(x, 9, oas=oas)
    rc = to_np(got[0])
    assert np.array_equal(np.unique(rc), np.arange(256)), "row codes miss some bytes"
    assert np.array_equal(rc[0], np.arange(256, dtype=np.uint8))
    for g_, w, name in zip(got, want, ("row codes", "row scales", "col codes", "col scales")):
        assert_bits_equal(to_np(g_), w, "double quantization " + name)
