"""MXFP4 GEMM on the block-scaled tensor cores (mxfp4_gemm) against the
oracle's fp64 product of the dequantized operands.

Bound: every product of two dequantized values is exact in fp32 (two E2M1
magnitudes times powers of two), so the only error is fp32 accumulation; for
a sum of k terms in any order it is at most (k - 1) u sum_j |a_j b_j| with
u = 2^-24 (recursive summation bound). Where every partial sum is a
multiple of 2^-2 below 2^22, no addition rounds and the result is exact.
"""
import numpy as np
import pytest
import torch

import mxfp4_block_quantization_quantizer_b200 as m
import oracle as O
from mxfp4_block_quantization_quantizer_b200 import workloads as W
from gpu_util import to_dev, to_np

pytestmark = pytest.mark.gpu


def gpu_gemm(ca, sa, cb, sb, k):
    return to_np(m.gemm(to_dev(ca), m.scales_to_blocked(to_dev(sa)),
                        to_dev(cb), m.scales_to_blocked(to_dev(sb)), k))


def assert_within_accumulation_bound(got, ca, sa, cb, sb, k):
    want = O.gemm(ca, sa, cb, sb, k)
    rows_a = O.dequantize(ca, sa, ca.shape[0], k, O.ROWS, "f32").astype(np.float64)
    rows_b = O.dequantize(cb, sb, cb.shape[0], k, O.ROWS, "f32").astype(np.float64)
    bound = (k - 1) * 2.0 ** -24 * (np.abs(rows_a) @ np.abs(rows_b).T)
    err = np.abs(got.astype(np.float64) - want)
    assert np.all(err <= bound), "max error / bound %g" % (err / np.maximum(bound, 1e-300)).max()


def test_gemm_exact_with_unit_scales():
    g = np.random.Generator(np.random.PCG64(1))
    ca = g.integers(0, 256, size=(128, 128), dtype=np.uint8)   # every code
    cb = g.integers(0, 256, size=(256, 128), dtype=np.uint8)
    s = np.full((256, 8), 127, np.uint8)
    got = gpu_gemm(ca, s[:128], cb, s, 256)
    assert np.array_equal(got, O.gemm(ca, s[:128], cb, s, 256).astype(np.float32))


def test_gemm_single_scale_moves_single_row_and_group():
    ones = np.full((128, 128), 0x22, np.uint8)  # every value 1.0
    sa = np.full((128, 8), 127, np.uint8)
    sb = sa.copy()
    for r, gi, b in [(0, 0, 128), (33, 1, 129), (64, 5, 126), (127, 7, 130)]:
        sa[r, gi] = b
    got = gpu_gemm(ones, sa, ones, sb, 256)
    assert np.array_equal(got, O.gemm(ones, sa, ones, sb, 256).astype(np.float32))
    sb[90, 3] = 131
    got = gpu_gemm(ones, sa, ones, sb, 256)
    assert np.array_equal(got, O.gemm(ones, sa, ones, sb, 256).astype(np.float32))


@pytest.mark.parametrize("mnk", [(128, 128, 256), (200, 136, 96), (64, 40, 32),
                                 (384, 256, 1024), (130, 520, 800),
                                 # the persistent TMA kernel (k % 256 == 0) on
                                 # partial tiles: clipped TMA stores, a missing
                                 # second B scale tile, direct stores (n % 4)
                                 (200, 136, 512), (130, 130, 768), (64, 8, 256),
                                 (1000, 600, 2048), (300, 1030, 256)])
def test_gemm_quantized_operands(mnk):
    M, N, K = mnk
    x = W.normal_bf16(M, K, M + 1, 0.01, 20.0)
    y = W.normal_bf16(N, K, N + 2)
    ca, sa = O.quantize(x, O.ROWS, O.RNE)
    cb, sb = O.quantize(y, O.ROWS, O.SR, 5)
    assert_within_accumulation_bound(gpu_gemm(ca, sa, cb, sb, K), ca, sa, cb, sb, K)


def test_gemm_random_scales_wide_range():
    g = np.random.Generator(np.random.PCG64(2))
    ca = g.integers(0, 256, size=(256, 512), dtype=np.uint8)
    cb = g.integers(0, 256, size=(128, 512), dtype=np.uint8)
    sa = g.integers(100, 150, size=(256, 32), dtype=np.uint8)
    sb = g.integers(100, 150, size=(128, 32), dtype=np.uint8)
    assert_within_accumulation_bound(gpu_gemm(ca, sa, cb, sb, 1024), ca, sa, cb, sb, 1024)


def test_gemm_on_quantizer_outputs_forward_and_backward():
    """Forward Y = Q_D(X) Q_D(W)^T from ROWS quantizations; backward
    dW = Q(dY)^T Q(X) from the column output of the double quantizer and a
    COLS quantization, all produced by the CUDA path and consumed as is."""
    X = W.normal_bf16(256, 384, 30)
    Wt = W.normal_bf16(160, 384, 31)
    dY = W.normal_bf16(256, 160, 32)
    xd, wd, gd = to_dev(X), to_dev(Wt), to_dev(dY)
    xc, xs = m.quantize(xd, m.ROWS, m.RNE)
    wc, ws = m.quantize(wd, m.ROWS, m.RNE)
    y = to_np(m.gemm(xc, m.scales_to_blocked(xs), wc, m.scales_to_blocked(ws), 384))
    assert_within_accumulation_bound(y, to_np(xc), to_np(xs), to_np(wc), to_np(ws), 384)
    _, _, xcc, xcs = m.double_quantize(xd, seed=3)       # X^T: [384, 256/2]
    gcc, gcs = m.quantize(gd, m.COLS, m.SR, seed=4)       # dY^T: [160, 256/2]
    dw = to_np(m.gemm(gcc, m.scales_to_blocked(gcs), xcc, m.scales_to_blocked(xcs), 256))
    assert_within_accumulation_bound(dw, to_np(gcc), to_np(gcs), to_np(xcc), to_np(xcs), 256)


def test_gemm_large_sampled_rows():
    """4096 x 4096 x 4096 from quantized normal data: every row band of 128
    checked at 8 sampled rows against the oracle (one launch)."""
    M = N = K = 4096
    x = W.normal_bf16(M, K, 40)
    y = W.normal_bf16(N, K, 41)
    xc, xs = m.quantize(to_dev(x), m.ROWS, m.RNE)
    yc, ys = m.quantize(to_dev(y), m.ROWS, m.RNE)
    c = to_np(m.gemm(xc, m.scales_to_blocked(xs), yc, m.scales_to_blocked(ys), K))
    g = np.random.Generator(np.random.PCG64(42))
    rows = np.sort(np.concatenate([b * 128 + g.choice(128, 8, replace=False)
                                   for b in range(M // 128)]))
    ca, sa, cb, sb = to_np(xc)[rows], to_np(xs)[rows], to_np(yc), to_np(ys)
    assert_within_accumulation_bound(c[rows], ca, sa, cb, sb, K)
