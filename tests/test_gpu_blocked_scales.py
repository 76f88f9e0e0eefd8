"""Blocked scale order for block-scaled GEMMs (mxfp4_scales_to_blocked)
against the oracle, bit for bit: aligned and unaligned scale pointers,
ragged row and group counts, the scales of every quantizer output, and the
full-size scales of the 8192x28672 sweep."""
import numpy as np
import pytest
import torch

import mxfp4_block_quantization_quantizer_b200 as m
import oracle as O
from mxfp4_block_quantization_quantizer_b200 import workloads as W
from gpu_util import assert_bits_equal, to_dev, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", [(1, 1), (1, 4), (127, 3), (128, 4), (130, 5),
                                   (300, 13), (256, 896), (4096, 7)])
def test_blocked_matches_oracle(shape):
    g = np.random.Generator(np.random.PCG64(shape[0] * 31 + shape[1]))
    s = g.integers(0, 256, size=shape, dtype=np.uint8)
    got = m.scales_to_blocked(to_dev(s))
    assert tuple(got.shape) == O.scales_to_blocked(s).shape
    assert_bits_equal(to_np(got), O.scales_to_blocked(s), "blocked %s" % (shape,))


def test_blocked_from_unaligned_scales():
    # a scale array starting 1 byte into its allocation: the byte-wise path
    g = np.random.Generator(np.random.PCG64(7))
    s = g.integers(0, 256, size=(260, 12), dtype=np.uint8)
    buf = torch.zeros(260 * 12 + 16, dtype=torch.uint8, device="cuda")
    view = buf[1:1 + 260 * 12].view(260, 12)
    view.copy_(to_dev(s))
    assert view.data_ptr() % 4 == 1
    assert_bits_equal(to_np(m.scales_to_blocked(view)), O.scales_to_blocked(s),
                      "blocked from unaligned scales")


def test_blocked_scales_of_every_quantizer_output():
    x = W.normal_bf16(384, 224, 21, 0.01, 30.0)
    xd = to_dev(x)
    _, rs = m.quantize(xd, m.ROWS, m.RNE)
    _, cs = m.quantize(xd, m.COLS, m.SR, seed=3)
    _, drs, _, dcs = m.double_quantize(xd, seed=4)
    for s in (rs, cs, drs, dcs):
        assert_bits_equal(to_np(m.scales_to_blocked(s)),
                          O.scales_to_blocked(to_np(s)), "blocked quantizer scales")


def test_blocked_sweep_scales_full_size():
    x = to_dev(W.sweep())
    _, s = m.quantize(x, m.ROWS, m.RNE)
    assert_bits_equal(to_np(m.scales_to_blocked(s)), O.scales_to_blocked(to_np(s)),
                      "sweep blocked scales")
