"""mxfp4_quantize_oas (overflow-aware scale: the smallest e with
absmax 2^-e <= 6) against the oracle, bit for bit: both axes, both roundings,
bf16 and fp32, ragged shapes, groups whose maximum sits exactly on, just
above and just below 6 * 2^k, non-finite, zero and subnormal groups, and a
band of the 8192x28672 sweep."""
import numpy as np
import pytest

import mxfp4_block_quantization_quantizer_b200 as m
import oracle as O
from mxfp4_block_quantization_quantizer_b200 import workloads as W
from gpu_util import BF16, assert_bits_equal, to_dev, to_np
from test_gpu_parity import edge_tensor, rand_tensor

pytestmark = pytest.mark.gpu


def check_oas(x, axis, rnd, seed):
    c, s = m.quantize(to_dev(x), axis, rnd, seed, oas=True)
    oc, os_ = O.quantize(x, axis, rnd, seed, oas=True)
    assert_bits_equal(to_np(c), oc, "oas codes")
    assert_bits_equal(to_np(s), os_, "oas scales")
    return to_np(s)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rnd", [O.RNE, O.SR])
@pytest.mark.parametrize("axis", [O.ROWS, O.COLS])
@pytest.mark.parametrize("shape", [(32, 32), (160, 96), (288, 416), (96, 1000)])
def test_oas_matches_oracle(shape, axis, rnd, dtype):
    if axis == O.ROWS and shape[1] % 32:
        shape = (shape[0], 992)
    x = rand_tensor(shape, dtype, sum(shape) + axis, spread=20)
    s = check_oas(x, axis, rnd, 9)
    _, s_ocp = O.quantize(x, axis, rnd, 9)
    diff = s.astype(int) - s_ocp.astype(int)
    assert set(np.unique(diff)) <= {0, 1} and diff.any()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rnd", [O.RNE, O.SR])
def test_oas_boundary_and_edge_groups(dtype, rnd):
    rows = []
    for k in (-120, -3, 0, 7, 100):
        for f in (6.0, 6.0 * (1 + 2.0 ** -7), 6.0 * (1 - 2.0 ** -8), 7.99, 4.0, 5.0):
            r = np.linspace(-1.0, 1.0, 32) * f * 2.0 ** k
            rows.append(r)
    x = np.concatenate([np.stack(rows).astype(np.float32),
                        edge_tensor(dtype).astype(np.float32)])
    x = x.astype(BF16) if dtype == "bf16" else x
    for axis in (O.ROWS, O.COLS):
        xx = x if axis == O.ROWS else np.ascontiguousarray(
            np.concatenate([x, x[:32 - len(x) % 32]]).T)
        check_oas(xx, axis, rnd, 3)


def test_oas_sweep_band():
    x = W.sweep()
    xd = to_dev(x)
    for axis, rnd in ((O.ROWS, O.RNE), (O.COLS, O.SR)):
        c, s = m.quantize(xd, axis, rnd, 5, oas=True)
        c, s = to_np(c), to_np(s)
        r0 = 4096
        oc, os_ = O.quantize(x[r0:r0 + 32], axis, rnd, 5, row0=r0, oas=True)
        if axis == O.ROWS:
            assert_bits_equal(c[r0:r0 + 32], oc, "sweep oas rows codes")
            assert_bits_equal(s[r0:r0 + 32], os_, "sweep oas rows scales")
        else:
            assert_bits_equal(c[:, r0 // 2:r0 // 2 + 16], oc, "sweep oas cols codes")
            assert_bits_equal(s[:, r0 // 32:r0 // 32 + 1], os_, "sweep oas cols scales")
