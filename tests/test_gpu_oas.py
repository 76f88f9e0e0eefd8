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


# ---------------------------------------------------------------------------
# The overflow-aware scale in the double quantizer and the rotation
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [(32, 32), (160, 96), (288, 416), (1024, 160)])
def test_double_quant_oas_matches_oracle(shape, dtype):
    x = rand_tensor(shape, dtype, sum(shape) + 5, spread=12)
    got = m.double_quantize(to_dev(x), seed=6, oas=True)
    want = O.double_quantize(x, 6, oas=True)
    for g, w, name in zip(got, want, ("row codes", "row scales", "col codes",
                                      "col scales")):
        assert_bits_equal(to_np(g), w, "oas double " + name)
    # the overflow-aware rule moved some row scales
    assert np.any(to_np(got[1]) != O.double_quantize(x, 6)[1])


def test_double_quant_oas_edges():
    x = np.concatenate([edge_tensor("bf16")] * 4)[:32]
    x = np.ascontiguousarray(np.concatenate([x, x[::-1]], axis=1))  # 32 x 64
    got = m.double_quantize(to_dev(x), seed=4, oas=True)
    for g, w in zip(got, O.double_quantize(x, 4, oas=True)):
        assert_bits_equal(to_np(g), w, "oas double quant edges")


def test_double_quant_oas_sweep_band():
    x = W.sweep()
    got = m.double_quantize(to_dev(x), seed=5, oas=True)
    want = O.double_quantize(x[:32], 5, oas=True)
    assert_bits_equal(to_np(got[0][:32]), want[0], "oas sweep row codes")
    assert_bits_equal(to_np(got[1][:32]), want[1], "oas sweep row scales")
    assert_bits_equal(to_np(got[2][:, :16]), want[2], "oas sweep col codes")
    assert_bits_equal(to_np(got[3][:, :1]), want[3], "oas sweep col scales")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rnd", [O.RNE, O.SR])
@pytest.mark.parametrize("shape", [(33, 96), (128, 320), (200, 4096)])
def test_rht_oas(shape, rnd, dtype):
    """The codes and scales are the overflow-aware quantization of the
    device's rotated values (the rotation itself is checked against the
    oracle's in test_gpu_parity), equal with and without the rotated output,
    and the rule moves some scales."""
    g = np.random.Generator(np.random.PCG64(shape[0] * 7 + shape[1]))
    x = (g.standard_t(3, size=shape) * 0.02).astype(np.float32)
    if dtype == "bf16":
        x = x.astype(BF16)
    codes, scales, rot = m.rht_quantize(to_dev(x), 2, rnd, 2, want_rotated=True, oas=True)
    r = to_np(rot)
    qc, qs = O.quantize(r, O.ROWS, rnd, 2, oas=True)
    assert_bits_equal(to_np(codes), qc, "oas rotated codes")
    assert_bits_equal(to_np(scales), qs, "oas rotated scales")
    c2, s2, _ = m.rht_quantize(to_dev(x), 2, rnd, 2, oas=True)
    assert_bits_equal(to_np(c2), to_np(codes), "oas codes without the rotated output")
    assert_bits_equal(to_np(s2), to_np(scales), "oas scales without the rotated output")
    _, s_ocp, _ = m.rht_quantize(to_dev(x), 2, rnd, 2)
    assert np.any(to_np(s_ocp) != to_np(scales))
