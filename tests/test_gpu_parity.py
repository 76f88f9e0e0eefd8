"""GPU parity: the CUDA path through the C ABI against the CPU oracle, element
by element, on seeded inputs small enough for the oracle to finish in
seconds but spanning several tiles with ragged tails; plus every edge case
(zero, subnormal, NaN/Inf, saturating and maximal groups), an exhaustive
encode table and output guard bands. Bit-exact for codes, scales, decoded
values and tracker state; the rotation within 1e-6 of the group's scale.
"""
import math

import numpy as np
import pytest
import torch

import mxfp4_block_quantization_quantizer_b200 as m
from mxfp4_block_quantization_quantizer_b200 import workloads as W
import oracle as O
from golden_io import hand_groups, unpack_nibbles
from gpu_util import (BF16, assert_bits_equal, assert_f32_equal_or_both_nan,
                      to_dev, to_np)

pytestmark = pytest.mark.gpu

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def rand_tensor(shape, dtype, seed, spread=8):
    g = np.random.Generator(np.random.PCG64(seed))
    x = g.standard_normal(shape) * np.exp2(g.integers(-spread, spread, size=shape))
    x = x.astype(np.float32)
    return x.astype(BF16) if dtype == "bf16" else x


def check_quantize(x, axis, rnd, seed):
    c, s = m.quantize(to_dev(x), axis, rnd, seed)
    oc, os_ = O.quantize(x, axis, rnd, seed)
    assert_bits_equal(to_np(c), oc, "codes")
    assert_bits_equal(to_np(s), os_, "scales")
    return c, s, oc, os_


# ---------------------------------------------------------------------------
# Exhaustive encode table: every finite bf16 under every reachable scale
# ---------------------------------------------------------------------------

def exhaustive_groups():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        v = bits.view(BF16).astype(np.float64)
    v = v[np.isfinite(v)]
    groups = []
    for e in range(-127, 126):
        A = math.ldexp(7.96875, e)
        xs = v[np.abs(v) <= A]
        xs = np.concatenate([xs, np.zeros((-len(xs)) % 31)]).reshape(-1, 31)
        groups.append(np.concatenate([np.full((len(xs), 1), A), xs], axis=1))
    return np.concatenate(groups).astype(np.float32).astype(BF16)


@pytest.mark.parametrize("rnd", [O.RNE, O.SR])
def test_exhaustive_encode_rows(rnd):
    x = exhaustive_groups()
    check_quantize(x, O.ROWS, rnd, 11)


def test_exhaustive_encode_cols_and_fp32():
    x = exhaustive_groups()
    xt = np.ascontiguousarray(x[:20000].T)  # 32 x 20000: one group per column
    check_quantize(xt, O.COLS, O.RNE, 0)
    check_quantize(xt, O.COLS, O.SR, 5)
    check_quantize(x[:20000].astype(np.float32), O.ROWS, O.RNE, 0)


def test_hand_worked_groups_on_gpu():
    for name, x, sb, codes in hand_groups():
        for dt in ("bf16", "f32"):
            xx = x.reshape(1, 32) if dt == "bf16" else x.astype(np.float32).reshape(1, 32)
            c, s = m.quantize(to_dev(xx), m.ROWS, m.RNE)
            assert to_np(s)[0, 0] == sb, (name, dt)
            assert np.array_equal(unpack_nibbles(to_np(c))[0], codes), (name, dt)
            c, s = m.quantize(to_dev(np.ascontiguousarray(xx.T)), m.COLS, m.RNE)
            assert to_np(s)[0, 0] == sb, (name, dt, "cols")
            assert np.array_equal(unpack_nibbles(to_np(c))[0], codes), (name, dt)


# ---------------------------------------------------------------------------
# Rows / columns on ragged shapes
# ---------------------------------------------------------------------------

ROW_SHAPES = [(1, 32), (3, 64), (96, 160), (257, 512), (1000, 96), (37, 4096)]
COL_SHAPES = [(32, 1), (64, 3), (32, 8), (96, 130), (160, 96), (288, 200),
              (512, 257), (64, 1030)]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rnd", [O.RNE, O.SR])
@pytest.mark.parametrize("shape", ROW_SHAPES)
def test_rows(shape, rnd, dtype):
    check_quantize(rand_tensor(shape, dtype, shape[0] * 7 + shape[1]), O.ROWS,
                   rnd, 1234)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rnd", [O.RNE, O.SR])
@pytest.mark.parametrize("shape", COL_SHAPES)
def test_cols(shape, rnd, dtype):
    check_quantize(rand_tensor(shape, dtype, shape[0] * 5 + shape[1]), O.COLS,
                   rnd, 99)


def test_seed_changes_sr_codes():
    x = to_dev(rand_tensor((64, 256), "bf16", 3))
    a, _ = m.quantize(x, m.ROWS, m.SR, 1)
    b, _ = m.quantize(x, m.ROWS, m.SR, 2)
    assert not torch.equal(a, b)


# ---------------------------------------------------------------------------
# Edge cases: zero, subnormal, NaN / Inf, saturation, extremes
# ---------------------------------------------------------------------------

def edge_tensor(dtype):
    rows = []
    z = np.zeros(32)
    rows.append(z)                                   # all zero
    r = z.copy(); r[[3, 9]] = -0.0; rows.append(r)   # negative zeros
    rows.append(np.full(32, 2.0 ** -133) * np.arange(32))  # subnormal bf16
    rows.append(np.linspace(-2.0 ** -126, 2.0 ** -126, 32))  # around min normal
    r = np.linspace(-7.9, 7.9, 32); rows.append(r)   # saturating grid scale
    r = np.full(32, 1.0); r[5] = np.nan; rows.append(r)
    r = np.full(32, 1.0); r[0] = np.inf; rows.append(r)
    r = np.full(32, 1.0); r[31] = -np.inf; rows.append(r)
    big = float(np.finfo(np.float32).max) if dtype == "f32" else float(
        np.array(3.3895313892515355e38, np.float32).astype(BF16))
    r = np.linspace(-big, big, 32); rows.append(r)   # largest finite values
    r = GRID[np.arange(32) % 8] * (-1.0) ** np.arange(32) * 2.0 ** 100
    rows.append(r)                                   # exact grid values
    x = np.stack(rows).astype(np.float32)
    if dtype == "bf16":
        return x.astype(BF16)
    x[2] = np.float32(1e-45) * np.arange(32)          # fp32 subnormals
    return x


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rnd", [O.RNE, O.SR])
def test_edge_groups(dtype, rnd):
    x = edge_tensor(dtype)
    c, s, oc, os_ = check_quantize(x, O.ROWS, rnd, 5)
    assert to_np(s)[5, 0] == 0xFF and to_np(s)[6, 0] == 0xFF
    check_quantize(np.ascontiguousarray(x.T), O.COLS, rnd, 5)
    for out_dtype, od in ((torch.bfloat16, "bf16"), (torch.float32, "f32")):
        y = m.dequantize(c, s, *x.shape, m.ROWS, out_dtype=out_dtype)
        want = O.dequantize(oc, os_, *x.shape, O.ROWS, out_dtype=od)
        assert_bits_equal(to_np(y), want, "edge dequantize " + od)


# ---------------------------------------------------------------------------
# Column stochastic rounding at extreme scales: scale bytes 2 .. 252 round
# the unscaled value (the power of two folded into the rounding), bytes 0
# and 1 scale first; both must give the oracle's codes.
# ---------------------------------------------------------------------------

EXTREME_PEAKS = [(1.5 * 2.0 ** -124, 1), (1.5 * 2.0 ** -123, 2), (1.5 * 2.0 ** -122, 3),
                 (1.5 * 2.0 ** -121, 4), (7.875 * 2.0 ** 125, 252)]


def extreme_scale_columns(dtype, seed, rows=128, per_band=64):
    """rows x (5 * per_band): one band of columns per peak of EXTREME_PEAKS,
    each 32x1 group uniform in [-peak, peak] with its peak present, plus
    subnormal, tiny and signed-zero entries."""
    g = np.random.Generator(np.random.PCG64(seed))
    bands = []
    for peak, _ in EXTREME_PEAKS:
        b = g.uniform(-1.0, 1.0, (rows, per_band)) * peak
        b[g.integers(0, 32, per_band) + 32 * g.integers(0, rows // 32, per_band),
          np.arange(per_band)] = peak * np.where(np.arange(per_band) % 2, 1.0, -1.0)
        tiny = [2.0 ** -133, -2.0 ** -140, 2.0 ** -126, -0.0, 0.0] + (
            [2.0 ** -149, -2.0 ** -145] if dtype == "f32" else [])
        for k, t in enumerate(tiny):
            b[(7 * k + 3) % rows, (5 * k + 1) % per_band :: 3] = t
        bands.append(b)
    x = np.concatenate(bands, axis=1).astype(np.float32)
    # the band peaks survive the rounding to bf16 (all are bf16 values)
    return x.astype(BF16) if dtype == "bf16" else x


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("oas", [False, True])
def test_column_sr_extreme_scales(dtype, oas):
    x = extreme_scale_columns(dtype, 11)
    c, s = m.quantize(to_dev(x), m.COLS, m.SR, 6, oas=oas)
    oc, os_ = O.quantize(x, O.COLS, O.SR, 6, oas=oas)
    if not oas:  # every band sits at its intended scale byte
        for i, (_, sb) in enumerate(EXTREME_PEAKS):
            assert (os_[64 * i:64 * (i + 1)] == sb).all()
    assert_bits_equal(to_np(c), oc, "extreme-scale column codes")
    assert_bits_equal(to_np(s), os_, "extreme-scale column scales")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rnd", [O.RNE, O.SR])
@pytest.mark.parametrize("oas", [False, True])
def test_row_quant_extreme_scales(dtype, rnd, oas):
    # the same groups along rows: the row kernel folds the scale into
    # stochastic rounding for bytes 2..252 and multiplies otherwise
    x = np.ascontiguousarray(extreme_scale_columns(dtype, 14).T)
    c, s = m.quantize(to_dev(x), m.ROWS, rnd, 8, oas=oas)
    oc, os_ = O.quantize(x, O.ROWS, rnd, 8, oas=oas)
    if not oas:
        for i, (_, sb) in enumerate(EXTREME_PEAKS):
            assert (os_[64 * i:64 * (i + 1)] == sb).all()
    assert_bits_equal(to_np(c), oc, "extreme-scale row codes")
    assert_bits_equal(to_np(s), os_, "extreme-scale row scales")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("oas", [False, True])
def test_double_quant_extreme_scales(oas, dtype):
    # overflow-aware row scales reach 2^126 here, where Q_D(X) holds 4 2^126
    # and 6 2^126: above the largest fp32 value, exact in the oracle
    x = extreme_scale_columns(dtype, 12)
    got = m.double_quantize(to_dev(x), seed=7, oas=oas)
    want = O.double_quantize(x, 7, oas=oas)
    assert set(np.unique(want[3])) >= {1, 2, 3}
    for g_, w, name in zip(got, want, ("row codes", "row scales", "col codes", "col scales")):
        assert_bits_equal(to_np(g_), w, "extreme-scale double quant " + name)


@pytest.mark.parametrize("oas", [False, True])
def test_column_kernels_multi_tile_ragged(oas):
    """2080 x 4000: 17 x 32 tiles of 128 x 128 with a ragged last row and
    column tile, more tiles than resident blocks (each block walks several,
    interior tiles on the unchecked staging path), compared in full."""
    x = rand_tensor((2080, 4000), "bf16", 21, spread=12)
    c, s = m.quantize(to_dev(x), m.COLS, m.SR, 13, oas=oas)
    oc, os_ = O.quantize(x, O.COLS, O.SR, 13, oas=oas)
    assert_bits_equal(to_np(c), oc, "multi-tile column codes")
    assert_bits_equal(to_np(s), os_, "multi-tile column scales")
    got = m.double_quantize(to_dev(x), seed=13, oas=oas)
    want = O.double_quantize(x, 13, oas=oas)
    for g_, w, name in zip(got, want, ("row codes", "row scales", "col codes", "col scales")):
        assert_bits_equal(to_np(g_), w, "multi-tile double quant " + name)


# ---------------------------------------------------------------------------
# Dequantize
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("axis", [O.ROWS, O.COLS])
@pytest.mark.parametrize("od", ["bf16", "f32"])
def test_dequantize(axis, od):
    x = rand_tensor((160, 96), "bf16", 8, spread=60)
    x[3, 40] = np.nan
    oc, os_ = O.quantize(x, axis, O.SR, 3)
    y = m.dequantize(to_dev(oc), to_dev(os_), 160, 96, axis,
                     out_dtype=torch.bfloat16 if od == "bf16" else torch.float32)
    assert_bits_equal(to_np(y), O.dequantize(oc, os_, 160, 96, axis, od),
                      "dequantize")


def test_dequantize_every_code_and_scale():
    # codes 0..15 under every scale byte 0..255
    R = 256
    codes = np.tile(np.array([0x10 * (2 * k + 1 & 15) + (2 * k & 15)
                              for k in range(16)], np.uint8), (R, 1))
    scales = np.arange(256, dtype=np.uint8).reshape(R, 1)
    y = m.dequantize(to_dev(codes), to_dev(scales), R, 32, m.ROWS,
                     out_dtype=torch.float32)
    assert_bits_equal(to_np(y), O.dequantize(codes, scales, R, 32, O.ROWS, "f32"),
                      "every code and scale f32")
    y = m.dequantize(to_dev(codes), to_dev(scales), R, 32, m.ROWS)
    assert_bits_equal(to_np(y), O.dequantize(codes, scales, R, 32, O.ROWS),
                      "every code and scale bf16")


# ---------------------------------------------------------------------------
# Double quantization
# ---------------------------------------------------------------------------

DQ_SHAPES = [(32, 32), (64, 96), (160, 96), (128, 128), (288, 416), (1024, 160)]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", DQ_SHAPES)
def test_double_quant(shape, dtype):
    x = rand_tensor(shape, dtype, sum(shape), spread=12)
    got = m.double_quantize(to_dev(x), seed=1)
    want = O.double_quantize(x, 1)
    for g, w, name in zip(got, want, ("row codes", "row scales", "col codes",
                                      "col scales")):
        assert_bits_equal(to_np(g), w, name)


def test_double_quant_edges():
    x = np.concatenate([edge_tensor("bf16")] * 4)[:32]
    x = np.ascontiguousarray(np.concatenate([x, x[::-1]], axis=1))  # 32 x 64
    got = m.double_quantize(to_dev(x), seed=4)
    for g, w in zip(got, O.double_quantize(x, 4)):
        assert_bits_equal(to_np(g), w, "double quant edges")


# ---------------------------------------------------------------------------
# Randomized Hadamard rotation + quantize
# ---------------------------------------------------------------------------

def check_rht(x, sign_seed, rnd, sr_seed, codes, scales, rot, row0=0):
    """rot within tolerance of the oracle's fp64 rotation; codes bit-exact
    as the quantization of rot; differences from the oracle's own codes only
    where its value lies within the tolerance of a decision boundary."""
    y_ref = O.rht_rotate(x, sign_seed).astype(np.float64)
    xg = x.astype(np.float64).reshape(-1, 32)
    rms = np.repeat(np.linalg.norm(xg, axis=1) / math.sqrt(32), 32).reshape(y_ref.shape)
    tol = 1e-6 * np.maximum(np.abs(y_ref), rms)
    err = np.abs(rot.astype(np.float64) - y_ref)
    assert np.all(err <= tol), "rotation error %g > tol" % (err / np.maximum(tol, 1e-300)).max()
    # the strict per-element relative error, where the group's signed sum
    # does not cancel (condition number sum|x| / (sqrt(32) |y|) <= 2) and y
    # is far from the subnormals: within 1e-6 of y itself
    cond = np.repeat(np.abs(xg).sum(axis=1) / math.sqrt(32), 32).reshape(y_ref.shape)
    ay = np.abs(y_ref)
    sel = (ay >= 2.0 ** -102) & (cond <= 2.0 * ay)
    if sel.any():
        strict = (err[sel] / ay[sel]).max()
        assert strict <= 1e-6, "strict relative rotation error %g" % strict
    qc, qs = O.quantize(rot, O.ROWS, rnd, sr_seed, row0)
    assert_bits_equal(codes, qc, "codes of the rotated values")
    assert_bits_equal(scales, qs, "scales of the rotated values")
    rc, rs, _ = O.rht_quantize(x, sign_seed, rnd, sr_seed, row0)
    # scales may differ only where the oracle's absmax sits on a power of two
    amax = np.abs(y_ref).reshape(-1, 32).max(axis=1)
    gtol = tol.reshape(-1, 32).max(axis=1)
    sdiff = rs.reshape(-1) != scales.reshape(-1)
    near_pow2 = np.abs(amax - np.exp2(np.round(np.log2(np.maximum(amax, 1e-300))))) <= gtol
    assert np.all(near_pow2[sdiff])
    cg, cr = unpack_nibbles(codes).reshape(-1, 32), unpack_nibbles(rc).reshape(-1, 32)
    bad = np.argwhere((cg != cr) & ~sdiff[:, None])
    R, C = x.shape
    for gi, j in bad:
        e = int(rs.reshape(-1)[gi]) - 127
        yv = y_ref.reshape(-1, 32)[gi, j]
        t = tol.reshape(-1, 32)[gi, j]
        a = abs(yv) * 2.0 ** -e
        if rnd == O.RNE:
            bounds = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
        else:
            i = (row0 + gi // (C // 32)) * C + (gi % (C // 32)) * 32 + j
            r = O.rand16(sr_seed, 0, i)
            lo = GRID[GRID <= a].max()
            hi = GRID[min(np.searchsorted(GRID, lo) + 1, 7)]
            bounds = np.array([lo + (r + 0.5) / 65536 * (hi - lo), lo, hi])
        assert np.min(np.abs(a - bounds)) * 2.0 ** e <= t, (gi, j, a)
    return len(bad)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rnd", [O.RNE, O.SR])
@pytest.mark.parametrize("shape", [(1, 32), (33, 96), (64, 320), (100, 4096)])
def test_rht(shape, rnd, dtype):
    g = np.random.Generator(np.random.PCG64(shape[0] + shape[1]))
    x = (g.standard_t(3, size=shape) * 0.02).astype(np.float32)
    if dtype == "bf16":
        x = x.astype(BF16)
    codes, scales, rot = m.rht_quantize(to_dev(x), 2, rnd, 2, want_rotated=True)
    check_rht(x, 2, rnd, 2, to_np(codes), to_np(scales), to_np(rot))
    c2, s2, none = m.rht_quantize(to_dev(x), 2, rnd, 2, want_rotated=False)
    assert none is None
    assert torch.equal(c2, codes) and torch.equal(s2, scales)


def test_rht_outlier_spreads_and_edges():
    x = np.zeros((4, 64), np.float32)
    x[0, 7] = 100.0                  # one outlier
    x[1, :] = np.nan                 # non-finite group
    x[2, 33] = np.inf
    x = x.astype(BF16)
    codes, scales, rot = m.rht_quantize(to_dev(x), 9, m.RNE, 0, want_rotated=True)
    r = to_np(rot)
    assert np.allclose(np.abs(r[0, :32]), 100.0 / math.sqrt(32), rtol=1e-6)
    s = to_np(scales)
    assert s[1, 0] == 0xFF and s[1, 1] == 0xFF and s[2, 1] == 0xFF
    rc, rs = O.quantize(r, O.ROWS, O.RNE, 0)
    assert_bits_equal(to_np(codes), rc, "rht edge codes")
    assert_bits_equal(s, rs, "rht edge scales")


# ---------------------------------------------------------------------------
# Oscillation tracker
# ---------------------------------------------------------------------------

def run_osc(w_np, steps, seed, threshold=4.0, rows_check=None):
    dev = "cuda"
    w = to_dev(w_np)
    ws, dw, dq = w.clone(), torch.zeros_like(w), torch.zeros_like(w)
    nflag = torch.zeros(1, dtype=torch.int64, device=dev)
    for t in range(steps):
        m.osc_synthetic_update(w, seed, t)
        m.osc_step(w, ws, dw, dq, window_end=(t == steps - 1), threshold=threshold,
                   n_flagged=nflag)
    return [to_np(a) for a in (w, ws, dw, dq)], int(nflag.item())


def run_osc_oracle(w_np, steps, seed, threshold=4.0, row0=0):
    w = w_np.copy()
    ws, dw, dq = w.copy(), np.zeros_like(w), np.zeros_like(w)
    flagged = 0
    for t in range(steps):
        O.osc_synthetic_update(w, seed, t, row0=row0)
        flagged += O.osc_step(w, ws, dw, dq, window_end=(t == steps - 1),
                              threshold=threshold)
    return [w, ws, dw, dq], flagged


@pytest.mark.parametrize("steps,threshold", [(200, 4.0), (37, 16.0), (1, 4.0)])
def test_osc_window(steps, threshold):
    w_np = W.osc_w(seed=3, rows=64, cols=512)
    got, nflag = run_osc(w_np, steps, 3, threshold)
    want, wflag = run_osc_oracle(w_np, steps, 3, threshold)
    for g, wv, name in zip(got, want, ("w", "w_snap", "d_w", "d_q")):
        assert_f32_equal_or_both_nan(g, wv, name)
    assert nflag == wflag
    if steps == 200:
        assert nflag > 0


def test_osc_crafted_crossings():
    """One step on hand-built groups: crossings of the 2.5, 0.75 and 0.25
    edges, a jump of several bins, a changed group scale and a plain 1 -> 2
    move must each add |DQ(w) - DQ(w_snap)| to d_q."""
    w = np.zeros((4, 32), np.float32)
    w[:, 0] = 0.1
    ws = w.copy()
    w[0, 1], ws[0, 1] = np.float32(-2.4998364 / 64), np.float32(-2.5000865 / 64)
    w[0, 2], ws[0, 2] = np.float32(0.75 / 64 * 1.001), np.float32(0.75 / 64 * 0.999)
    w[0, 3], ws[0, 3] = np.float32(0.25 / 64 * 1.0001), np.float32(0.25 / 64 * 0.9999)
    w[1, 1], ws[1, 1] = 1.0 / 64, 3.0 / 64
    ws[2, 0] = 0.01  # only the snapshot's group scale differs
    w[2, 5] = ws[2, 5] = 0.004
    w[3, :] = 0.0
    ws[3, :] = 0.0
    w[3, 1], ws[3, 1] = 1.0, 2.0
    dev = [to_dev(a.copy()) for a in (w, ws, np.zeros_like(w), np.zeros_like(w))]
    m.osc_step(*dev)
    ref = [w.copy(), ws.copy(), np.zeros_like(w), np.zeros_like(w)]
    O.osc_step(*ref)
    for g, r, name in zip(dev, ref, ("w", "w_snap", "d_w", "d_q")):
        assert_f32_equal_or_both_nan(to_np(g), r, name)
    assert np.count_nonzero(ref[3]) >= 6


def test_osc_mid_window_state():
    w_np = W.osc_w(seed=4, rows=32, cols=256)
    w = to_dev(w_np)
    ws, dw, dq = w.clone(), torch.zeros_like(w), torch.zeros_like(w)
    ow, ows, odw, odq = w_np.copy(), w_np.copy(), np.zeros_like(w_np), np.zeros_like(w_np)
    for t in range(50):
        m.osc_synthetic_update(w, 4, t)
        m.osc_step(w, ws, dw, dq)
        O.osc_synthetic_update(ow, 4, t)
        O.osc_step(ow, ows, odw, odq)
    for g, wv in zip((w, ws, dw, dq), (ow, ows, odw, odq)):
        assert_f32_equal_or_both_nan(to_np(g), wv, "mid-window state")
    assert np.any(odq > 0)


def qramp_deltas(w0, n, seed):
    """Seeded updates of the tracker workload: +-1e-4 |w0| with random signs,
    and a quarter of the weights alternating sign every iteration (they sit
    near a rounding edge, so these oscillate)."""
    g = np.random.Generator(np.random.PCG64(seed))
    osc = g.random(w0.shape) < 0.25
    mag = (np.float32(1e-4) * np.abs(w0)).astype(np.float32)
    out = []
    for t in range(n):
        s = np.where(osc, 1.0 if t % 2 == 0 else -1.0,
                     np.where(g.random(w0.shape) < 0.5, -1.0, 1.0))
        out.append((s * mag).astype(np.float32))
    return out


@pytest.mark.parametrize("track,k2", [(5, 3), (6, 1), (0, 4)])
def test_qramp_epochs(track, k2):
    """Three epochs of 9 iterations: every array bit for bit, and the flag
    counts, after every iteration."""
    w_np = W.osc_w(seed=5, rows=64, cols=256)
    deltas = qramp_deltas(w_np, 27, 11)
    z = np.zeros_like(w_np)
    ref = [w_np.copy(), z.copy(), z.copy(), z.copy(), z.copy(), np.zeros(w_np.shape, np.uint8)]
    dev = [to_dev(a.copy()) for a in ref]
    nflag = torch.zeros(1, dtype=torch.int64, device="cuda")
    total = 0
    for t, d in enumerate(deltas):
        it = t % 9
        dd = to_dev(d)
        m.qramp_step(dev[0], dd, dev[1], dev[2], dev[3], dev[4], dev[5], it,
                     track_iters=track, k1=16.0, k2=k2, n_flagged=nflag)
        total += O.qramp_step(ref[0], d, ref[1], ref[2], ref[3], ref[4], ref[5], it,
                              track_iters=track, k1=16.0, k2=k2)
        for g, r, name in zip(dev, ref, ("w", "w_snap", "d_w", "d_q", "acc", "flag")):
            if name == "flag":
                assert_bits_equal(to_np(g), r, "flag at %d" % t)
            else:
                assert_f32_equal_or_both_nan(to_np(g), r, "%s at %d" % (name, t))
    assert int(nflag.item()) == total
    if track:
        assert total > 0


def test_qramp_flag_count_with_a_ragged_last_block():
    """96 groups (not a multiple of a block's 64): the threads past the last
    group must not add to the flag count (they recompute group 0's flags
    without storing them). Group 0 oscillates, so it has flags to count."""
    w_np = W.osc_w(seed=6, rows=32, cols=96)
    deltas = qramp_deltas(w_np, 4, 12)
    for d in deltas:
        d[0, :32] = np.where(np.arange(32) % 2 == 0, 1.0, -1.0) * np.float32(4e-3)
    z = np.zeros_like(w_np)
    ref = [w_np.copy(), z.copy(), z.copy(), z.copy(), z.copy(), np.zeros(w_np.shape, np.uint8)]
    dev = [to_dev(a.copy()) for a in ref]
    nflag = torch.zeros(1, dtype=torch.int64, device="cuda")
    total = 0
    for it, d in enumerate(deltas):
        m.qramp_step(dev[0], to_dev(d), *dev[1:], it, track_iters=4, k1=0.5, k2=2,
                     n_flagged=nflag)
        total += O.qramp_step(ref[0], d, *ref[1:], it, track_iters=4, k1=0.5, k2=2)
    assert_bits_equal(to_np(dev[5]), ref[5], "flags")
    assert ref[5][0, :32].any()
    assert int(nflag.item()) == total == int(ref[5].sum())


def test_osc_update_alone_and_ragged_length():
    g = np.random.Generator(np.random.PCG64(2))
    w_np = g.normal(0, 0.02, size=(7, 13)).astype(np.float32)  # 91 elements
    w = to_dev(w_np)
    m.osc_synthetic_update(w, 9, 5, 1e-3)
    O.osc_synthetic_update(w_np, 9, 5, 1e-3)
    assert_bits_equal(to_np(w), w_np, "synthetic update")


# ---------------------------------------------------------------------------
# Guard bands and streams
# ---------------------------------------------------------------------------

def test_outputs_stay_inside_their_buffers():
    x_np = rand_tensor((96, 160), "bf16", 17)
    x = to_dev(x_np)
    R, C = x.shape
    pad = 4096
    canary = 0xA5

    def guarded(n):
        buf = torch.full((n + 2 * pad,), canary, dtype=torch.uint8, device="cuda")
        return buf, buf[pad:pad + n]

    for axis in (m.ROWS, m.COLS):
        cb, c = guarded(R * C // 2)
        sbuf, s = guarded(R * C // 32)
        shp_c = (R, C // 2) if axis == m.ROWS else (C, R // 2)
        shp_s = (R, C // 32) if axis == m.ROWS else (C, R // 32)
        m.quantize(x, axis, m.SR, 1, out=(c.view(shp_c), s.view(shp_s)))
        for b in (cb, sbuf):
            h = to_np(b)
            assert np.all(h[:pad] == canary) and np.all(h[-pad:] == canary)
    bufs = [guarded(R * C // 2), guarded(R * C // 32), guarded(R * C // 2),
            guarded(R * C // 32)]
    m.double_quantize(x, 1, out=(bufs[0][1].view(R, C // 2), bufs[1][1].view(R, C // 32),
                                 bufs[2][1].view(C, R // 2), bufs[3][1].view(C, R // 32)))
    for b, _ in bufs:
        h = to_np(b)
        assert np.all(h[:pad] == canary) and np.all(h[-pad:] == canary)


def test_runs_on_a_side_stream():
    x_np = rand_tensor((256, 512), "bf16", 21)
    x = to_dev(x_np)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        c, sc = m.quantize(x, m.COLS, m.SR, 8)
    s.synchronize()
    oc, os_ = O.quantize(x_np, O.COLS, O.SR, 8)
    assert_bits_equal(to_np(c), oc, "side-stream codes")


def test_c_abi_statuses_on_device_pointers():
    L = m.lib()
    x = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    c = torch.zeros(64 * 32 + 16, dtype=torch.uint8, device="cuda")
    s = torch.zeros(128, dtype=torch.uint8, device="cuda")
    import ctypes
    p = lambda t, off=0: ctypes.c_void_p(t.data_ptr() + off)  # noqa: E731
    assert L.mxfp4_quantize(p(x), 1, 64, 64, 0, 0, 0, p(c), p(s), None) == 0
    assert L.mxfp4_quantize(p(x, 2), 1, 64, 64, 0, 0, 0, p(c), p(s), None) == 3
    assert L.mxfp4_quantize(p(x), 1, 64, 64, 0, 0, 0, p(c, 4), p(s), None) == 3
    torch.cuda.synchronize()


# ---------------------------------------------------------------------------
# Q-EMA: EMA update fused with 1x32 RNE quantization
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("shape", [(1, 32), (37, 96), (256, 512)])
@pytest.mark.parametrize("beta", [0.998, 0.9, 0.0, 1.0])
def test_qema_steps(shape, beta):
    g = np.random.Generator(np.random.PCG64(shape[0] + 7))
    w_np = g.normal(0, 0.02, size=shape).astype(np.float32)
    e_np = g.normal(0, 0.02, size=shape).astype(np.float32)
    w, e = to_dev(w_np), to_dev(e_np)
    for step in range(5):
        c, s = m.qema_quantize(w, e, beta)
        oc, os_ = O.qema_quantize(w_np, e_np, beta)
        assert_bits_equal(to_np(e), e_np, "ema step %d" % step)
        assert_bits_equal(to_np(c), oc, "codes step %d" % step)
        assert_bits_equal(to_np(s), os_, "scales step %d" % step)
        w_np = (w_np * np.float32(1.01)).astype(np.float32)
        w = to_dev(w_np)


def test_qema_edge_groups():
    x = edge_tensor("f32")
    e = np.zeros_like(x)
    got_e = to_dev(e)
    c, s = m.qema_quantize(to_dev(x), got_e, 0.5)
    oc, os_ = O.qema_quantize(x, e, 0.5)
    assert_f32_equal_or_both_nan(to_np(got_e), e, "ema")
    assert_bits_equal(to_np(c), oc, "codes")
    assert_bits_equal(to_np(s), os_, "scales")


# ---------------------------------------------------------------------------
# Graph capture and concurrent streams
# ---------------------------------------------------------------------------

def test_calls_replay_from_a_cuda_graph():
    """The entry points allocate nothing and only launch kernels on the
    caller's stream, so a captured sequence replays to the same results."""
    x_np = rand_tensor((256, 512), "bf16", 41)
    x = to_dev(x_np)
    R, C = x.shape
    u8 = lambda *s: torch.empty(s, dtype=torch.uint8, device="cuda")  # noqa: E731
    rows = (u8(R, C // 2), u8(R, C // 32))
    dq = (u8(R, C // 2), u8(R, C // 32), u8(C, R // 2), u8(C, R // 32))
    y = torch.empty(R, C, dtype=torch.bfloat16, device="cuda")
    # warm up outside capture (first calls set kernel attributes)
    m.quantize(x, m.ROWS, m.SR, 3, out=rows)
    m.double_quantize(x, 4, out=dq)
    m.dequantize(rows[0], rows[1], R, C, out=y)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        m.quantize(x, m.ROWS, m.SR, 3, out=rows)
        m.double_quantize(x, 4, out=dq)
        m.dequantize(rows[0], rows[1], R, C, out=y)
    for t in rows + dq:
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    oc, os_ = O.quantize(x_np, O.ROWS, O.SR, 3)
    assert_bits_equal(to_np(rows[0]), oc, "graph row codes")
    for got, want in zip(dq, O.double_quantize(x_np, 4)):
        assert_bits_equal(to_np(got), want, "graph double quantization")
    assert_bits_equal(to_np(y), O.dequantize(oc, os_, R, C), "graph dequantize")


def test_two_streams_at_once():
    a_np = rand_tensor((512, 1024), "bf16", 42)
    b_np = rand_tensor((512, 1024), "bf16", 43)
    a, b = to_dev(a_np), to_dev(b_np)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    s1.wait_stream(torch.cuda.current_stream())
    s2.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s1):
        ra = m.double_quantize(a, seed=9)
    with torch.cuda.stream(s2):
        rb = m.double_quantize(b, seed=9)
    torch.cuda.synchronize()
    for got, want in zip(ra, O.double_quantize(a_np, 9)):
        assert_bits_equal(to_np(got), want, "stream 1")
    for got, want in zip(rb, O.double_quantize(b_np, 9)):
        assert_bits_equal(to_np(got), want, "stream 2")
