"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times. Where the oracle finishes in seconds the whole output is
compared; otherwise the oracle recomputes sampled 32-row bands (every group
and every random number is keyed by its global index, so a band is exact on
its own). Bit-exact except the rotation (1e-6 of the group scale).
"""
import numpy as np
import pytest
import torch

import mxfp4_block_quantization_quantizer_b200 as m
from mxfp4_block_quantization_quantizer_b200 import workloads as W
import oracle as O
from gpu_util import assert_bits_equal, assert_f32_equal_or_both_nan, to_dev, to_np
from test_gpu_parity import check_rht

pytestmark = pytest.mark.gpu


def test_small_256x512_quantize_dequantize():
    x = W.small(seed=0)
    xd = to_dev(x)
    c, s = m.quantize(xd, m.ROWS, m.RNE)
    oc, os_ = O.quantize(x, O.ROWS, O.RNE)
    assert_bits_equal(to_np(c), oc, "codes")
    assert_bits_equal(to_np(s), os_, "scales")
    assert to_np(s)[0, 0] == 0  # the all-zero group
    y = m.dequantize(c, s, 256, 512)
    assert_bits_equal(to_np(y), O.dequantize(oc, os_, 256, 512), "dequantized")


def test_deit_activation_double_quant_full():
    x = W.deit_act(seed=1)  # 12608 x 1536
    got = m.double_quantize(to_dev(x), seed=1)
    want = O.double_quantize(x, 1)
    for g, w, name in zip(got, want, ("row codes", "row scales", "col codes",
                                      "col scales")):
        assert_bits_equal(to_np(g), w, name)


def rht_check_rows(rows, seed):
    """Rows of the 4096x14336 weight for the boundary check: four per 128-row
    tile (one in each 32-row lane quarter the epilogue warps read, at seeded
    offsets), so every tile, and with it every CTA's run of tiles, is
    covered across the full width."""
    g = np.random.Generator(np.random.PCG64(seed))
    out = []
    for t in range(rows // 128):
        for q in range(4):
            out.append(128 * t + 32 * q + int(g.integers(0, 32)))
    return out


def test_llm_weight_rht_sr_full():
    """Every code and scale of the 4096x14336 rotation + SR equals the
    oracle's quantization of the device's rotated values (bit for bit), and
    on 128 rows spread over every tile the rotated values are within the
    tolerance of the oracle's fp64 rotation, with code differences from the
    oracle's own only at decision boundaries."""
    x = W.llm_w(seed=2)  # 4096 x 14336
    codes, scales, rot = m.rht_quantize(to_dev(x), 2, m.SR, 2, want_rotated=True)
    codes, scales, rot = to_np(codes), to_np(scales), to_np(rot)
    qc, qs = O.quantize(rot, O.ROWS, O.SR, 2)
    assert_bits_equal(codes, qc, "codes of the rotated values (all rows)")
    assert_bits_equal(scales, qs, "scales of the rotated values (all rows)")
    n_near = 0
    rows = rht_check_rows(4096, 2)
    assert len(rows) == 128
    for r in rows:
        n_near += check_rht(x[r:r + 1], 2, O.SR, 2, codes[r:r + 1],
                            scales[r:r + 1], rot[r:r + 1], row0=r)
    assert n_near <= 160  # boundary cases are rare


@pytest.mark.parametrize("rnd", [O.RNE, O.SR])
def test_llm_weight_rht_without_rotated_output(rnd):
    """The benchmark's form (no rotated output; nearest rounding stages its
    codes for whole-row stores): on the 4096x14336 weight every CTA runs
    several tiles across column blocks; the codes and scales equal those of
    the call that also writes the rotated values, which are checked against
    the oracle on sampled rows."""
    x = W.llm_w(seed=2)
    xd = to_dev(x)
    codes, scales, rot = m.rht_quantize(xd, 2, rnd, 2, want_rotated=True)
    c2, s2, none = m.rht_quantize(xd, 2, rnd, 2)
    assert none is None
    assert torch.equal(c2, codes) and torch.equal(s2, scales)
    codes, scales, rot = to_np(codes), to_np(scales), to_np(rot)
    for r in (0, 127, 128, 2048, 4095):
        check_rht(x[r:r + 1], 2, rnd, 2, codes[r:r + 1], scales[r:r + 1],
                  rot[r:r + 1], row0=r)


def test_osc_weight_200_steps_sampled_bands():
    w_np = W.osc_w(seed=3)  # 4096 x 4096
    w = to_dev(w_np)
    ws, dw, dq = w.clone(), torch.zeros_like(w), torch.zeros_like(w)
    nflag = torch.zeros(1, dtype=torch.int64, device="cuda")
    for t in range(200):
        m.osc_synthetic_update(w, 3, t)
        m.osc_step(w, ws, dw, dq, window_end=(t == 199), n_flagged=nflag)
    got = [to_np(a) for a in (w, ws, dw, dq)]
    total = int(nflag.item())
    assert total > 0
    flagged_in_bands = 0
    # first rows (the grid's first wave), last rows (its last wave) and
    # seeded bands in between
    mid = np.random.Generator(np.random.PCG64(3)).integers(1, 255, 6)
    for r0 in [0, 4080] + [16 * int(b) for b in mid]:
        band = w_np[r0:r0 + 16].copy()
        ow, ows, odw, odq = band.copy(), band.copy(), np.zeros_like(band), np.zeros_like(band)
        for t in range(200):
            O.osc_synthetic_update(ow, 3, t, row0=r0)
            flagged_in_bands += O.osc_step(ow, ows, odw, odq, window_end=(t == 199))
        for g, wv, name in zip(got, (ow, ows, odw, odq), ("w", "w_snap", "d_w", "d_q")):
            assert_f32_equal_or_both_nan(g[r0:r0 + 16], wv, name)
    # the bands' share of the flags agrees with the device count's scale
    assert flagged_in_bands > 0


def test_osc_weight_qramp_epoch_sampled_bands():
    """One 40-iteration epoch of Q-Ramping (window 30, k1 16, k2 5) on the
    4096x4096 tracker workload; first, last and seeded middle bands."""
    from test_gpu_parity import qramp_deltas
    w_np = W.osc_w(seed=3)
    bands = [0, 4080] + [16 * int(b) for b in np.random.Generator(
        np.random.PCG64(7)).integers(1, 255, 4)]
    g_d = qramp_deltas(w_np[:16], 1, 0)  # shape check of the generator
    assert g_d[0].shape == (16, 4096)
    z = np.zeros_like(w_np)
    dev = [to_dev(a) for a in (w_np, z, z, z, z)] + [
        torch.zeros(w_np.shape, dtype=torch.uint8, device="cuda")]
    nflag = torch.zeros(1, dtype=torch.int64, device="cuda")
    deltas = qramp_deltas(w_np, 40, 21)
    for it, d in enumerate(deltas):
        m.qramp_step(*dev[:1], to_dev(d), *dev[1:], it, track_iters=30, k1=16.0, k2=5,
                     n_flagged=nflag)
    got = [to_np(a) for a in dev]
    assert int(nflag.item()) > 0
    for r0 in bands:
        sl = slice(r0, r0 + 16)
        ref = [w_np[sl].copy(), np.zeros_like(w_np[sl]), np.zeros_like(w_np[sl]),
               np.zeros_like(w_np[sl]), np.zeros_like(w_np[sl]),
               np.zeros((16, 4096), np.uint8)]
        for it, d in enumerate(deltas):
            O.qramp_step(ref[0], np.ascontiguousarray(d[sl]), *ref[1:], it, track_iters=30,
                         k1=16.0, k2=5)
        for g, r, name in zip(got, ref, ("w", "w_snap", "d_w", "d_q", "acc", "flag")):
            if name == "flag":
                assert_bits_equal(g[sl], r, "flag band %d" % r0)
            else:
                assert_f32_equal_or_both_nan(g[sl], r, "%s band %d" % (name, r0))


@pytest.fixture(scope="module")
def sweep():
    x = W.sweep(seed=5)  # 8192 x 28672 bf16
    return x, to_dev(x)


# 32-row bands: the first, the last and 16 seeded ones in between (the
# column and double-quantize kernels walk 128x128 tiles persistently, so the
# bands land in different waves and tile positions of the grid)
BANDS = [0, 255] + sorted(int(b) for b in np.random.Generator(
    np.random.PCG64(5)).choice(np.arange(1, 255), 16, replace=False))


def test_sweep_rows_rne(sweep):
    x, xd = sweep
    c, s = (to_np(t) for t in m.quantize(xd, m.ROWS, m.RNE))
    for b in BANDS:
        oc, os_ = O.quantize(x[32 * b:32 * b + 32], O.ROWS, O.RNE, 0, row0=32 * b)
        assert_bits_equal(c[32 * b:32 * b + 32], oc, "row codes band %d" % b)
        assert_bits_equal(s[32 * b:32 * b + 32], os_, "row scales band %d" % b)


def test_sweep_rows_sr(sweep):
    x, xd = sweep
    c, s = (to_np(t) for t in m.quantize(xd, m.ROWS, m.SR, 5))
    for b in BANDS:
        oc, os_ = O.quantize(x[32 * b:32 * b + 32], O.ROWS, O.SR, 5, row0=32 * b)
        assert_bits_equal(c[32 * b:32 * b + 32], oc, "row codes band %d" % b)
        assert_bits_equal(s[32 * b:32 * b + 32], os_, "row scales band %d" % b)


def test_sweep_rht_sr(sweep):
    """The step's rotation on the sweep: the benchmark's form (no rotated
    output) equals the form that writes the rotated values, and those pass
    the rotation's rule on every band."""
    x, xd = sweep
    c2, s2, _ = m.rht_quantize(xd, 2, m.SR, 5)
    codes, scales, rot = m.rht_quantize(xd, 2, m.SR, 5, want_rotated=True)
    assert torch.equal(c2, codes) and torch.equal(s2, scales)
    del c2, s2
    for b in BANDS:
        sl = slice(32 * b, 32 * b + 32)
        check_rht(x[sl], 2, O.SR, 5, to_np(codes[sl]), to_np(scales[sl]), to_np(rot[sl]),
                  row0=32 * b)


def test_sweep_cols_sr(sweep):
    x, xd = sweep
    c, s = (to_np(t) for t in m.quantize(xd, m.COLS, m.SR, 5))
    for b in BANDS:
        oc, os_ = O.quantize(x[32 * b:32 * b + 32], O.COLS, O.SR, 5, row0=32 * b)
        assert_bits_equal(c[:, 16 * b:16 * b + 16], oc, "col codes band %d" % b)
        assert_bits_equal(s[:, b:b + 1], os_, "col scales band %d" % b)


def test_sweep_double_quant(sweep):
    x, xd = sweep
    rc, rs, cc, cs = (to_np(t) for t in m.double_quantize(xd, seed=5))
    for b in BANDS:
        orc, ors, occ, ocs = O.double_quantize(x[32 * b:32 * b + 32], 5, row0=32 * b)
        assert_bits_equal(rc[32 * b:32 * b + 32], orc, "row codes band %d" % b)
        assert_bits_equal(rs[32 * b:32 * b + 32], ors, "row scales band %d" % b)
        assert_bits_equal(cc[:, 16 * b:16 * b + 16], occ, "col codes band %d" % b)
        assert_bits_equal(cs[:, b:b + 1], ocs, "col scales band %d" % b)


def test_sweep_dequantize_rows(sweep):
    x, xd = sweep
    c, s = m.quantize(xd, m.ROWS, m.RNE)
    y = to_np(m.dequantize(c, s, *x.shape))
    c, s = to_np(c), to_np(s)
    for b in BANDS:
        sl = slice(32 * b, 32 * b + 32)
        want = O.dequantize(c[sl], s[sl], 32, x.shape[1])
        assert_bits_equal(y[sl], want, "dequantized band %d" % b)


def test_beyond_2_pow_33_elements():
    """2^33 + 2^21 elements: the pair counter's high word becomes 1 in the
    last band, which every random-number path must carry."""
    R, C = (1 << 18) + 64, 1 << 15
    block = W.normal_bf16(64, C, seed=6, outlier_frac=0.001, outlier_scale=100.0)
    xd = to_dev(block).repeat(R // 64, 1)
    bands = [0, (R - 64) // 32, (R - 32) // 32]  # pairs below and above 2^32
    for op in ("rows", "cols", "double", "rht"):
        if op == "rows":
            out = m.quantize(xd, m.ROWS, m.SR, 77)
        elif op == "cols":
            out = m.quantize(xd, m.COLS, m.SR, 77)
        elif op == "double":
            out = m.double_quantize(xd, seed=77)
        else:
            out = m.rht_quantize(xd, 3, m.SR, 77, want_rotated=True)
        for b in bands:
            r0 = 32 * b
            xb = block[r0 % 64:r0 % 64 + 32]
            rows_ = slice(r0, r0 + 32)
            if op == "rows":
                want = O.quantize(xb, O.ROWS, O.SR, 77, row0=r0)
                got = (out[0][rows_], out[1][rows_])
            elif op == "cols":
                want = O.quantize(xb, O.COLS, O.SR, 77, row0=r0)
                got = (out[0][:, 16 * b:16 * b + 16], out[1][:, b:b + 1])
            elif op == "double":
                want = O.double_quantize(xb, 77, row0=r0)
                got = (out[0][rows_], out[1][rows_],
                       out[2][:, 16 * b:16 * b + 16], out[3][:, b:b + 1])
            else:
                # the rotation's own rule: tolerance on the rotated values,
                # codes exact for them, boundary-only differences
                check_rht(xb, 3, O.SR, 77, to_np(out[0][rows_]), to_np(out[1][rows_]),
                          to_np(out[2][rows_]), row0=r0)
                continue
            got = [to_np(g) for g in got]
            for g, w in zip(got, want):
                assert_bits_equal(g, w, "%s band %d" % (op, b))
        del out
    del xd
    torch.cuda.empty_cache()


def test_master_weight_qema_sampled_bands():
    w_np = W.master_w(seed=7)                 # 4096 x 14336 fp32
    e_np = W.master_w(seed=8)
    w, e = to_dev(w_np), to_dev(e_np)
    for _ in range(3):
        c, s = m.qema_quantize(w, e, 0.998)
    c, s, e_got = to_np(c), to_np(s), to_np(e)
    for r0 in (0, 2048, 4064):
        band_w, band_e = w_np[r0:r0 + 32].copy(), e_np[r0:r0 + 32].copy()
        for _ in range(3):
            oc, os_ = O.qema_quantize(band_w, band_e, 0.998)
        assert_bits_equal(e_got[r0:r0 + 32], band_e, "ema band %d" % r0)
        assert_bits_equal(c[r0:r0 + 32], oc, "codes band %d" % r0)
        assert_bits_equal(s[r0:r0 + 32], os_, "scales band %d" % r0)
