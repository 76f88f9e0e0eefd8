"""Seeded random sweep over shapes, dtypes, value distributions, seeds and
scale rules: every quantizer entry point against the oracle, bit for bit
(the rotation through its own rule), and the fused GEMM against the
two-step path; the tracker, Q-Ramping and Q-EMA state bit for bit. Each
case is small enough for the oracle; together they
cover many ragged tile positions, grid sizes and special values that the
hand-picked cases do not.
"""
import numpy as np
import pytest
import torch

import mxfp4_block_quantization_quantizer_b200 as m
import oracle as O
from gpu_util import BF16, assert_bits_equal, assert_f32_equal_or_both_nan, to_dev, to_np
from test_gpu_parity import check_rht

pytestmark = pytest.mark.gpu

N_CASES = 64


def random_tensor(g, rows, cols, dtype):
    """A mix the kernels must handle alike: a random log-uniform spread of
    magnitudes, exact zeros, signed zeros, subnormals, huge values, and now
    and then an inf or NaN group."""
    x = g.standard_normal((rows, cols)) * np.exp2(g.integers(-20, 20, size=(rows, cols)))
    kind = g.integers(0, 6)
    if kind == 1:
        x[g.random((rows, cols)) < 0.2] = 0.0
        x[g.random((rows, cols)) < 0.05] = -0.0
    elif kind == 2:
        x *= 2.0 ** -130                      # subnormal territory
    elif kind == 3:
        x *= 2.0 ** 100                       # near the top of the range
    elif kind == 4:
        r, c = g.integers(0, rows), g.integers(0, cols)
        x[r, c] = [np.inf, -np.inf, np.nan][g.integers(0, 3)]
    x = x.astype(np.float32)
    return x.astype(BF16) if dtype == "bf16" else x


def cases(seed):
    g = np.random.Generator(np.random.PCG64(seed))
    out = []
    for i in range(N_CASES):
        rows = int(32 * g.integers(1, 20))
        cols = int(32 * g.integers(1, 40))
        out.append((i, rows, cols, ["bf16", "f32"][g.integers(0, 2)],
                    int(g.integers(0, 2**32)), bool(g.integers(0, 2))))
    return out


@pytest.mark.parametrize("case", cases(101), ids=lambda c: "case%d" % c[0])
def test_fuzz_quantize_and_dequantize(case):
    i, rows, cols, dtype, seed, oas = case
    g = np.random.Generator(np.random.PCG64(1000 + i))
    x = random_tensor(g, rows, cols, dtype)
    xd = to_dev(x)
    for axis in (m.ROWS, m.COLS):
        for rnd in (m.RNE, m.SR):
            c, s = m.quantize(xd, axis, rnd, seed, oas=oas)
            oc, os_ = O.quantize(x, axis, rnd, seed, oas=oas)
            assert_bits_equal(to_np(c), oc, "codes axis %d rnd %d" % (axis, rnd))
            assert_bits_equal(to_np(s), os_, "scales axis %d rnd %d" % (axis, rnd))
            for od, oname in ((torch.bfloat16, "bf16"), (torch.float32, "f32")):
                y = m.dequantize(c, s, rows, cols, axis, out_dtype=od)
                want = O.dequantize(oc, os_, rows, cols, axis, oname)
                assert_bits_equal(to_np(y), want, "dequantized axis %d" % axis)


@pytest.mark.parametrize("case", cases(202), ids=lambda c: "case%d" % c[0])
def test_fuzz_double_quantize(case):
    i, rows, cols, dtype, seed, oas = case
    g = np.random.Generator(np.random.PCG64(2000 + i))
    x = random_tensor(g, rows, cols, dtype)
    got = m.double_quantize(to_dev(x), seed=seed, oas=oas)
    for gt, w, name in zip(got, O.double_quantize(x, seed, oas=oas),
                           ("row codes", "row scales", "col codes", "col scales")):
        assert_bits_equal(to_np(gt), w, "double quantization " + name)


@pytest.mark.parametrize("case", cases(303)[:24], ids=lambda c: "case%d" % c[0])
def test_fuzz_rotation(case):
    """Finite inputs of moderate range (the rotation's parity claim)."""
    i, rows, cols, dtype, seed, oas = case
    g = np.random.Generator(np.random.PCG64(3000 + i))
    x = (g.standard_normal((rows, cols)) * np.exp2(g.integers(-6, 6, size=(rows, cols))))
    x = x.astype(np.float32)
    x = x.astype(BF16) if dtype == "bf16" else x
    for rnd in (m.RNE, m.SR):
        codes, scales, rot = m.rht_quantize(to_dev(x), seed % 97, rnd, seed, want_rotated=True)
        check_rht(x, seed % 97, rnd, seed, to_np(codes), to_np(scales), to_np(rot))


@pytest.mark.parametrize("case", cases(404)[:24], ids=lambda c: "case%d" % c[0])
def test_fuzz_fused_gemm(case):
    i, rows, cols, dtype, seed, oas = case
    g = np.random.Generator(np.random.PCG64(4000 + i))
    k = 256 * int(g.integers(1, 5))
    n = int(g.integers(1, 600))
    x = (g.standard_normal((rows, k)) * np.exp2(g.integers(-8, 8, size=(rows, k))))
    xd = to_dev(x.astype(np.float32).astype(BF16))
    w = to_dev(g.standard_normal((n, k)).astype(np.float32).astype(BF16))
    wc, ws = m.quantize(w, m.ROWS, m.RNE)
    wb = m.scales_to_blocked(ws)
    for rnd in (m.RNE, m.SR):
        c, ac, as_ = m.gemm_quantize_a(xd, wc, wb, rounding=rnd, seed=seed, want_a=True)
        qc, qs = m.quantize(xd, m.ROWS, rnd, seed)
        assert torch.equal(ac, qc) and torch.equal(as_, qs)
        ref = m.gemm(qc, m.scales_to_blocked(qs), wc, wb, k)
        assert torch.equal(c.view(torch.int32), ref.view(torch.int32))


@pytest.mark.parametrize("i", range(16), ids=lambda i: "case%d" % i)
def test_fuzz_fused_gemm_clusters(i):
    """More than one column tile of C (clusters of 2 or 4 CTAs sharing the
    quantization of their rows), 64- or 128-row tiles, ragged m and n."""
    g = np.random.Generator(np.random.PCG64(4500 + i))
    mm = int(g.integers(1, 12000))
    n = int(g.integers(257, 2100))
    k = 256 * int(g.integers(1, 5))
    seed = int(g.integers(0, 2**32))
    x = g.standard_normal((mm, k)) * np.exp2(g.integers(-8, 8, size=(mm, k)))
    xd = to_dev(x.astype(np.float32).astype(BF16))
    wc, ws = m.quantize(to_dev(g.standard_normal((n, k)).astype(np.float32).astype(BF16)),
                        m.ROWS, m.RNE)
    wb = m.scales_to_blocked(ws)
    for rnd in (m.RNE, m.SR):
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        c, ac, as_ = m.gemm_quantize_a(xd, wc, wb, rounding=rnd, seed=seed, want_a=True,
                                       status=st)
        assert int(st.item()) == 0
        qc, qs = m.quantize(xd, m.ROWS, rnd, seed)
        assert torch.equal(ac, qc) and torch.equal(as_, qs)
        ref = m.gemm(qc, m.scales_to_blocked(qs), wc, wb, k)
        assert torch.equal(c.view(torch.int32), ref.view(torch.int32))


def tracker_weights(g, rows, cols):
    """fp32 weights with one group maximum per group (a fixed scale) and many
    values near a rounding edge, like the tracker workload."""
    w = (g.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    w = np.clip(w, -2.0 ** -4, 2.0 ** -4)
    w.reshape(-1, 32)[:, 0] = np.float32(2.0 ** -4 * 1.5)
    edges = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]) * 2.0 ** -6
    pick = g.random((rows, cols)) < 0.3
    near = g.choice(edges, size=(rows, cols)) * (1 + g.uniform(-1e-3, 1e-3, (rows, cols)))
    w[pick] = (near * np.sign(g.standard_normal((rows, cols))))[pick].astype(np.float32)
    w.reshape(-1, 32)[:, 0] = np.float32(2.0 ** -4 * 1.5)
    return w


@pytest.mark.parametrize("case", cases(505)[:16], ids=lambda c: "case%d" % c[0])
def test_fuzz_tracker_and_qramp(case):
    """The tracker over a random window with a random threshold, and
    Q-Ramping with random window, k1 and k2 over two epochs: every state
    array and flag count bit for bit after every iteration."""
    i, rows, cols, dtype, seed, oas = case
    g = np.random.Generator(np.random.PCG64(5000 + i))
    w0 = tracker_weights(g, min(rows, 128), cols)
    # the tracker
    steps = int(g.integers(1, 30))
    threshold = float(g.choice([0.5, 2.0, 4.0, 16.0]))
    w, ws = to_dev(w0.copy()), to_dev(w0.copy())
    dw, dq = torch.zeros_like(w), torch.zeros_like(w)
    nflag = torch.zeros(1, dtype=torch.int64, device="cuda")
    ow, ows, odw, odq = w0.copy(), w0.copy(), np.zeros_like(w0), np.zeros_like(w0)
    flagged = 0
    for t in range(steps):
        end = t == steps - 1 or g.random() < 0.1
        m.osc_synthetic_update(w, seed, t)
        m.osc_step(w, ws, dw, dq, window_end=end, threshold=threshold, n_flagged=nflag)
        O.osc_synthetic_update(ow, seed, t)
        flagged += O.osc_step(ow, ows, odw, odq, window_end=end, threshold=threshold)
    for gt, wv, name in zip((w, ws, dw, dq), (ow, ows, odw, odq), ("w", "w_snap", "d_w", "d_q")):
        assert_bits_equal(to_np(gt), wv, "tracker " + name)
    assert int(nflag.item()) == flagged
    # Q-Ramping
    track, k2, k1 = int(g.integers(0, 8)), int(g.integers(1, 7)), float(g.choice([2.0, 16.0]))
    epoch = int(g.integers(1, 12))
    z = np.zeros_like(w0)
    ref = [w0.copy(), z.copy(), z.copy(), z.copy(), z.copy(), np.zeros(w0.shape, np.uint8)]
    dev = [to_dev(a.copy()) for a in ref]
    nflag.zero_()
    total = 0
    mag = (np.float32(1e-4) * np.abs(w0)).astype(np.float32)
    for t in range(2 * epoch):
        d = (np.where(g.random(w0.shape) < 0.5, -1.0, 1.0) * mag).astype(np.float32)
        it = t % epoch
        m.qramp_step(dev[0], to_dev(d), *dev[1:], it, track_iters=track, k1=k1, k2=k2,
                     n_flagged=nflag)
        total += O.qramp_step(ref[0], d, *ref[1:], it, track_iters=track, k1=k1, k2=k2)
        for gt, r, name in zip(dev, ref, ("w", "w_snap", "d_w", "d_q", "acc", "flag")):
            assert_bits_equal(to_np(gt), r, "qramp %s at %d" % (name, t))
    assert int(nflag.item()) == total


@pytest.mark.parametrize("case", cases(606)[:16], ids=lambda c: "case%d" % c[0])
def test_fuzz_qema(case):
    i, rows, cols, dtype, seed, oas = case
    g = np.random.Generator(np.random.PCG64(6000 + i))
    w_np = random_tensor(g, rows, cols, "f32")
    e_np = random_tensor(g, rows, cols, "f32")
    beta = float(g.choice([0.0, 0.5, 0.9, 0.998, 1.0]))
    e = to_dev(e_np)
    c, s = m.qema_quantize(to_dev(w_np), e, beta)
    oc, os_ = O.qema_quantize(w_np, e_np, beta)
    assert_f32_equal_or_both_nan(to_np(e), e_np, "ema")   # NaN payloads may differ
    assert_bits_equal(to_np(c), oc, "codes")
    assert_bits_equal(to_np(s), os_, "scales")


@pytest.mark.parametrize("case", cases(707)[:24], ids=lambda c: "case%d" % c[0])
def test_fuzz_blocked_scales_and_gemm(case):
    """Random m, n and k (a multiple of 32: both GEMM kernels): the blocked
    scale order byte for byte, and C within the fp32 accumulation bound of
    the oracle's product."""
    i, rows, cols, dtype, seed, oas = case
    g = np.random.Generator(np.random.PCG64(7000 + i))
    mm, nn, k = int(g.integers(1, 300)), int(g.integers(1, 300)), int(32 * g.integers(1, 24))
    ca = g.integers(0, 256, size=(mm, k // 2), dtype=np.uint8)
    cb = g.integers(0, 256, size=(nn, k // 2), dtype=np.uint8)
    sa = g.integers(110, 145, size=(mm, k // 32), dtype=np.uint8)
    sb = g.integers(110, 145, size=(nn, k // 32), dtype=np.uint8)
    ba, bb = m.scales_to_blocked(to_dev(sa)), m.scales_to_blocked(to_dev(sb))
    assert_bits_equal(to_np(ba), O.scales_to_blocked(sa), "blocked A scales")
    assert_bits_equal(to_np(bb), O.scales_to_blocked(sb), "blocked B scales")
    got = to_np(m.gemm(to_dev(ca), ba, to_dev(cb), bb, k)).astype(np.float64)
    want = O.gemm(ca, sa, cb, sb, k)
    da = np.abs(O.dequantize(ca, sa, mm, k, O.ROWS, "f32").astype(np.float64))
    db = np.abs(O.dequantize(cb, sb, nn, k, O.ROWS, "f32").astype(np.float64))
    assert np.all(np.abs(got - want) <= (k - 1) * 2.0 ** -24 * (da @ db.T))
