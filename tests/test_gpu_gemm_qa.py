"""The GEMM with the activation quantized in its load stage
(mxfp4_gemm_quantize_a, C = Q(X) B^T, Q nearest-even or stochastic) against
the two-step path it replaces and against the oracle.

- Q(X) as the fused kernel writes it out equals mxfp4_quantize's ROWS codes
  and scales (same rounding and seed) byte for byte, and the oracle's;
- C equals mxfp4_gemm on those codes bit for bit (same tiles, same MMA
  sequence) and lies within the fp32 accumulation bound of the oracle's
  exact product: (k - 1) 2^-24 sum_j |a_j b_j|.

The shapes reach every tile form of the kernel: 64- and 128-row tiles, alone
or in clusters of 2 or 4 CTAs that share the quantization of their rows
(more than one column tile of 256), with column tiles of a cluster past n.
"""
import numpy as np
import pytest
import torch

import mxfp4_block_quantization_quantizer_b200 as m
import oracle as O
from mxfp4_block_quantization_quantizer_b200 import workloads as W
from gpu_util import to_dev, to_np

pytestmark = pytest.mark.gpu


def weight(n, k, seed):
    """A pre-quantized weight: ROWS RNE codes and scales of N(0,1) bf16."""
    w = W.normal_bf16(n, k, seed)
    wc, ws = m.quantize(to_dev(w), m.ROWS, m.RNE)
    return wc, ws


def check_against_oracle(c, xc, xs, wc, ws, k, rows=None):
    """C (rows `rows` of it) within the accumulation bound of the oracle's
    fp64 product of the dequantized operands."""
    if rows is not None:
        xc, xs, c = xc[rows], xs[rows], c[rows]
    want = O.gemm(xc, xs, wc, ws, k)
    da = np.abs(O.dequantize(xc, xs, xc.shape[0], k, O.ROWS, "f32").astype(np.float64))
    db = np.abs(O.dequantize(wc, ws, wc.shape[0], k, O.ROWS, "f32").astype(np.float64))
    bound = (k - 1) * 2.0 ** -24 * (da @ db.T)
    err = np.abs(c.astype(np.float64) - want)
    assert np.all(err <= bound), "max error / bound %g" % (err / np.maximum(bound, 1e-300)).max()


@pytest.mark.parametrize("mnk", [(128, 256, 256),    # one tile, one stage
                                 (200, 136, 512),    # ragged rows and columns
                                 # 3 x 3 tiles, a 8-column edge tile (64-row
                                 # tiles in clusters of 2)
                                 (384, 520, 768),
                                 (1000, 64, 1024),   # narrow output, many row tiles
                                 (256, 768, 2560),   # 10 stages: the rings wrap
                                 # several tiles per CTA (or cluster) with one stage
                                 # each (the accumulator drained after the next
                                 # tile's only stage): one CTA per tile, clusters of 2;
                                 # one tile per cluster of 2
                                 (40000, 200, 256), (20000, 520, 256), (9000, 512, 256),
                                 # one row; two weight rows; n not a multiple of 4
                                 # (scalar stores of C)
                                 (1, 256, 256), (65, 2, 512), (100, 130, 256),
                                 # 128-row tiles without clusters (149 row tiles)
                                 (19000, 200, 256),
                                 # clusters of 4 CTAs sharing the quantization of
                                 # their rows: 64-row tiles; 128-row tiles with the
                                 # second cluster's last three column tiles past n
                                 (300, 1024, 512), (5000, 1100, 512),
                                 # clusters of 2 over 3 column tiles (one CTA of the
                                 # last cluster past n), rows not a multiple of 64
                                 (4100, 700, 768)])
def test_fused_equals_quantize_then_gemm(mnk):
    mm, nn, k = mnk
    x = W.normal_bf16(mm, k, 21, 0.005, 50.0)
    x[0, :32] = 0          # an all-zero group
    xd = to_dev(x)
    wc, ws = weight(nn, k, 22)
    wb = m.scales_to_blocked(ws)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    c, ac, as_ = m.gemm_quantize_a(xd, wc, wb, want_a=True, status=st)
    assert int(st.item()) == 0
    qc, qs = m.quantize(xd, m.ROWS, m.RNE)
    assert torch.equal(ac, qc) and torch.equal(as_, qs)
    oc, os_ = O.quantize(x, O.ROWS, O.RNE)
    assert np.array_equal(to_np(ac), oc) and np.array_equal(to_np(as_), os_)
    ref = m.gemm(qc, m.scales_to_blocked(qs), wc, wb, k)
    assert torch.equal(c.view(torch.int32), ref.view(torch.int32))
    check_against_oracle(to_np(c), oc, os_, to_np(wc), to_np(ws), k)
    # without the optional outputs: the same C
    c2 = m.gemm_quantize_a(xd, wc, wb)
    assert torch.equal(c2.view(torch.int32), c.view(torch.int32))


def test_special_values_follow_the_quantizer():
    """Groups whose maximum is inf or NaN get scale byte 0xFF (NaN) in the
    quantizer; the fused GEMM quantizes them the same way."""
    k = 256
    x = W.normal_bf16(128, k, 23)
    xi = x.view(np.uint16)
    xi[3, 5] = 0x7F80      # +inf
    xi[9, 40] = 0xFFC1     # NaN
    xi[17, 100] = 0x0001   # subnormal in an otherwise normal group
    xd = to_dev(x)
    wc, ws = weight(256, k, 24)
    c, ac, as_ = m.gemm_quantize_a(xd, wc, m.scales_to_blocked(ws), want_a=True)
    qc, qs = m.quantize(xd, m.ROWS, m.RNE)
    assert torch.equal(ac, qc) and torch.equal(as_, qs)
    ref = m.gemm(qc, m.scales_to_blocked(qs), wc, m.scales_to_blocked(ws), k)
    assert torch.equal(c.view(torch.int32), ref.view(torch.int32))
    assert torch.isnan(c[3]).all() and torch.isnan(c[9]).all()


@pytest.mark.parametrize("n", [256, 512, 1024])
def test_fused_on_the_sweep_activation(n):
    """The benchmark's activation (8192 x 28672 bf16 with outliers) against
    a weight of n rows: all of C and all of Q_D(X) against the two-step path
    on the GPU, and sampled rows of C against the oracle."""
    x = W.sweep(seed=5)
    xd = to_dev(x)
    K = x.shape[1]
    wc, ws = weight(n, K, 6)
    wb = m.scales_to_blocked(ws)
    c, ac, as_ = m.gemm_quantize_a(xd, wc, wb, want_a=True)
    qc, qs = m.quantize(xd, m.ROWS, m.RNE)
    assert torch.equal(ac, qc) and torch.equal(as_, qs)
    ref = m.gemm(qc, m.scales_to_blocked(qs), wc, wb, K)
    assert torch.equal(c.view(torch.int32), ref.view(torch.int32))
    rows = np.array([0, 1, 127, 128, 4095, 4096, 8190, 8191])
    oc, os_ = O.quantize(x[rows], O.ROWS, O.RNE, row0=0)
    # the oracle's row quantization of sampled rows is the GPU's
    assert np.array_equal(to_np(ac)[rows], oc) and np.array_equal(to_np(as_)[rows], os_)
    check_against_oracle(to_np(c)[rows], oc, os_, to_np(wc), to_np(ws), K)


@pytest.mark.parametrize("mnk", [(200, 136, 512), (9000, 512, 256), (20000, 520, 256),
                                 (384, 1024, 2560), (5000, 1100, 512), (19000, 200, 256)])
def test_fused_stochastic_rounding(mnk):
    """Q_S(X) in the load stage (a gradient for a backward GEMM): the codes of
    mxfp4_quantize with the same seed, and the two-step C."""
    mm, nn, k = mnk
    x = W.normal_bf16(mm, k, 25, 0.005, 50.0)
    xd = to_dev(x)
    wc, ws = weight(nn, k, 26)
    wb = m.scales_to_blocked(ws)
    c, ac, as_ = m.gemm_quantize_a(xd, wc, wb, rounding=m.SR, seed=17, want_a=True)
    qc, qs = m.quantize(xd, m.ROWS, m.SR, 17)
    assert torch.equal(ac, qc) and torch.equal(as_, qs)
    oc, os_ = O.quantize(x, O.ROWS, O.SR, 17)
    assert np.array_equal(to_np(ac), oc) and np.array_equal(to_np(as_), os_)
    ref = m.gemm(qc, m.scales_to_blocked(qs), wc, wb, k)
    assert torch.equal(c.view(torch.int32), ref.view(torch.int32))
    check_against_oracle(to_np(c), oc, os_, to_np(wc), to_np(ws), k)
    # another seed gives other codes
    c2, ac2, _ = m.gemm_quantize_a(xd, wc, wb, rounding=m.SR, seed=18, want_a=True)
    assert not torch.equal(ac2, ac)


def test_fused_stochastic_rounding_on_the_sweep():
    x = W.sweep(seed=5)
    xd = to_dev(x)
    K = x.shape[1]
    wc, ws = weight(256, K, 6)
    wb = m.scales_to_blocked(ws)
    c, ac, as_ = m.gemm_quantize_a(xd, wc, wb, rounding=m.SR, seed=5, want_a=True)
    qc, qs = m.quantize(xd, m.ROWS, m.SR, 5)
    assert torch.equal(ac, qc) and torch.equal(as_, qs)
    ref = m.gemm(qc, m.scales_to_blocked(qs), wc, wb, K)
    assert torch.equal(c.view(torch.int32), ref.view(torch.int32))
    # sampled rows against the oracle (its counters start at row0)
    acn, asn, cn = to_np(ac), to_np(as_), to_np(c)
    for r in (0, 4097, 8191):
        oc, os_ = O.quantize(x[r:r + 1], O.ROWS, O.SR, 5, row0=r)
        assert np.array_equal(acn[r:r + 1], oc) and np.array_equal(asn[r:r + 1], os_)
        check_against_oracle(cn[r:r + 1], oc, os_, to_np(wc), to_np(ws), K)


@pytest.mark.parametrize("mnk", [(200, 136, 512),     # one CTA per tile
                                 (384, 520, 768),     # clusters of 2, a CTA past n
                                 (300, 1100, 512),    # clusters of 4, three CTAs past n
                                 (5000, 1100, 256)])  # the same with 128-row tiles
def test_fused_outputs_stay_inside_their_buffers(mnk):
    """C and the optional Q(X) outputs written into guarded buffers: the
    canary bytes around each are untouched (rows past m, column tiles of a
    cluster past n) and the results equal an unguarded call."""
    mm, nn, k = mnk
    xd = to_dev(W.normal_bf16(mm, k, 27, 0.005, 50.0))
    wc, ws = weight(nn, k, 28)
    wb = m.scales_to_blocked(ws)
    pad, canary = 4096, 0xA5

    def guarded(nbytes):
        buf = torch.full((nbytes + 2 * pad,), canary, dtype=torch.uint8, device="cuda")
        return buf, buf[pad:pad + nbytes]

    cbuf, cv = guarded(4 * mm * nn)
    abuf, av = guarded(mm * k // 2)
    sbuf, sv = guarded(mm * k // 32)
    out = (cv.view(torch.float32).view(mm, nn), av.view(mm, k // 2), sv.view(mm, k // 32))
    for rnd in (m.RNE, m.SR):
        m.gemm_quantize_a(xd, wc, wb, rounding=rnd, seed=3, out=out, want_a=True)
        ref_c, ref_a, ref_s = m.gemm_quantize_a(xd, wc, wb, rounding=rnd, seed=3, want_a=True)
        for b in (cbuf, abuf, sbuf):
            h = to_np(b)
            assert np.all(h[:pad] == canary) and np.all(h[-pad:] == canary)
        assert torch.equal(out[0].view(torch.int32), ref_c.view(torch.int32))
        assert torch.equal(out[1], ref_a) and torch.equal(out[2], ref_s)
