"""The status word of the tensor-core entry points (mxfp4_gemm,
mxfp4_rht_quantize, mxfp4_gemm_quantize_a): clear after every normal run; set, with the documented
poison values in the outputs, by a test build whose accumulator waits give
up at once (MXFP4_ACC_WAIT_POLLS=0). That build fails no hardware operation:
each CTA stops waiting, lets the copies and MMAs it issued finish, frees its
tensor memory and returns, so the context stays usable, which the last step
of each test checks with the normal library.
"""
import ctypes

import numpy as np
import pytest
import torch

import mxfp4_block_quantization_quantizer_b200 as m
import oracle as O
from mxfp4_block_quantization_quantizer_b200 import build as B
from mxfp4_block_quantization_quantizer_b200 import workloads as W
from gpu_util import to_dev, to_np

pytestmark = pytest.mark.gpu

GEMM_CASES = [(384, 512, 512),   # persistent TMA kernel (k % 256 == 0), 6 tiles
              (200, 136, 96)]    # one-tile-per-CTA kernel, ragged edges
RHT_CASES = [(m.SR, True), (m.RNE, False)]   # fp32 rotation out / staged codes


def gemm_operands(mm, nn, k, seed):
    g = np.random.Generator(np.random.PCG64(seed))
    ca = g.integers(0, 256, size=(mm, k // 2), dtype=np.uint8)
    cb = g.integers(0, 256, size=(nn, k // 2), dtype=np.uint8)
    sa = g.integers(120, 135, size=(mm, k // 32), dtype=np.uint8)
    sb = g.integers(120, 135, size=(nn, k // 32), dtype=np.uint8)
    return ca, sa, cb, sb


def zero_status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


@pytest.fixture(scope="module")
def short_wait_lib(tmp_path_factory):
    path = str(tmp_path_factory.mktemp("shortwait") / "libmxfp4_shortwait.so")
    B.build_variant(path, ["MXFP4_ACC_WAIT_POLLS=0"])
    L = ctypes.CDLL(path)
    vp, i32, i64, u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64
    L.mxfp4_gemm.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, vp, vp]
    L.mxfp4_rht_quantize.argtypes = [vp, i32, i64, i64, u64, i32, u64, vp, vp, vp, vp, vp]
    L.mxfp4_gemm_quantize_a.argtypes = [vp, i64, i64, i64, i32, u64, vp, vp, vp, vp, vp, vp,
                                        vp]
    for f in (L.mxfp4_gemm, L.mxfp4_rht_quantize, L.mxfp4_gemm_quantize_a):
        f.restype = i32
    return L


def ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("mnk", GEMM_CASES)
def test_gemm_status_clear_on_normal_runs(mnk):
    mm, nn, k = mnk
    ca, sa, cb, sb = gemm_operands(mm, nn, k, 11)
    st = zero_status()
    got = to_np(m.gemm(to_dev(ca), m.scales_to_blocked(to_dev(sa)), to_dev(cb),
                       m.scales_to_blocked(to_dev(sb)), k, status=st))
    assert int(st.item()) == 0
    want = O.gemm(ca, sa, cb, sb, k)
    da = np.abs(O.dequantize(ca, sa, mm, k, O.ROWS, "f32").astype(np.float64))
    db = np.abs(O.dequantize(cb, sb, nn, k, O.ROWS, "f32").astype(np.float64))
    assert np.all(np.abs(got - want) <= (k - 1) * 2.0 ** -24 * (da @ db.T))


@pytest.mark.parametrize("rnd,rot", RHT_CASES)
def test_rht_status_clear_on_normal_runs(rnd, rot):
    x = W.normal_bf16(256, 1024, 4)
    st = zero_status()
    codes, scales, rotated = m.rht_quantize(to_dev(x), 2, rnd, 3, want_rotated=rot, status=st)
    assert int(st.item()) == 0
    if rot:   # codes are those of the rotation the kernel computed
        oc, os_ = O.quantize(to_np(rotated), O.ROWS, rnd, 3)
        assert np.array_equal(to_np(codes), oc) and np.array_equal(to_np(scales), os_)
    c0, s0, _ = m.rht_quantize(to_dev(x), 2, rnd, 3, want_rotated=rot)
    assert torch.equal(codes, c0) and torch.equal(scales, s0)


@pytest.mark.parametrize("mnk", GEMM_CASES)
def test_gemm_timeout_sets_status_and_poisons_tiles(short_wait_lib, mnk):
    mm, nn, k = mnk
    ca, sa, cb, sb = gemm_operands(mm, nn, k, 12)
    a, b = to_dev(ca), to_dev(cb)
    ab, bb = m.scales_to_blocked(to_dev(sa)), m.scales_to_blocked(to_dev(sb))
    c = torch.zeros((mm, nn), dtype=torch.float32, device="cuda")
    st = zero_status()
    rc = short_wait_lib.mxfp4_gemm(ptr(a), ptr(ab), ptr(b), ptr(bb), mm, nn, k, ptr(c),
                                   ptr(st), stream())
    assert rc == 0
    torch.cuda.synchronize()
    assert int(st.item()) == m.STATUS_WAIT_TIMEOUT
    assert torch.isnan(c).all()
    # the context is intact: the normal library still computes the product
    st2 = zero_status()
    again = to_np(m.gemm(a, ab, b, bb, k, status=st2))
    assert int(st2.item()) == 0 and np.isfinite(again).all()
    assert np.array_equal(again, to_np(m.gemm(a, ab, b, bb, k)))


@pytest.mark.parametrize("rnd,rot", RHT_CASES)
def test_rht_timeout_sets_status_and_poisons_groups(short_wait_lib, rnd, rot):
    x = W.normal_bf16(256, 1024, 5)
    xd = to_dev(x)
    R, C = x.shape
    codes = torch.full((R, C // 2), 0x55, dtype=torch.uint8, device="cuda")
    scales = torch.zeros((R, C // 32), dtype=torch.uint8, device="cuda")
    rotated = torch.zeros((R, C), dtype=torch.float32, device="cuda") if rot else None
    st = zero_status()
    rc = short_wait_lib.mxfp4_rht_quantize(ptr(xd), m.BF16, R, C, 2, rnd, 3, ptr(codes),
                                           ptr(scales), ptr(rotated), ptr(st), stream())
    assert rc == 0
    torch.cuda.synchronize()
    assert int(st.item()) == m.STATUS_WAIT_TIMEOUT
    assert (scales == 0xFF).all() and (codes == 0).all()
    if rot:
        assert torch.isnan(rotated).all()
    # the context is intact: the normal library quantizes the rotation
    st2 = zero_status()
    c2, s2, r2 = m.rht_quantize(xd, 2, rnd, 3, want_rotated=True, status=st2)
    assert int(st2.item()) == 0 and torch.isfinite(r2).all()
    oc, os_ = O.quantize(to_np(r2), O.ROWS, rnd, 3)
    assert np.array_equal(to_np(c2), oc) and np.array_equal(to_np(s2), os_)


def test_fused_gemm_timeout_sets_status_and_poisons_tiles(short_wait_lib):
    x = W.normal_bf16(384, 768, 7)
    xd = to_dev(x)
    wc, ws = m.quantize(to_dev(W.normal_bf16(520, 768, 8)), m.ROWS, m.RNE)
    wb = m.scales_to_blocked(ws)
    c = torch.zeros((384, 520), dtype=torch.float32, device="cuda")
    st = zero_status()
    rc = short_wait_lib.mxfp4_gemm_quantize_a(ptr(xd), 384, 520, 768, m.RNE, 0, ptr(wc),
                                              ptr(wb), ptr(c), None, None, ptr(st), stream())
    assert rc == 0
    torch.cuda.synchronize()
    assert int(st.item()) == m.STATUS_WAIT_TIMEOUT
    assert torch.isnan(c).all()
    st2 = zero_status()
    again = m.gemm_quantize_a(xd, wc, wb, status=st2)
    assert int(st2.item()) == 0 and torch.isfinite(again).all()
    qc, qs = m.quantize(xd, m.ROWS, m.RNE)
    ref = m.gemm(qc, m.scales_to_blocked(qs), wc, wb, 768)
    assert torch.equal(again.view(torch.int32), ref.view(torch.int32))
