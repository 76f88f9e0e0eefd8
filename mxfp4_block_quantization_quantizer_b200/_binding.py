"""ctypes binding of libmxfp4 (include/mxfp4.h).

Argument marshalling only: tensors become device pointers and sizes, the
current torch stream becomes the cudaStream_t, output buffers are allocated
with torch. Every step of the computation runs in the library's kernels.
There is no fallback: if the library is missing, or a tensor is not on a CUDA
device, the call raises.
"""
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmxfp4.so")

F32, BF16 = 0, 1
ROWS, COLS = 0, 1
RNE, SR = 0, 1
# Bit of the tensor-core entry points' status word: a bounded wait ran out.
STATUS_WAIT_TIMEOUT = 1

# Every symbol include/mxfp4.h declares.
SYMBOLS = ("mxfp4_quantize", "mxfp4_quantize_oas", "mxfp4_dequantize",
           "mxfp4_double_quantize", "mxfp4_double_quantize_oas",
           "mxfp4_rht_quantize", "mxfp4_rht_quantize_oas", "mxfp4_osc_step",
           "mxfp4_osc_synthetic_update", "mxfp4_qramp_step", "mxfp4_qema_quantize",
           "mxfp4_scales_to_blocked", "mxfp4_gemm", "mxfp4_gemm_quantize_a",
           "mxfp4_status_string")


class Mxfp4Error(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__("%s: %s (status %d)" % (what, status_string(status), status))


_lib = None


def lib():
    """The loaded libmxfp4 (ctypes.CDLL). Raises if it was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                "libmxfp4.so is not built (expected at %s); run "
                "__graft_entry__.build() or python -m "
                "mxfp4_block_quantization_quantizer_b200.build" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, u64, u32, i32 = (ctypes.c_void_p, ctypes.c_int64,
                                  ctypes.c_uint64, ctypes.c_uint32,
                                  ctypes.c_int)
        sig = {
            "mxfp4_quantize": [vp, i32, i64, i64, i32, i32, u64, vp, vp, vp],
            "mxfp4_quantize_oas": [vp, i32, i64, i64, i32, i32, u64, vp, vp, vp],
            "mxfp4_dequantize": [vp, vp, i64, i64, i32, vp, i32, vp],
            "mxfp4_double_quantize": [vp, i32, i64, i64, u64, vp, vp, vp, vp,
                                      vp],
            "mxfp4_double_quantize_oas": [vp, i32, i64, i64, u64, vp, vp, vp,
                                          vp, vp],
            "mxfp4_rht_quantize": [vp, i32, i64, i64, u64, i32, u64, vp, vp,
                                   vp, vp, vp],
            "mxfp4_rht_quantize_oas": [vp, i32, i64, i64, u64, i32, u64, vp,
                                       vp, vp, vp, vp],
            "mxfp4_osc_step": [vp, vp, vp, vp, i64, i64, i32, ctypes.c_float,
                               vp, vp],
            "mxfp4_osc_synthetic_update": [vp, i64, i64, u64, u32,
                                           ctypes.c_float, vp],
            "mxfp4_qema_quantize": [vp, vp, i64, i64, ctypes.c_float, vp, vp,
                                    vp],
            "mxfp4_qramp_step": [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64,
                                 ctypes.c_float, i64, vp, vp],
            "mxfp4_scales_to_blocked": [vp, i64, i64, vp, vp],
            "mxfp4_gemm": [vp, vp, vp, vp, i64, i64, i64, vp, vp, vp],
            "mxfp4_gemm_quantize_a": [vp, i64, i64, i64, i32, u64, vp, vp, vp, vp,
                                      vp, vp, vp],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes, f.restype = args, i32
        L.mxfp4_status_string.argtypes = [i32]
        L.mxfp4_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(status):
    return lib().mxfp4_status_string(status).decode()


def _check(status, what):
    if status != 0:
        raise Mxfp4Error(status, what)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError("expected a bfloat16 or float32 tensor, got %s" % t.dtype)


def _on_device(t, name, device=None):
    """t is a CUDA tensor (on `device` when one is given)."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if device is not None and t.device != device:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, device))


def _cuda2d(t, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dim() != 2 or not t.is_contiguous():
        raise ValueError("%s must be a contiguous 2-D tensor" % name)
    _on_device(t, name)
    return t


def _buffer(t, name, dtype, numel, device):
    """Check a buffer before its pointer reaches the C ABI, which cannot see
    sizes: the library reads and writes exactly the bytes the header states
    for the given shape, so a smaller, strided, mistyped or foreign-device
    buffer would be read or written out of bounds. Raises before any launch."""
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a tensor" % name)
    if t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if t.numel() != numel:
        raise ValueError("%s must hold %d elements, got %d" % (name, numel, t.numel()))
    _on_device(t, name, device)
    return t


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device, stream=None):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _empty_u8(shape, device):
    return torch.empty(shape, dtype=torch.uint8, device=device)


def quantize(x, axis=ROWS, rounding=RNE, seed=0, out=None, stream=None,
             oas=False):
    """mxfp4_quantize (mxfp4_quantize_oas with oas=True): returns (codes,
    scales) in the layout of `axis`: ROWS -> codes [R, C/2], scales
    [R, C/32]; COLS -> codes [C, R/2], scales [C, R/32]."""
    _cuda2d(x, "x")
    R, C = x.shape
    if out is None:
        shape_c = (R, C // 2) if axis == ROWS else (C, R // 2)
        shape_s = (R, C // 32) if axis == ROWS else (C, R // 32)
        out = (_empty_u8(shape_c, x.device), _empty_u8(shape_s, x.device))
    codes, scales = out
    _buffer(codes, "codes", torch.uint8, R * C // 2, x.device)
    _buffer(scales, "scales", torch.uint8, R * C // 32, x.device)
    fn = lib().mxfp4_quantize_oas if oas else lib().mxfp4_quantize
    _check(fn(_ptr(x), _dtype_code(x), R, C, axis, rounding, seed, _ptr(codes),
              _ptr(scales), _stream(x.device, stream)), "mxfp4_quantize")
    return codes, scales


def dequantize(codes, scales, rows, cols, axis=ROWS, out_dtype=torch.bfloat16,
               out=None, stream=None):
    """mxfp4_dequantize: values [rows, cols] (ROWS) or [cols, rows] (COLS)."""
    _on_device(codes, "codes")
    n = int(rows) * int(cols)
    _buffer(codes, "codes", torch.uint8, n // 2, codes.device)
    _buffer(scales, "scales", torch.uint8, n // 32, codes.device)
    if out is None:
        shape = (rows, cols) if axis == ROWS else (cols, rows)
        out = torch.empty(shape, dtype=out_dtype, device=codes.device)
    _dtype_code(out)
    _buffer(out, "out", out.dtype, n, codes.device)
    _check(lib().mxfp4_dequantize(_ptr(codes), _ptr(scales), rows, cols, axis,
                                  _ptr(out), _dtype_code(out),
                                  _stream(codes.device, stream)),
           "mxfp4_dequantize")
    return out


def double_quantize(x, seed=0, out=None, stream=None, oas=False):
    """mxfp4_double_quantize (mxfp4_double_quantize_oas when oas):
    (row_codes, row_scales, col_codes, col_scales)."""
    _cuda2d(x, "x")
    R, C = x.shape
    if out is None:
        d = x.device
        out = (_empty_u8((R, C // 2), d), _empty_u8((R, C // 32), d),
               _empty_u8((C, R // 2), d), _empty_u8((C, R // 32), d))
    rc, rs, cc, cs = out
    for t, nm, n in ((rc, "row_codes", R * C // 2), (rs, "row_scales", R * C // 32),
                     (cc, "col_codes", R * C // 2), (cs, "col_scales", R * C // 32)):
        _buffer(t, nm, torch.uint8, n, x.device)
    name = "mxfp4_double_quantize_oas" if oas else "mxfp4_double_quantize"
    _check(getattr(lib(), name)(_ptr(x), _dtype_code(x), R, C, seed, _ptr(rc),
                                _ptr(rs), _ptr(cc), _ptr(cs),
                                _stream(x.device, stream)),
           name)
    return out


def _status_word(status, device):
    """The optional device status word of the tensor-core entry points: an
    int32 tensor of one element on `device` (the kernels OR
    MXFP4_STATUS_WAIT_TIMEOUT = 1 into it; the caller zeroes it)."""
    if status is not None:
        _buffer(status, "status", torch.int32, 1, device)
    return _ptr(status)


def rht_quantize(x, sign_seed=0, rounding=RNE, sr_seed=0, want_rotated=False,
                 out=None, stream=None, oas=False, status=None):
    """mxfp4_rht_quantize (mxfp4_rht_quantize_oas when oas): (codes, scales,
    rotated or None), ROWS layout. status: optional int32 CUDA tensor of one
    element, the timeout status word."""
    _cuda2d(x, "x")
    R, C = x.shape
    if out is None:
        d = x.device
        rot = torch.empty((R, C), dtype=torch.float32, device=d) if want_rotated else None
        out = (_empty_u8((R, C // 2), d), _empty_u8((R, C // 32), d), rot)
    codes, scales, rot = out
    _buffer(codes, "codes", torch.uint8, R * C // 2, x.device)
    _buffer(scales, "scales", torch.uint8, R * C // 32, x.device)
    if rot is not None:
        _buffer(rot, "rotated", torch.float32, R * C, x.device)
    st = _status_word(status, x.device)
    name = "mxfp4_rht_quantize_oas" if oas else "mxfp4_rht_quantize"
    _check(getattr(lib(), name)(_ptr(x), _dtype_code(x), R, C, sign_seed, rounding,
                                sr_seed, _ptr(codes), _ptr(scales), _ptr(rot), st,
                                _stream(x.device, stream)),
           name)
    return out


def osc_step(w, w_snap, d_w, d_q, window_end=False, threshold=4.0,
             n_flagged=None, stream=None):
    """mxfp4_osc_step on fp32 tensors, in place. n_flagged: optional int64
    CUDA tensor of one element to which the flag count is added."""
    for name, t in (("w", w), ("w_snap", w_snap), ("d_w", d_w), ("d_q", d_q)):
        _cuda2d(t, name)
        if t.dtype != torch.float32 or t.shape != w.shape:
            raise TypeError("%s must be float32 with the shape of w" % name)
        _on_device(t, name, w.device)
    if n_flagged is not None:
        _buffer(n_flagged, "n_flagged", torch.int64 if n_flagged.dtype != torch.uint64
                else torch.uint64, 1, w.device)
    R, C = w.shape
    _check(lib().mxfp4_osc_step(_ptr(w), _ptr(w_snap), _ptr(d_w), _ptr(d_q),
                                R, C, int(bool(window_end)), threshold,
                                _ptr(n_flagged), _stream(w.device, stream)),
           "mxfp4_osc_step")


def qramp_step(w, delta, w_snap, d_w, d_q, acc, flag, it, track_iters=30, k1=16.0,
               k2=5, n_flagged=None, stream=None):
    """mxfp4_qramp_step: one Q-Ramping iteration, in place. w, delta,
    w_snap, d_w, d_q, acc: fp32 CUDA tensors of one shape; flag: uint8 of
    that shape; n_flagged: optional int64 CUDA tensor of one element."""
    _cuda2d(w, "w")
    if w.dtype != torch.float32:
        raise TypeError("w must be float32")
    for name, t in (("delta", delta), ("w_snap", w_snap), ("d_w", d_w), ("d_q", d_q),
                    ("acc", acc)):
        _buffer(t, name, torch.float32, w.numel(), w.device)
    _buffer(flag, "flag", torch.uint8, w.numel(), w.device)
    if n_flagged is not None:
        _buffer(n_flagged, "n_flagged", torch.int64 if n_flagged.dtype != torch.uint64
                else torch.uint64, 1, w.device)
    R, C = w.shape
    _check(lib().mxfp4_qramp_step(_ptr(w), _ptr(delta), _ptr(w_snap), _ptr(d_w), _ptr(d_q),
                                  _ptr(acc), _ptr(flag), R, C, int(it), int(track_iters),
                                  float(k1), int(k2), _ptr(n_flagged),
                                  _stream(w.device, stream)),
           "mxfp4_qramp_step")


def osc_synthetic_update(w, seed, step, rel_step=1e-4, stream=None):
    """mxfp4_osc_synthetic_update on an fp32 CUDA tensor, in place."""
    _cuda2d(w, "w")
    if w.dtype != torch.float32:
        raise TypeError("w must be float32")
    R, C = w.shape
    _check(lib().mxfp4_osc_synthetic_update(_ptr(w), R, C, seed, step,
                                            rel_step, _stream(w.device, stream)),
           "mxfp4_osc_synthetic_update")


def qema_quantize(w, w_ema, beta=0.998, out=None, stream=None):
    """mxfp4_qema_quantize: update w_ema in place (fp32 CUDA tensors) and
    return the ROWS-layout (codes, scales) of the new w_ema."""
    for name, t in (("w", w), ("w_ema", w_ema)):
        _cuda2d(t, name)
        if t.dtype != torch.float32 or t.shape != w.shape:
            raise TypeError("%s must be float32 with the shape of w" % name)
    _on_device(w_ema, "w_ema", w.device)
    R, C = w.shape
    if out is None:
        out = (_empty_u8((R, C // 2), w.device), _empty_u8((R, C // 32), w.device))
    codes, scales = out
    _buffer(codes, "codes", torch.uint8, R * C // 2, w.device)
    _buffer(scales, "scales", torch.uint8, R * C // 32, w.device)
    _check(lib().mxfp4_qema_quantize(_ptr(w), _ptr(w_ema), R, C, beta,
                                     _ptr(codes), _ptr(scales),
                                     _stream(w.device, stream)),
           "mxfp4_qema_quantize")
    return codes, scales


def scales_to_blocked(scales, out=None, stream=None):
    """mxfp4_scales_to_blocked: the [rows, groups] uint8 CUDA scales in the
    blocked order of block-scaled GEMMs, returned as a
    [ceil(rows/128)*128, ceil(groups/4)*4] uint8 tensor (storage order)."""
    _cuda2d(scales, "scales")
    if scales.dtype != torch.uint8:
        raise TypeError("scales must be uint8")
    rows, groups = scales.shape
    if out is None:
        out = _empty_u8((-(-rows // 128) * 128, -(-groups // 4) * 4),
                        scales.device)
    _buffer(out, "out", torch.uint8, -(-rows // 128) * 128 * (-(-groups // 4) * 4),
            scales.device)
    _check(lib().mxfp4_scales_to_blocked(_ptr(scales), rows, groups, _ptr(out),
                                         _stream(scales.device, stream)),
           "mxfp4_scales_to_blocked")
    return out


def gemm(a_codes, a_blocked, b_codes, b_blocked, k, out=None, stream=None, status=None):
    """mxfp4_gemm: C = A B^T in fp32 for MXFP4 operands given as K-major
    codes [rows, k/2] and blocked scales (from scales_to_blocked). status:
    optional int32 CUDA tensor of one element, the timeout status word."""
    for name, t in (("a_codes", a_codes), ("a_blocked", a_blocked),
                    ("b_codes", b_codes), ("b_blocked", b_blocked)):
        _cuda2d(t, name)
        if t.dtype != torch.uint8:
            raise TypeError("%s must be uint8" % name)
    m, n = a_codes.shape[0], b_codes.shape[0]
    if a_codes.shape[1] * 2 != k or b_codes.shape[1] * 2 != k:
        raise ValueError("codes must have k/2 bytes per row")
    for name, t, rows in (("a_blocked", a_blocked, m), ("b_blocked", b_blocked, n)):
        need = -(-rows // 128) * 128 * (-(-k // 128) * 4)
        if t.numel() != need:
            raise ValueError("%s must hold %d bytes" % (name, need))
    for name, t in (("a_blocked", a_blocked), ("b_codes", b_codes),
                    ("b_blocked", b_blocked)):
        _on_device(t, name, a_codes.device)
    if out is None:
        out = torch.empty((m, n), dtype=torch.float32, device=a_codes.device)
    _buffer(out, "out", torch.float32, m * n, a_codes.device)
    st = _status_word(status, a_codes.device)
    _check(lib().mxfp4_gemm(_ptr(a_codes), _ptr(a_blocked), _ptr(b_codes),
                            _ptr(b_blocked), m, n, k, _ptr(out), st,
                            _stream(a_codes.device, stream)), "mxfp4_gemm")
    return out


def gemm_quantize_a(x, b_codes, b_blocked, rounding=RNE, seed=0, out=None, want_a=False,
                    stream=None, status=None):
    """mxfp4_gemm_quantize_a: C = Q(x) B^T in fp32, x bf16 [m, k] (k a
    multiple of 256) quantized 1x32 (rounding RNE, or SR keyed by seed)
    inside the GEMM's load stage, B given as K-major codes [n, k/2] and
    blocked scales. Returns C, or (C, a_codes, a_scales) with want_a (Q(x)
    in the ROWS layout)."""
    _cuda2d(x, "x")
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    m, k = x.shape
    for name, t in (("b_codes", b_codes), ("b_blocked", b_blocked)):
        _cuda2d(t, name)
        if t.dtype != torch.uint8:
            raise TypeError("%s must be uint8" % name)
        _on_device(t, name, x.device)
    n = b_codes.shape[0]
    if b_codes.shape[1] * 2 != k:
        raise ValueError("b_codes must have k/2 bytes per row")
    need = -(-n // 128) * 128 * (-(-k // 128) * 4)
    if b_blocked.numel() != need:
        raise ValueError("b_blocked must hold %d bytes" % need)
    d = x.device
    if out is None:
        out = torch.empty((m, n), dtype=torch.float32, device=d)
        if want_a:
            out = (out, _empty_u8((m, k // 2), d), _empty_u8((m, k // 32), d))
    c, ac, as_ = (out if want_a else (out, None, None))
    _buffer(c, "out", torch.float32, m * n, d)
    if want_a:
        _buffer(ac, "a_codes", torch.uint8, m * k // 2, d)
        _buffer(as_, "a_scales", torch.uint8, m * k // 32, d)
    st = _status_word(status, d)
    _check(lib().mxfp4_gemm_quantize_a(_ptr(x), m, n, k, rounding, seed, _ptr(b_codes),
                                       _ptr(b_blocked), _ptr(c), _ptr(ac), _ptr(as_), st,
                                       _stream(d, stream)), "mxfp4_gemm_quantize_a")
    return out


# The C names, for callers that prefer them.
mxfp4_quantize = quantize


def mxfp4_quantize_oas(x, axis=ROWS, rounding=RNE, seed=0, out=None, stream=None):
    return quantize(x, axis, rounding, seed, out, stream, oas=True)


mxfp4_dequantize = dequantize
mxfp4_double_quantize = double_quantize
mxfp4_rht_quantize = rht_quantize
mxfp4_osc_step = osc_step
mxfp4_osc_synthetic_update = osc_synthetic_update
mxfp4_qramp_step = qramp_step
mxfp4_qema_quantize = qema_quantize
mxfp4_scales_to_blocked = scales_to_blocked
mxfp4_gemm = gemm
mxfp4_gemm_quantize_a = gemm_quantize_a
mxfp4_status_string = status_string
