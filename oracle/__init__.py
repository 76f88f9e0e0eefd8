"""CPU oracle for the MXFP4 block quantizer — TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct restatement of the quantizer in C (fp64),
wrapped for numpy arrays. Only the tests, the smoke check and the benchmark's
CPU baseline use it; the product path never imports it, and it shares no code
with the CUDA library. ``mxfp4_oracle.c`` names the passage each function
follows.

Arrays: bf16 tensors are numpy arrays of ``ml_dtypes.bfloat16`` (or raw
``uint16`` bits); fp32 tensors are ``float32``. Shapes are ``[rows, cols]``.

The module-level functions use the oracle built from ``mxfp4_oracle.c``;
``Oracle(path)`` wraps another build of it (the mutation tests load
deliberately broken copies this way).
"""
import ctypes
import numpy as np
import ml_dtypes

from . import build as _build

DT_F32, DT_BF16 = 0, 1
ROWS, COLS = 0, 1
RNE, SR = 0, 1

_u8p = ctypes.POINTER(ctypes.c_uint8)
_fp = ctypes.POINTER(ctypes.c_float)


def _u8(a):
    return a.ctypes.data_as(_u8p)


def _f32(a):
    return a.ctypes.data_as(_fp)


def _as_input(x):
    """Return (contiguous array, dtype code) for a bf16 or fp32 tensor."""
    x = np.ascontiguousarray(x)
    if x.dtype == ml_dtypes.bfloat16 or x.dtype == np.uint16:
        return x.view(np.uint16), DT_BF16
    if x.dtype == np.float32:
        return x, DT_F32
    raise TypeError("oracle input must be bfloat16 or float32, got %s" % x.dtype)


def _declare(L):
    vp, i64, u64, u32, i32 = (ctypes.c_void_p, ctypes.c_int64,
                              ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int)
    dbl = ctypes.c_double
    sig = {
        "orc_mix32": ([u32], u32),
        "orc_key": ([u64, u32], u32),
        "orc_counter_hash": ([u32, u64], u32),
        "orc_rand16": ([u64, u32, u64], u32),
        "orc_rand16_range": ([u64, u32, u64, i64,
                              ctypes.POINTER(ctypes.c_uint32)], None),
        "orc_scale_exponent": ([dbl], i32),
        "orc_scale_exponent_oas": ([dbl], i32),
        "orc_quantize_oas": ([vp, i32, i64, i64, i64, i32, i32, u64, _u8p, _u8p],
                             i32),
        "orc_rne_index": ([dbl], i32),
        "orc_sr_index": ([dbl, u32], i32),
        "orc_sr_count_up": ([dbl], i32),
        "orc_encode": ([dbl, i32, i32, u32], i32),
        "orc_decode": ([i32, i32], dbl),
        "orc_rht_sign": ([u64, u32], i32),
        "orc_quantize": ([vp, i32, i64, i64, i64, i32, i32, u64, _u8p, _u8p],
                         i32),
        "orc_dequantize": ([_u8p, _u8p, i64, i64, i32, vp, i32], i32),
        "orc_double_quantize": ([vp, i32, i64, i64, i64, u64, _u8p, _u8p,
                                 _u8p, _u8p], i32),
        "orc_double_quantize_oas": ([vp, i32, i64, i64, i64, u64, _u8p, _u8p,
                                     _u8p, _u8p], i32),
        "orc_rht_rotate": ([vp, i32, i64, i64, u64, _fp], i32),
        "orc_rht_quantize": ([vp, i32, i64, i64, i64, u64, i32, u64, _u8p,
                              _u8p, _fp], i32),
        "orc_rht_quantize_oas": ([vp, i32, i64, i64, i64, u64, i32, u64, _u8p,
                                  _u8p, _fp], i32),
        "orc_qramp_step": ([_fp, _fp, _fp, _fp, _fp, _fp, _u8p, i64, i64, i64, i64,
                            ctypes.c_float, i64], i64),
        "orc_osc_step": ([_fp, _fp, _fp, _fp, i64, i64, i32, ctypes.c_float],
                         i64),
        "orc_osc_synthetic_update": ([_fp, i64, i64, i64, u64, u32,
                                      ctypes.c_float], i32),
        "orc_qema_quantize": ([_fp, _fp, i64, i64, ctypes.c_float, _u8p,
                               _u8p], i32),
        "orc_scales_to_blocked": ([_u8p, i64, i64, _u8p], i32),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes, f.restype = args, res


class Oracle:
    """numpy-facing wrapper over one build of the C oracle."""

    DT_F32, DT_BF16, ROWS, COLS, RNE, SR = DT_F32, DT_BF16, ROWS, COLS, RNE, SR

    def __init__(self, path=None):
        self.path = path or _build.build()
        self.L = ctypes.CDLL(self.path)
        _declare(self.L)

    # --- scalar pieces ---------------------------------------------------
    def mix32(self, h):
        return self.L.orc_mix32(h & 0xFFFFFFFF)

    def key(self, seed, stream):
        return self.L.orc_key(seed, stream)

    def counter_hash(self, k, n):
        return self.L.orc_counter_hash(k, n)

    def rand16(self, seed, stream, i):
        return self.L.orc_rand16(seed, stream, i)

    def rand16_range(self, seed, stream, first, n):
        out = np.zeros(n, np.uint32)
        self.L.orc_rand16_range(seed, stream, first, n,
                                out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint32)))
        return out

    def scale_exponent(self, absmax):
        return self.L.orc_scale_exponent(float(absmax))

    def scale_exponent_oas(self, absmax):
        return self.L.orc_scale_exponent_oas(absmax)

    def rne_index(self, a):
        return self.L.orc_rne_index(float(a))

    def sr_index(self, a, r16):
        return self.L.orc_sr_index(float(a), r16)

    def sr_count_up(self, a):
        return self.L.orc_sr_count_up(float(a))

    def encode(self, x, e, rounding=RNE, r16=0):
        return self.L.orc_encode(float(x), e, rounding, r16)

    def decode(self, code, scale_byte):
        return self.L.orc_decode(code, scale_byte)

    def rht_sign(self, sign_seed, c):
        return self.L.orc_rht_sign(sign_seed, c)

    # --- tensor entry points ---------------------------------------------
    def quantize(self, x, axis=ROWS, rounding=RNE, seed=0, row0=0, oas=False):
        """Block quantize x [R, C]; returns (codes, scales), axis layout.
        x may be rows row0.. of a larger tensor (random numbers are keyed by
        the index in that tensor). oas: the overflow-aware scale rule."""
        x, dt = _as_input(x)
        R, C = x.shape
        codes = np.zeros(R * C // 2, np.uint8)
        scales = np.zeros(R * C // 32, np.uint8)
        fn = self.L.orc_quantize_oas if oas else self.L.orc_quantize
        rc = fn(x.ctypes.data, dt, R, C, row0, axis, rounding, seed, _u8(codes),
                _u8(scales))
        if rc != 0:
            raise ValueError("bad shape for the oracle quantizer: %s" % (x.shape,))
        if axis == ROWS:
            return codes.reshape(R, C // 2), scales.reshape(R, C // 32)
        return codes.reshape(C, R // 2), scales.reshape(C, R // 32)

    def dequantize(self, codes, scales, rows, cols, axis=ROWS,
                   out_dtype="bf16"):
        """Decode to [rows, cols] (ROWS) or [cols, rows] (COLS)."""
        codes = np.ascontiguousarray(codes, np.uint8).reshape(-1)
        scales = np.ascontiguousarray(scales, np.uint8).reshape(-1)
        shape = (rows, cols) if axis == ROWS else (cols, rows)
        if out_dtype == "bf16":
            y, dt = np.zeros(shape, np.uint16), DT_BF16
        else:
            y, dt = np.zeros(shape, np.float32), DT_F32
        self.L.orc_dequantize(_u8(codes), _u8(scales), rows, cols, axis,
                              y.ctypes.data, dt)
        return y.view(ml_dtypes.bfloat16) if dt == DT_BF16 else y

    def double_quantize(self, x, seed, row0=0, oas=False):
        """Q_S(32x1)(Q_D(1x32)(x)): (row codes, row scales, col codes,
        col scales); oas: the overflow-aware scale in both passes."""
        x, dt = _as_input(x)
        R, C = x.shape
        out = [np.zeros(R * C // 2, np.uint8), np.zeros(R * C // 32, np.uint8),
               np.zeros(R * C // 2, np.uint8), np.zeros(R * C // 32, np.uint8)]
        fn = self.L.orc_double_quantize_oas if oas else self.L.orc_double_quantize
        rc = fn(x.ctypes.data, dt, R, C, row0, seed, *[_u8(a) for a in out])
        if rc != 0:
            raise ValueError("bad shape for the oracle double quantizer")
        return (out[0].reshape(R, C // 2), out[1].reshape(R, C // 32),
                out[2].reshape(C, R // 2), out[3].reshape(C, R // 32))

    def rht_rotate(self, x, sign_seed):
        x, dt = _as_input(x)
        R, C = x.shape
        y = np.zeros((R, C), np.float32)
        if self.L.orc_rht_rotate(x.ctypes.data, dt, R, C, sign_seed, _f32(y)):
            raise ValueError("bad shape for the oracle rotation")
        return y

    def rht_quantize(self, x, sign_seed, rounding, sr_seed, row0=0, oas=False):
        """Rotate each 1x32 row group, quantize along rows: (codes, scales,
        rotated fp32); oas: the overflow-aware scale."""
        x, dt = _as_input(x)
        R, C = x.shape
        codes = np.zeros(R * C // 2, np.uint8)
        scales = np.zeros(R * C // 32, np.uint8)
        y = np.zeros((R, C), np.float32)
        fn = self.L.orc_rht_quantize_oas if oas else self.L.orc_rht_quantize
        if fn(x.ctypes.data, dt, R, C, row0, sign_seed, rounding, sr_seed, _u8(codes),
              _u8(scales), _f32(y)):
            raise ValueError("bad shape for the oracle rotation")
        return codes.reshape(R, C // 2), scales.reshape(R, C // 32), y

    def osc_step(self, w, w_snap, d_w, d_q, window_end=False, threshold=4.0):
        """One tracker step on fp32 arrays, in place; returns the flags."""
        for a in (w, w_snap, d_w, d_q):
            if a.dtype != np.float32 or not a.flags.c_contiguous:
                raise TypeError("oscillation state must be contiguous float32")
        R, C = w.shape
        n = self.L.orc_osc_step(_f32(w), _f32(w_snap), _f32(d_w), _f32(d_q),
                                R, C, int(bool(window_end)), threshold)
        if n < 0:
            raise ValueError("bad shape for the oracle tracker")
        return int(n)

    def qramp_step(self, w, delta, w_snap, d_w, d_q, acc, flag, it, track_iters=30,
                   k1=16.0, k2=5):
        """One Q-Ramping iteration on fp32 arrays (flag: uint8), in place;
        returns the number of weights flagged at this iteration."""
        for a in (w, delta, w_snap, d_w, d_q, acc):
            if a.dtype != np.float32 or not a.flags.c_contiguous or a.shape != w.shape:
                raise TypeError("Q-Ramping state must be contiguous float32 of w's shape")
        if flag.dtype != np.uint8 or not flag.flags.c_contiguous or flag.shape != w.shape:
            raise TypeError("flag must be contiguous uint8 of w's shape")
        R, C = w.shape
        n = self.L.orc_qramp_step(_f32(w), _f32(delta), _f32(w_snap), _f32(d_w), _f32(d_q),
                                  _f32(acc), _u8(flag), R, C, it, track_iters, k1, k2)
        if n < 0:
            raise ValueError("bad arguments for the oracle Q-Ramping step")
        return int(n)

    def osc_synthetic_update(self, w, seed, step, rel_step=1e-4, row0=0):
        if w.dtype != np.float32 or not w.flags.c_contiguous:
            raise TypeError("w must be contiguous float32")
        R, C = w.shape
        self.L.orc_osc_synthetic_update(_f32(w), R, C, row0, seed, step,
                                        rel_step)


    def qema_quantize(self, w, w_ema, beta=0.998):
        """Q-EMA: update w_ema in place, return its 1x32 RNE (codes, scales)."""
        for a in (w, w_ema):
            if a.dtype != np.float32 or not a.flags.c_contiguous:
                raise TypeError("Q-EMA arrays must be contiguous float32")
        R, C = w.shape
        codes = np.zeros(R * C // 2, np.uint8)
        scales = np.zeros(R * C // 32, np.uint8)
        if self.L.orc_qema_quantize(_f32(w), _f32(w_ema), R, C, beta,
                                    _u8(codes), _u8(scales)):
            raise ValueError("bad shape for the oracle Q-EMA")
        return codes.reshape(R, C // 2), scales.reshape(R, C // 32)

    def scales_to_blocked(self, scales):
        """The [rows, groups] scale bytes in the blocked layout of
        block-scaled GEMMs, as a [ceil(rows/128)*128, ceil(groups/4)*4]
        uint8 array (the bytes in storage order)."""
        s = np.ascontiguousarray(scales, np.uint8)
        rows, groups = s.shape
        pr, pg = -(-rows // 128) * 128, -(-groups // 4) * 4
        out = np.zeros(pr * pg, np.uint8)
        if self.L.orc_scales_to_blocked(_u8(s.reshape(-1)), rows, groups, _u8(out)):
            raise ValueError("bad shape for the blocked scale layout")
        return out.reshape(pr, pg)


    def gemm(self, a_codes, a_scales, b_codes, b_scales, k):
        """C = A B^T in fp64 for two K-major MXFP4 operands given as codes
        [rows, k/2] and plain scales [rows, k/32]: both are dequantized
        exactly (each value is an E2M1 magnitude times a power of two) and
        multiplied with numpy's fp64 matmul."""
        m, n = a_codes.shape[0], b_codes.shape[0]
        da = self.dequantize(a_codes, a_scales, m, k, ROWS, "f32").astype(np.float64)
        db = self.dequantize(b_codes, b_scales, n, k, ROWS, "f32").astype(np.float64)
        return da @ db.T


_default = None


def default():
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def __getattr__(name):
    # Module-level access (oracle.quantize, ...) goes to the default build.
    if not name.startswith("_") and hasattr(Oracle, name):
        return getattr(default(), name)
    raise AttributeError(name)
