// C ABI of libmxfp4: argument validation on the host, then one kernel
// launch on the caller's stream. The contract of every entry point (layouts,
// ownership, errors) is stated in include/mxfp4.h.
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/mxfp4.h"
#include "launch.cuh"

namespace {

bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

// The optional status word (NULL passes).
bool aligned4(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 3u) == 0;
}

// rows, cols > 0, each at most MXFP4_MAX_DIM, product below 2^46.
bool dims_ok(int64_t rows, int64_t cols) {
  if (rows <= 0 || cols <= 0) return false;
  if (rows > MXFP4_MAX_DIM || cols > MXFP4_MAX_DIM) return false;
  return rows <= (int64_t(1) << 46) / cols;
}

bool dtype_ok(int dt) { return dt == MXFP4_F32 || dt == MXFP4_BF16; }
bool axis_ok(int a) { return a == MXFP4_ROWS || a == MXFP4_COLS; }
bool rounding_ok(int r) { return r == MXFP4_RNE || r == MXFP4_SR; }

mxfp4_status from_cuda(cudaError_t e) {
  return e == cudaSuccess ? MXFP4_OK : MXFP4_ERR_CUDA;
}

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

}  // namespace

extern "C" {

namespace {

mxfp4_status quantize_with_rule(const void* x, int dtype, int64_t rows,
                                int64_t cols, int axis, int rounding,
                                uint64_t seed, uint8_t* codes,
                                uint8_t* scales, void* stream, bool oas) {
  if (!dtype_ok(dtype) || !axis_ok(axis) || !rounding_ok(rounding))
    return MXFP4_ERR_ENUM;
  if (!x || !codes || !scales) return MXFP4_ERR_NULL;
  if (!dims_ok(rows, cols)) return MXFP4_ERR_SHAPE;
  if ((axis == MXFP4_ROWS ? cols : rows) % 32 != 0) return MXFP4_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(codes)) return MXFP4_ERR_ALIGN;
  const bool bf16 = dtype == MXFP4_BF16, sr = rounding == MXFP4_SR;
  if (axis == MXFP4_ROWS)
    return from_cuda(mxfp4::launch_quant_rows(x, bf16, rows, cols, sr, seed,
                                              codes, scales, as_stream(stream),
                                              oas));
  return from_cuda(mxfp4::launch_quant_cols(x, bf16, rows, cols, sr, seed,
                                            codes, scales, as_stream(stream),
                                            oas));
}

}  // namespace

mxfp4_status mxfp4_quantize(const void* x, int dtype, int64_t rows,
                            int64_t cols, int axis, int rounding,
                            uint64_t seed, uint8_t* codes, uint8_t* scales,
                            void* stream) {
  return quantize_with_rule(x, dtype, rows, cols, axis, rounding, seed, codes,
                            scales, stream, false);
}

mxfp4_status mxfp4_quantize_oas(const void* x, int dtype, int64_t rows,
                                int64_t cols, int axis, int rounding,
                                uint64_t seed, uint8_t* codes, uint8_t* scales,
                                void* stream) {
  return quantize_with_rule(x, dtype, rows, cols, axis, rounding, seed, codes,
                            scales, stream, true);
}

mxfp4_status mxfp4_dequantize(const uint8_t* codes, const uint8_t* scales,
                              int64_t rows, int64_t cols, int axis, void* y,
                              int out_dtype, void* stream) {
  if (!dtype_ok(out_dtype) || !axis_ok(axis)) return MXFP4_ERR_ENUM;
  if (!codes || !scales || !y) return MXFP4_ERR_NULL;
  if (!dims_ok(rows, cols)) return MXFP4_ERR_SHAPE;
  if ((axis == MXFP4_ROWS ? cols : rows) % 32 != 0) return MXFP4_ERR_SHAPE;
  if (!aligned16(codes) || !aligned16(y)) return MXFP4_ERR_ALIGN;
  return from_cuda(mxfp4::launch_dequant(codes, scales, rows * cols / 32, y,
                                         out_dtype == MXFP4_BF16,
                                         as_stream(stream)));
}

static mxfp4_status double_quantize_with_rule(const void* x, int dtype, int64_t rows,
                                              int64_t cols, uint64_t seed,
                                              uint8_t* row_codes, uint8_t* row_scales,
                                              uint8_t* col_codes, uint8_t* col_scales,
                                              void* stream, bool oas) {
  if (!dtype_ok(dtype)) return MXFP4_ERR_ENUM;
  if (!x || !row_codes || !row_scales || !col_codes || !col_scales)
    return MXFP4_ERR_NULL;
  if (!dims_ok(rows, cols) || rows % 32 || cols % 32) return MXFP4_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(row_codes) || !aligned16(col_codes))
    return MXFP4_ERR_ALIGN;
  return from_cuda(mxfp4::launch_double_quant(
      x, dtype == MXFP4_BF16, rows, cols, seed, row_codes, row_scales,
      col_codes, col_scales, as_stream(stream), oas));
}

mxfp4_status mxfp4_double_quantize(const void* x, int dtype, int64_t rows,
                                   int64_t cols, uint64_t seed,
                                   uint8_t* row_codes, uint8_t* row_scales,
                                   uint8_t* col_codes, uint8_t* col_scales,
                                   void* stream) {
  return double_quantize_with_rule(x, dtype, rows, cols, seed, row_codes, row_scales,
                                   col_codes, col_scales, stream, false);
}

mxfp4_status mxfp4_double_quantize_oas(const void* x, int dtype, int64_t rows,
                                       int64_t cols, uint64_t seed,
                                       uint8_t* row_codes, uint8_t* row_scales,
                                       uint8_t* col_codes, uint8_t* col_scales,
                                       void* stream) {
  return double_quantize_with_rule(x, dtype, rows, cols, seed, row_codes, row_scales,
                                   col_codes, col_scales, stream, true);
}

static mxfp4_status rht_quantize_with_rule(const void* x, int dtype, int64_t rows,
                                           int64_t cols, uint64_t sign_seed,
                                           int rounding, uint64_t sr_seed,
                                           uint8_t* codes, uint8_t* scales,
                                           float* rotated, int* status, void* stream,
                                           bool oas) {
  if (!dtype_ok(dtype) || !rounding_ok(rounding)) return MXFP4_ERR_ENUM;
  if (!x || !codes || !scales) return MXFP4_ERR_NULL;
  if (!dims_ok(rows, cols) || cols % 32) return MXFP4_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(codes) || (rotated && !aligned16(rotated)) ||
      !aligned4(status))
    return MXFP4_ERR_ALIGN;
  return from_cuda(mxfp4::launch_rht_quant(
      x, dtype == MXFP4_BF16, rows, cols, sign_seed, rounding == MXFP4_SR,
      sr_seed, codes, scales, rotated, status, as_stream(stream), oas));
}

mxfp4_status mxfp4_rht_quantize(const void* x, int dtype, int64_t rows,
                                int64_t cols, uint64_t sign_seed,
                                int rounding, uint64_t sr_seed,
                                uint8_t* codes, uint8_t* scales,
                                float* rotated, int* status, void* stream) {
  return rht_quantize_with_rule(x, dtype, rows, cols, sign_seed, rounding, sr_seed, codes,
                                scales, rotated, status, stream, false);
}

mxfp4_status mxfp4_rht_quantize_oas(const void* x, int dtype, int64_t rows,
                                    int64_t cols, uint64_t sign_seed,
                                    int rounding, uint64_t sr_seed,
                                    uint8_t* codes, uint8_t* scales,
                                    float* rotated, int* status, void* stream) {
  return rht_quantize_with_rule(x, dtype, rows, cols, sign_seed, rounding, sr_seed, codes,
                                scales, rotated, status, stream, true);
}

mxfp4_status mxfp4_osc_step(float* w, float* w_snap, float* d_w, float* d_q,
                            int64_t rows, int64_t cols, int window_end,
                            float threshold, unsigned long long* n_flagged,
                            void* stream) {
  if (!w || !w_snap || !d_w || !d_q) return MXFP4_ERR_NULL;
  if (!dims_ok(rows, cols) || cols % 32) return MXFP4_ERR_SHAPE;
  if (!aligned16(w) || !aligned16(w_snap) || !aligned16(d_w) ||
      !aligned16(d_q))
    return MXFP4_ERR_ALIGN;
  return from_cuda(mxfp4::launch_osc_step(w, w_snap, d_w, d_q, rows, cols,
                                          window_end != 0, threshold,
                                          n_flagged, as_stream(stream)));
}

mxfp4_status mxfp4_qramp_step(float* w, const float* delta, float* w_snap,
                              float* d_w, float* d_q, float* acc, uint8_t* flag,
                              int64_t rows, int64_t cols, int64_t iter,
                              int64_t track_iters, float k1, int64_t k2,
                              unsigned long long* n_flagged, void* stream) {
  if (!w || !delta || !w_snap || !d_w || !d_q || !acc || !flag) return MXFP4_ERR_NULL;
  if (!dims_ok(rows, cols) || cols % 32) return MXFP4_ERR_SHAPE;
  if (iter < 0 || track_iters < 0 || k2 < 1) return MXFP4_ERR_SHAPE;
  if (!aligned16(w) || !aligned16(delta) || !aligned16(w_snap) || !aligned16(d_w) ||
      !aligned16(d_q) || !aligned16(acc) || !aligned16(flag))
    return MXFP4_ERR_ALIGN;
  return from_cuda(mxfp4::launch_qramp_step(w, delta, w_snap, d_w, d_q, acc, flag, rows,
                                            cols, iter, track_iters, k1, k2, n_flagged,
                                            as_stream(stream)));
}

mxfp4_status mxfp4_osc_synthetic_update(float* w, int64_t rows, int64_t cols,
                                        uint64_t seed, uint32_t step,
                                        float rel_step, void* stream) {
  if (!w) return MXFP4_ERR_NULL;
  if (!dims_ok(rows, cols)) return MXFP4_ERR_SHAPE;
  if (!aligned16(w)) return MXFP4_ERR_ALIGN;
  return from_cuda(mxfp4::launch_osc_update(w, rows * cols, seed, step,
                                            rel_step, as_stream(stream)));
}

mxfp4_status mxfp4_qema_quantize(const float* w, float* w_ema, int64_t rows,
                                 int64_t cols, float beta, uint8_t* codes,
                                 uint8_t* scales, void* stream) {
  if (!w || !w_ema || !codes || !scales) return MXFP4_ERR_NULL;
  if (!dims_ok(rows, cols) || cols % 32) return MXFP4_ERR_SHAPE;
  if (!aligned16(w) || !aligned16(w_ema) || !aligned16(codes))
    return MXFP4_ERR_ALIGN;
  return from_cuda(mxfp4::launch_qema_quant(w, w_ema, rows, cols, beta,
                                            codes, scales, as_stream(stream)));
}

mxfp4_status mxfp4_scales_to_blocked(const uint8_t* scales, int64_t rows,
                                     int64_t groups, uint8_t* blocked,
                                     void* stream) {
  if (!scales || !blocked) return MXFP4_ERR_NULL;
  if (!dims_ok(rows, groups)) return MXFP4_ERR_SHAPE;
  if (!aligned16(blocked)) return MXFP4_ERR_ALIGN;
  return from_cuda(mxfp4::launch_scales_blocked(scales, rows, groups, blocked,
                                                as_stream(stream)));
}

mxfp4_status mxfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales,
                        const uint8_t* b_codes, const uint8_t* b_scales,
                        int64_t m, int64_t n, int64_t k, float* c,
                        int* status, void* stream) {
  if (!a_codes || !a_scales || !b_codes || !b_scales || !c)
    return MXFP4_ERR_NULL;
  if (!dims_ok(m, k) || !dims_ok(n, k) || !dims_ok(m, n) || k % 32)
    return MXFP4_ERR_SHAPE;
  if ((m + 127) / 128 > 65535) return MXFP4_ERR_SHAPE;  // grid y
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(b_codes) ||
      !aligned16(b_scales) || !aligned16(c) || !aligned4(status))
    return MXFP4_ERR_ALIGN;
  return from_cuda(mxfp4::launch_gemm_mxf4(a_codes, a_scales, b_codes,
                                           b_scales, m, n, k, c, status,
                                           as_stream(stream)));
}

mxfp4_status mxfp4_gemm_quantize_a(const void* x, int64_t m, int64_t n, int64_t k,
                                   int rounding, uint64_t seed, const uint8_t* b_codes,
                                   const uint8_t* b_scales, float* c, uint8_t* a_codes,
                                   uint8_t* a_scales, int* status, void* stream) {
  if (!rounding_ok(rounding)) return MXFP4_ERR_ENUM;
  if (!x || !b_codes || !b_scales || !c || (a_codes == nullptr) != (a_scales == nullptr))
    return MXFP4_ERR_NULL;
  if (!dims_ok(m, k) || !dims_ok(n, k) || !dims_ok(m, n) || k % 256)
    return MXFP4_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(b_codes) || !aligned16(b_scales) || !aligned16(c) ||
      !aligned16(a_codes) || !aligned4(status))
    return MXFP4_ERR_ALIGN;
  return from_cuda(mxfp4::launch_gemm_qa(x, m, n, k, rounding == MXFP4_SR, seed, b_codes,
                                         b_scales, c, a_codes, a_scales, status,
                                         as_stream(stream)));
}

const char* mxfp4_status_string(int status) {
  switch (status) {
    case MXFP4_OK: return "ok";
    case MXFP4_ERR_NULL: return "a required pointer is NULL";
    case MXFP4_ERR_SHAPE:
      return "bad shape: rows/cols must be positive, within the size limit, "
             "and the group axis a multiple of 32 (of 256 for the fused GEMM)";
    case MXFP4_ERR_ALIGN:
      return "a tensor pointer is not 16-byte aligned (a status word: 4-byte)";
    case MXFP4_ERR_ENUM: return "dtype, axis or rounding out of range";
    case MXFP4_ERR_CUDA: return "CUDA launch failed";
    default: return "unknown status";
  }
}

}  // extern "C"
