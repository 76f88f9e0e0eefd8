// Kernel launchers of libmxfp4 (internal; the C ABI in capi.cu validates
// arguments and calls these). Each returns the cudaError_t of its launch.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace mxfp4 {

// Grid size for a grid-stride kernel: resident blocks per SM x SMs of the
// current device, capped by the amount of work.
int persistent_grid(const void* kernel, int threads, size_t smem,
                    int64_t work_blocks);

// oas: the overflow-aware scale rule instead of the OCP one.
cudaError_t launch_quant_rows(const void* x, bool bf16, int64_t rows,
                              int64_t cols, bool sr, uint64_t seed,
                              uint8_t* codes, uint8_t* scales, cudaStream_t s,
                              bool oas = false);

cudaError_t launch_quant_cols(const void* x, bool bf16, int64_t rows,
                              int64_t cols, bool sr, uint64_t seed,
                              uint8_t* codes, uint8_t* scales, cudaStream_t s,
                              bool oas = false);

// Flat decode of n_groups groups (rows of the output are contiguous runs of
// whole groups in both layouts).
cudaError_t launch_dequant(const uint8_t* codes, const uint8_t* scales,
                           int64_t n_groups, void* y, bool bf16_out,
                           cudaStream_t s);

// oas: the overflow-aware scale rule in both passes.
cudaError_t launch_double_quant(const void* x, bool bf16, int64_t rows,
                                int64_t cols, uint64_t seed,
                                uint8_t* row_codes, uint8_t* row_scales,
                                uint8_t* col_codes, uint8_t* col_scales,
                                cudaStream_t s, bool oas = false);

// status: device word or nullptr; the tensor-core kernel ORs 1 into it when
// one of its bounded waits ran out.
cudaError_t launch_rht_quant(const void* x, bool bf16, int64_t rows,
                             int64_t cols, uint64_t sign_seed, bool sr,
                             uint64_t sr_seed, uint8_t* codes,
                             uint8_t* scales, float* rotated, int* status,
                             cudaStream_t s, bool oas = false);

cudaError_t launch_osc_step(float* w, float* w_snap, float* d_w, float* d_q,
                            int64_t rows, int64_t cols, bool window_end,
                            float threshold, unsigned long long* n_flagged,
                            cudaStream_t s);

// One Q-Ramping iteration (see mxfp4_qramp_step).
cudaError_t launch_qramp_step(float* w, const float* delta, float* w_snap, float* d_w,
                              float* d_q, float* acc, uint8_t* flag, int64_t rows,
                              int64_t cols, int64_t iter, int64_t track_iters, float k1,
                              int64_t k2, unsigned long long* n_flagged, cudaStream_t s);

cudaError_t launch_qema_quant(const float* w, float* w_ema, int64_t rows,
                              int64_t cols, float beta, uint8_t* codes,
                              uint8_t* scales, cudaStream_t s);

cudaError_t launch_osc_update(float* w, int64_t n, uint64_t seed,
                              uint32_t step, float rel_step, cudaStream_t s);

// Scales [rows][groups] -> the blocked order of block-scaled GEMMs.
cudaError_t launch_scales_blocked(const uint8_t* scales, int64_t rows,
                                  int64_t groups, uint8_t* blocked,
                                  cudaStream_t s);

// C[m][n] = sum_k A[m][k] B[n][k] on MXFP4 operands (K-major codes,
// blocked scales), fp32 out, on the block-scaled tensor cores; status as for
// launch_rht_quant.
cudaError_t launch_gemm_mxf4(const uint8_t* a, const uint8_t* a_scales,
                             const uint8_t* b, const uint8_t* b_scales,
                             int64_t m, int64_t n, int64_t k, float* c,
                             int* status, cudaStream_t s);

// C = Q(X) B^T with X (bf16 [m][k], k a multiple of 256) quantized 1x32
// (nearest-even, or stochastic keyed by seed) inside the GEMM's load stage;
// a_codes / a_scales (ROWS layout) receive that quantization when not null.
cudaError_t launch_gemm_qa(const void* x, int64_t m, int64_t n, int64_t k, bool sr,
                           uint64_t seed, const uint8_t* b, const uint8_t* b_scales, float* c,
                           uint8_t* a_codes, uint8_t* a_scales, int* status,
                           cudaStream_t s);

}  // namespace mxfp4
