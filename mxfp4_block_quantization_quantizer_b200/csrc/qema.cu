// Q-EMA step fused with the 1x32 RNE quantization of the averaged weight
// (sm_100a).
//
// Source: "Oscillation-Reduced MXFP4 Training for Vision Transformers"
// rebuttal, Question 4 (the forward pass quantizes an exponential moving
// average of each linear layer's weight, updated with the parameters) and
// the hyper-parameter answers (beta in [0.997, 0.999], default 0.998).
//
// One pass over fp32 w and w_ema: w_ema = beta * w_ema + (1 - beta) * w
// (two fp32 products and an fp32 sum, no fused multiply-add), stored back,
// and the new values quantized along 1x32 row groups (RNE, saturating)
// straight from registers. 12.53 bytes move per element. Four threads share
// a group (8 elements, two 16-byte loads per array); the group maximum comes
// from quad shuffles. Each quad loads kQemaU groups before any arithmetic.
#include "launch.cuh"
#include "mxfp4_device.cuh"

namespace mxfp4 {

namespace {

constexpr int kQemaThreads = 256;
constexpr int kQemaU = 4;  // groups per quad in flight (1: 4% slower)

__global__ void __launch_bounds__(kQemaThreads)
    k_qema_quant(const float* __restrict__ w, float* __restrict__ w_ema,
                 int64_t n_groups, float beta, uint8_t* __restrict__ codes,
                 uint8_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int sub = lane & 3;
  const int64_t warp = (int64_t(blockIdx.x) * kQemaThreads + threadIdx.x) >> 5;
  const int64_t chunk = (int64_t(gridDim.x) * kQemaThreads) >> 2;
  const int64_t my = warp * 8 + (lane >> 2);
  const float omb = __fsub_rn(1.0f, beta);
  for (int64_t base = 0; base < n_groups; base += chunk * kQemaU) {
    // every load of this pass first: kQemaU groups per quad in flight
    uint4 w0[kQemaU], w1[kQemaU], m0[kQemaU], m1[kQemaU];
#pragma unroll
    for (int u = 0; u < kQemaU; ++u) {
      const int64_t g = base + u * chunk + my;
      const int64_t e = (g < n_groups ? g : 0) * 32 + sub * 8;
      w0[u] = ld_l1(w + e), w1[u] = ld_l1(w + e + 4);
      m0[u] = ld_l1(w_ema + e), m1[u] = ld_l1(w_ema + e + 4);
    }
#pragma unroll
    for (int u = 0; u < kQemaU; ++u) {
      const int64_t g = base + u * chunk + my;
      const bool ok = g < n_groups;
      const int64_t e = (ok ? g : 0) * 32 + sub * 8;
      const uint32_t wb[8] = {w0[u].x, w0[u].y, w0[u].z, w0[u].w,
                              w1[u].x, w1[u].y, w1[u].z, w1[u].w};
      const uint32_t mb[8] = {m0[u].x, m0[u].y, m0[u].z, m0[u].w,
                              m1[u].x, m1[u].y, m1[u].z, m1[u].w};
      float v[8];
      uint32_t amax = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        v[j] = __fadd_rn(__fmul_rn(beta, __uint_as_float(mb[j])),
                         __fmul_rn(omb, __uint_as_float(wb[j])));
        amax = max(amax, __float_as_uint(v[j]) & 0x7FFFFFFFu);
      }
      amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
      amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
      if (!ok) continue;
      float4* out = reinterpret_cast<float4*>(w_ema + e);
      __stcs(out, make_float4(v[0], v[1], v[2], v[3]));
      __stcs(out + 1, make_float4(v[4], v[5], v[6], v[7]));
      const uint32_t sb = scale_byte(amax);
      const float mul = inv_scale(sb);
      float q[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) q[j] = v[j] * mul;
      const uint32_t word = sb == 0xFFu ? 0u : e2m1x8_rn(q);
      reinterpret_cast<uint32_t*>(codes)[g * 4 + sub] = word;
      if (sub == 0) scales[g] = static_cast<uint8_t>(sb);
    }
  }
}

}  // namespace

cudaError_t launch_qema_quant(const float* w, float* w_ema, int64_t rows,
                              int64_t cols, float beta, uint8_t* codes,
                              uint8_t* scales, cudaStream_t s) {
  const int64_t n_groups = rows * cols / kGroup;
  const int64_t per_block = int64_t(kQemaThreads / 4) * kQemaU;
  const int64_t blocks = (n_groups + per_block - 1) / per_block;
  const int grid = persistent_grid(reinterpret_cast<const void*>(k_qema_quant),
                                   kQemaThreads, 0, blocks);
  k_qema_quant<<<grid, kQemaThreads, 0, s>>>(w, w_ema, n_groups, beta, codes,
                                             scales);
  return cudaGetLastError();
}

}  // namespace mxfp4
