// Randomized Hadamard rotation of 1x32 row groups fused with MXFP4 1x32
// quantization (sm_100a).
//
// Sources: "ALTO MXFP4 training — Weight de-oscillation — What does it
// mean?", Jargon: Randomized Hadamard transform (a random rotation before
// quantizing spreads one large value over many entries); "Microscaling FP4
// Quantization: MR-GPTQ Achieves 6x Speedup", section "FP4 Quantization with
// Micro-Rotated GPTQ Algorithm" (block-wise Hadamard transforms, fused so
// that the rotation costs no extra pass).
//
// y_g = (1/sqrt(32)) * H32 * (s .* x_g) with H32 the Sylvester matrix
// (H[j][k] = (-1)^popcount(j & k)) and s_c = -1 iff bit 31 of
// mix(K(sign_seed, 1) + c) is set. One thread owns one group: the signs are
// folded into the loaded bits as an XOR, the transform is an in-register
// radix-2 butterfly (5 stages x 16 add/sub pairs, no shuffles), the absmax
// needs no reduction across threads, and the thread writes its group's 16
// code bytes and scale. A CTA covers 8 column groups x 32 rows and walks down
// the rows, so the 256 sign bits of its columns are hashed once per CTA (one
// hash per thread, combined with a warp ballot).
#include "launch.cuh"
#include "mxfp4_device.cuh"

namespace mxfp4 {

namespace {

constexpr int kRhtThreads = 256;
constexpr int kRhtGroupsX = 8;  // column groups per CTA
constexpr int kRhtRowsY = 32;   // rows per CTA step

// fp32 nearest to 1/sqrt(32).
constexpr float kInvSqrt32 = 0.17677669529663687f;

template <bool BF16, bool SR, bool ROT>
__global__ void __launch_bounds__(kRhtThreads, BF16 ? 4 : 2)
    k_rht_quant(const void* __restrict__ x, int64_t rows, int64_t cols,
                uint32_t sign_key, RngKey key, uint8_t* __restrict__ codes,
                uint8_t* __restrict__ scales, float* __restrict__ rotated) {
  __shared__ uint32_t sign_bits[kRhtGroupsX];
  const int64_t n_cgroups = cols / 32;
  {
    // warp w hashes the 32 column signs of column group blockIdx.x*8 + w
    // (bit 31 of mix32 is bit 31 of mix32_pre)
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t c = uint32_t((int64_t(blockIdx.x) * kRhtGroupsX + w) * 32 + lane);
    const unsigned neg = __ballot_sync(0xFFFFFFFFu, (mix32_pre(sign_key + c) >> 31) != 0);
    if (lane == 0) sign_bits[w] = neg;
  }
  __syncthreads();
  const int kk = threadIdx.x & (kRhtGroupsX - 1);
  const int rr = threadIdx.x / kRhtGroupsX;
  const int64_t k = int64_t(blockIdx.x) * kRhtGroupsX + kk;
  if (k >= n_cgroups) return;
  const uint32_t neg = sign_bits[kk];
  // XOR masks that flip the sign bit of the elements whose column sign is -1
  uint32_t flip[BF16 ? 16 : 32];
  if (BF16) {
#pragma unroll
    for (int i = 0; i < 16; ++i)
      flip[i] = ((neg >> (2 * i)) & 1u) << 15 | ((neg >> (2 * i + 1)) & 1u) << 31;
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) flip[i] = ((neg >> i) & 1u) << 31;
  }
  for (int64_t r = int64_t(blockIdx.y) * kRhtRowsY + rr; r < rows;
       r += int64_t(gridDim.y) * kRhtRowsY) {
    const int64_t e0 = r * cols + k * 32;  // first element of the group
    float y[32];
    if (BF16) {
      const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + e0);
      uint4 q[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) q[i] = ld_l1(p + i);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t w4[4] = {q[i].x ^ flip[4 * i], q[i].y ^ flip[4 * i + 1],
                                q[i].z ^ flip[4 * i + 2], q[i].w ^ flip[4 * i + 3]};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          y[8 * i + 2 * j] = bf16_lo(w4[j]);
          y[8 * i + 2 * j + 1] = bf16_hi(w4[j]);
        }
      }
    } else {
      const uint4* p = reinterpret_cast<const uint4*>(static_cast<const float*>(x) + e0);
      uint4 q[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) q[i] = ld_l1(p + i);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        y[4 * i] = __uint_as_float(q[i].x ^ flip[4 * i]);
        y[4 * i + 1] = __uint_as_float(q[i].y ^ flip[4 * i + 1]);
        y[4 * i + 2] = __uint_as_float(q[i].z ^ flip[4 * i + 2]);
        y[4 * i + 3] = __uint_as_float(q[i].w ^ flip[4 * i + 3]);
      }
    }
    // Sylvester Hadamard butterfly: stage h pairs j with j + h (j & h == 0).
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if ((j & h) == 0) {
          const float a = y[j], b = y[j + h];
          y[j] = a + b;
          y[j + h] = a - b;
        }
      }
    }
    // The rotated value is fl(z * c), z the butterfly output and c = 1/sqrt(32),
    // and the quantizer scales it by 2^-e. Without the rotated output both
    // multiplies fold into one, fl(z * (c 2^-e)) = fl(z c) 2^-e (a power of
    // two commutes with rounding; a result below the normal range only
    // differs in values that quantize to 0 either way), and the group
    // maximum is fl(max|z| c), rounding being monotonic.
    uint32_t amax;
    if (ROT) {
      amax = 0;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        y[j] *= kInvSqrt32;
        amax = max(amax, __float_as_uint(y[j]) & 0x7FFFFFFFu);
      }
      float4* o = reinterpret_cast<float4*>(rotated + e0);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        __stcs(o + i, make_float4(y[4 * i], y[4 * i + 1], y[4 * i + 2], y[4 * i + 3]));
    } else {
      float zmax = 0.0f;
#pragma unroll
      for (int j = 0; j < 32; ++j) zmax = absmax_nan(y[j], zmax);
      amax = __float_as_uint(zmax * kInvSqrt32);
    }
    const uint32_t sb = scale_byte(amax);
    const float mul = ROT ? inv_scale(sb) : inv_scale(sb) * kInvSqrt32;
    uint32_t wq[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = y[8 * q + j] * mul;
      if (SR) {
        const uint64_t p0 = uint64_t(e0 >> 1) + 4 * q;
        const uint32_t kh = inner_key(key, uint32_t(p0 >> 32));
        uint32_t h[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) h[t] = mix32_pre(kh + uint32_t(p0) + t);
        wq[q] = e2m1x8_sr(v, h);
      } else {
        wq[q] = e2m1x8_rn(v);
      }
    }
    if (sb == 0xFFu) wq[0] = wq[1] = wq[2] = wq[3] = 0;
    *reinterpret_cast<uint4*>(codes + e0 / 2) = make_uint4(wq[0], wq[1], wq[2], wq[3]);
    scales[e0 / 32] = uint8_t(sb);
  }
}

template <bool BF16, bool SR, bool ROT>
cudaError_t rht_impl(const void* x, int64_t rows, int64_t cols,
                     uint32_t sign_key, RngKey key, uint8_t* codes,
                     uint8_t* scales, float* rotated, cudaStream_t s) {
  auto kern = k_rht_quant<BF16, SR, ROT>;
  const int64_t gx = (cols / 32 + kRhtGroupsX - 1) / kRhtGroupsX;
  const int64_t row_blocks = (rows + kRhtRowsY - 1) / kRhtRowsY;
  const int target = persistent_grid(reinterpret_cast<const void*>(kern),
                                     kRhtThreads, 0, int64_t(1) << 40);
  int64_t gy = (target + gx - 1) / gx;
  if (gy > row_blocks) gy = row_blocks;
  if (gy > 65535) gy = 65535;
  if (gy < 1) gy = 1;
  if (gx > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  kern<<<grid, kRhtThreads, 0, s>>>(x, rows, cols, sign_key, key, codes,
                                    scales, rotated);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rht_quant(const void* x, bool bf16, int64_t rows,
                             int64_t cols, uint64_t sign_seed, bool sr,
                             uint64_t sr_seed, uint8_t* codes,
                             uint8_t* scales, float* rotated,
                             cudaStream_t s) {
  const uint32_t sign_key = stream_key(sign_seed, 1);
  const RngKey key = make_key(sr_seed, 0);
  const bool rot = rotated != nullptr;
#define MXFP4_RHT(B, S, R) \
  return rht_impl<B, S, R>(x, rows, cols, sign_key, key, codes, scales, rotated, s)
  if (bf16) {
    if (sr) {
      if (rot) MXFP4_RHT(true, true, true);
      MXFP4_RHT(true, true, false);
    }
    if (rot) MXFP4_RHT(true, false, true);
    MXFP4_RHT(true, false, false);
  }
  if (sr) {
    if (rot) MXFP4_RHT(false, true, true);
    MXFP4_RHT(false, true, false);
  }
  if (rot) MXFP4_RHT(false, false, true);
  MXFP4_RHT(false, false, false);
#undef MXFP4_RHT
}

}  // namespace mxfp4
