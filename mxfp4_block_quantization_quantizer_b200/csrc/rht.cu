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
// hash per thread, combined with a warp ballot). This kernel serves fp32
// inputs; bf16 inputs take the tensor-core kernel below.
#include "launch.cuh"
#include "mxfp4_device.cuh"
#include "tc_common.cuh"

namespace mxfp4 {

namespace {

constexpr int kRhtThreads = 256;
constexpr int kRhtGroupsX = 8;  // column groups per CTA
constexpr int kRhtRowsY = 32;   // rows per CTA step

// fp32 nearest to 1/sqrt(32).
constexpr float kInvSqrt32 = 0.17677669529663687f;

// Stochastic codes of the 8 values y[j] mul (mul > 0), pair k taking its
// random numbers from the hash of counter c0 + k, as e2m1x8_sr: the
// magnitude is formed as |y[j]| mul, the same product as |y[j] mul|
// (nearest rounding is symmetric), so the absolute value rides on the
// multiply, and the sign comes from y[j]; each pair's hash is formed where
// it is used.
__device__ __forceinline__ uint32_t e2m1x8_sr_mul(const float* y, float mul, uint32_t c0) {
  uint32_t out = 0;
#pragma unroll
  for (int k = 3; k >= 0; --k) {
    uint32_t ne, no;
    sr_noise64_pair(mix32_pre(mad_u32(uint32_t(k), 1u, c0)), ne, no);
#pragma unroll
    for (int par = 1; par >= 0; --par) {
      const float yv = y[2 * k + par];
      const float a = fabsf(yv) * mul;
      float ry = fmaxf(a, __fmaf_ru(a, 0.5f, 0.5f));
      ry = fminf(ry, 6.0f);  // |v| >= 6 saturates to 6
      out = push_code(out, (__float_as_uint(ry) * 64u + (par ? no : ne)) |
                               (__float_as_uint(yv) & 0x80000000u));
    }
  }
  return out;
}

// fp32 inputs (bf16 inputs take the tensor-core kernel below).
template <bool SR, bool ROT, bool OAS>
__global__ void __launch_bounds__(kRhtThreads, 2)
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
  uint32_t flip[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) flip[i] = ((neg >> i) & 1u) << 31;
  for (int64_t r = int64_t(blockIdx.y) * kRhtRowsY + rr; r < rows;
       r += int64_t(gridDim.y) * kRhtRowsY) {
    const int64_t e0 = r * cols + k * 32;  // first element of the group
    float y[32];
    {
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
    const uint32_t sb = OAS ? scale_byte_oas(amax) : scale_byte(amax);
    const float mul = ROT ? inv_scale(sb) : inv_scale(sb) * kInvSqrt32;
    // the group's 16 pairs share the high word of their index
    const uint64_t pg = uint64_t(e0 >> 1);
    const uint32_t kh = SR ? inner_key(key, uint32_t(pg >> 32)) : 0u;
    uint32_t wq[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (SR) {
        wq[q] = e2m1x8_sr_mul(y + 8 * q, mul, kh + uint32_t(pg) + 4 * q);
      } else {
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = y[8 * q + j] * mul;
        wq[q] = e2m1x8_rn(v);
      }
    }
    if (sb == 0xFFu) wq[0] = wq[1] = wq[2] = wq[3] = 0;
    *reinterpret_cast<uint4*>(codes + e0 / 2) = make_uint4(wq[0], wq[1], wq[2], wq[3]);
    scales[e0 / 32] = uint8_t(sb);
  }
}

// ---------------------------------------------------------------------------
// The rotation on the tensor cores (bf16 inputs). Over a tile of 128 rows
// and 8 column groups the rotation of group g is D_g = X_g B_g^T with
// B_g = H diag(s_g): X_g the group's 128 x 32 bf16 inputs, B_g 32 x 32
// entries +-1 (exact in bf16), D_g the unnormalised z of all 128 rows, an
// M = 128, N = 32, K = 32 product (two K = 16 tcgen05.mma of kind::f16 with
// fp32 accumulation in tensor memory). The products are exact and only the
// order of the fp32 additions differs from the butterfly's. z then goes
// through the same quantization as above.
//   warp 0: B_g of the tile's column block (all lanes, rebuilt only when
//           the block changes) and TMA loads of X (lane 0) into a 2-stage
//           ring, X as four 128-byte-swizzled boxes of 128 rows x 64
//           columns (two groups per 128-byte row);
//   warp 1: one thread issues a tile's 16 MMAs into one of two 256-column
//           accumulators;
//   warps 2-17: epilogue; warp w reads lane quarter w % 4 (32 rows, the
//           quarter a warp can reach) of groups 2 ((w - 2) / 4) and the next
//           with tcgen05.ld, one group per thread at a time.
// CTA i takes a contiguous run of the tiles ordered column block first, so
// its column block (and B) rarely changes. STAGED (nearest rounding without
// the rotated output, whose quantization is short): the four warps of a lane
// quarter stage their codes in shared memory and write whole 128-byte row
// segments; otherwise each thread stores its group's 16 bytes directly,
// which lets the longer stochastic quantization of the warps overlap.
// ---------------------------------------------------------------------------

constexpr int kRtStages = 2;
constexpr int kRtEpiWarps = 16;
constexpr int kRtThreads = 32 * (2 + kRtEpiWarps);
constexpr int kRtGroups = 8;          // 1x32 groups per tile row
constexpr int kRtAccBufs = 2;         // 256-column accumulators
// kind::f16 instruction descriptor: fp32 D (bit 4), bf16 A and B (bits 7,
// 10), both K-major, N/8 at bit 17, M/16 at bit 24
constexpr uint32_t kIdescBf16M128N32 = (1u << 4) | (1u << 7) | (1u << 10) |
                                       (uint32_t(32 >> 3) << 17) | (uint32_t(128 >> 4) << 24);

struct __align__(1024) RhtSmem {
  uint8_t x[kRtStages][kRtGroups / 2][128][128];  // X: group pairs, 128 rows x 128 B
  uint8_t h[kRtStages][kRtGroups][4][32][16];     // B_g: K chunks x 32 rows x 16 B
  uint4 out_codes[2][4][32][kRtGroups];           // staged codes [tile parity][quarter][row]
  uint8_t out_scales[2][4][32][kRtGroups];
  unsigned long long full[kRtStages], empty[kRtStages], acc_full[kRtAccBufs],
      acc_empty[kRtAccBufs], drain;
  uint32_t tmem_base;
  int failed;
};

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// 32 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* d) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, "
      "%7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, "
      "%21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]), "=r"(d[4]), "=r"(d[5]),
        "=r"(d[6]), "=r"(d[7]), "=r"(d[8]), "=r"(d[9]), "=r"(d[10]), "=r"(d[11]),
        "=r"(d[12]), "=r"(d[13]), "=r"(d[14]), "=r"(d[15]), "=r"(d[16]), "=r"(d[17]),
        "=r"(d[18]), "=r"(d[19]), "=r"(d[20]), "=r"(d[21]), "=r"(d[22]), "=r"(d[23]),
        "=r"(d[24]), "=r"(d[25]), "=r"(d[26]), "=r"(d[27]), "=r"(d[28]), "=r"(d[29]),
        "=r"(d[30]), "=r"(d[31])
      : "r"(taddr));
}

// Quantize the rotated group z (unnormalised) of row r, columns c0 ..
// c0+31, as k_rht_quant does; the codes and scale go to *oc / *os when
// STAGED, else to global memory; ROT also writes z / sqrt(32).
template <bool SR, bool ROT, bool STAGED, bool OAS>
__device__ __forceinline__ void rht_tc_quantize_group(float* y, int64_t r, int64_t c0,
                                                      int64_t cols, RngKey key, bool failed,
                                                      uint8_t* __restrict__ codes,
                                                      uint8_t* __restrict__ scales,
                                                      float* __restrict__ rotated, uint4* oc,
                                                      uint8_t* os) {
  const int64_t e0 = r * cols + c0;
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
    for (int j = 0; j < 32; j += 2) zmax = absmax3_nan(y[j], y[j + 1], zmax);
    amax = __float_as_uint(zmax * kInvSqrt32);
  }
  const uint32_t sb = failed ? 0xFFu : (OAS ? scale_byte_oas(amax) : scale_byte(amax));
  const float mul = ROT ? inv_scale(sb) : inv_scale(sb) * kInvSqrt32;
  // the group's 16 pairs start at a multiple of 16, so they share the high
  // word of their index (2^32 is a multiple of 16): one inner key
  const uint64_t pg = uint64_t(e0 >> 1);
  const uint32_t kh = SR ? inner_key(key, uint32_t(pg >> 32)) : 0u;
  uint32_t wq[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    if (SR) {
      wq[q] = e2m1x8_sr_mul(y + 8 * q, mul, kh + uint32_t(pg) + 4 * q);
    } else {
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = y[8 * q + j] * mul;
      wq[q] = e2m1x8_rn(v);
    }
  }
  if (sb == 0xFFu) wq[0] = wq[1] = wq[2] = wq[3] = 0;
  if (STAGED) {
    *oc = make_uint4(wq[0], wq[1], wq[2], wq[3]);
    *os = uint8_t(sb);
  } else {
    *reinterpret_cast<uint4*>(codes + e0 / 2) = make_uint4(wq[0], wq[1], wq[2], wq[3]);
    scales[e0 / 32] = uint8_t(sb);
  }
}

template <bool SR, bool ROT, bool STAGED, bool OAS>
__global__ void __launch_bounds__(kRtThreads, 1)
    k_rht_tc(const __grid_constant__ CUtensorMap tm_x, int64_t rows, int64_t cols,
             uint32_t sign_key, RngKey key, uint8_t* __restrict__ codes,
             uint8_t* __restrict__ scales, float* __restrict__ rotated,
             int* __restrict__ status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the 128-byte swizzle wants 1024-byte aligned tiles (1 KB of slack)
  RhtSmem& sm = *reinterpret_cast<RhtSmem*>(
      smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n_rt = (rows + 127) / 128;
  const int64_t n_cb = (cols + 32 * kRtGroups - 1) / (32 * kRtGroups);
  const int64_t n_tiles = n_rt * n_cb;
  const int64_t t_begin = n_tiles * blockIdx.x / gridDim.x;
  const int64_t t_end = n_tiles * (blockIdx.x + 1) / gridDim.x;

  if (tid == 0) {
    for (int s = 0; s < kRtStages; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.full[s])));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.empty[s])));
    }
    for (int b = 0; b < kRtAccBufs; ++b) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.acc_full[b])));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(&sm.acc_empty[b])),
                   "r"(kRtEpiWarps));
    }
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.drain)));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    sm.failed = 0;
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&sm.tmem_base)), "r"(32 * kRtGroups * kRtAccBufs));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;");
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // row j = lane of H: bit k set iff popcount(j & k) is odd
    uint32_t hpar = 0;
#pragma unroll
    for (int k = 0; k < 32; ++k) hpar |= uint32_t(__popc(lane & k) & 1) << k;
    int64_t slot_cb[kRtStages];
#pragma unroll
    for (int s = 0; s < kRtStages; ++s) slot_cb[s] = -1;
    uint32_t s = 0, ph = 0;
    // stages with a load issued and the phase parity of each one's last
    // load (the same in every lane): every load lands before the CTA ends
    uint32_t issued = 0, last_ph = 0;
    int64_t cb = t_begin / n_rt, rt = t_begin % n_rt;
    for (int64_t t = t_begin; t < t_end; ++t, rt = rt + 1 == n_rt ? 0 : rt + 1,
                 cb += rt == 0 ? 1 : 0) {
      // runs ahead of the epilogue; the lanes agree on the outcome
      if (!__all_sync(0xFFFFFFFFu,
                      wait_parity_or_failed<true>(&sm.empty[s], ph ^ 1u, &sm.failed))) {
        atomicExch(&sm.failed, 1);
        break;
      }
      if (slot_cb[s] != cb) {
        // column signs (bit 31 of mix32 is bit 31 of mix32_pre), one ballot
        // per group, then row `lane` of every B_g
        uint32_t neg[kRtGroups];
#pragma unroll
        for (int g = 0; g < kRtGroups; ++g) {
          const int64_t c = cb * (32 * kRtGroups) + 32 * g + lane;
          const bool n = c < cols && (mix32_pre(sign_key + uint32_t(c)) >> 31) != 0;
          neg[g] = __ballot_sync(0xFFFFFFFFu, n);
        }
#pragma unroll
        for (int g = 0; g < kRtGroups; ++g) {
          const uint32_t nb = hpar ^ neg[g];  // bit k: B_g[lane][k] < 0
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int k = 8 * cc + 2 * i;
              w[i] = (0x3F80u | (((nb >> k) & 1u) << 15)) |
                     ((0x3F80u | (((nb >> (k + 1)) & 1u) << 15)) << 16);
            }
            *reinterpret_cast<uint4*>(&sm.h[s][g][cc][lane][0]) =
                make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
        slot_cb[s] = cb;
      }
      // B_g was written through the generic proxy; the MMAs read it through
      // the async proxy
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      issued |= 1u << s;
      last_ph = (last_ph & ~(1u << s)) | (ph << s);
      if (lane == 0) {
        expect_tx(&sm.full[s], (kRtGroups / 2) * 128 * 128);
#pragma unroll
        for (int p = 0; p < kRtGroups / 2; ++p)
          tma_load_2d(&sm.x[s][p][0][0], &tm_x, int((cb * (32 * kRtGroups) + 64 * p) * 2),
                      int(rt * 128), &sm.full[s]);
      }
      __syncwarp();
      if (++s == kRtStages) {
        s = 0;
        ph ^= 1u;
      }
    }
    // drain (immediate unless a wait ran out)
    if (lane == 0)
      for (uint32_t st = 0; st < kRtStages; ++st)
        if ((issued >> st) & 1u) wait_parity(&sm.full[st], (last_ph >> st) & 1u);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint64_t x_d0 = smem_desc_sw128(&sm.x[0][0][0][0]);
      const uint64_t h_d0 = smem_desc(&sm.h[0][0][0][0][0], 32 * 16, 128);
      // start-address steps (16-byte units): X stage, group pair, second
      // group of a pair (64 B into the 128-byte row), K = 16 (32 B); B
      // stage, group, K = 16 (two 512-byte K chunks)
      constexpr uint32_t kXs = ((kRtGroups / 2) * 128 * 128) >> 4, kXp = (128 * 128) >> 4,
                         kXh = 64 >> 4, kXk = 32 >> 4;
      constexpr uint32_t kHs = (kRtGroups * 4 * 32 * 16) >> 4, kHg = (4 * 32 * 16) >> 4,
                         kHk = (2 * 32 * 16) >> 4;
      uint32_t s = 0, ph = 0, b = 0, bph = 0;
      for (int64_t t = t_begin; t < t_end; ++t) {
        if (!wait_parity_or_failed<true>(&sm.full[s], ph, &sm.failed) ||
            !wait_parity_or_failed<true>(&sm.acc_empty[b], bph ^ 1u, &sm.failed)) {
          atomicExch(&sm.failed, 1);
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;");
#pragma unroll
        for (int g = 0; g < kRtGroups; ++g)
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_bf16(tmem + 32u * kRtGroups * b + 32u * g,
                     x_d0 + (s * kXs + (g >> 1) * kXp + (g & 1) * kXh + kk * kXk),
                     h_d0 + (s * kHs + g * kHg + kk * kHk), kIdescBf16M128N32,
                     kk > 0 ? 1u : 0u);
        commit_to(&sm.empty[s]);
        commit_to(&sm.acc_full[b]);
        if (++s == kRtStages) {
          s = 0;
          ph ^= 1u;
        }
        if (++b == kRtAccBufs) {
          b = 0;
          bph ^= 1u;
        }
      }
      // drain: every MMA issued has completed before the stages or the
      // tensor memory can go away
      commit_to(&sm.drain);
      if (!wait_parity(&sm.drain, 0)) atomicExch(&sm.failed, 1);
    }
    __syncwarp();
  } else {
    // a warp reaches the tensor-memory lanes of its quarter, 32 (warp % 4)
    const int q = warp & 3, gs = (warp - 2) >> 2;
    constexpr int kPer = kRtGroups / 4;  // groups per thread and tile
    uint32_t b = 0, bph = 0;
    int64_t cb = t_begin / n_rt, rt = t_begin % n_rt;
    for (int64_t t = t_begin; t < t_end; ++t, rt = rt + 1 == n_rt ? 0 : rt + 1,
                 cb += rt == 0 ? 1 : 0) {
      const int64_t r = rt * 128 + 32 * q + lane;
      // after a failure every warp still runs every tile, without waiting
      // and without touching tensor memory (NaN rotations, zero codes,
      // scale 0xFF), so the quarter barriers of the staged stores stay
      // matched
      const bool ok = __all_sync(0xFFFFFFFFu, !failed_flag(&sm.failed) &&
                                                  wait_parity(&sm.acc_full[b], bph,
                                                              kAccWaitLimit));
      if (!ok) atomicExch(&sm.failed, 1);
      if (ok) asm volatile("tcgen05.fence::after_thread_sync;");
#pragma unroll 1
      for (int gi = 0; gi < kPer; ++gi) {
        const int g = kPer * gs + gi;
        uint32_t zb[32];
        if (ok) {
          tmem_ld32(tmem + (uint32_t(32 * q) << 16) + 32u * kRtGroups * b + 32u * uint32_t(g),
                    zb);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) zb[j] = kNaNf32;
        }
        if (ok && gi == kPer - 1) {  // the accumulator is read: release it
          asm volatile("tcgen05.fence::before_thread_sync;");
          __syncwarp();
          if (lane == 0)
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(
                             smem_u32(&sm.acc_empty[b]))
                         : "memory");
        }
        const int64_t c0 = cb * (32 * kRtGroups) + 32 * g;
        // staged slot: 16-byte chunks swizzled by row (conflict-free)
        uint4* oc = &sm.out_codes[t & 1][q][lane][g ^ (lane & (kRtGroups - 1))];
        uint8_t* os = &sm.out_scales[t & 1][q][lane][g];
        if (r < rows && c0 < cols) {
          float y[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) y[j] = __uint_as_float(zb[j]);
          rht_tc_quantize_group<SR, ROT, STAGED, OAS>(y, r, c0, cols, key,
                                                 !ok || failed_flag(&sm.failed), codes,
                                                 scales, rotated, oc, os);
        }
      }
      if (STAGED) {
        // the four warps of this lane quarter write its 32 rows x 8 groups
        // as whole 128-byte row segments (the stage alternates with the
        // tile, and this barrier of the next tile orders its reuse)
        asm volatile("bar.sync %0, 128;" ::"r"(1 + q) : "memory");
        const int lt = 32 * gs + lane;  // 0 .. 127 within the quarter
        const int64_t rbase = rt * 128 + 32 * q;
#pragma unroll
        for (int i = 0; i < 32 * kRtGroups / 128; ++i) {
          const int idx = lt + 128 * i;
          const int row = idx / kRtGroups, ch = idx % kRtGroups;
          const int64_t rr = rbase + row, cc = cb * (32 * kRtGroups) + 32 * ch;
          if (rr < rows && cc < cols)
            *reinterpret_cast<uint4*>(codes + (rr * cols + cc) / 2) =
                sm.out_codes[t & 1][q][row][ch ^ (row & (kRtGroups - 1))];
        }
        if (lt < 32) {
          const int64_t rr = rbase + lt, cc = cb * (32 * kRtGroups);
          if (rr < rows) {
            uint8_t* dst = scales + (rr * cols + cc) / 32;
            if (cols % (32 * kRtGroups) == 0 && (reinterpret_cast<uintptr_t>(dst) & 7) == 0) {
              *reinterpret_cast<uint2*>(dst) =
                  *reinterpret_cast<const uint2*>(&sm.out_scales[t & 1][q][lt][0]);
            } else {
              for (int j = 0; j < kRtGroups; ++j)
                if (cc + 32 * j < cols) dst[j] = sm.out_scales[t & 1][q][lt][j];
            }
          }
        }
      }
      if (++b == kRtAccBufs) {
        b = 0;
        bph ^= 1u;
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;");
  __syncthreads();
  report_failure(status, &sm.failed);
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(32 * kRtGroups * kRtAccBufs));
}

template <bool SR, bool ROT, bool STAGED, bool OAS>
cudaError_t rht_tc_impl(const CUtensorMap& mx, int64_t rows, int64_t cols,
                        uint32_t sign_key, RngKey key, uint8_t* codes, uint8_t* scales,
                        float* rotated, int* status, cudaStream_t s) {
  auto kern = k_rht_tc<SR, ROT, STAGED, OAS>;
  constexpr size_t smem = sizeof(RhtSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(kern),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int64_t tiles = ((rows + 127) / 128) * ((cols + 32 * kRtGroups - 1) / (32 * kRtGroups));
  const int grid = persistent_grid(reinterpret_cast<const void*>(kern), kRtThreads, smem, tiles);
  kern<<<grid, kRtThreads, smem, s>>>(mx, rows, cols, sign_key, key, codes, scales, rotated,
                                      status);
  return cudaGetLastError();
}

template <bool SR, bool ROT, bool OAS>
cudaError_t rht_impl(const void* x, int64_t rows, int64_t cols,
                     uint32_t sign_key, RngKey key, uint8_t* codes,
                     uint8_t* scales, float* rotated, cudaStream_t s) {
  auto kern = k_rht_quant<SR, ROT, OAS>;
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

template <bool OAS>
static cudaError_t rht_dispatch(const void* x, bool bf16, int64_t rows, int64_t cols,
                                uint32_t sign_key, RngKey key, bool sr, uint8_t* codes,
                                uint8_t* scales, float* rotated, int* status,
                                cudaStream_t s) {
  const bool rot = rotated != nullptr;
  if (bf16) {
    // X as a byte array [rows][2 cols] for the TMA: 128-byte boxes
    CUtensorMap mx;
    if (!encode_rows_sw128(&mx, x, rows, 2 * cols, 128)) return cudaErrorInvalidValue;
    if (sr)
      return rot ? rht_tc_impl<true, true, false, OAS>(mx, rows, cols, sign_key, key, codes,
                                                       scales, rotated, status, s)
                 : rht_tc_impl<true, false, false, OAS>(mx, rows, cols, sign_key, key, codes,
                                                        scales, rotated, status, s);
    return rot ? rht_tc_impl<false, true, false, OAS>(mx, rows, cols, sign_key, key, codes,
                                                      scales, rotated, status, s)
               : rht_tc_impl<false, false, true, OAS>(mx, rows, cols, sign_key, key, codes,
                                                      scales, rotated, status, s);
  }
  if (sr)
    return rot ? rht_impl<true, true, OAS>(x, rows, cols, sign_key, key, codes,
                                                  scales, rotated, s)
               : rht_impl<true, false, OAS>(x, rows, cols, sign_key, key, codes,
                                                   scales, rotated, s);
  return rot ? rht_impl<false, true, OAS>(x, rows, cols, sign_key, key, codes, scales,
                                                 rotated, s)
             : rht_impl<false, false, OAS>(x, rows, cols, sign_key, key, codes, scales,
                                                  rotated, s);
}

cudaError_t launch_rht_quant(const void* x, bool bf16, int64_t rows,
                             int64_t cols, uint64_t sign_seed, bool sr,
                             uint64_t sr_seed, uint8_t* codes,
                             uint8_t* scales, float* rotated, int* status,
                             cudaStream_t s, bool oas) {
  const uint32_t sign_key = stream_key(sign_seed, 1);
  const RngKey key = make_key(sr_seed, 0);
  return oas ? rht_dispatch<true>(x, bf16, rows, cols, sign_key, key, sr, codes, scales,
                                  rotated, status, s)
             : rht_dispatch<false>(x, bf16, rows, cols, sign_key, key, sr, codes, scales,
                                   rotated, status, s);
}

}  // namespace mxfp4
