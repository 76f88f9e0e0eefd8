// MXFP4 block quantize (1x32 row groups and 32x1 column groups) and
// dequantize kernels for sm_100a.
//
// Sources: "ALTO MXFP4 training — Weight de-oscillation — What does it
// mean?", Jargon (MXFP4, E2M1, Bin, Stochastic rounding);
// "Oscillation-Reduced MXFP4 Training for Vision Transformers", rebuttal,
// Question 2 (Q_D along 1x32 groups for the forward GEMM, 32x1 groups for the
// backward GEMM).
//
// Row groups: a [rows, cols] tensor with cols % 32 == 0 is a flat array of
// rows*cols/32 groups, so the row kernel is a grid-stride loop over groups,
// one thread per group: its 16-byte loads of a group (L1-allocating, so the
// warp's loads together read whole sectors) are all issued, for U groups,
// before any arithmetic; the maximum and the scale are computed once per
// group and its 32 codes leave in one 16-byte store. (A form with four
// threads per group, one 16-byte load each and quad shuffles, ran 12%
// slower for nearest rounding and 22% slower for stochastic rounding.)
//
// Column groups: a CTA stages a 128-row tile (128 bf16 or 64 fp32 columns)
// in shared memory, then each thread reduces two adjacent columns over 32
// rows (one 32-bit shared word per row; a warp reads 32 consecutive words of
// one row: no bank conflicts) and writes 16 code bytes per column. The four
// row groups of a column in the tile write one contiguous 64-byte run, so
// every DRAM sector of the transposed output is written whole.
#include "launch.cuh"
#include "mxfp4_device.cuh"

namespace mxfp4 {

namespace {

// ---------------------------------------------------------------------------
// Row groups
// ---------------------------------------------------------------------------

constexpr int kRowThreads = 256;

// One thread per whole 1x32 group: the group's maximum and scale are
// computed once, by the thread that rounds all 32 values, with no shuffles.
// Consecutive threads take consecutive groups; a group's 64 (bf16) or 128
// (fp32) bytes arrive as 16-byte L1-allocating loads, which together cover
// whole sectors, U groups in flight per thread; each group leaves as one
// 16-byte code store and its scale byte.
template <bool BF16, bool SR, int U, bool OAS = false>
__global__ void __launch_bounds__(kRowThreads)
    k_quant_rows(const void* __restrict__ x, int64_t n_groups, RngKey key,
                 uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  constexpr int kLoads = BF16 ? 4 : 8;  // 16-byte pieces per group
  const int64_t stride = int64_t(gridDim.x) * kRowThreads;
  for (int64_t base = int64_t(blockIdx.x) * kRowThreads + threadIdx.x; base < n_groups;
       base += stride * U) {
    uint4 w[U][kLoads];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t g = base + u * stride;
      const uint4* p = reinterpret_cast<const uint4*>(static_cast<const char*>(x) +
                                                      g * (BF16 ? 64 : 128));
#pragma unroll
      for (int k = 0; k < kLoads; ++k)
        w[u][k] = g < n_groups ? ld_l1(p + k) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t g = base + u * stride;
      if (g >= n_groups) break;
      float v[32];
      uint32_t amax;
      if (BF16) {
        uint32_t m[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint4 q = w[u][k];
          v[8 * k] = bf16_lo(q.x), v[8 * k + 1] = bf16_hi(q.x);
          v[8 * k + 2] = bf16_lo(q.y), v[8 * k + 3] = bf16_hi(q.y);
          v[8 * k + 4] = bf16_lo(q.z), v[8 * k + 5] = bf16_hi(q.z);
          v[8 * k + 6] = bf16_lo(q.w), v[8 * k + 7] = bf16_hi(q.w);
          m[2 * k] = bf16x2_absmax_nan(q.x, q.y);
          m[2 * k + 1] = bf16x2_absmax_nan(q.z, q.w);
        }
#pragma unroll
        for (int n = 4; n >= 1; n /= 2)
#pragma unroll
          for (int i = 0; i < n; ++i) m[i] = bf16x2_absmax_nan(m[i], m[i + n]);
        const uint32_t mm = m[0] & 0x7FFF7FFFu;
        amax = max(mm << 16, mm & 0xFFFF0000u);
      } else {
        amax = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint4 q = w[u][k];
          v[4 * k] = __uint_as_float(q.x), v[4 * k + 1] = __uint_as_float(q.y);
          v[4 * k + 2] = __uint_as_float(q.z), v[4 * k + 3] = __uint_as_float(q.w);
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) amax = max(amax, __float_as_uint(v[j]) & 0x7FFFFFFFu);
      }
      const uint32_t sb = OAS ? scale_byte_oas(amax) : scale_byte(amax);
      // the group's 16 pairs start at a multiple of 16: one inner key
      const uint64_t p0 = uint64_t(g) * 16;
      const uint32_t kh = inner_key(key, uint32_t(p0 >> 32)) + uint32_t(p0);
      uint32_t word[4];
      if (!SR) {
        const float mul = inv_scale(sb);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] *= mul;
#pragma unroll
        for (int q = 0; q < 4; ++q) word[q] = sb == 0xFFu ? 0u : e2m1x8_rn(v + 8 * q);
      } else if (BF16 && sb != 0xFFu) {
        // bf16: the pair form on the packed input words (bf16x8_sr_word)
        const unsigned short s16 = bf16_inv_scale(sb);
        const uint32_t sat2 = bf16x2_six_scale(sb);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          word[q] = bf16x8_sr_word<OAS>(reinterpret_cast<const uint32_t*>(&w[u][q]), s16, sat2,
                                        kh, uint32_t(q));
      } else if (sb >= 2u && sb != 0xFFu) {
        // the power of two rides on the rounding (e2m1_sr_top_scaled)
        const float half = scale_half(sb), sat = OAS ? 0.0f : scale_six(sb);
        const uint32_t nb = sr_noise64_base(sb);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t h[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) h[k] = mix32_pre(kh + uint32_t(4 * q + k));
          word[q] = e2m1x8_sr_scaled<!OAS>(v + 8 * q, h, half, sat, nb);
        }
      } else {
        const float mul = inv_scale(sb);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] *= mul;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t h[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) h[k] = mix32_pre(kh + uint32_t(4 * q + k));
          word[q] = sb == 0xFFu ? 0u : e2m1x8_sr(v + 8 * q, h);
        }
      }
      reinterpret_cast<uint4*>(codes)[g] = make_uint4(word[0], word[1], word[2], word[3]);
      scales[g] = static_cast<uint8_t>(sb);
    }
  }
}

// ---------------------------------------------------------------------------
// Column groups
// ---------------------------------------------------------------------------

constexpr int kTileRows = 128;

template <bool BF16>
struct ColTile {
  static constexpr int kCols = BF16 ? 128 : 64;           // tile columns
  static constexpr int kThreads = (kCols / 2) * (kTileRows / 32);
  static constexpr int kElemBytes = BF16 ? 2 : 4;
  static constexpr int kChunkElems = 16 / kElemBytes;     // per 16-byte load
  static constexpr int kChunksPerRow = kCols / kChunkElems;
};

// Random-number noise (sr_noise64) of the two adjacent elements (r0+j, c0),
// (r0+j, c0+1) of a column pass. Element (r, c) has index i = r*cols + c; c0
// is even. EVEN (cols even): i is even, so both elements are the halves of
// pair i/2, and the pair index of row r0+j is p0 + j*cols/2. Otherwise odd
// rows split the two elements over adjacent pairs. BIG: the tensor has 2^33
// elements or more, so the high word of a pair index can be nonzero.
template <bool EVEN, bool BIG>
__device__ __forceinline__ void column_noise(RngKey key, uint64_t i0,
                                             int64_t cols, int j, uint32_t& na,
                                             uint32_t& nb) {
  if (EVEN && !BIG) {
    const uint32_t h = mix32_pre(key.k0 + uint32_t(i0 >> 1) +
                                 uint32_t(j) * uint32_t(uint64_t(cols) >> 1));
    sr_noise64_pair(h, na, nb);
  } else {
    const uint64_t i = i0 + uint64_t(j) * uint64_t(cols);
    const uint64_t p = i >> 1;
    const uint32_t h = mix32_pre(inner_key(key, uint32_t(p >> 32)) + uint32_t(p));
    if ((i & 1) == 0) {
      sr_noise64_pair(h, na, nb);
    } else {
      const uint64_t p2 = p + 1;
      const uint32_t h2 = mix32_pre(inner_key(key, uint32_t(p2 >> 32)) + uint32_t(p2));
      uint32_t unused;
      sr_noise64_pair(h, unused, na);
      sr_noise64_pair(h2, nb, unused);
    }
  }
}

// Codes and scale bytes of two adjacent columns over one 32-row group: wa/wb
// hold the 32 codes of each column (row r0+j in nibble j%8 of word j/8).
struct ColPair {
  uint32_t wa[4], wb[4];
  uint32_t sa, sb;
};

// The multiplier that scales a value v held at half its size (HALF) by
// 2^-e, e = sb - 127, in one or two exact steps: 2^(1-e) for sb >= 1, and
// 2 then 2^127 for sb = 0 (where 2^128 is not an fp32 value).
struct HalfScale {
  float m1, m2;
  __device__ __forceinline__ explicit HalfScale(uint32_t sb) {
    m1 = sb == 0u ? 2.0f : 1.0f;
    m2 = __uint_as_float((sb == 0u ? 254u : 255u - min(sb, 254u)) << 23);
  }
  __device__ __forceinline__ float operator()(float v) const { return (v * m1) * m2; }
};

// Quantize the two adjacent columns c0, c0+1 over the 32 rows r0 .. r0+31.
// get(j) returns the values of row r0+j (x: column c0, y: column c0+1); ma
// and mb are the fp32 bit patterns of the two columns' absolute maxima.
// HALF: get() returns every value at half its size (see half_scale_value),
// and ma, mb are the halved maxima.
template <bool SR, bool EVEN, bool BIG, bool SAT = true, bool OAS = false,
          bool HALF = false, typename Get>
__device__ __forceinline__ ColPair column_pair_codes(Get get, uint32_t ma,
                                                     uint32_t mb, int64_t r0,
                                                     int64_t c0, int64_t cols,
                                                     RngKey key) {
  ColPair o;
  if (HALF) {
    o.sa = OAS ? scale_byte_oas_of_double(ma) : scale_byte_of_double(ma);
    o.sb = OAS ? scale_byte_oas_of_double(mb) : scale_byte_of_double(mb);
  } else {
    o.sa = OAS ? scale_byte_oas(ma) : scale_byte(ma);
    o.sb = OAS ? scale_byte_oas(mb) : scale_byte(mb);
  }
  const float mula = inv_scale(o.sa), mulb = inv_scale(o.sb);
  const HalfScale hsa(o.sa), hsb(o.sb);
  auto scale_a = [&](float v) { return HALF ? hsa(v) : v * mula; };
  auto scale_b = [&](float v) { return HALF ? hsb(v) : v * mulb; };
  // the scale byte of the values as get() returns them
  constexpr uint32_t kHeld = HALF ? 1u : 0u;
#pragma unroll
  for (int q = 0; q < 4; ++q) o.wa[q] = o.wb[q] = 0;
  if (SR && EVEN && !BIG && o.sa >= 2u + kHeld && o.sb >= 2u + kHeld && o.sa != 0xFFu &&
      o.sb != 0xFFu) {
    // Scales of at least 2^-125 (for the values as held): the power of two
    // rides on the rounding (e2m1_sr_top_scaled) instead of a multiply per
    // element. Overflow-aware scales never leave a value above 6, so they
    // skip the saturation.
    constexpr bool kSat = SAT && !OAS;
    const uint32_t ua = o.sa - kHeld, ub = o.sb - kHeld;
    const float ha = scale_half(ua), hb = scale_half(ub);
    const float xa = kSat ? scale_six(ua) : 0.0f, xb = kSat ? scale_six(ub) : 0.0f;
    const uint32_t ka = sr_noise64_base(ua), kb = sr_noise64_base(ub);
    const uint32_t p0 = key.k0 + uint32_t((uint64_t(r0) * uint64_t(cols) + uint64_t(c0)) >> 1);
    const uint32_t hc = uint32_t(uint64_t(cols) >> 1);
#pragma unroll
    for (int j = 31; j >= 0; --j) {  // push_code fills nibbles 7 .. 0
      uint32_t na, nb;
      sr_noise64_pair_based(mix32_pre(p0 + uint32_t(j) * hc), ka, kb, na, nb);
      const float2 v = get(j);
      o.wa[j >> 3] = push_code(o.wa[j >> 3], e2m1_sr_top_scaled<kSat>(v.x, ha, xa, na));
      o.wb[j >> 3] = push_code(o.wb[j >> 3], e2m1_sr_top_scaled<kSat>(v.y, hb, xb, nb));
    }
  } else if (SR) {
    const uint64_t i0 = uint64_t(r0) * uint64_t(cols) + uint64_t(c0);
#pragma unroll
    for (int j = 31; j >= 0; --j) {  // push_code fills nibbles 7 .. 0
      uint32_t na, nb;
      column_noise<EVEN, BIG>(key, i0, cols, j, na, nb);
      const float2 v = get(j);
      o.wa[j >> 3] = push_code(o.wa[j >> 3], e2m1_sr_top<SAT>(scale_a(v.x), na));
      o.wb[j >> 3] = push_code(o.wb[j >> 3], e2m1_sr_top<SAT>(scale_b(v.y), nb));
    }
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float va[8], vb[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float2 v = get(8 * q + j);
        va[j] = scale_a(v.x);
        vb[j] = scale_b(v.y);
      }
      o.wa[q] = e2m1x8_rn(va);
      o.wb[q] = e2m1x8_rn(vb);
    }
  }
  if (o.sa == 0xFFu) o.wa[0] = o.wa[1] = o.wa[2] = o.wa[3] = 0;
  if (o.sb == 0xFFu) o.wb[0] = o.wb[1] = o.wb[2] = o.wb[3] = 0;
  return o;
}

// Store a column pair straight to the COLS layout (16 bytes per column).
__device__ __forceinline__ void store_column_pair(
    const ColPair& o, int64_t r0, int64_t c0, int64_t rows, int64_t cols,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const int64_t half_rows = rows / 2;
  if (c0 < cols) {
    *reinterpret_cast<uint4*>(codes + c0 * half_rows + r0 / 2) =
        make_uint4(o.wa[0], o.wa[1], o.wa[2], o.wa[3]);
    scales[c0 * (rows / 32) + r0 / 32] = static_cast<uint8_t>(o.sa);
  }
  if (c0 + 1 < cols) {
    *reinterpret_cast<uint4*>(codes + (c0 + 1) * half_rows + r0 / 2) =
        make_uint4(o.wb[0], o.wb[1], o.wb[2], o.wb[3]);
    scales[(c0 + 1) * (rows / 32) + r0 / 32] = static_cast<uint8_t>(o.sb);
  }
}

// Column outputs of one 128-row tile, staged in shared memory so that each
// column's 64-byte run of codes leaves in one piece: the 16-byte chunk of
// column pair cp, side s (0: even column), row group rg sits at uint4 index
// 9cp + 4s + rg (the ninth chunk of each pair is padding, so the stores of
// consecutive cp fall in distinct bank groups); scale bytes at 4c + rg for
// tile column c.
template <int kCols>
struct ColStage {
  static constexpr int kChunks = (kCols / 2) * 9;
  static constexpr int kBytes = kChunks * 16 + kCols * 4;
};

__device__ __forceinline__ void stage_column_pair(const ColPair& o, int cp,
                                                  int rg, uint4* s_col,
                                                  uint8_t* s_sc) {
  s_col[9 * cp + rg] = make_uint4(o.wa[0], o.wa[1], o.wa[2], o.wa[3]);
  s_col[9 * cp + 4 + rg] = make_uint4(o.wb[0], o.wb[1], o.wb[2], o.wb[3]);
  s_sc[8 * cp + rg] = static_cast<uint8_t>(o.sa);
  s_sc[8 * cp + 4 + rg] = static_cast<uint8_t>(o.sb);
}

// Write a staged tile to the COLS layout: four consecutive threads write one
// column's 64 contiguous code bytes, and one thread its 4 scale bytes (one
// 32-bit store when rows is a multiple of 128, which also aligns it).
template <int kCols, int kThreads>
__device__ __forceinline__ void store_staged_columns(
    const uint4* s_col, const uint8_t* s_sc, int64_t tile_r, int64_t tile_c,
    int64_t rows, int64_t cols, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales) {
  static_assert(kCols * 4 % kThreads == 0 && kCols <= kThreads, "stage shape");
  const int64_t half_rows = rows / 2, groups = rows / 32;
#pragma unroll
  for (int i = 0; i < kCols * 4 / kThreads; ++i) {
    const int k = i * kThreads + threadIdx.x;
    const int cp = k >> 3, side = (k >> 2) & 1, part = k & 3;
    const int64_t c = tile_c + 2 * cp + side, r = tile_r + 32 * part;
    if (c < cols && r < rows)
      *reinterpret_cast<uint4*>(codes + c * half_rows + r / 2) =
          s_col[9 * cp + 4 * side + part];
  }
  const int k = threadIdx.x;
  const int64_t c = tile_c + k;
  if (k < kCols && c < cols) {
    uint8_t* dst = scales + c * groups + tile_r / 32;
    if (rows % kTileRows == 0) {
      *reinterpret_cast<uint32_t*>(dst) = reinterpret_cast<const uint32_t*>(s_sc)[k];
    } else {
#pragma unroll
      for (int part = 0; part < 4; ++part)
        if (tile_r + 32 * part < rows) dst[part] = s_sc[4 * k + part];
    }
  }
}

// Stochastic 32x1 codes of two adjacent columns from their 32 row words
// wr[j] (bf16 pairs, the even column in the low half), the columns' scale
// bytes sa, sb (not 0xFF) and the pair counter of row 0, kp0 (key.k0 plus
// the pair index; row j adds j * hc), for tensors below 2^33 elements. As
// the bf16 row kernel: one exact mixed-precision product per value (each
// column its own power of two), saturation on the packed pairs when SAT,
// the codes of rows 2k (x4 sum) and 2k+1 (x64 sum) merged into one byte per
// column, signs gathered from the row words. HELD: the words hold half of
// the values (the double quantizer's Q_D(X) / 2), so the power of two is
// 2^(1-e) and sa, sb must be at least 1.
template <bool SAT, bool HELD>
__device__ __forceinline__ ColPair column_pair_sr_bf16(const uint32_t* wr, uint32_t sa,
                                                       uint32_t sb, uint32_t kp0,
                                                       uint32_t hc) {
  ColPair o;
  o.sa = sa;
  o.sb = sb;
  const unsigned short s16a = bf16_inv_scale(HELD ? sa - 1u : sa);
  const unsigned short s16b = bf16_inv_scale(HELD ? sb - 1u : sb);
  const uint32_t sat2 = SAT ? bitsel(bf16x2_six_scale(sa), bf16x2_six_scale(sb), 0xFFFFu) : 0u;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t pa[4], pb[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t t[2][2];
#pragma unroll
      for (int par = 0; par < 2; ++par) {  // row 8q+2k+par
        const int j = 8 * q + 2 * k + par;
        uint32_t re, ro;
        pair_randoms(mix32_pre(mad_u32(uint32_t(j), hc, kp0)), re, ro);
        const uint32_t ws = SAT ? bf16x2_clamp_abs(wr[j], sat2) : wr[j];
        const uint32_t mul = par ? 64u : 4u;
        const uint32_t nm = par ? 0xFFFFF000u : 0xFFFFFF00u;
        const uint32_t nbase = par ? kSrBase64 : kSrBase4;
        t[par][0] = mad_u32(sr_operand(bf16lo_mul(ws, s16a)), mul, mad_u32(re, nm, nbase));
        t[par][1] = mad_u32(sr_operand(bf16hi_mul(ws, s16b)), mul, mad_u32(ro, nm, nbase));
      }
      pa[k] = pair_byte(t[1][0], t[0][0]);
      pb[k] = pair_byte(t[1][1], t[0][1]);
    }
    uint32_t ta, tb;
    sign_nibbles_cols(wr + 8 * q, ta, tb);
    o.wa[q] = pack_pair_bytes(pa[0], pa[1], pa[2], pa[3]) | ta;
    o.wb[q] = pack_pair_bytes(pb[0], pb[1], pb[2], pb[3]) | tb;
  }
  return o;
}

// Column pass over a staged tile: thread (rg, cp) quantizes the columns
// 2cp, 2cp+1 over tile rows 32rg .. 32rg+31 (rows below the tensor's end:
// the caller checks tile_r + 32rg < rows). The tile is read twice (maxima,
// then codes) rather than held in registers. A warp reads 32 consecutive
// 32-bit words (bf16) or 64-bit words (fp32) of one row: no bank conflicts.
template <bool BF16, bool SR, bool EVEN, bool BIG, bool OAS = false>
__device__ __forceinline__ ColPair column_tile_pass(const uint4* tile,
                                                    int kcols, int rg, int cp,
                                                    int64_t tile_r,
                                                    int64_t tile_c,
                                                    int64_t cols, RngKey key) {
  const int64_t r0 = tile_r + 32 * rg;
  uint32_t ma = 0, mb = 0;
  if (BF16) {
    const uint32_t* s = reinterpret_cast<const uint32_t*>(tile) + 32 * rg * (kcols / 2) + cp;
    uint32_t m = 0, wr[32];  // the column pair's 32 rows, kept for the codes
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      wr[j] = s[j * (kcols / 2)];
      m = bf16x2_absmax_nan(m, wr[j]);
    }
    m &= 0x7FFF7FFFu;
    ma = m << 16;
    mb = m & 0xFFFF0000u;
    if (SR && EVEN && !BIG) {
      const uint32_t sa = OAS ? scale_byte_oas(ma) : scale_byte(ma);
      const uint32_t sb = OAS ? scale_byte_oas(mb) : scale_byte(mb);
      if (sa != 0xFFu && sb != 0xFFu) {
        const int64_t c0 = tile_c + 2 * cp;
        return column_pair_sr_bf16<!OAS, false>(
            wr, sa, sb,
            key.k0 + uint32_t((uint64_t(r0) * uint64_t(cols) + uint64_t(c0)) >> 1),
            uint32_t(uint64_t(cols) >> 1));
      }
    }
    return column_pair_codes<SR, EVEN, BIG, true, OAS>(
        [&](int j) {
          const uint32_t w = wr[j];
          return make_float2(bf16_lo(w), bf16_hi(w));
        },
        ma, mb, r0, tile_c + 2 * cp, cols, key);
  }
  const float2* s = reinterpret_cast<const float2*>(tile) + 32 * rg * (kcols / 2) + cp;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float2 w = s[j * (kcols / 2)];
    ma = max(ma, __float_as_uint(w.x) & 0x7FFFFFFFu);
    mb = max(mb, __float_as_uint(w.y) & 0x7FFFFFFFu);
  }
  return column_pair_codes<SR, EVEN, BIG, true, OAS>([&](int j) { return s[j * (kcols / 2)]; },
                                          ma, mb, r0, tile_c + 2 * cp, cols, key);
}

// Load one [128 x kCols] tile into shared memory (zero outside the tensor).
// VEC: every row starts 16-byte aligned and cols is a multiple of the
// 16-byte chunk, so chunks are either wholly inside or wholly outside.
template <bool BF16, bool VEC>
__device__ __forceinline__ void load_tile(const void* __restrict__ x,
                                          int64_t rows, int64_t cols,
                                          int64_t tile_r, int64_t tile_c,
                                          uint4* tile) {
  using T = ColTile<BF16>;
  constexpr int kChunks = kTileRows * T::kChunksPerRow;
  constexpr int kPer = kChunks / T::kThreads;
  uint4 buf[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int idx = k * T::kThreads + threadIdx.x;
    const int r = idx / T::kChunksPerRow, ch = idx % T::kChunksPerRow;
    const int64_t gr = tile_r + r, gc = tile_c + int64_t(ch) * T::kChunkElems;
    if (VEC) {
      buf[k] = (gr < rows && gc < cols)
                   ? ld_stream(static_cast<const char*>(x) +
                               (gr * cols + gc) * T::kElemBytes)
                   : make_uint4(0, 0, 0, 0);
    } else {
      uint32_t e[4] = {0, 0, 0, 0};
      if (BF16) {
        const uint16_t* p = static_cast<const uint16_t*>(x);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (gr < rows && gc + j < cols)
            e[j / 2] |= uint32_t(p[gr * cols + gc + j]) << (16 * (j & 1));
      } else {
        const uint32_t* p = static_cast<const uint32_t*>(x);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (gr < rows && gc + j < cols) e[j] = p[gr * cols + gc + j];
      }
      buf[k] = make_uint4(e[0], e[1], e[2], e[3]);
    }
  }
#pragma unroll
  for (int k = 0; k < kPer; ++k) tile[k * T::kThreads + threadIdx.x] = buf[k];
}

// Stage one [128 x kCols] tile of a tensor whose rows are 16-byte aligned
// and whose cols are a whole number of 16-byte chunks, with asynchronous
// copies (zero-filled outside the tensor), and commit them as one group.
// Tiles wholly inside the tensor skip the per-chunk range checks.
// SWZ (bf16 only): chunk ch of tile row r lands in slot
// ch ^ dq_swizzle(ch >> 2, r) of that row, so that the double quantizer's
// row pass, where four consecutive threads read the four 64-byte groups of
// a row chunk by chunk, hits 32 distinct banks per 8-thread phase.
__device__ __forceinline__ int dq_swizzle(int group, int row) {
  return (group & 2) | (row & 1);
}

template <bool BF16, bool SWZ = false>
__device__ __forceinline__ void stage_tile_async(const void* __restrict__ x,
                                                 int64_t rows, int64_t cols,
                                                 int64_t tile_r, int64_t tile_c,
                                                 uint4* tile) {
  using T = ColTile<BF16>;
  constexpr int kPer = kTileRows * T::kChunksPerRow / T::kThreads;
  static_assert(T::kThreads % T::kChunksPerRow == 0, "whole rows per pass");
  constexpr int kRowStep = T::kThreads / T::kChunksPerRow;  // rows per pass
  // this thread's chunk column is the same in every pass
  const int r0 = threadIdx.x / T::kChunksPerRow, ch = threadIdx.x % T::kChunksPerRow;
  const int64_t gc = tile_c + int64_t(ch) * T::kChunkElems;
  const bool col_ok = gc < cols;
  const char* src = static_cast<const char*>(x) + ((tile_r + r0) * cols + gc) * T::kElemBytes;
  const int64_t step = int64_t(kRowStep) * cols * T::kElemBytes;
  static_assert(!SWZ || (BF16 && kRowStep % 2 == 0), "swizzle: bf16 tiles, even row step");
  uint4* dst = tile + r0 * T::kChunksPerRow + (SWZ ? ch ^ dq_swizzle(ch >> 2, r0) : ch);
  if (tile_r + kTileRows <= rows && tile_c + T::kCols <= cols) {
#pragma unroll
    for (int k = 0; k < kPer; ++k, src += step) cp_async16(dst + k * T::kThreads, src, true);
  } else {
#pragma unroll
    for (int k = 0; k < kPer; ++k, src += step) {
      const bool ok = col_ok && tile_r + r0 + k * kRowStep < rows;
      cp_async16(dst + k * T::kThreads, ok ? src : x, ok);
    }
  }
  cp_async_commit();
}

// Column groups, general shapes: one staged tile at a time, plain loads.
template <bool BF16, bool SR, bool EVEN, bool BIG, bool OAS = false>
__global__ void __launch_bounds__(ColTile<BF16>::kThreads)
    k_quant_cols(const void* __restrict__ x, int64_t rows, int64_t cols,
                 RngKey key, uint8_t* __restrict__ codes,
                 uint8_t* __restrict__ scales) {
  using T = ColTile<BF16>;
  __shared__ uint4 tile[kTileRows * T::kChunksPerRow];
  const int64_t tiles_c = (cols + T::kCols - 1) / T::kCols;
  const int64_t n_tiles = ((rows + kTileRows - 1) / kTileRows) * tiles_c;
  const int cp = threadIdx.x % (T::kCols / 2);
  const int rg = threadIdx.x / (T::kCols / 2);
  for (int64_t t = blockIdx.x; t < n_tiles; t += gridDim.x) {
    const int64_t tile_r = (t / tiles_c) * kTileRows;
    const int64_t tile_c = (t % tiles_c) * T::kCols;
    load_tile<BF16, false>(x, rows, cols, tile_r, tile_c, tile);
    __syncthreads();
    const int64_t r0 = tile_r + 32 * rg;
    if (r0 < rows)
      store_column_pair(column_tile_pass<BF16, SR, EVEN, BIG, OAS>(
                            tile, T::kCols, rg, cp, tile_r, tile_c, cols, key),
                        r0, tile_c + 2 * cp, rows, cols, codes, scales);
    __syncthreads();
  }
}

// Row and column of the tiles first, first + stride, ... of a grid with
// n_c tile columns (tile t = row * n_c + column), advanced without a 64-bit
// division per step (one division when constructed).
struct TileWalk {
  int64_t r, c, dr, dc, n_c;
  __device__ __forceinline__ TileWalk(int64_t first, int64_t stride, int64_t nc) : n_c(nc) {
    r = first / nc;
    c = first - r * nc;
    dr = stride / nc;
    dc = stride - dr * nc;
  }
  __device__ __forceinline__ void next() {
    r += dr;
    c += dc;
    if (c >= n_c) {
      c -= n_c;
      ++r;
    }
  }
};

// Column groups, 16-byte aligned rows: double-buffered. The copies of the
// CTA's next tile are in flight while the current tile is quantized; the
// tile's column codes are staged and leave as whole 64-byte runs.
template <bool BF16, bool SR, bool EVEN, bool BIG, bool OAS = false>
__global__ void __launch_bounds__(ColTile<BF16>::kThreads, 3)
    k_quant_cols_pipe(const void* __restrict__ x, int64_t rows, int64_t cols,
                      RngKey key, uint8_t* __restrict__ codes,
                      uint8_t* __restrict__ scales) {
  using T = ColTile<BF16>;
  using S = ColStage<T::kCols>;
  constexpr int kChunks = kTileRows * T::kChunksPerRow;
  extern __shared__ uint4 smem[];  // two tiles, then the column stage
  uint4* s_col = smem + 2 * kChunks;
  uint8_t* s_sc = reinterpret_cast<uint8_t*>(s_col + S::kChunks);
  const int64_t tiles_c = (cols + T::kCols - 1) / T::kCols;
  const int64_t n_tiles = ((rows + kTileRows - 1) / kTileRows) * tiles_c;
  const int cp = threadIdx.x % (T::kCols / 2);
  const int rg = threadIdx.x / (T::kCols / 2);
  int64_t t = blockIdx.x;
  if (t >= n_tiles) return;
  TileWalk cur(t, gridDim.x, tiles_c), nxt = cur;
  nxt.next();
  stage_tile_async<BF16>(x, rows, cols, cur.r * kTileRows, cur.c * T::kCols, smem);
  for (int buf = 0; t < n_tiles; t += gridDim.x, buf ^= 1, cur = nxt, nxt.next()) {
    // this tile's copies are done and visible, and every thread has left the
    // previous tile (whose buffer and column stage are reused below)
    cp_async_wait<0>();
    __syncthreads();
    if (t + gridDim.x < n_tiles)
      stage_tile_async<BF16>(x, rows, cols, nxt.r * kTileRows, nxt.c * T::kCols,
                             smem + (buf ^ 1) * kChunks);
    const int64_t tile_r = cur.r * kTileRows;
    const int64_t tile_c = cur.c * T::kCols;
    if (tile_r + 32 * rg < rows)
      stage_column_pair(column_tile_pass<BF16, SR, EVEN, BIG, OAS>(
                            smem + buf * kChunks, T::kCols, rg, cp, tile_r,
                            tile_c, cols, key),
                        cp, rg, s_col, s_sc);
    __syncthreads();
    store_staged_columns<T::kCols, T::kThreads>(s_col, s_sc, tile_r, tile_c,
                                                rows, cols, codes, scales);
  }
}

// ---------------------------------------------------------------------------
// Dequantize (flat groups; both layouts)
// ---------------------------------------------------------------------------

template <bool BF16OUT, int U>
__global__ void __launch_bounds__(kRowThreads)
    k_dequant(const uint8_t* __restrict__ codes,
              const uint8_t* __restrict__ scales, int64_t n_groups,
              void* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int sub = lane & 3;
  const int64_t warp = (int64_t(blockIdx.x) * kRowThreads + threadIdx.x) >> 5;
  const int64_t chunk = (int64_t(gridDim.x) * kRowThreads) >> 2;
  const int64_t my = warp * 8 + (lane >> 2);
  for (int64_t base = 0; base < n_groups; base += chunk * U) {
    uint32_t w[U], sb[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t g = base + u * chunk + my;
      const bool ok = g < n_groups;
      w[u] = ok ? __ldcs(reinterpret_cast<const uint32_t*>(codes) + g * 4 + sub)
                : 0u;
      sb[u] = ok ? __ldcs(scales + g) : 0u;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t g = base + u * chunk + my;
      if (g >= n_groups) continue;
      float f[8];
      e2m1x8_decode(w[u], f);
      const float s = scale_value(sb[u]);
#pragma unroll
      for (int j = 0; j < 8; ++j) f[j] *= s;
      if (BF16OUT) {
        uint4 o = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                             pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
        if (sb[u] == 0xFFu) o = make_uint4(kNaNbf16x2, kNaNbf16x2, kNaNbf16x2,
                                           kNaNbf16x2);
        __stcs(reinterpret_cast<uint4*>(static_cast<uint16_t*>(y) + g * 32 +
                                        sub * 8),
               o);
      } else {
        float4 o0 = make_float4(f[0], f[1], f[2], f[3]);
        float4 o1 = make_float4(f[4], f[5], f[6], f[7]);
        if (sb[u] == 0xFFu) {
          const float n = __uint_as_float(kNaNf32);
          o0 = o1 = make_float4(n, n, n, n);
        }
        float4* p = reinterpret_cast<float4*>(static_cast<float*>(y) + g * 32 +
                                              sub * 8);
        __stcs(p, o0);
        __stcs(p + 1, o1);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Fused double quantization (TetraJet rebuttal, Question 2): one pass over a
// 128x128 tile computes the row layout of Q_D(1x32)(X) (RNE) in registers and
// writes it; the same codes and row scales are staged in shared memory (4.5
// bits per element), and the column pass decodes them, exactly, back to the
// values of Q_D(X) and quantizes those along 32x1 columns with stochastic
// rounding. X is read once; no transpose pass, no intermediate in global
// memory.
// ---------------------------------------------------------------------------

constexpr int kDqThreads = 256;
constexpr int kDqCols = 128;
// Staged row-group scale values of the pipelined double quantizer, group
// major: value (row r, group g) at g * kDqScaleStride + r. The column pass
// reads four consecutive rows in one 16-byte load; the padding (8 words)
// spreads the row pass's stores (8 rows x 4 groups per warp) over 32 banks.
constexpr int kDqScaleStride = kTileRows + 8;

template <bool BF16, bool BIG, bool OAS>
__global__ void __launch_bounds__(kDqThreads)
    k_double_quant(const void* __restrict__ x, int64_t rows, int64_t cols,
                   RngKey key, uint8_t* __restrict__ row_codes,
                   uint8_t* __restrict__ row_scales,
                   uint8_t* __restrict__ col_codes,
                   uint8_t* __restrict__ col_scales) {
  // Q_D(X) of the tile: codes [128 rows][64 bytes] and the scale byte of
  // every 1x32 row group [128 rows][4].
  __shared__ uint32_t s_codes[kTileRows * (kDqCols / 8)];
  __shared__ uint8_t s_scales[kTileRows * (kDqCols / 32)];
  const int64_t tiles_c = (cols + kDqCols - 1) / kDqCols;
  const int64_t n_tiles = ((rows + kTileRows - 1) / kTileRows) * tiles_c;
  const int ch = threadIdx.x & 15;   // 8-column chunk of a tile row
  const int rr = threadIdx.x >> 4;   // tile row, plus 16 per pass
  const int cp = threadIdx.x & 63;   // column pair of the column pass
  const int rg = threadIdx.x >> 6;   // 32-row group of the column pass
  constexpr int kPasses = kTileRows / 16;
  for (int64_t t = blockIdx.x; t < n_tiles; t += gridDim.x) {
    const int64_t tile_r = (t / tiles_c) * kTileRows;
    const int64_t tile_c = (t % tiles_c) * kDqCols;
    const int64_t gc = tile_c + 8 * ch;
    // Row pass: all loads first, then quad-reduced 1x32 groups.
    uint4 raw[kPasses][BF16 ? 1 : 2];
#pragma unroll
    for (int k = 0; k < kPasses; ++k) {
      const int64_t gr = tile_r + rr + 16 * k;
      const bool ok = gr < rows && gc < cols;
      if (BF16) {
        raw[k][0] = ok ? ld_stream(static_cast<const uint16_t*>(x) + gr * cols + gc)
                       : make_uint4(0, 0, 0, 0);
      } else {
        const float* p = static_cast<const float*>(x) + gr * cols + gc;
        raw[k][0] = ok ? ld_stream(p) : make_uint4(0, 0, 0, 0);
        raw[k][BF16 ? 0 : 1] = ok ? ld_stream(p + 4) : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int k = 0; k < kPasses; ++k) {
      const int64_t gr = tile_r + rr + 16 * k;
      const bool ok = gr < rows && gc < cols;
      float v[8];
      if (BF16) {
        const uint4 w = raw[k][0];
        v[0] = bf16_lo(w.x), v[1] = bf16_hi(w.x), v[2] = bf16_lo(w.y);
        v[3] = bf16_hi(w.y), v[4] = bf16_lo(w.z), v[5] = bf16_hi(w.z);
        v[6] = bf16_lo(w.w), v[7] = bf16_hi(w.w);
      } else {
        const uint4 a = raw[k][0], b = raw[k][BF16 ? 0 : 1];
        v[0] = __uint_as_float(a.x), v[1] = __uint_as_float(a.y);
        v[2] = __uint_as_float(a.z), v[3] = __uint_as_float(a.w);
        v[4] = __uint_as_float(b.x), v[5] = __uint_as_float(b.y);
        v[6] = __uint_as_float(b.z), v[7] = __uint_as_float(b.w);
      }
      uint32_t amax = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        amax = max(amax, __float_as_uint(v[j]) & 0x7FFFFFFFu);
      amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
      amax = max(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
      const uint32_t sb = OAS ? scale_byte_oas(amax) : scale_byte(amax);
      const float mul = inv_scale(sb);
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] *= mul;
      uint32_t word = e2m1x8_rn(v);
      if (sb == 0xFFu) word = 0;
      if (ok) {
        *reinterpret_cast<uint32_t*>(row_codes + gr * (cols / 2) + gc / 2) = word;
        if ((ch & 3) == 0) row_scales[gr * (cols / 32) + gc / 32] = uint8_t(sb);
      }
      s_codes[(rr + 16 * k) * (kDqCols / 8) + ch] = word;
      if ((ch & 3) == 0) s_scales[(rr + 16 * k) * (kDqCols / 32) + ch / 4] = uint8_t(sb);
    }
    __syncthreads();
    // Column pass: decode Q_D(X) / 2 for columns 2cp, 2cp+1 over 32 rows
    // (one shared byte per row holds both codes), then stochastic rounding
    // along the 32x1 groups. A row group of scale 0xFF decodes to NaN (0 x inf).
    const int64_t r0 = tile_r + 32 * rg;
    if (r0 < rows) {
      const uint8_t* sc = reinterpret_cast<const uint8_t*>(s_codes);
      float a[32], b[32];
      uint32_t ma = 0, mb = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        uint32_t w4 = 0;
        float sv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = 32 * rg + 4 * q + i;
          w4 |= uint32_t(sc[r * (kDqCols / 2) + cp]) << (8 * i);
          sv[i] = half_scale_value(s_scales[r * (kDqCols / 32) + cp / 16]);
        }
        float f[8];
        e2m1x8_decode(w4, f);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          a[4 * q + i] = f[2 * i] * sv[i];
          b[4 * q + i] = f[2 * i + 1] * sv[i];
          ma = max(ma, __float_as_uint(a[4 * q + i]) & 0x7FFFFFFFu);
          mb = max(mb, __float_as_uint(b[4 * q + i]) & 0x7FFFFFFFu);
        }
      }
      // cols is a multiple of 32 here, so every pair index is even-aligned
      store_column_pair(column_pair_codes<true, true, BIG, true, OAS, true>(
                            [&](int j) { return make_float2(a[j], b[j]); }, ma,
                            mb, r0, tile_c + 2 * cp, cols, key),
                        r0, tile_c + 2 * cp, rows, cols, col_codes, col_scales);
    }
    __syncthreads();
  }
}

// Row pass of one whole 1x32 group: group g of the staged raw tile row
// `row` (tile row tr; chunks swizzled as the staging placed them). Writes
// the 32 row codes and the scale byte to global memory (when in range) and
// stages the codes and the halved scale value 2^(e-1) (half_scale_value) in
// shared memory for the column pass.
template <bool OAS>
__device__ __forceinline__ void dq_row_group(const uint4* row, int g, int tr, bool ok,
                                             uint8_t* __restrict__ rc,
                                             uint8_t* __restrict__ rs, uint4* s_code,
                                             float* s_scale) {
  uint32_t w[16];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 q = row[4 * g + (c ^ dq_swizzle(g, tr))];
    w[4 * c] = q.x, w[4 * c + 1] = q.y, w[4 * c + 2] = q.z, w[4 * c + 3] = q.w;
  }
  uint32_t m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = bf16x2_absmax_nan(w[2 * i], w[2 * i + 1]);
#pragma unroll
  for (int n = 4; n >= 1; n /= 2)
#pragma unroll
    for (int i = 0; i < n; ++i) m[i] = bf16x2_absmax_nan(m[i], m[i + n]);
  const uint32_t mm = m[0] & 0x7FFF7FFFu;
  const uint32_t amax = max(mm << 16, mm & 0xFFFF0000u);
  const uint32_t sb = OAS ? scale_byte_oas(amax) : scale_byte(amax);
  const float mul = inv_scale(sb);
  uint32_t word[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float v[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] = bf16_lo(w[4 * c + j]) * mul;
      v[2 * j + 1] = bf16_hi(w[4 * c + j]) * mul;
    }
    word[c] = sb == 0xFFu ? 0u : e2m1x8_rn(v);
  }
  const uint4 out = make_uint4(word[0], word[1], word[2], word[3]);
  if (ok) {
    *reinterpret_cast<uint4*>(rc) = out;
    *rs = uint8_t(sb);
  }
  *s_code = out;
  *s_scale = half_scale_value(sb);
}

// Column pass of the double quantizer over the staged Q_D(X) codes: decode
// columns 2cp, 2cp+1 of rows 32rg.. (one shared byte per row holds both
// codes) and multiply by the row groups' staged halved scale values, which
// gives Q_D(X) / 2 exactly (a row group of scale 0xFF has the value +inf and
// codes 0, so it decodes to NaN, and the NaN-propagating maximum carries it
// into the column scale), then stochastic rounding along the 32x1 groups
// (column_pair_codes with HALF). The caller checks that the row group lies
// inside the tensor.
//
// No saturation is needed: every decoded value is G[m] 2^k, two significant
// bits, and the column scale puts the column maximum in [4, 8), so a scaled
// value is at most 6 (the only such values in [4, 8) are 4 and 6).
template <bool BIG, bool OAS>
__device__ __forceinline__ ColPair dq_column_pass(
    const uint32_t* s_codes, const float* s_scales, int rg, int cp,
    int64_t tile_r, int64_t tile_c, int64_t cols, RngKey key) {
  const int64_t r0 = tile_r + 32 * rg;
  const uint8_t* sc = reinterpret_cast<const uint8_t*>(s_codes);
  float a[32], b[32];
  float ma = 0.0f, mb = 0.0f;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    uint32_t w4 = 0;
    const float4 sv4 = *reinterpret_cast<const float4*>(
        s_scales + (cp / 16) * kDqScaleStride + 32 * rg + 4 * q);
    const float sv[4] = {sv4.x, sv4.y, sv4.z, sv4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = 32 * rg + 4 * q + i;
      w4 |= uint32_t(sc[r * (kDqCols / 2) + cp]) << (8 * i);
    }
    float f[8];
    e2m1x8_decode(w4, f);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      a[4 * q + i] = f[2 * i] * sv[i];
      b[4 * q + i] = f[2 * i + 1] * sv[i];
    }
#pragma unroll
    for (int i = 0; i < 4; i += 2) {
      ma = absmax3_nan(a[4 * q + i], a[4 * q + i + 1], ma);
      mb = absmax3_nan(b[4 * q + i], b[4 * q + i + 1], mb);
    }
  }
  // cols is a multiple of 32 here, so every pair index is even-aligned
  return column_pair_codes<true, true, BIG, false, OAS, true>(
      [&](int j) { return make_float2(a[j], b[j]); }, __float_as_uint(ma),
      __float_as_uint(mb), r0, tile_c + 2 * cp, cols, key);
}

// Fused double quantization of bf16 X, double-buffered: the raw tiles are
// staged with asynchronous copies, so the next tile streams in while the
// current one is quantized along rows and then along columns. Once the row
// pass is done the current raw tile is free and holds the column stage.
template <bool BIG, bool OAS>
__global__ void __launch_bounds__(kDqThreads, 3)
    k_double_quant_pipe(const void* __restrict__ x, int64_t rows, int64_t cols,
                        RngKey key, uint8_t* __restrict__ row_codes,
                        uint8_t* __restrict__ row_scales,
                        uint8_t* __restrict__ col_codes,
                        uint8_t* __restrict__ col_scales) {
  constexpr int kChunks = kTileRows * (kDqCols / 8);
  extern __shared__ uint4 smem[];  // two raw tiles, then the staged Q_D(X)
  uint32_t* s_codes = reinterpret_cast<uint32_t*>(smem + 2 * kChunks);
  float* s_scales = reinterpret_cast<float*>(s_codes + kTileRows * (kDqCols / 8));
  const int64_t tiles_c = (cols + kDqCols - 1) / kDqCols;
  const int64_t n_tiles = ((rows + kTileRows - 1) / kTileRows) * tiles_c;
  const int g = threadIdx.x & 3, tr = threadIdx.x >> 2;  // row pass
  const int cp = threadIdx.x & 63, rg = threadIdx.x >> 6;  // column pass
  int64_t t = blockIdx.x;
  if (t >= n_tiles) return;
  TileWalk cur(t, gridDim.x, tiles_c), nxt = cur;
  nxt.next();
  stage_tile_async<true, true>(x, rows, cols, cur.r * kTileRows, cur.c * kDqCols, smem);
  for (int buf = 0; t < n_tiles; t += gridDim.x, buf ^= 1, cur = nxt, nxt.next()) {
    // this tile's copies are done and visible, and every thread has left the
    // previous tile (whose buffer the next copies overwrite)
    cp_async_wait<0>();
    __syncthreads();
    if (t + gridDim.x < n_tiles)
      stage_tile_async<true, true>(x, rows, cols, nxt.r * kTileRows, nxt.c * kDqCols,
                                   smem + (buf ^ 1) * kChunks);
    const int64_t tile_r = cur.r * kTileRows;
    const int64_t tile_c = cur.c * kDqCols;
    const uint4* raw = smem + buf * kChunks;
    // this thread's row outputs: group g of tile rows tr and tr + 64
    uint8_t* rc = row_codes + (tile_r + tr) * (cols / 2) + (tile_c + 32 * g) / 2;
    uint8_t* rs = row_scales + (tile_r + tr) * (cols / 32) + (tile_c + 32 * g) / 32;
    const bool g_ok = tile_c + 32 * g < cols;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int r = tr + 64 * k;
      dq_row_group<OAS>(raw + r * (kDqCols / 8), g, r, g_ok && tile_r + r < rows,
                        rc + k * 64 * (cols / 2), rs + k * 64 * (cols / 32),
                        reinterpret_cast<uint4*>(s_codes) + r * (kDqCols / 32) + g,
                        s_scales + g * kDqScaleStride + r);
    }
    __syncthreads();
    static_assert(ColStage<kDqCols>::kBytes <= kChunks * 16, "stage fits a tile");
    uint4* s_col = smem + buf * kChunks;
    uint8_t* s_sc = reinterpret_cast<uint8_t*>(s_col + ColStage<kDqCols>::kChunks);
    if (tile_r + 32 * rg < rows)
      stage_column_pair(dq_column_pass<BIG, OAS>(s_codes, s_scales, rg, cp, tile_r,
                                            tile_c, cols, key),
                        cp, rg, s_col, s_sc);
    __syncthreads();
    store_staged_columns<kDqCols, kDqThreads>(s_col, s_sc, tile_r, tile_c,
                                              rows, cols, col_codes, col_scales);
  }
}

// Fused double quantization of bf16 X, second form. The row pass writes,
// in place of each 1x32 group it read from the staged tile, the group's
// Q_D(X) / 2 as bf16 (exact: a decoded value has two significant bits and
// an exponent of at least -130), decoded from the codes it stores (through
// shared memory: codes are only decoded from memory). The column pass then
// runs the bf16 column kernel's stochastic rounding on those words (no
// saturation: a decoded value never scales past 6). X is read once.
constexpr int kDq3StageBytes = ColStage<kDqCols>::kBytes;

template <bool OAS>
__device__ __forceinline__ void dq3_row_group(uint4* row, int g, int tr, bool ok,
                                              uint8_t* __restrict__ rc,
                                              uint8_t* __restrict__ rs, uint4* s_code) {
  uint32_t w[16];
  const int sw = dq_swizzle(g, tr);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 q = row[4 * g + (c ^ sw)];
    w[4 * c] = q.x, w[4 * c + 1] = q.y, w[4 * c + 2] = q.z, w[4 * c + 3] = q.w;
  }
  uint32_t m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = bf16x2_absmax_nan(w[2 * i], w[2 * i + 1]);
#pragma unroll
  for (int n = 4; n >= 1; n /= 2)
#pragma unroll
    for (int i = 0; i < n; ++i) m[i] = bf16x2_absmax_nan(m[i], m[i + n]);
  const uint32_t mm = m[0] & 0x7FFF7FFFu;
  const uint32_t amax = max(mm << 16, mm & 0xFFFF0000u);
  const uint32_t sb = OAS ? scale_byte_oas(amax) : scale_byte(amax);
  const unsigned short s16 = bf16_inv_scale(min(sb, 253u));
  uint32_t word[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float v[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] = bf16lo_mul(w[4 * c + j], s16);
      v[2 * j + 1] = bf16hi_mul(w[4 * c + j], s16);
    }
    word[c] = sb == 0xFFu ? 0u : e2m1x8_rn(v);
  }
  const uint4 out = make_uint4(word[0], word[1], word[2], word[3]);
  if (ok) {
    *reinterpret_cast<uint4*>(rc) = out;
    *rs = uint8_t(sb);
  }
  // decode from shared memory: Q_D(X) / 2 = G[m] 2^(e-1) (a group of scale
  // 0xFF has codes 0 and the value +inf: it decodes to NaN)
  *s_code = out;
  uint32_t wb[4];  // a load the compiler cannot replace by the stored registers
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(wb[0]), "=r"(wb[1]), "=r"(wb[2]), "=r"(wb[3])
               : "r"(smem_addr(s_code))
               : "memory");
  const float sv = half_scale_value(sb);
  const unsigned short one = 0x3C00;  // 1.0 as f16
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t h[4];
    e2m1x4_decode_rows(wb[c], h);  // elements 8c+2i, 8c+2i+1 in h[i]
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      o[i] = prmt(__float_as_uint(f16lo_f32(h[i], one) * sv),
                  __float_as_uint(f16hi_f32(h[i], one) * sv), 0x7632u);
    row[4 * g + (c ^ sw)] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

template <bool OAS>
__global__ void __launch_bounds__(kDqThreads, 3)
    k_double_quant_pipe3(const void* __restrict__ x, int64_t rows, int64_t cols,
                         RngKey key, uint8_t* __restrict__ row_codes,
                         uint8_t* __restrict__ row_scales,
                         uint8_t* __restrict__ col_codes,
                         uint8_t* __restrict__ col_scales) {
  constexpr int kChunks = kTileRows * (kDqCols / 8);
  extern __shared__ uint4 smem[];  // two raw tiles, then the codes / column stage
  uint4* s_codes = smem + 2 * kChunks;
  uint4* s_col = s_codes;  // the column stage reuses the codes' space
  uint8_t* s_sc = reinterpret_cast<uint8_t*>(s_col + ColStage<kDqCols>::kChunks);
  const int64_t tiles_c = (cols + kDqCols - 1) / kDqCols;
  const int64_t n_tiles = ((rows + kTileRows - 1) / kTileRows) * tiles_c;
  const int g = threadIdx.x & 3, tr = threadIdx.x >> 2;    // row pass
  const int cp = threadIdx.x & 63, rg = threadIdx.x >> 6;  // column pass
  // the column pass's word offsets within a row (the chunk slot depends on
  // the row's parity through the staging swizzle)
  const int chunk = cp >> 2, cg = chunk >> 2;
  const int off_even = ((chunk ^ dq_swizzle(cg, 0)) << 2) + (cp & 3);
  const int off_odd = ((chunk ^ dq_swizzle(cg, 1)) << 2) + (cp & 3);
  const uint32_t hc = uint32_t(uint64_t(cols) >> 1);
  int64_t t = blockIdx.x;
  if (t >= n_tiles) return;
  TileWalk cur(t, gridDim.x, tiles_c), nxt = cur;
  nxt.next();
  stage_tile_async<true, true>(x, rows, cols, cur.r * kTileRows, cur.c * kDqCols, smem);
  for (int buf = 0; t < n_tiles; t += gridDim.x, buf ^= 1, cur = nxt, nxt.next()) {
    cp_async_wait<0>();
    __syncthreads();
    if (t + gridDim.x < n_tiles)
      stage_tile_async<true, true>(x, rows, cols, nxt.r * kTileRows, nxt.c * kDqCols,
                                   smem + (buf ^ 1) * kChunks);
    const int64_t tile_r = cur.r * kTileRows;
    const int64_t tile_c = cur.c * kDqCols;
    uint4* raw = smem + buf * kChunks;
    uint8_t* rc = row_codes + (tile_r + tr) * (cols / 2) + (tile_c + 32 * g) / 2;
    uint8_t* rs = row_scales + (tile_r + tr) * (cols / 32) + (tile_c + 32 * g) / 32;
    const bool g_ok = tile_c + 32 * g < cols;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int r = tr + 64 * k;
      dq3_row_group<OAS>(raw + r * (kDqCols / 8), g, r, g_ok && tile_r + r < rows,
                         rc + k * 64 * (cols / 2), rs + k * 64 * (cols / 32),
                         s_codes + r * (kDqCols / 32) + g);
    }
    __syncthreads();
    if (tile_r + 32 * rg < rows) {
      const uint32_t* s = reinterpret_cast<const uint32_t*>(raw) + 32 * rg * (kDqCols / 2);
      uint32_t m = 0, wr[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        wr[j] = s[j * (kDqCols / 2) + ((j & 1) ? off_odd : off_even)];
        m = bf16x2_absmax_nan(m, wr[j]);
      }
      m &= 0x7FFF7FFFu;
      const uint32_t ma = m << 16, mb = m & 0xFFFF0000u;
      const uint32_t sa = OAS ? scale_byte_oas_of_double(ma) : scale_byte_of_double(ma);
      const uint32_t sb = OAS ? scale_byte_oas_of_double(mb) : scale_byte_of_double(mb);
      const int64_t r0 = tile_r + 32 * rg, c0 = tile_c + 2 * cp;
      ColPair o;
      if (sa >= 1u && sb >= 1u && sa != 0xFFu && sb != 0xFFu) {
        o = column_pair_sr_bf16<false, true>(
            wr, sa, sb,
            key.k0 + uint32_t((uint64_t(r0) * uint64_t(cols) + uint64_t(c0)) >> 1), hc);
      } else {
        o = column_pair_codes<true, true, false, false, OAS, true>(
            [&](int j) { return make_float2(bf16_lo(wr[j]), bf16_hi(wr[j])); }, ma, mb, r0,
            c0, cols, key);
      }
      stage_column_pair(o, cp, rg, s_col, s_sc);
    }
    __syncthreads();
    store_staged_columns<kDqCols, kDqThreads>(s_col, s_sc, tile_r, tile_c,
                                              rows, cols, col_codes, col_scales);
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------

int persistent_grid(const void* kernel, int threads, size_t smem,
                    int64_t work_blocks) {
  int dev = 0, sms = 148, per_sm = 1;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads,
                                                    smem) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  int64_t g = int64_t(sms) * per_sm;
  if (work_blocks < g) g = work_blocks;
  return static_cast<int>(g < 1 ? 1 : g);
}

template <bool BF16, bool SR, bool OAS>
static cudaError_t quant_rows_impl(const void* x, int64_t n_groups,
                                   RngKey key, uint8_t* codes,
                                   uint8_t* scales, cudaStream_t s) {
  // bf16 groups in flight per thread: two for nearest rounding (memory
  // bound), one for stochastic rounding (issue bound: the fewer registers
  // measured 2% faster than two or three)
  constexpr int U = BF16 ? (SR ? 1 : 2) : 1;
  auto kern = k_quant_rows<BF16, SR, U, OAS>;
  const int64_t groups_per_block = int64_t(kRowThreads) * U;
  const int grid = persistent_grid(reinterpret_cast<const void*>(kern), kRowThreads, 0,
                                   (n_groups + groups_per_block - 1) / groups_per_block);
  kern<<<grid, kRowThreads, 0, s>>>(x, n_groups, key, codes, scales);
  return cudaGetLastError();
}

template <bool OAS>
static cudaError_t quant_rows_rule(const void* x, bool bf16, int64_t n_groups,
                                   bool sr, RngKey key, uint8_t* codes,
                                   uint8_t* scales, cudaStream_t s) {
  if (bf16)
    return sr ? quant_rows_impl<true, true, OAS>(x, n_groups, key, codes, scales, s)
              : quant_rows_impl<true, false, OAS>(x, n_groups, key, codes, scales, s);
  return sr ? quant_rows_impl<false, true, OAS>(x, n_groups, key, codes, scales, s)
            : quant_rows_impl<false, false, OAS>(x, n_groups, key, codes, scales, s);
}

cudaError_t launch_quant_rows(const void* x, bool bf16, int64_t rows,
                              int64_t cols, bool sr, uint64_t seed,
                              uint8_t* codes, uint8_t* scales,
                              cudaStream_t s, bool oas) {
  const int64_t n_groups = rows * cols / kGroup;
  const RngKey key = make_key(seed, 0);
  return oas ? quant_rows_rule<true>(x, bf16, n_groups, sr, key, codes, scales, s)
             : quant_rows_rule<false>(x, bf16, n_groups, sr, key, codes, scales, s);
}

template <bool BF16, bool SR, bool VEC, bool EVEN, bool BIG, bool OAS>
static cudaError_t quant_cols_impl(const void* x, int64_t rows, int64_t cols,
                                   RngKey key, uint8_t* codes,
                                   uint8_t* scales, cudaStream_t s) {
  using T = ColTile<BF16>;
  const int64_t n_tiles = ((rows + kTileRows - 1) / kTileRows) *
                          ((cols + T::kCols - 1) / T::kCols);
  if (VEC) {
    auto kern = k_quant_cols_pipe<BF16, SR, EVEN, BIG, OAS>;
    constexpr size_t smem = 2 * kTileRows * T::kChunksPerRow * sizeof(uint4) +
                            ColStage<T::kCols>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(
        reinterpret_cast<const void*>(kern),
        cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    const int grid = persistent_grid(reinterpret_cast<const void*>(kern),
                                     T::kThreads, smem, n_tiles);
    kern<<<grid, T::kThreads, smem, s>>>(x, rows, cols, key, codes, scales);
  } else {
    auto kern = k_quant_cols<BF16, SR, EVEN, BIG, OAS>;
    const int grid = persistent_grid(reinterpret_cast<const void*>(kern),
                                     T::kThreads, 0, n_tiles);
    kern<<<grid, T::kThreads, 0, s>>>(x, rows, cols, key, codes, scales);
  }
  return cudaGetLastError();
}

// 2^33 elements or more: pair indices reach 2^32.
static bool big_tensor(int64_t rows, int64_t cols) {
  return rows * cols >= (int64_t(1) << 33);
}

template <bool BF16, bool OAS>
static cudaError_t quant_cols_dispatch(const void* x, int64_t rows,
                                       int64_t cols, bool sr, RngKey key,
                                       uint8_t* codes, uint8_t* scales,
                                       cudaStream_t s) {
  const bool vec = cols % (BF16 ? 8 : 4) == 0;
  if (!sr)
    return vec ? quant_cols_impl<BF16, false, true, true, false, OAS>(x, rows, cols, key, codes, scales, s)
               : quant_cols_impl<BF16, false, false, true, false, OAS>(x, rows, cols, key, codes, scales, s);
  if (cols % 2 != 0)  // odd rows split column pairs over two hashes
    return quant_cols_impl<BF16, true, false, false, true, OAS>(x, rows, cols, key, codes, scales, s);
  if (big_tensor(rows, cols))
    return vec ? quant_cols_impl<BF16, true, true, true, true, OAS>(x, rows, cols, key, codes, scales, s)
               : quant_cols_impl<BF16, true, false, true, true, OAS>(x, rows, cols, key, codes, scales, s);
  return vec ? quant_cols_impl<BF16, true, true, true, false, OAS>(x, rows, cols, key, codes, scales, s)
             : quant_cols_impl<BF16, true, false, true, false, OAS>(x, rows, cols, key, codes, scales, s);
}

cudaError_t launch_quant_cols(const void* x, bool bf16, int64_t rows,
                              int64_t cols, bool sr, uint64_t seed,
                              uint8_t* codes, uint8_t* scales,
                              cudaStream_t s, bool oas) {
  const RngKey key = make_key(seed, 0);
  if (oas)
    return bf16 ? quant_cols_dispatch<true, true>(x, rows, cols, sr, key, codes, scales, s)
                : quant_cols_dispatch<false, true>(x, rows, cols, sr, key, codes, scales, s);
  return bf16 ? quant_cols_dispatch<true, false>(x, rows, cols, sr, key, codes, scales, s)
              : quant_cols_dispatch<false, false>(x, rows, cols, sr, key, codes, scales, s);
}

cudaError_t launch_dequant(const uint8_t* codes, const uint8_t* scales,
                           int64_t n_groups, void* y, bool bf16_out,
                           cudaStream_t s) {
  constexpr int U = 8;
  const int64_t groups_per_block = (kRowThreads / 4) * U;
  const int64_t blocks = (n_groups + groups_per_block - 1) / groups_per_block;
  if (bf16_out) {
    auto kern = k_dequant<true, U>;
    const int grid = persistent_grid(reinterpret_cast<const void*>(kern),
                                     kRowThreads, 0, blocks);
    kern<<<grid, kRowThreads, 0, s>>>(codes, scales, n_groups, y);
  } else {
    auto kern = k_dequant<false, U>;
    const int grid = persistent_grid(reinterpret_cast<const void*>(kern),
                                     kRowThreads, 0, blocks);
    kern<<<grid, kRowThreads, 0, s>>>(codes, scales, n_groups, y);
  }
  return cudaGetLastError();
}

}  // namespace mxfp4

namespace mxfp4 {

template <bool OAS>
static cudaError_t double_quant_impl(const void* x, bool bf16, int64_t rows,
                                     int64_t cols, RngKey key, uint8_t* row_codes,
                                     uint8_t* row_scales, uint8_t* col_codes,
                                     uint8_t* col_scales, cudaStream_t s) {
  const int64_t n_tiles = ((rows + kTileRows - 1) / kTileRows) *
                          ((cols + kDqCols - 1) / kDqCols);
  const bool big = big_tensor(rows, cols);
  if (bf16 && !big) {
    auto kern = k_double_quant_pipe3<OAS>;
    constexpr size_t smem = 2 * kTileRows * (kDqCols / 8) * sizeof(uint4) + kDq3StageBytes;
    static_assert(kDq3StageBytes >= kTileRows * (kDqCols / 8) * 4, "codes fit the stage");
    cudaError_t e = cudaFuncSetAttribute(
        reinterpret_cast<const void*>(kern),
        cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    const int grid = persistent_grid(reinterpret_cast<const void*>(kern),
                                     kDqThreads, smem, n_tiles);
    kern<<<grid, kDqThreads, smem, s>>>(x, rows, cols, key, row_codes,
                                        row_scales, col_codes, col_scales);
    return cudaGetLastError();
  }
  if (bf16) {
    auto kern = big ? k_double_quant_pipe<true, OAS> : k_double_quant_pipe<false, OAS>;
    constexpr size_t smem = 2 * kTileRows * (kDqCols / 8) * sizeof(uint4) +
                            kTileRows * (kDqCols / 8) * 4 +
                            (kDqCols / 32) * kDqScaleStride * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(
        reinterpret_cast<const void*>(kern),
        cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    const int grid = persistent_grid(reinterpret_cast<const void*>(kern),
                                     kDqThreads, smem, n_tiles);
    kern<<<grid, kDqThreads, smem, s>>>(x, rows, cols, key, row_codes,
                                        row_scales, col_codes, col_scales);
    return cudaGetLastError();
  }
  auto kern = big ? k_double_quant<false, true, OAS> : k_double_quant<false, false, OAS>;
  const int grid = persistent_grid(reinterpret_cast<const void*>(kern),
                                   kDqThreads, 0, n_tiles);
  kern<<<grid, kDqThreads, 0, s>>>(x, rows, cols, key, row_codes, row_scales,
                                   col_codes, col_scales);
  return cudaGetLastError();
}

cudaError_t launch_double_quant(const void* x, bool bf16, int64_t rows,
                                int64_t cols, uint64_t seed,
                                uint8_t* row_codes, uint8_t* row_scales,
                                uint8_t* col_codes, uint8_t* col_scales,
                                cudaStream_t s, bool oas) {
  const RngKey key = make_key(seed, 0);
  return oas ? double_quant_impl<true>(x, bf16, rows, cols, key, row_codes, row_scales,
                                       col_codes, col_scales, s)
             : double_quant_impl<false>(x, bf16, rows, cols, key, row_codes, row_scales,
                                        col_codes, col_scales, s);
}

}  // namespace mxfp4
