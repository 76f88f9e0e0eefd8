// Device-side building blocks of the MXFP4 block quantizer (sm_100a).
//
// Format (ALTO explainer, "ALTO MXFP4 training — Weight de-oscillation",
// Jargon: MXFP4, E2M1, Bin; "Unveiling the Potential of Quantization with
// MXFP4", abstract: power-of-two block scaling):
//   - one E8M0 scale byte per 32-element group, byte = e + 127 with
//     e = floor(log2(absmax)) - 2 clamped to [-127, 127]; 0 for a zero group,
//     0xFF (codes 0) for a group holding Inf/NaN;
//   - 4-bit E2M1 codes: sign in bit 3, magnitude index m of
//     {0, .5, 1, 1.5, 2, 3, 4, 6} in bits 0..2; the even element of a pair
//     in the low nibble.
//
// All arithmetic that decides a code is exact: scaling multiplies by a power
// of two, rounding to nearest-even uses the hardware E2M1 conversion, and
// stochastic rounding compares integer bit fields. The library is built
// without fast-math and with FMA contraction off, so subnormal inputs are
// not flushed.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace mxfp4 {

constexpr int kGroup = 32;

// ---------------------------------------------------------------------------
// Counter-based random numbers. mix() is the MurmurHash3 32-bit finalizer.
// K(seed, s) = mix(lo32(seed) ^ mix(hi32(seed) + s * 0x9E3779B9));
// pair p: h = mix(mix(K ^ hi32(p)) + lo32(p)); the element with even
// row-major index i = 2p takes h & 0xFFFF, the odd one takes h >> 16.
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ uint32_t mix32(uint32_t h) {
  h ^= h >> 16;
  h *= 0x85EBCA6Bu;
  h ^= h >> 13;
  h *= 0xC2B2AE35u;
  h ^= h >> 16;
  return h;
}

__host__ __device__ __forceinline__ uint32_t stream_key(uint64_t seed,
                                                        uint32_t stream) {
  return mix32(static_cast<uint32_t>(seed) ^
               mix32(static_cast<uint32_t>(seed >> 32) + stream * 0x9E3779B9u));
}

// Per-key constants handed to kernels: the key and mix(key ^ 0), the inner
// hash of every counter below 2^32.
struct RngKey {
  uint32_t k;
  uint32_t k0;
};

__host__ __forceinline__ RngKey make_key(uint64_t seed, uint32_t stream) {
  RngKey r;
  r.k = stream_key(seed, stream);
  r.k0 = mix32(r.k ^ 0u);
  return r;
}

// mix32 on the device, in two parts: mix32_pre is every step but the last
// xor-shift, so mix32(x) = g ^ (g >> 16) with g = mix32_pre(x). Consumers of
// the two 16-bit halves take them from g directly: the high half of mix32 is
// g >> 16 (the xor only touches the low half) and the low half is
// (g ^ (g >> 16)) & 0xFFFF; the top bit of mix32 is the top bit of g. The
// stochastic-rounding kernels are bound by the integer logic pipe and the
// multiply pipe together; the two multiplies already load the latter, so the
// shifts stay plain shifts (measured: issuing them on the multiply pipe as
// high halves of products was slower).
__device__ __forceinline__ uint32_t mix32_pre(uint32_t h) {
  h ^= h >> 16;
  h *= 0x85EBCA6Bu;
  h ^= h >> 13;
  h *= 0xC2B2AE35u;
  return h;
}
__device__ __forceinline__ uint32_t mix32_d(uint32_t h) {
  const uint32_t g = mix32_pre(h);
  return g ^ (g >> 16);
}

// Inner hash for counters whose high word is `hi` (0 for every tensor below
// 2^33 elements).
__device__ __forceinline__ uint32_t inner_key(RngKey key, uint32_t hi) {
  return hi == 0 ? key.k0 : mix32_d(key.k ^ hi);
}

// ---------------------------------------------------------------------------
// Scale
// ---------------------------------------------------------------------------

// E8M0 byte from the fp32 bit pattern of |absmax| (bf16 inputs are widened
// first: same exponent field). With E the biased exponent field,
// floor(log2 absmax) = E - 127 for normal values, so byte = E - 2, clamped at
// 0, which also covers zero and subnormal maxima (e clamps to -127).
__device__ __forceinline__ uint32_t scale_byte(uint32_t abs_bits) {
  uint32_t E = abs_bits >> 23;
  return abs_bits >= 0x7F800000u ? 0xFFu : (E > 2u ? E - 2u : 0u);
}

// Overflow-aware variant ("Unveiling the Potential of Quantization with
// MXFP4", abstract: overflow-aware scaling): the smallest e with
// absmax 2^-e <= 6. The OCP exponent leaves absmax 2^-e in [4, 8); it moves
// up by one exactly when that exceeds 6, i.e. when the mantissa of absmax is
// above 1.5 (mantissa field > 0x400000). Below the exponent field 2 the OCP
// byte is clamped at 0 and the scaled maximum stays under 4.
__device__ __forceinline__ uint32_t scale_byte_oas(uint32_t abs_bits) {
  const uint32_t sb = scale_byte(abs_bits);
  const bool up = abs_bits >= (2u << 23) && abs_bits < 0x7F800000u &&
                  (abs_bits & 0x7FFFFFu) > 0x400000u;
  return sb + (up ? 1u : 0u);
}

// 2^-e as fp32 for byte sb = e + 127 <= 253 (the OCP rule reaches 252, the
// overflow-aware one 253): biased exponent 254 - sb, normal throughout.
__device__ __forceinline__ float inv_scale(uint32_t sb) {
  uint32_t b = sb > 253u ? 253u : sb;
  return __uint_as_float((254u - b) << 23);
}

// The double quantizer carries its decoded row groups at half their size,
// G[m] 2^(e-1), so that the largest, 6 2^126 under the overflow-aware rule,
// stays finite (exact: at least 0.5 2^-128). half_scale_value(sb) = 2^(e-1)
// (sb 0 and 1: the subnormals 2^-128, 2^-127; sb 0xFF: +inf), and the
// column scale bytes of such halved values: scale_byte / scale_byte_oas of
// twice the maximum, from the fp32 bit pattern of the halved maximum (one
// exponent step down; below 2^-125 the OCP byte is 0 either way).
__device__ __forceinline__ float half_scale_value(uint32_t sb) {
  return __uint_as_float(sb == 0xFFu ? 0x7F800000u
                                     : (sb >= 2u ? (sb - 1u) << 23 : 0x00200000u << sb));
}
__device__ __forceinline__ uint32_t scale_byte_of_double(uint32_t half_bits) {
  const uint32_t E = half_bits >> 23;
  return half_bits >= 0x7F800000u ? 0xFFu : (E > 1u ? E - 1u : 0u);
}
__device__ __forceinline__ uint32_t scale_byte_oas_of_double(uint32_t half_bits) {
  const bool up = half_bits >= (1u << 23) && half_bits < 0x7F800000u &&
                  (half_bits & 0x7FFFFFu) > 0x400000u;
  return scale_byte_of_double(half_bits) + (up ? 1u : 0u);
}

// 2^(e-1) and 6 2^e as fp32 for byte sb = e + 127 in [2, 252].
__device__ __forceinline__ float scale_half(uint32_t sb) {
  return __uint_as_float((sb - 1u) << 23);
}
__device__ __forceinline__ float scale_six(uint32_t sb) {
  return __uint_as_float(((sb + 2u) << 23) | 0x400000u);
}

// 2^e as fp32 for byte sb (sb = 0 gives the subnormal 2^-127, whose pattern
// 0x00400000 lies below every normal one; sb = 0xFF gives +inf).
__device__ __forceinline__ float scale_value(uint32_t sb) {
  return __uint_as_float(max(sb << 23, 0x00400000u));
}

// ---------------------------------------------------------------------------
// E2M1 rounding
// ---------------------------------------------------------------------------

// Round 8 scaled values to nearest-even E2M1 with saturation to +-6 (the
// hardware conversion); element j lands in nibble j of the result.
__device__ __forceinline__ uint32_t e2m1x8_rn(const float* v) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]),
        "f"(v[6]), "f"(v[7]));
  return out;
}

// Stochastic E2M1 code of one scaled value v (exact): lo = largest grid
// value <= |v|, hi = the next one; the result is hi iff
// (r + 0.5) * 2^-16 < (|v| - lo) / (hi - lo), r the element's 16-bit random
// number; |v| >= 6 gives 6.
//
// In every binade [2^k, 2^k+1) with k >= 0 the grid keeps one mantissa bit,
// so the low 22 mantissa bits of |v| are frac * 2^22 exactly, and the code is
// the top bits of |v| minus those of 0.5. Below 1 the grid step is 0.5
// throughout; (1 + |v|) / 2 rounded up maps [0, 1) onto [0.5, 1] with the
// same structure (and is the smaller of the two for |v| >= 1, the larger
// below), and rounding up keeps the test exact because the threshold lies on
// the 2^-18 grid. The test frac * 2^22 > 64r + 32 is an addition: with
// noise = 2^22 - 33 - 64r, the mantissa field plus noise carries into bit 22
// exactly when the value goes up (the carry may run on into the exponent:
// 1.5 -> 2, 3 -> 4). The bias 0.5 = 0x3F000000 is folded into the noise.
//
// The sum lies in [31, 2^25), magnitude index in bits 22..24; it is formed
// times 64 (one multiply-add), which puts the index in bits 28..30 with bit
// 31 clear for the sign: the code is the top nibble, and codes are packed by
// funnel shifts of those nibbles. sr_noise64(r) = 64 (2^22 - 33 - 64r) -
// 64 * 0x3F000000 mod 2^32.
__device__ __forceinline__ uint32_t sr_noise64(uint32_t r) {
  return r * 0xFFFFF000u + 0x4FFFF7C0u;
}
// The noises of the pair whose hash is mix32 = g ^ (g >> 16), g = mix32_pre
// of its counter: the even element takes the low half, the odd one the high
// half (g >> 16: the xor only touches the low half).
__device__ __forceinline__ void sr_noise64_pair(uint32_t g, uint32_t& n_even,
                                                uint32_t& n_odd) {
  const uint32_t hi = g >> 16;
  n_even = sr_noise64((g ^ hi) & 0xFFFFu);
  n_odd = sr_noise64(hi);
}

// The same noise for a value left unscaled by 2^-e, e = sb - 127, and its
// pair form: with y the rounding operand of v 2^-e (normal) and y' = 2^e y
// that of v (normal when e >= -125), bits(y) = bits(y') - e 2^23, so
// 64 bits(y) + sr_noise64(r) = 64 bits(y') + (r * 0xFFFFF000 + base).
__device__ __forceinline__ uint32_t sr_noise64_base(uint32_t sb) {
  return 0x4FFFF7C0u - ((sb - 127u) << 29);
}
__device__ __forceinline__ void sr_noise64_pair_based(uint32_t g, uint32_t base_even,
                                                      uint32_t base_odd, uint32_t& n_even,
                                                      uint32_t& n_odd) {
  const uint32_t hi = g >> 16;
  n_even = ((g ^ hi) & 0xFFFFu) * 0xFFFFF000u + base_even;
  n_odd = hi * 0xFFFFF000u + base_odd;
}

// The stochastic code of v in bits 28..31 (sign in bit 31; the bits below
// are not part of it). SAT = false leaves out the saturation, for callers
// whose |v| never exceeds 6.
template <bool SAT = true>
__device__ __forceinline__ uint32_t e2m1_sr_top(float v, uint32_t noise64) {
  const float a = fabsf(v);
  float y = fmaxf(a, __fmaf_ru(a, 0.5f, 0.5f));
  if (SAT) y = fminf(y, 6.0f);  // |v| >= 6 saturates to 6
  return (__float_as_uint(y) * 64u + noise64) |
         (__float_as_uint(v) & 0x80000000u);
}

// e2m1_sr_top of v 2^-e computed on the unscaled v, for scale bytes
// sb = e + 127 in [2, 252]: half = 2^(e-1), sat = 6 2^e (scale_half,
// scale_six), noise from sr_noise64_pair_based with base
// sr_noise64_base(sb). Every step is the unscaled one times 2^e, and each
// result is normal (y' >= 2^(e-1) >= 2^-126), so the rounding up and the
// comparisons are those of the scaled value; a value whose scaled form
// would underflow is below 2^-126 and gives the same code (the carry needs
// a scaled value of at least 33 2^-23).
template <bool SAT>
__device__ __forceinline__ uint32_t e2m1_sr_top_scaled(float v, float half, float sat,
                                                      uint32_t noise) {
  const float a = fabsf(v);
  float y = fmaxf(a, __fmaf_ru(a, 0.5f, half));
  if (SAT) y = fminf(y, sat);
  return (__float_as_uint(y) * 64u + noise) | (__float_as_uint(v) & 0x80000000u);
}

// e2m1x8_sr on 8 unscaled values (e2m1_sr_top_scaled; scale byte in
// [2, 252], or up to 253 with SAT = false).
template <bool SAT>
__device__ __forceinline__ uint32_t e2m1x8_sr_scaled(const float* v, const uint32_t* g,
                                                    float half, float sat, uint32_t base);

// Shift a packed code word up by one nibble and append the code held in the
// top nibble of t: codes pushed in the order 7, 6, .., 0 land in nibbles
// 7 .. 0.
__device__ __forceinline__ uint32_t push_code(uint32_t acc, uint32_t t) {
  return __funnelshift_l(t, acc, 4);
}

// Stochastic codes of 8 values; pair k of the 8 values takes its two random
// numbers from the hash whose mix32_pre is g[k] (low half for the even
// element).
__device__ __forceinline__ uint32_t e2m1x8_sr(const float* v,
                                              const uint32_t* g) {
  uint32_t out = 0;
#pragma unroll
  for (int k = 3; k >= 0; --k) {
    uint32_t ne, no;
    sr_noise64_pair(g[k], ne, no);
    out = push_code(out, e2m1_sr_top(v[2 * k + 1], no));
    out = push_code(out, e2m1_sr_top(v[2 * k], ne));
  }
  return out;
}

template <bool SAT>
__device__ __forceinline__ uint32_t e2m1x8_sr_scaled(const float* v, const uint32_t* g,
                                                    float half, float sat, uint32_t base) {
  uint32_t out = 0;
#pragma unroll
  for (int k = 3; k >= 0; --k) {
    uint32_t ne, no;
    sr_noise64_pair_based(g[k], base, base, ne, no);
    out = push_code(out, e2m1_sr_top_scaled<SAT>(v[2 * k + 1], half, sat, no));
    out = push_code(out, e2m1_sr_top_scaled<SAT>(v[2 * k], half, sat, ne));
  }
  return out;
}

// Nearest-even E2M1 value of a scaled v (exact, no codes): with K the power
// of two 2^(max(E,0) + 22), E the binade of |v|, the fp32 sum |v| + K has an
// ulp equal to the E2M1 grid step at |v| (2^(E-1), or 0.5 below 1), so the
// round-to-nearest-even addition lands on the nearest grid value with ties to
// the even one and the subtraction is exact; values from 6 up saturate to 6.
// The sign of v is kept (a negative value that rounds to 0 gives -0).
__device__ __forceinline__ float e2m1_rn_value(float v) {
  const uint32_t vb = __float_as_uint(v);
  const uint32_t ab = vb & 0x7FFFFFFFu;
  const uint32_t eb = ab & 0x7F800000u;
  const float K = __uint_as_float((eb > 0x3F800000u ? eb : 0x3F800000u) + 0x0B000000u);
  const float a = __uint_as_float(ab);
  float q = __fsub_rn(__fadd_rn(a, K), K);
  q = fminf(q, 6.0f);
  return __uint_as_float(__float_as_uint(q) | (vb & 0x80000000u));
}

// ---------------------------------------------------------------------------
// Decode
// ---------------------------------------------------------------------------

// The 8 codes of one 32-bit word as fp32 values G[m] with their signs
// (hardware E2M1 -> f16 conversion, exact), element j from nibble j.
// Decode only words that were loaded from memory (global or shared): feeding
// the result of e2m1x8_rn straight into this conversion in registers produced
// wrong values in one kernel shape on this toolchain, so no kernel does that.
__device__ __forceinline__ void e2m1x8_decode(uint32_t w, float* out) {
  uint32_t h0, h1, h2, h3;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
      : "r"(w));
  const uint32_t h[4] = {h0, h1, h2, h3};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float lo, hi;
    asm("{\n\t.reg .f16 l, u;\n\t"
        "mov.b32 {l, u}, %2;\n\t"
        "cvt.f32.f16 %0, l;\n\t"
        "cvt.f32.f16 %1, u;\n\t}"
        : "=f"(lo), "=f"(hi)
        : "r"(h[k]));
    out[2 * k] = lo;
    out[2 * k + 1] = hi;
  }
}

// ---------------------------------------------------------------------------
// Packed bf16 helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ float bf16_lo(uint32_t w) {
  return __uint_as_float(w * 65536u);
}
__device__ __forceinline__ float bf16_hi(uint32_t w) {
  return __uint_as_float(w & 0xFFFF0000u);
}

// max(|a|, m) for m >= 0 or NaN, propagating NaN (a NaN a or m gives NaN).
__device__ __forceinline__ float absmax_nan(float a, float m) {
  float d;
  asm("{\n\t.reg .f32 t;\n\tabs.f32 t, %1;\n\tmax.NaN.f32 %0, t, %2;\n\t}"
      : "=f"(d)
      : "f"(a), "f"(m));
  return d;
}

// max(|a|, |b|, m) for m >= 0 or NaN, propagating NaN.
__device__ __forceinline__ float absmax3_nan(float a, float b, float m) {
  float d;
  asm("{\n\t.reg .f32 t, u;\n\tabs.f32 t, %1;\n\tabs.f32 u, %2;\n\t"
      "max.NaN.f32 %0, t, u, %3;\n\t}"
      : "=f"(d)
      : "f"(a), "f"(b), "f"(m));
  return d;
}

// Per-half unsigned max of two packed 16-bit pairs.
__device__ __forceinline__ uint32_t umax16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Per-half max(|a|, |b|) of two packed bf16 pairs, propagating NaN (a NaN
// half gives the canonical NaN); the sign bits of the result are not
// defined, callers mask them.
__device__ __forceinline__ uint32_t bf16x2_absmax_nan(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// fp32 bit pattern of the largest |value| among 8 packed bf16 values (any
// Inf/NaN gives a pattern of at least 0x7F800000): the absolute bit patterns
// order like the magnitudes, so the two halves combine with an integer max.
__device__ __forceinline__ uint32_t bf16x8_absmax(uint4 w) {
  const uint32_t m = bf16x2_absmax_nan(bf16x2_absmax_nan(w.x, w.y),
                                       bf16x2_absmax_nan(w.z, w.w)) &
                     0x7FFF7FFFu;
  return max(m << 16, m & 0xFFFF0000u);
}

// Two exact fp32 values -> packed bf16x2 (low element in the low half).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// Shared-state-space address of a generic pointer into shared memory.
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte load of read-once data: no L1 allocation.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

// Asynchronous 16-byte global -> shared copy (bypassing L1). When !valid
// nothing is read and the 16 shared bytes are zero-filled; src must still be
// a mapped global address.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* src,
                                           bool valid) {
  const unsigned dst = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst),
               "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
// Wait until at most N committed groups of this thread are still pending.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// 16-byte read-only load that allocates in L1: for threads that read 32 or
// more contiguous bytes in 16-byte steps, where one warp instruction covers
// only half of each 32-byte sector and the next instruction the other half.
__device__ __forceinline__ uint4 ld_l1(const void* p) {
  uint4 r;
  asm("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

// ---------------------------------------------------------------------------
// Stochastic rounding of bf16 inputs with few integer-logic instructions.
//
// On sm_100a the integer-logic pipe (logic ops, shifts, byte permutes,
// minimum/maximum, the E2M1 conversions) issues at half the rate of the FMA
// pipes and bounds the stochastic-rounding kernels, so these helpers move
// work onto the FMA pipes: a bf16 value is widened and scaled by 2^-e in
// one exact mixed-precision product, the saturation runs on packed bf16
// pairs, two codes share one byte-merge, and the signs are gathered from
// the input words by byte permutes, eight codes at a time.
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
// (a & c) | (b & ~c)
__device__ __forceinline__ uint32_t bitsel(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// (a & b) | c
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// a * b + c on the multiply pipe (an integer add there would take a logic
// pipe slot)
__device__ __forceinline__ uint32_t mad_u32(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// Per half: the sign of w with magnitude min(|w|, sat), sat >= 0 (the
// saturation at 6 2^e, a bf16 value, applied to two inputs at once).
__device__ __forceinline__ uint32_t bf16x2_clamp_abs(uint32_t w, uint32_t sat2) {
  uint32_t d;
  asm("min.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(w), "r"(sat2));
  return d;
}
// The low / high bf16 half of w times s16 (a bf16 power of two), as fp32:
// one exact mixed-precision product on the FMA pipe (both factors have at
// most 8 significant bits; no flush of subnormals).
__device__ __forceinline__ float bf16lo_mul(uint32_t w, unsigned short s16) {
  float d;
  asm("{.reg .b16 l, h; mov.b32 {l, h}, %1;\n\t"
      "fma.rn.f32.bf16 %0, l, %2, %3;}" : "=f"(d) : "r"(w), "h"(s16), "f"(-0.0f));
  return d;
}
__device__ __forceinline__ float bf16hi_mul(uint32_t w, unsigned short s16) {
  float d;
  asm("{.reg .b16 l, h; mov.b32 {l, h}, %1;\n\t"
      "fma.rn.f32.bf16 %0, h, %2, %3;}" : "=f"(d) : "r"(w), "h"(s16), "f"(-0.0f));
  return d;
}
// 2^-e as bf16 bits for scale byte sb = e + 127 in [0, 253].
__device__ __forceinline__ unsigned short bf16_inv_scale(uint32_t sb) {
  return static_cast<unsigned short>((254u - sb) << 7);
}
// 6 2^e as bf16 bits in both halves (sb in [0, 252]).
__device__ __forceinline__ uint32_t bf16x2_six_scale(uint32_t sb) {
  return (((sb + 2u) << 7) | 0x40u) * 0x10001u;
}

// The rounding operand y of the carry test (e2m1_sr_top) of a scaled value
// v, without saturation (callers clamp beforehand) and without the sign.
__device__ __forceinline__ uint32_t sr_operand(float v) {
  const float a = fabsf(v);
  return __float_as_uint(fmaxf(a, __fmaf_ru(a, 0.5f, 0.5f)));
}
// The same for v held unscaled, half = 2^(e-1) (e2m1_sr_top_scaled).
__device__ __forceinline__ uint32_t sr_operand_scaled(float v, float half) {
  const float a = fabsf(v);
  return __float_as_uint(fmaxf(a, __fmaf_ru(a, 0.5f, half)));
}

// Two forms of the carry test's sum for scaled values: x64 (the sum times
// 64, magnitude index in bits 28..30, the bits below are not part of it) =
// y * 64 + r * 0xFFFFF000 + kSrBase64, and x4 (the sum times 4: index in
// bits 24..26, bits 27..31 zero, since the sum is below 2^25) = y * 4 +
// r * 0xFFFFFF00 + kSrBase4; r the element's 16-bit random number.
constexpr uint32_t kSrBase64 = 64u * (0x400000u - 33u) - (0x3F000000u << 6);
constexpr uint32_t kSrBase4 = 4u * (0x400000u - 33u) - (0x3F000000u << 2);
// The bases for operands held unscaled by 2^e, e = u - 127 (see
// sr_noise64_base): the sum is the same integer.
__device__ __forceinline__ uint32_t sr_base64(uint32_t u) {
  return 64u * (0x400000u - 33u) - ((0x3F000000u + ((u - 127u) << 23)) << 6);
}
__device__ __forceinline__ uint32_t sr_base4(uint32_t u) {
  return 4u * (0x400000u - 33u) - ((0x3F000000u + ((u - 127u) << 23)) << 2);
}

// The byte of a pair of codes, in bits 24..31 (the bits below are not part
// of it): the odd element's x64 sum over the even element's x4 sum, whose
// bits above its index are zero; signs are added afterwards.
__device__ __forceinline__ uint32_t pair_byte(uint32_t t_odd64, uint32_t t_even4) {
  return and_or(t_odd64, 0xF0000000u, t_even4);
}
// Four pair bytes (pairs 0..3 of eight consecutive codes) into one code word.
__device__ __forceinline__ uint32_t pack_pair_bytes(uint32_t b0, uint32_t b1, uint32_t b2,
                                                    uint32_t b3) {
  return prmt(prmt(b0, b1, 0x0073u), prmt(b2, b3, 0x7300u), 0x7610u);
}

// Sign bits (bit 4i+3) of the codes of 8 bf16 values held in 4 words,
// element 2k in the low half of word k: byte permutes replicate each sign
// over a byte, a bit select merges the even and odd elements' bytes.
__device__ __forceinline__ uint32_t sign_nibbles_rows(uint32_t w0, uint32_t w1, uint32_t w2,
                                                      uint32_t w3) {
  const uint32_t p01 = prmt(w0, w1, 0xFDB9u), p23 = prmt(w2, w3, 0xFDB9u);
  const uint32_t e = prmt(p01, p23, 0x6420u), o = prmt(p01, p23, 0x7531u);
  return bitsel(e, o, 0x0F0F0F0Fu) & 0x88888888u;
}
// The same for two columns over 8 rows: word w[j] of row j holds column a
// in its low half and column b in its high half (bf16 or f16); ta, tb get
// the sign of row i in bit 4i+3.
__device__ __forceinline__ void sign_nibbles_cols(const uint32_t* w, uint32_t& ta, uint32_t& tb) {
  const uint32_t qlo = prmt(w[0], w[2], 0xFBD9u), rlo = prmt(w[1], w[3], 0xFBD9u);
  const uint32_t qhi = prmt(w[4], w[6], 0xFBD9u), rhi = prmt(w[5], w[7], 0xFBD9u);
  const uint32_t mlo = bitsel(qlo, rlo, 0x0F0F0F0Fu), mhi = bitsel(qhi, rhi, 0x0F0F0F0Fu);
  ta = prmt(mlo, mhi, 0x5410u) & 0x88888888u;
  tb = prmt(mlo, mhi, 0x7632u) & 0x88888888u;
}

// The two 16-bit random numbers of a pair whose hash has mix32_pre g (low
// half, after the finalizer's last xorshift, for the even element).
__device__ __forceinline__ void pair_randoms(uint32_t g, uint32_t& r_even, uint32_t& r_odd) {
  r_odd = g >> 16;
  r_even = (g ^ r_odd) & 0xFFFFu;
}

// Stochastic codes of 8 bf16 values of a 1x32 group (four packed words wq,
// element 2k in the low half of wq[k]) whose scale byte sb is not 0xFF, as
// the row quantizer forms them: each value is widened and scaled by 2^-e in
// one exact mixed-precision product (s16 = bf16_inv_scale(sb)), after the
// packed pairs are saturated at 6 2^e (sat2 = bf16x2_six_scale(sb); the
// overflow-aware rule never exceeds 6); pair k of the 8 takes its random
// numbers from the hash of counter kh + 4 q + k; the codes of a pair share
// one byte merge and the signs come from the input words.
template <bool OAS>
__device__ __forceinline__ uint32_t bf16x8_sr_word(const uint32_t* wq, unsigned short s16,
                                                   uint32_t sat2, uint32_t kh, uint32_t q) {
  uint32_t pb[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t ws = OAS ? wq[k] : bf16x2_clamp_abs(wq[k], sat2);
    uint32_t re, ro;
    pair_randoms(mix32_pre(mad_u32(4u * q + uint32_t(k), 1u, kh)), re, ro);
    const uint32_t te = mad_u32(sr_operand(bf16lo_mul(ws, s16)), 4u,
                                mad_u32(re, 0xFFFFFF00u, kSrBase4));
    const uint32_t to = mad_u32(sr_operand(bf16hi_mul(ws, s16)), 64u,
                                mad_u32(ro, 0xFFFFF000u, kSrBase64));
    pb[k] = pair_byte(to, te);
  }
  return pack_pair_bytes(pb[0], pb[1], pb[2], pb[3]) |
         sign_nibbles_rows(wq[0], wq[1], wq[2], wq[3]);
}

// f16 halves as fp32 by an exact mixed-precision product with one (f16 1.0)
// on the FMA pipe.
__device__ __forceinline__ float f16lo_f32(uint32_t h, unsigned short one) {
  float d;
  asm("{.reg .b16 l, u; mov.b32 {l, u}, %1;\n\t"
      "fma.rn.f32.f16 %0, l, %2, %3;}" : "=f"(d) : "r"(h), "h"(one), "f"(-0.0f));
  return d;
}
__device__ __forceinline__ float f16hi_f32(uint32_t h, unsigned short one) {
  float d;
  asm("{.reg .b16 l, u; mov.b32 {l, u}, %1;\n\t"
      "fma.rn.f32.f16 %0, u, %2, %3;}" : "=f"(d) : "r"(h), "h"(one), "f"(-0.0f));
  return d;
}
// The 4 bytes of w as 4 f16x2 words of E2M1 values (byte i's low nibble in
// the low half of h[i]). Decode only words loaded from memory (see
// e2m1x8_decode).
__device__ __forceinline__ void e2m1x4_decode_rows(uint32_t w, uint32_t* h) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3]) : "r"(w));
}

constexpr uint32_t kNaNbf16x2 = 0x7FC07FC0u;
constexpr uint32_t kNaNf32 = 0x7FC00000u;

}  // namespace mxfp4
