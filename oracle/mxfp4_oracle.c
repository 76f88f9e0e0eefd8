/*
 * MXFP4 block quantizer — CPU ORACLE. TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously correct restatement of what the quantizer
 * computes, used only by the tests, the smoke check and the CPU baseline of
 * the benchmark. The product path never calls it. It shares no code, header,
 * table or helper with the CUDA library.
 *
 * Arithmetic is fp64 throughout. Where the method's own state is fp32 (the
 * oscillation tracker's caller-owned arrays) each update is computed in fp64
 * and rounded to fp32 once, which is the same as the fp32 operation.
 * Build with -O2 -ffp-contract=off (no fused multiply-add, no fast-math).
 *
 * Sources ("the pages"):
 *  [ALTO]  "ALTO MXFP4 training — Weight de-oscillation — What does it mean?"
 *          Jargon (MXFP4, E2M1, Bin, Randomized Hadamard transform,
 *          Stochastic rounding); the paragraphs on the block scale set by the
 *          largest magnitude, on the d_Q/d_w ratio, and the worked example.
 *  [TJ]    "Oscillation-Reduced MXFP4 Training for Vision Transformers",
 *          rebuttal, Question 2 (double quantization, group shapes).
 *  [OAS]   "Unveiling the Potential of Quantization with MXFP4", abstract
 *          (power-of-two block scaling).
 *  [MR]    "Microscaling FP4 Quantization: MR-GPTQ Achieves 6x Speedup",
 *          section "FP4 Quantization with Micro-Rotated GPTQ Algorithm"
 *          (block-wise Hadamard transforms).
 *
 * Where the pages are silent, the readings used here are:
 *  - scale exponent e = floor(log2(absmax)) - 2, clamped to [-127, 127],
 *    stored as the byte e + 127; an all-zero group stores byte 0;
 *  - a group holding Inf or NaN stores byte 0xFF and codes 0;
 *  - the sign bit of a code is the sign bit of the input, also when the
 *    magnitude rounds to 0;
 *  - the even element of a byte sits in the low nibble;
 *  - stochastic rounding goes up iff (r + 0.5) * 2^-16 < frac, r the 16-bit
 *    random number of the element, from the counter hash below;
 *  - the Hadamard transform is 1-D along each 1x32 row group;
 *  - the "bin centre" of a weight is its dequantized value;
 *  - the overflow-aware scale ([OAS]) is the smallest e with
 *    absmax * 2^-e <= 6. The page names the idea without a formula: the
 *    rule is pinned by its own properties (exhaustive minimality and
 *    non-saturation, unbiased stochastic rounding), but its agreement with
 *    the paper's OAS is parity unpinned.
 *
 * Parity pins: every function here is checked by tests against something
 * other than itself (a library E2M1 cast, exact comparisons with powers of
 * two, exhaustive enumeration of the random numbers, a library Hadamard
 * matrix, published hash test vectors, the worked oscillation example).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* E2M1 magnitudes: 2 exponent bits with bias 1 and 1 mantissa bit; the top
 * value is 6 ([ALTO] Jargon: E2M1, "roughly between -6 and 6"). */
static const double GRID[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

enum { DT_F32 = 0, DT_BF16 = 1 };
enum { AX_ROWS = 0, AX_COLS = 1 };
enum { RND_RNE = 0, RND_SR = 1 };

/* ------------------------------------------------------------------ */
/* Counter-based random numbers (the pages give none; this is our own   */
/* specification). mix() is the MurmurHash3 32-bit finalizer, from its  */
/* published definition.                                                */
/* ------------------------------------------------------------------ */

uint32_t orc_mix32(uint32_t h) {
  h ^= h >> 16;
  h *= 0x85EBCA6Bu;
  h ^= h >> 13;
  h *= 0xC2B2AE35u;
  h ^= h >> 16;
  return h;
}

uint32_t orc_key(uint64_t seed, uint32_t stream) {
  uint32_t lo = (uint32_t)(seed & 0xFFFFFFFFu);
  uint32_t hi = (uint32_t)(seed >> 32);
  return orc_mix32(lo ^ orc_mix32(hi + stream * 0x9E3779B9u));
}

/* 32-bit hash of counter n under key k. */
uint32_t orc_counter_hash(uint32_t k, uint64_t n) {
  uint32_t hi = (uint32_t)(n >> 32);
  uint32_t lo = (uint32_t)(n & 0xFFFFFFFFu);
  return orc_mix32(orc_mix32(k ^ hi) + lo);
}

/* 16-bit random number of the element with row-major input index i. */
uint32_t orc_rand16(uint64_t seed, uint32_t stream, uint64_t i) {
  uint32_t h = orc_counter_hash(orc_key(seed, stream), i >> 1);
  return (i & 1) ? (h >> 16) : (h & 0xFFFFu);
}

/* ------------------------------------------------------------------ */
/* Element access                                                       */
/* ------------------------------------------------------------------ */

static double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* Exact for values with at most 8 significant bits in the bf16 range
 * (every dequantized MXFP4 value); the low half of the fp32 is zero. */
static uint16_t double_to_bf16_exact(double v) {
  float f = (float)v;
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

static double load(const void* x, int dtype, int64_t idx) {
  if (dtype == DT_BF16) return bf16_to_double(((const uint16_t*)x)[idx]);
  return (double)((const float*)x)[idx];
}

/* ------------------------------------------------------------------ */
/* Scale ([ALTO] block scale set by the largest magnitude; [OAS]        */
/* power-of-two scale)                                                  */
/* ------------------------------------------------------------------ */

/* e = floor(log2(absmax)) - 2 clamped to [-127, 127]; absmax > 0 finite.
 * frexp gives absmax = f * 2^E with f in [0.5, 1), so floor(log2) = E - 1. */
int orc_scale_exponent(double absmax) {
  int E;
  if (absmax == 0.0) return -127;
  (void)frexp(absmax, &E);
  int e = (E - 1) - 2;
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

/* Overflow-aware scale ([OAS] abstract: overflow-aware scaling under
 * power-of-two block scales; the page gives no formula, so this is a
 * reading, parity unpinned by the pages): the smallest e in [-127, 127] with
 * absmax * 2^-e <= 6, so no element of the group saturates. Found by exact
 * comparisons, starting below the OCP exponent. */
int orc_scale_exponent_oas(double absmax) {
  int e = orc_scale_exponent(absmax) - 1;
  if (e < -127) e = -127;
  while (e < 127 && ldexp(absmax, -e) > 6.0) ++e;
  return e;
}

enum { SCALE_OCP = 0, SCALE_OAS = 1 };

/* E8M0 byte of a group: 0xFF if any element is not finite, else e + 127
 * with e from the OCP rule or the overflow-aware one. */
static int group_scale_byte(const double* g, int scale_rule) {
  double absmax = 0.0;
  for (int j = 0; j < 32; ++j) {
    if (!isfinite(g[j])) return 0xFF;
    if (fabs(g[j]) > absmax) absmax = fabs(g[j]);
  }
  return (scale_rule == SCALE_OAS ? orc_scale_exponent_oas(absmax)
                                  : orc_scale_exponent(absmax)) + 127;
}

/* ------------------------------------------------------------------ */
/* Element encoding ([ALTO] Jargon: Bin — rounding to the nearest bin;  */
/* Stochastic rounding — odds set by the distance to each neighbour)    */
/* ------------------------------------------------------------------ */

/* Q_D: the grid index nearest to a = |v|; a tie goes to the even index.
 * Values past 6 take index 7 (saturation). */
int orc_rne_index(double a) {
  int best = 0;
  for (int m = 1; m < 8; ++m) {
    double dm = fabs(a - GRID[m]);
    double db = fabs(a - GRID[best]);
    if (dm < db || (dm == db && (m % 2) == 0)) best = m;
  }
  return best;
}

/* Q_S: lo = largest grid value <= a, hi = next; up iff
 * (r + 0.5) * 2^-16 < (a - lo) / (hi - lo). a >= 6 saturates to 6. */
int orc_sr_index(double a, uint32_t r16) {
  if (a >= 6.0) return 7;
  int lo = 0;
  for (int m = 0; m < 8; ++m)
    if (GRID[m] <= a) lo = m;
  double frac = (a - GRID[lo]) / (GRID[lo + 1] - GRID[lo]);
  double t = ((double)r16 + 0.5) / 65536.0;
  return (t < frac) ? lo + 1 : lo;
}

/* Code of element x under exponent e: sign of x in bit 3, index in 0..2. */
int orc_encode(double x, int e, int rounding, uint32_t r16) {
  double a = fabs(ldexp(x, -e));
  int m = (rounding == RND_SR) ? orc_sr_index(a, r16) : orc_rne_index(a);
  return (signbit(x) ? 8 : 0) | m;
}

/* Value of a code under scale byte sb ([ALTO] Jargon: MXFP4). */
double orc_decode(int code, int sb) {
  if (sb == 0xFF) return NAN;
  double v = ldexp(GRID[code & 7], sb - 127);
  return (code & 8) ? -v : v;
}

/* ------------------------------------------------------------------ */
/* Group walk: quantize one group g[0..31] (values), writing 32 codes.  */
/* ------------------------------------------------------------------ */

static int quantize_group(const double* g, int rounding, uint64_t seed,
                          const uint64_t* idx, int scale_rule, int* codes_out) {
  int sb = group_scale_byte(g, scale_rule);
  for (int j = 0; j < 32; ++j) {
    if (sb == 0xFF) {
      codes_out[j] = 0;
      continue;
    }
    uint32_t r = (rounding == RND_SR) ? orc_rand16(seed, 0, idx[j]) : 0;
    codes_out[j] = orc_encode(g[j], sb - 127, rounding, r);
  }
  return sb;
}

static void put_nibble(uint8_t* codes, int64_t byte, int high, int code) {
  if (high)
    codes[byte] = (uint8_t)((codes[byte] & 0x0F) | (code << 4));
  else
    codes[byte] = (uint8_t)((codes[byte] & 0xF0) | code);
}

/* Quantize values xv[rows*cols] (row-major doubles). The tensor is rows
 * row0 .. row0+rows-1 of a larger one with the same cols: random numbers
 * are keyed by the element's index in that larger tensor. */
static void quantize_values(const double* xv, int64_t rows, int64_t cols,
                            int64_t row0, int axis, int rounding,
                            uint64_t seed, int scale_rule, uint8_t* codes,
                            uint8_t* scales) {
  double g[32];
  uint64_t idx[32];
  int cq[32];
  if (axis == AX_ROWS) {
    for (int64_t r = 0; r < rows; ++r)
      for (int64_t k = 0; k < cols / 32; ++k) {
        for (int j = 0; j < 32; ++j) {
          int64_t c = 32 * k + j;
          idx[j] = (uint64_t)((row0 + r) * cols + c);
          g[j] = xv[r * cols + c];
        }
        scales[r * (cols / 32) + k] =
            (uint8_t)quantize_group(g, rounding, seed, idx, scale_rule, cq);
        for (int j = 0; j < 32; ++j) {
          int64_t c = 32 * k + j;
          put_nibble(codes, r * (cols / 2) + c / 2, (int)(c & 1), cq[j]);
        }
      }
  } else {
    for (int64_t c = 0; c < cols; ++c)
      for (int64_t k = 0; k < rows / 32; ++k) {
        for (int j = 0; j < 32; ++j) {
          int64_t r = 32 * k + j;
          idx[j] = (uint64_t)((row0 + r) * cols + c);
          g[j] = xv[r * cols + c];
        }
        scales[c * (rows / 32) + k] =
            (uint8_t)quantize_group(g, rounding, seed, idx, scale_rule, cq);
        for (int j = 0; j < 32; ++j) {
          int64_t r = 32 * k + j;
          put_nibble(codes, c * (rows / 2) + r / 2, (int)(r & 1), cq[j]);
        }
      }
  }
}

static double* load_all(const void* x, int dtype, int64_t n) {
  double* xv = (double*)malloc((size_t)n * sizeof(double));
  for (int64_t i = 0; i < n; ++i) xv[i] = load(x, dtype, i);
  return xv;
}

/* ------------------------------------------------------------------ */
/* Public oracle entry points                                           */
/* ------------------------------------------------------------------ */

/* Block quantize x[rows][cols] along axis (rows row0.. of a larger tensor,
 * see quantize_values). Returns 0, or -1 on bad shape. */
int orc_quantize(const void* x, int dtype, int64_t rows, int64_t cols,
                 int64_t row0, int axis, int rounding, uint64_t seed,
                 uint8_t* codes, uint8_t* scales) {
  if (rows <= 0 || cols <= 0) return -1;
  if ((axis == AX_ROWS ? cols : rows) % 32 != 0) return -1;
  double* xv = load_all(x, dtype, rows * cols);
  quantize_values(xv, rows, cols, row0, axis, rounding, seed, SCALE_OCP, codes,
                  scales);
  free(xv);
  return 0;
}

/* orc_quantize with the overflow-aware scale (see orc_scale_exponent_oas):
 * every scaled value is at most 6, so nothing saturates and stochastic
 * rounding is unbiased for every input. */
int orc_quantize_oas(const void* x, int dtype, int64_t rows, int64_t cols,
                     int64_t row0, int axis, int rounding, uint64_t seed,
                     uint8_t* codes, uint8_t* scales) {
  if (rows <= 0 || cols <= 0) return -1;
  if ((axis == AX_ROWS ? cols : rows) % 32 != 0) return -1;
  double* xv = load_all(x, dtype, rows * cols);
  quantize_values(xv, rows, cols, row0, axis, rounding, seed, SCALE_OAS, codes,
                  scales);
  free(xv);
  return 0;
}

/* Decode the codes of a [rows][cols] tensor quantized along axis into a
 * double array in the output layout ([rows][cols] for ROWS, [cols][rows]
 * for COLS). */
static void dequantize_values(const uint8_t* codes, const uint8_t* scales,
                              int64_t rows, int64_t cols, int axis,
                              double* out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      int64_t byte, sidx, o;
      int high;
      if (axis == AX_ROWS) {
        byte = r * (cols / 2) + c / 2;
        high = (int)(c & 1);
        sidx = r * (cols / 32) + c / 32;
        o = r * cols + c;
      } else {
        byte = c * (rows / 2) + r / 2;
        high = (int)(r & 1);
        sidx = c * (rows / 32) + r / 32;
        o = c * rows + r;
      }
      int code = high ? (codes[byte] >> 4) : (codes[byte] & 0x0F);
      out[o] = orc_decode(code, scales[sidx]);
    }
}

int orc_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t rows,
                   int64_t cols, int axis, void* y, int out_dtype) {
  if (rows <= 0 || cols <= 0) return -1;
  int64_t n = rows * cols;
  double* v = (double*)malloc((size_t)n * sizeof(double));
  dequantize_values(codes, scales, rows, cols, axis, v);
  for (int64_t i = 0; i < n; ++i) {
    if (out_dtype == DT_BF16)
      ((uint16_t*)y)[i] = double_to_bf16_exact(v[i]);
    else
      ((float*)y)[i] = (float)v[i];
  }
  free(v);
  return 0;
}

/* [TJ] Question 2: Q_S along 32x1 groups of the dequantized Q_D(1x32)(X),
 * both passes with the scale rule given. */
static int double_quantize_rule(const void* x, int dtype, int64_t rows, int64_t cols,
                                int64_t row0, uint64_t seed, int scale_rule,
                                uint8_t* row_codes, uint8_t* row_scales,
                                uint8_t* col_codes, uint8_t* col_scales) {
  if (rows <= 0 || cols <= 0 || rows % 32 || cols % 32) return -1;
  int64_t n = rows * cols;
  double* xv = load_all(x, dtype, n);
  quantize_values(xv, rows, cols, row0, AX_ROWS, RND_RNE, 0, scale_rule, row_codes,
                  row_scales);
  double* d = (double*)malloc((size_t)n * sizeof(double));
  dequantize_values(row_codes, row_scales, rows, cols, AX_ROWS, d);
  quantize_values(d, rows, cols, row0, AX_COLS, RND_SR, seed, scale_rule, col_codes,
                  col_scales);
  free(d);
  free(xv);
  return 0;
}

int orc_double_quantize(const void* x, int dtype, int64_t rows, int64_t cols,
                        int64_t row0, uint64_t seed, uint8_t* row_codes,
                        uint8_t* row_scales, uint8_t* col_codes,
                        uint8_t* col_scales) {
  return double_quantize_rule(x, dtype, rows, cols, row0, seed, SCALE_OCP, row_codes,
                              row_scales, col_codes, col_scales);
}

/* orc_double_quantize with the overflow-aware scale in both passes. */
int orc_double_quantize_oas(const void* x, int dtype, int64_t rows, int64_t cols,
                            int64_t row0, uint64_t seed, uint8_t* row_codes,
                            uint8_t* row_scales, uint8_t* col_codes,
                            uint8_t* col_scales) {
  return double_quantize_rule(x, dtype, rows, cols, row0, seed, SCALE_OAS, row_codes,
                              row_scales, col_codes, col_scales);
}

/* Sign of column c for the randomized Hadamard transform: -1 iff bit 31 of
 * mix(K(seed, 1) + c) is set. */
int orc_rht_sign(uint64_t sign_seed, uint32_t c) {
  return (orc_mix32(orc_key(sign_seed, 1) + c) >> 31) ? -1 : 1;
}

/* Sylvester Hadamard entry H[j][k] = (-1)^popcount(j & k). */
static int hadamard_entry(int j, int k) {
  int p = 0;
  for (int b = j & k; b; b >>= 1) p += b & 1;
  return (p & 1) ? -1 : 1;
}

/* [ALTO] Jargon: Randomized Hadamard transform; [MR] block-wise Hadamard:
 * y_g = (1/sqrt(32)) H (s .* x_g) for every 1x32 row group, as a plain
 * matrix-vector product in fp64, rounded once to fp32. */
int orc_rht_rotate(const void* x, int dtype, int64_t rows, int64_t cols,
                   uint64_t sign_seed, float* y) {
  if (rows <= 0 || cols <= 0 || cols % 32) return -1;
  const double inv_sqrt32 = 1.0 / sqrt(32.0);
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < cols / 32; ++k) {
      double sx[32];
      for (int j = 0; j < 32; ++j) {
        int64_t c = 32 * k + j;
        sx[j] = orc_rht_sign(sign_seed, (uint32_t)c) * load(x, dtype, r * cols + c);
      }
      for (int j = 0; j < 32; ++j) {
        double acc = 0.0;
        for (int m = 0; m < 32; ++m) acc += hadamard_entry(j, m) * sx[m];
        y[r * cols + 32 * k + j] = (float)(acc * inv_sqrt32);
      }
    }
  return 0;
}

/* Rotate, then quantize the fp32 rotated values along rows (OCP or
 * overflow-aware scale). `rotated` receives y when not NULL. */
static int rht_quantize_rule(const void* x, int dtype, int64_t rows, int64_t cols,
                             int64_t row0, uint64_t sign_seed, int rounding,
                             uint64_t sr_seed, int scale_rule, uint8_t* codes,
                             uint8_t* scales, float* rotated) {
  if (rows <= 0 || cols <= 0 || cols % 32) return -1;
  float* y = rotated ? rotated : (float*)malloc((size_t)(rows * cols) * 4);
  orc_rht_rotate(x, dtype, rows, cols, sign_seed, y);
  if (scale_rule == SCALE_OAS)
    orc_quantize_oas(y, DT_F32, rows, cols, row0, AX_ROWS, rounding, sr_seed, codes,
                     scales);
  else
    orc_quantize(y, DT_F32, rows, cols, row0, AX_ROWS, rounding, sr_seed, codes, scales);
  if (!rotated) free(y);
  return 0;
}

int orc_rht_quantize(const void* x, int dtype, int64_t rows, int64_t cols,
                     int64_t row0, uint64_t sign_seed, int rounding,
                     uint64_t sr_seed, uint8_t* codes, uint8_t* scales,
                     float* rotated) {
  return rht_quantize_rule(x, dtype, rows, cols, row0, sign_seed, rounding, sr_seed,
                           SCALE_OCP, codes, scales, rotated);
}

/* orc_rht_quantize with the overflow-aware scale. */
int orc_rht_quantize_oas(const void* x, int dtype, int64_t rows, int64_t cols,
                         int64_t row0, uint64_t sign_seed, int rounding,
                         uint64_t sr_seed, uint8_t* codes, uint8_t* scales,
                         float* rotated) {
  return rht_quantize_rule(x, dtype, rows, cols, row0, sign_seed, rounding, sr_seed,
                           SCALE_OAS, codes, scales, rotated);
}

/* ------------------------------------------------------------------ */
/* Weight-oscillation tracker ([ALTO] the d_Q/d_w ratio paragraph)      */
/* ------------------------------------------------------------------ */

/* DQ of every element of one fp32 row-major tensor: 1x32 RNE
 * quantize-dequantize. */
static void dq_rows(const float* w, int64_t rows, int64_t cols, double* out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < cols / 32; ++k) {
      double g[32];
      for (int j = 0; j < 32; ++j) g[j] = (double)w[r * cols + 32 * k + j];
      int sb = group_scale_byte(g, SCALE_OCP);
      for (int j = 0; j < 32; ++j) {
        double v;
        if (sb == 0xFF)
          v = NAN;
        else
          v = orc_decode(orc_encode(g[j], sb - 127, RND_RNE, 0), sb);
        out[r * cols + 32 * k + j] = v;
      }
    }
}

/* One tracker step; returns the number of flagged elements (window end) or
 * 0, or -1 on bad shape. */
int64_t orc_osc_step(float* w, float* w_snap, float* d_w, float* d_q,
                     int64_t rows, int64_t cols, int window_end,
                     float threshold) {
  if (rows <= 0 || cols <= 0 || cols % 32) return -1;
  int64_t n = rows * cols;
  double* qw = (double*)malloc((size_t)n * sizeof(double));
  double* qs = (double*)malloc((size_t)n * sizeof(double));
  dq_rows(w, rows, cols, qw);
  dq_rows(w_snap, rows, cols, qs);
  int64_t flagged = 0;
  for (int64_t i = 0; i < n; ++i) {
    float dist_w = (float)fabs((double)w[i] - (double)w_snap[i]);
    d_w[i] = (float)((double)d_w[i] + (double)dist_w);
    float dist_q = (float)fabs(qw[i] - qs[i]);
    d_q[i] = (float)((double)d_q[i] + (double)dist_q);
    w_snap[i] = w[i];
    if (window_end) {
      float limit = (float)((double)threshold * (double)d_w[i]);
      if (d_q[i] > limit) {
        w[i] = (float)qw[i];
        ++flagged;
      }
      d_w[i] = 0.0f;
      d_q[i] = 0.0f;
      w_snap[i] = w[i];
    }
  }
  free(qs);
  free(qw);
  return flagged;
}

/* Q-Ramping ([TJ] rebuttal, Weakness 2 and the hyper-parameter answers):
 * oscillations are tracked only in the first iterations of an epoch (30 of
 * about 2500), with an oscillation detection factor k1 (16 is a good
 * choice) and a weight update frequency factor k2 (3 to 5; 5 by default).
 * The page gives the parameters, not the rule; the reading here:
 *  - iteration `iter` counts from 0 at each epoch's start; there the
 *    updates a flagged weight still holds are applied, its flag is cleared
 *    and the tracking window starts (w_snap = w, d_w = d_q = 0);
 *  - every iteration applies the caller's update delta: an unflagged
 *    weight takes it at once (w += delta); a flagged one gathers it
 *    (acc += delta) and takes the gathered sum every k2-th iteration
 *    (iter % k2 == k2 - 1), i.e. it updates k2 times less often;
 *  - during the window (iter < track_iters) the ALTO tracker runs on the
 *    updated weight: d_w += |w - w_snap|, d_q += |Q(w) - Q(w_snap)| (1x32
 *    nearest rounding, value units), w_snap = w; at its last iteration a
 *    weight is flagged iff d_q > k1 * d_w (the [ALTO] ratio test with k1
 *    as the threshold) and d_w, d_q are reset.
 * Every update is one fp32 operation (here fp64 rounded once). Returns the
 * number of weights flagged at this iteration (0 outside the window end),
 * -1 for bad arguments. Parity unpinned by the pages. */
int64_t orc_qramp_step(float* w, const float* delta, float* w_snap, float* d_w,
                       float* d_q, float* acc, uint8_t* flag, int64_t rows,
                       int64_t cols, int64_t iter, int64_t track_iters,
                       float k1, int64_t k2) {
  if (rows <= 0 || cols <= 0 || cols % 32 || iter < 0 || track_iters < 0 ||
      k2 < 1)
    return -1;
  int64_t n = rows * cols;
  if (iter == 0) {
    for (int64_t i = 0; i < n; ++i) {
      if (flag[i]) w[i] = (float)((double)w[i] + (double)acc[i]);
      acc[i] = 0.0f;
      flag[i] = 0;
      w_snap[i] = w[i];
      d_w[i] = d_q[i] = 0.0f;
    }
  }
  for (int64_t i = 0; i < n; ++i) {
    if (flag[i]) {
      acc[i] = (float)((double)acc[i] + (double)delta[i]);
      if (iter % k2 == k2 - 1) {
        w[i] = (float)((double)w[i] + (double)acc[i]);
        acc[i] = 0.0f;
      }
    } else {
      w[i] = (float)((double)w[i] + (double)delta[i]);
    }
  }
  if (iter >= track_iters) return 0;
  double* qw = (double*)malloc((size_t)n * sizeof(double));
  double* qs = (double*)malloc((size_t)n * sizeof(double));
  dq_rows(w, rows, cols, qw);
  dq_rows(w_snap, rows, cols, qs);
  int64_t flagged = 0;
  for (int64_t i = 0; i < n; ++i) {
    float moved_w = (float)fabs((double)w[i] - (double)w_snap[i]);
    d_w[i] = (float)((double)d_w[i] + (double)moved_w);
    float moved_q = (float)fabs(qw[i] - qs[i]);
    d_q[i] = (float)((double)d_q[i] + (double)moved_q);
    w_snap[i] = w[i];
    if (iter == track_iters - 1) {
      float limit = (float)((double)k1 * (double)d_w[i]);
      flag[i] = d_q[i] > limit ? 1 : 0;
      flagged += flag[i];
      d_w[i] = d_q[i] = 0.0f;
    }
  }
  free(qs);
  free(qw);
  return flagged;
}

/* Synthetic update driving the tracker: w += s * (rel_step * |w|), as an
 * fp32 multiply then an fp32 add; s from stream 2 keyed by
 * seed + (step << 32), one hash per element index (rows row0.. of a larger
 * tensor with the same cols). */
int orc_osc_synthetic_update(float* w, int64_t rows, int64_t cols,
                             int64_t row0, uint64_t seed, uint32_t step,
                             float rel_step) {
  if (rows <= 0 || cols <= 0) return -1;
  uint32_t k = orc_key(seed + ((uint64_t)step << 32), 2);
  for (int64_t i = 0; i < rows * cols; ++i) {
    uint64_t gi = (uint64_t)(row0 * cols + i);
    double s = (orc_counter_hash(k, gi) >> 31) ? -1.0 : 1.0;
    float mag = (float)((double)rel_step * fabs((double)w[i]));
    w[i] = (float)((double)w[i] + s * (double)mag);
  }
  return 0;
}

/* ------------------------------------------------------------------ */
/* Helpers for the pin tests                                            */
/* ------------------------------------------------------------------ */

/* How many of the 65536 random numbers send a up to the next grid value
 * (Q_S index above the largest grid index whose value is <= a). */
int orc_sr_count_up(double a) {
  int lo = 0;
  for (int m = 0; m < 8; ++m)
    if (GRID[m] <= a) lo = m;
  int n = 0;
  for (uint32_t r = 0; r < 65536u; ++r)
    if (orc_sr_index(a, r) > lo) ++n;
  return n;
}

/* 16-bit random numbers of elements first .. first+n-1. */
void orc_rand16_range(uint64_t seed, uint32_t stream, uint64_t first,
                      int64_t n, uint32_t* out) {
  for (int64_t k = 0; k < n; ++k)
    out[k] = orc_rand16(seed, stream, first + (uint64_t)k);
}

/* ------------------------------------------------------------------ */
/* Q-EMA ([TJ] rebuttal, Question 4 and the hyper-parameter answers:   */
/* the forward pass quantizes an exponential moving average of the     */
/* weight, updated whenever the parameters are; beta around 0.998)     */
/* ------------------------------------------------------------------ */

/* w_ema = beta * w_ema + (1 - beta) * w per element, each product and the
 * sum rounded to fp32 (no fused multiply-add; 1 - beta itself rounded to
 * fp32 first), then the 1x32 RNE quantization of the new w_ema. */
int orc_qema_quantize(const float* w, float* w_ema, int64_t rows, int64_t cols,
                      float beta, uint8_t* codes, uint8_t* scales) {
  if (rows <= 0 || cols <= 0 || cols % 32) return -1;
  const float omb = (float)(1.0 - (double)beta);
  for (int64_t i = 0; i < rows * cols; ++i) {
    float keep = (float)((double)beta * (double)w_ema[i]);
    float take = (float)((double)omb * (double)w[i]);
    w_ema[i] = (float)((double)keep + (double)take);
  }
  return orc_quantize(w_ema, DT_F32, rows, cols, 0, AX_ROWS, RND_RNE, 0,
                      codes, scales);
}

/* ------------------------------------------------------------------ */
/* Blocked scale layout for block-scaled GEMMs. [TJ] abstract: the MX   */
/* format is supported by the Blackwell architecture; its block-scaled  */
/* tensor-core GEMMs (and NVIDIA's library GEMMs over them) read the    */
/* scales of an operand [rows, K], one byte per 32-element group along  */
/* K, in NVIDIA's published one-dimensional block-scaling-factor layout */
/* (a reading: the pages name the hardware, not the layout).            */
/* ------------------------------------------------------------------ */

/* The scale matrix [rows][groups] is cut into tiles of 128 rows by 4
 * groups, padded with zero bytes; tiles are stored one after another,
 * across the groups first, then for the next 128 rows; each tile is 512
 * bytes, and inside it the scale of tile row r and tile group g is byte
 * 16 * (r mod 32) + 4 * (r div 32) + g. out holds
 * ceil(rows/128) * 128 * ceil(groups/4) * 4 bytes. */
int orc_scales_to_blocked(const uint8_t* s, int64_t rows, int64_t groups,
                          uint8_t* out) {
  if (rows <= 0 || groups <= 0) return -1;
  const int64_t row_tiles = (rows + 127) / 128, group_tiles = (groups + 3) / 4;
  memset(out, 0, (size_t)(row_tiles * group_tiles * 512));
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t g = 0; g < groups; ++g) {
      const int64_t tile = (r / 128) * group_tiles + g / 4;
      const int64_t tr = r % 128, tg = g % 4;
      out[tile * 512 + 16 * (tr % 32) + 4 * (tr / 32) + tg] = s[r * groups + g];
    }
  }
  return 0;
}
