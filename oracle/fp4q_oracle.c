/*
 * fp4q_oracle.c -- plain CPU definition of block-scaled FP4 quantization.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the oracle that the CUDA library is
 * checked against.  Only the tests, the smoke check and the benchmark's CPU
 * baseline may load it; the library itself never does, and the two share no
 * code, headers, tables or constants.
 *
 * Every result is written out step by step, in IEEE binary32, in the order
 * stated next to each function.  Build with -O2 -ffp-contract=off and without
 * -ffast-math on x86-64 (SSE arithmetic, no excess precision), so that each
 * C float operation below is one correctly rounded binary32 operation
 * ("RN(.)" in the comments).  Speed is not a goal: scale and element codes are
 * found by enumerating the format's values.
 *
 * Sources (the pages this follows):
 *   [Q]  Qiita note on the NVFP4 pre-training paper (nishiha): sections
 *        "NVFP4データの変換" (E2M1 definition), "2D scaling", "ランダム
 *        アダマール変換" (RHT), "確率的丸め" (stochastic rounding),
 *        "NVFP4の表現できる最大値" (2688), "scaleの導出" (scale derivation).
 *   [G]  Ultralytics glossary "FP4": "FP4の仕組み" (MXFP4 / NVFP4 and the
 *        block-size worked example).
 *   [I]  gist.science explainer of "Adaptive Block-Scaled Data Types":
 *        section 2 "提案手法：IF4" (IF4 selection, sign-bit flag, 6/7 method).
 *   [F]  blog.ast.moe "FP6から考えるLLM量子化": remark that round-to-nearest-
 *        even matters when converting the shared scale to E8M0.
 * Where the pages are silent the plainest reading is taken; each such place is
 * marked READING below.
 *
 * The outer loops over rows, columns or tile rows carry OpenMP pragmas.  Each
 * iteration writes whole bytes of its own, so a build with -fopenmp (the
 * all-core CPU baseline) gives the same bytes as the plain single-threaded
 * build the tests use, where the pragmas are inert.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_BF16 0
#define ORC_FP32 1
#define ORC_ROWWISE 1u
#define ORC_COLWISE 2u
#define ORC_RNE 0
#define ORC_SR 1
#define ORC_SCALE_LINEAR 0
#define ORC_SCALE_SWIZZLED 1
#define ORC_E8M0_RNE 0
#define ORC_E8M0_CEIL 1
#define ORC_E8M0_OCP_FLOOR 2
#define ORC_FMT_NVFP4 0
#define ORC_FMT_MXFP4 1
#define ORC_FMT_IF4 2
#define ORC_FMT_MXFP6_E2M3 3
#define ORC_FMT_MXFP6_E3M2 4
#define ORC_FMT_IF6 5
#define ORC_FMT_IF3 6
#define ORC_FP6_E2M3 0
#define ORC_FP6_E3M2 1

/* ------------------------------------------------------------------------ */
/* Scalar helpers                                                            */
/* ------------------------------------------------------------------------ */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* BF16 -> FP32 is exact: the 16 bits are the high half of the FP32 word. */
float orc_bf16_to_f32(uint16_t b) { return f32_from_bits((uint32_t)b << 16); }

/* FP32 -> BF16, round to nearest even (finite inputs; NaN kept quiet). */
uint16_t orc_f32_to_bf16(float f) {
  uint32_t u = bits_from_f32(f);
  if (isnan(f)) return (uint16_t)((u >> 16) | 0x40);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

static float load_elem(const void *x, int dtype, int64_t ld, int64_t r, int64_t c) {
  if (dtype == ORC_BF16) return orc_bf16_to_f32(((const uint16_t *)x)[r * ld + c]);
  return ((const float *)x)[r * ld + c];
}

/* ------------------------------------------------------------------------ */
/* E2M1 (FP4) element format  [Q] "NVFP4データの変換", [G] "FP4の仕組み"       */
/*   value = (-1)^s (0 + m/2) 2^e           for e = 0                        */
/*   value = (-1)^s (1 + m/2) 2^(e-1)       for e > 0                        */
/* giving magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 for codes 0..7; bit 3 = sign.*/
/* ------------------------------------------------------------------------ */

float orc_e2m1_value(uint8_t code) {
  int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  double mag = (e == 0) ? (0.0 + 0.5 * m) : (1.0 + 0.5 * m) * ldexp(1.0, e - 1);
  return (float)(s ? -mag : mag);
}

/* Code (0..7) of the E2M1 magnitude nearest to a >= 0, found by trying all
 * eight magnitudes.  An exact tie between two magnitudes goes to the even
 * code when ties_to_even is set, else to the smaller magnitude.  a must be
 * below 6 or saturation is the caller's business (a NaN gives code 0). */
static int e2m1_nearest_magnitude(double a, int ties_to_even) {
  int best = 0;
  double best_d = INFINITY;
  for (int c = 0; c < 8; ++c) {
    double d = fabs(a - (double)orc_e2m1_value((uint8_t)c));
    if (d < best_d || (ties_to_even && d == best_d && (c % 2) == 0)) { best = c; best_d = d; }
  }
  return best;
}

/* Nearest E2M1 value to v; a tie goes to the even code (round to nearest
 * even); magnitudes beyond 6 saturate to 6.  READING: the sign bit copies the
 * sign of v, so a negative value that rounds to zero gives code 0x8. */
uint8_t orc_e2m1_rne(float v) {
  double a = fabs((double)v);
  int best = (a >= 6.0) ? 7 /* 6 is the nearest value to anything above it */
                        : e2m1_nearest_magnitude(a, 1);
  return (uint8_t)(best | (signbit(v) ? 8 : 0));
}

/* Stochastic rounding onto the E2M1 grid  [Q] "確率的丸め".
 * The page rounds x + U(-1/2, 1/2) on a unit grid, i.e. it rounds up with
 * probability equal to the distance from the lower neighbour.  READING: the
 * same rule on the non-uniform E2M1 grid with 16 random bits: between adjacent
 * magnitudes lo <= |v| < hi, t = (|v| - lo)/(hi - lo) (exact: Sterbenz and a
 * power-of-two divisor) and the magnitude rounds up iff u < t * 2^16.
 * |v| >= 6 saturates to 6.  The sign is copied. */
uint8_t orc_e2m1_sr(float v, uint32_t u16) {
  float a = fabsf(v);
  int code;
  if (a >= 6.0f) {
    code = 7;
  } else {
    int lo = 0;
    for (int c = 0; c < 8; ++c)
      if (orc_e2m1_value((uint8_t)c) <= a) lo = c;
    float lo_v = orc_e2m1_value((uint8_t)lo);
    float hi_v = orc_e2m1_value((uint8_t)(lo + 1));
    float t = (a - lo_v) / (hi_v - lo_v);
    int up = (float)(u16 & 0xFFFFu) < t * 65536.0f;
    code = lo + up;
  }
  return (uint8_t)(code | (signbit(v) ? 8 : 0));
}

/* ------------------------------------------------------------------------ */
/* E4M3 (FP8, "fn": no infinities, 0x7F/0xFF = NaN) block-scale format       */
/* [Q] "NVFP4の表現できる最大値": the largest E4M3 value is 448.             */
/* ------------------------------------------------------------------------ */

float orc_e4m3_value(uint8_t code) {
  int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
  if (e == 15 && m == 7) return NAN;
  double mag = (e == 0) ? m * ldexp(1.0, -9) : (1.0 + m / 8.0) * ldexp(1.0, e - 7);
  return (float)(s ? -mag : mag);
}

/* Nearest non-negative E4M3 value to s >= 0, ties to the even code, values
 * at or above 448 saturate to 448 (code 0x7E). */
uint8_t orc_e4m3_rne_sat(float s) {
  if (s >= 448.0f) return 0x7E;
  int best = 0;
  double best_d = INFINITY;
  for (int c = 0; c <= 0x7E; ++c) {
    double d = fabs((double)s - (double)orc_e4m3_value((uint8_t)c));
    if (d < best_d || (d == best_d && (c % 2) == 0)) { best = c; best_d = d; }
  }
  return (uint8_t)best;
}

/* ------------------------------------------------------------------------ */
/* E8M0 shared scale (MXFP4)  [G] "FP4の仕組み", [F] E8M0 rounding remark     */
/* Returns the unbiased exponent e of the scale 2^e, e in [-127, 127];       */
/* the stored byte is e + 127.                                               */
/* ------------------------------------------------------------------------ */

/* split a positive float into f * 2^E with f in [1, 2) (exact) */
static void split_pow2(float a, double *f, int *E) {
  int e2;
  double fr = frexp((double)a, &e2); /* fr in [0.5, 1) */
  *f = fr * 2.0;
  *E = e2 - 1;
}

/* The exponent for an element format whose largest magnitude is qmax =
 * 1.x * 2^emax (E2M1: 6 = 1.5 * 2^2; FP6 E2M3: 7.5 = 1.875 * 2^2; E3M2:
 * 28 = 1.75 * 2^4). */
static int e8m0_exponent_q(float block_amax, int mode, float qmax, int emax) {
  int e;
  if (!(block_amax > 0.0f)) return -127;
  if (mode == ORC_E8M0_OCP_FLOOR) {
    /* floor(log2(amax)) - emax */
    double f; int E;
    split_pow2(block_amax, &f, &E);
    e = E - emax;
  } else {
    /* map the block maximum to qmax: the scale before rounding is RN(amax/qmax) */
    float target = block_amax / qmax;
    if (!(target > 0.0f)) return -127;
    double f; int E;
    split_pow2(target, &f, &E);
    if (mode == ORC_E8M0_CEIL) {
      e = (f > 1.0) ? E + 1 : E;             /* smallest 2^e >= target */
    } else {
      /* nearest power of two (linear distance: the midpoint of 2^E and
       * 2^(E+1) is 1.5 * 2^E); at the exact midpoint take the even biased
       * exponent.  READING of "round-to-nearest-even" for E8M0. */
      if (f > 1.5) e = E + 1;
      else if (f < 1.5) e = E;
      else e = (((E + 127) & 1) == 0) ? E : E + 1;
    }
  }
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

int orc_e8m0_exponent(float block_amax, int mode) {
  return e8m0_exponent_q(block_amax, mode, 6.0f, 2);
}

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As   */
/* Easy as 1, 2, 3", SC'11): 10 rounds of the 4x32 S-box with multipliers    */
/* 0xD2511F53 / 0xCD9E8D57 and Weyl key increments 0x9E3779B9 / 0xBB67AE85.  */
/* ------------------------------------------------------------------------ */

void orc_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
  uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
  uint32_t k0 = key_in[0], k1 = key_in[1];
  for (int round = 0; round < 10; ++round) {
    if (round > 0) { k0 += 0x9E3779B9u; k1 += 0xBB67AE85u; }
    uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)c0;
    uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)c2;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c1 ^ k0, n1 = lo1, n2 = hi0 ^ c3 ^ k1, n3 = lo0;
    c0 = n0; c1 = n1; c2 = n2; c3 = n3;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* READING (the pages give no bit mapping): the 16 random bits of the element
 * with flat row-major index i of the input tensor come from the Philox call
 * with counter (g mod 2^32, g div 2^32, 0, 0), g = i div 8, keyed by
 * (seed mod 2^32, seed div 2^32); element i takes bits 16*(i mod 2) .. +15 of
 * output word (i mod 8) div 2. */
uint32_t orc_sr_bits16(uint64_t seed, uint64_t i) {
  uint64_t g = i / 8;
  uint32_t ctr[4] = {(uint32_t)g, (uint32_t)(g >> 32), 0u, 0u};
  uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  uint32_t w[4];
  orc_philox4x32_10(ctr, key, w);
  return (w[(i % 8) / 2] >> (16 * (i % 2))) & 0xFFFFu;
}

/* READING: the random diagonal S of the Hadamard transform is one sign vector
 * of length n per call, drawn from the Philox call with counter (0, 0, 1, 0):
 * S_k = -1 when bit k of the 128-bit output (word k div 32, bit k mod 32) is
 * set, else +1.  [Q] "ランダムアダマール変換": S_d has {1, -1} on its diagonal. */
void orc_rht_signs(uint64_t seed, int n, float *signs) {
  uint32_t ctr[4] = {0u, 0u, 1u, 0u};
  uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  uint32_t w[4];
  orc_philox4x32_10(ctr, key, w);
  for (int k = 0; k < n; ++k) signs[k] = ((w[k / 32] >> (k % 32)) & 1u) ? -1.0f : 1.0f;
}

/* ------------------------------------------------------------------------ */
/* Scale-factor layouts                                                      */
/* ------------------------------------------------------------------------ */

/* Size in bytes of a [rows, cols] scale matrix in the given layout.  The
 * swizzled layout is the 128 x 4 block-scale tile layout that NVIDIA
 * documents for block-scaled tensor-core operands: rows padded to 128, scale
 * columns padded to 4, each 128 x 4 tile stored as 512 contiguous bytes. */
int64_t orc_scale_bytes(int64_t rows, int64_t cols, int layout) {
  if (layout == ORC_SCALE_LINEAR) return rows * cols;
  int64_t rp = (rows + 127) / 128 * 128, cp = (cols + 3) / 4 * 4;
  return rp * cp;
}

int64_t orc_scale_offset(int64_t r, int64_t c, int64_t rows, int64_t cols, int layout) {
  (void)rows;
  if (layout == ORC_SCALE_LINEAR) return r * cols + c;
  int64_t col_tiles = (cols + 3) / 4;
  int64_t tile = (r / 128) * col_tiles + (c / 4);
  return tile * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + (c % 4);
}

/* ------------------------------------------------------------------------ */
/* Tensor amax and the two-level NVFP4 tensor scale                          */
/* [Q] "scaleの導出": global_scale = 6*448 / max|x|                          */
/* ------------------------------------------------------------------------ */

float orc_amax(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld) {
  float m = 0.0f;
  int any_nan = 0;
#pragma omp parallel for reduction(max : m) reduction(| : any_nan)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      float a = fabsf(load_elem(x, dtype, ld, r, c));
      if (isnan(a)) any_nan = 1;
      else if (a > m) m = a;
    }
  return any_nan ? NAN : m;
}

/* global (encode) scale s_enc = RN(2688 / amax), clamped to FLT_MAX, and
 * the stored (decode) scale s_dec = RN(amax / 2688).  amax == 0 gives 1, 1.
 * 2688 = 6 * 448 is the largest NVFP4 magnitude ([Q] "NVFP4の表現できる最大値"). */
/* The same with the largest scaled magnitude as a parameter: top = qmax *
 * 448 for a block grid whose maximum is qmax (6 for NVFP4, 4 for 4/6). */
static void tensor_scales_top(float amax, float top, float *s_enc, float *s_dec) {
  if (amax == 0.0f) { *s_enc = 1.0f; *s_dec = 1.0f; return; }
  float e = top / amax;
  if (e > FLT_MAX) e = FLT_MAX;
  *s_enc = e;
  *s_dec = amax / top;
}

void orc_tensor_scales(float amax, float *s_enc, float *s_dec) {
  tensor_scales_top(amax, 2688.0f, s_enc, s_dec);
}

/* One block scale  [Q] "scaleの導出": x2 = x * global_scale, the block's
 * local scale is max|x2| / qmax cast to E4M3 (qmax = 6 for NVFP4).  Because
 * RN is monotone, max|RN(x * s)| = RN(max|x| * s), so the block maximum is
 * taken on x. */
static uint8_t block_scale_q(float block_amax, float s_enc, float qmax) {
  float x2_max = block_amax * s_enc;
  float local = x2_max / qmax;
  return orc_e4m3_rne_sat(local);
}

static uint8_t nvfp4_block_scale(float block_amax, float s_enc) {
  return block_scale_q(block_amax, s_enc, 6.0f);
}

/* READING: the element step divides by the block scale once per block:
 * r = RN(s_enc / S) (0 when S == 0), then v = RN(x * r).  READING (the
 * pages do not consider overflow): like s_enc, r is clamped to FLT_MAX; it
 * can only overflow when the whole tensor is tiny (amax < ~4e-33), and the
 * clamp keeps v finite (x = 0 would otherwise give 0 * inf = NaN). */
static float nvfp4_block_factor(uint8_t sf, float s_enc) {
  float S = orc_e4m3_value((uint8_t)(sf & 0x7F));
  if (S == 0.0f) return 0.0f;
  float r = s_enc / S;
  return (r > FLT_MAX) ? FLT_MAX : r;
}

/* ------------------------------------------------------------------------ */
/* NVFP4 1x16 quantization, row-wise and/or column-wise                      */
/* [Q] "Blockwise" (16 values per 8-bit scale), "2D scaling" (activations    */
/* and gradients use 1x16), "誤差逆伝播と転置" (the backward pass needs the   */
/* transposed operand, hence the column-wise copy).                          */
/* Row-wise: blocks are 16 consecutive columns of a row; codes [rows, cols/2]*/
/*   (element 2j in the low nibble), scales [rows, cols/16].                 */
/* Column-wise: blocks are 16 consecutive rows of a column, written as the   */
/*   transposed matrix: codes [cols, rows/2], scales [cols, rows/16].        */
/* SR bits use the element's flat row-major index r*cols + c in the input.   */
/* ------------------------------------------------------------------------ */

static uint8_t encode_elem(float v, int round, uint64_t seed, uint64_t index) {
  return (round == ORC_SR) ? orc_e2m1_sr(v, orc_sr_bits16(seed, index)) : orc_e2m1_rne(v);
}

static void put_nibble(uint8_t *q, int64_t byte_index, int high, uint8_t code) {
  if (high) q[byte_index] = (uint8_t)((q[byte_index] & 0x0F) | ((code & 0xF) << 4));
  else q[byte_index] = (uint8_t)((q[byte_index] & 0xF0) | (code & 0xF));
}

/* 1x16 quantization with block grid maximum qmax (6: NVFP4, 4: 4/6).  x is */
/* rows row0 .. row0 + rows - 1 of a tensor with cols columns (row0 = 0: the */
/* whole tensor); only the SR bits see row0, through the flat index.        */
static int quantize_1x16(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                         unsigned layouts, int round, uint64_t seed, const float *amax_in,
                         float *s_dec_out, uint8_t *q_row, uint8_t *sf_row, uint8_t *q_col,
                         uint8_t *sf_col, int scale_layout, float qmax, int64_t row0) {
  if ((layouts & ORC_ROWWISE) && cols % 16 != 0) return 1;
  if ((layouts & ORC_COLWISE) && rows % 16 != 0) return 1;
  float amax = amax_in ? *amax_in : orc_amax(x, dtype, rows, cols, ld);
  float s_enc, s_dec;
  tensor_scales_top(amax, qmax * 448.0f, &s_enc, &s_dec);
  if (s_dec_out) *s_dec_out = s_dec;

  if (layouts & ORC_ROWWISE) {
#pragma omp parallel for
    for (int64_t r = 0; r < rows; ++r)
      for (int64_t b = 0; b < cols / 16; ++b) {
        float m = 0.0f;
        for (int k = 0; k < 16; ++k) {
          float a = fabsf(load_elem(x, dtype, ld, r, b * 16 + k));
          if (a > m) m = a;
        }
        uint8_t sf = block_scale_q(m, s_enc, qmax);
        float rf = nvfp4_block_factor(sf, s_enc);
        sf_row[orc_scale_offset(r, b, rows, cols / 16, scale_layout)] = sf;
        for (int k = 0; k < 16; ++k) {
          int64_t c = b * 16 + k;
          float v = load_elem(x, dtype, ld, r, c) * rf;
          uint8_t code = encode_elem(v, round, seed, (uint64_t)((row0 + r) * cols + c));
          put_nibble(q_row, r * (cols / 2) + c / 2, (int)(c & 1), code);
        }
      }
  }
  if (layouts & ORC_COLWISE) {
#pragma omp parallel for
    for (int64_t c = 0; c < cols; ++c)
      for (int64_t b = 0; b < rows / 16; ++b) {
        float m = 0.0f;
        for (int k = 0; k < 16; ++k) {
          float a = fabsf(load_elem(x, dtype, ld, b * 16 + k, c));
          if (a > m) m = a;
        }
        uint8_t sf = block_scale_q(m, s_enc, qmax);
        float rf = nvfp4_block_factor(sf, s_enc);
        sf_col[orc_scale_offset(c, b, cols, rows / 16, scale_layout)] = sf;
        for (int k = 0; k < 16; ++k) {
          int64_t r = b * 16 + k;
          float v = load_elem(x, dtype, ld, r, c) * rf;
          uint8_t code = encode_elem(v, round, seed, (uint64_t)((row0 + r) * cols + c));
          put_nibble(q_col, c * (rows / 2) + r / 2, (int)(r & 1), code);
        }
      }
  }
  return 0;
}

int orc_quantize_nvfp4(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                       unsigned layouts, int round, uint64_t seed, const float *amax_in,
                       float *s_dec_out, uint8_t *q_row, uint8_t *sf_row, uint8_t *q_col,
                       uint8_t *sf_col, int scale_layout) {
  return quantize_1x16(x, dtype, rows, cols, ld, layouts, round, seed, amax_in, s_dec_out,
                       q_row, sf_row, q_col, sf_col, scale_layout, 6.0f, 0);
}

/* The same for rows row0 .. row0 + rows - 1 of a larger tensor with cols     */
/* columns, given its amax: the SR bits use the whole tensor's flat index     */
/* (row0 + r) * cols + c, everything else is local to the rows (row-wise     */
/* blocks; column blocks when rows and row0 are multiples of 16).            */
int orc_quantize_nvfp4_rows(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                            unsigned layouts, int round, uint64_t seed, const float *amax_in,
                            float *s_dec_out, uint8_t *q_row, uint8_t *sf_row, uint8_t *q_col,
                            uint8_t *sf_col, int scale_layout, int64_t row0) {
  if (row0 < 0) return 1;
  return quantize_1x16(x, dtype, rows, cols, ld, layouts, round, seed, amax_in, s_dec_out,
                       q_row, sf_row, q_col, sf_col, scale_layout, 6.0f, row0);
}

/* ------------------------------------------------------------------------ */
/* Four over six ("4/6"), the remedy [I] section 1 contrasts IF4 with: the   */
/* block maximum is mapped to 4 instead of 6, which makes the grid finer     */
/* relative to the block at the cost of the codes +-6.                       */
/* READING: everything else is NVFP4 1x16 with 4 in place of 6: tensor       */
/* scales s_enc = RN(1792 / amax), s_dec = RN(amax / 1792) (1792 = 4 * 448,  */
/* so the block scales use the E4M3 range as NVFP4's do), block scale        */
/* S = E4M3_rne_sat(RN(RN(m * s_enc) / 4)), r = RN(s_enc / S),               */
/* v = RN(x * r), E2M1 round to nearest even.  |v| <= 4 (1 + 2^-4) < 5, so    */
/* no code reaches 6.  Dequantization is NVFP4's, y = RN(RN(g * S) * s_dec). */
/* ------------------------------------------------------------------------ */

int orc_quantize_four_over_six(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                               unsigned layouts, const float *amax_in, float *s_dec_out,
                               uint8_t *q_row, uint8_t *sf_row, uint8_t *q_col, uint8_t *sf_col,
                               int scale_layout) {
  return quantize_1x16(x, dtype, rows, cols, ld, layouts, ORC_RNE, 0, amax_in, s_dec_out,
                       q_row, sf_row, q_col, sf_col, scale_layout, 4.0f, 0);
}

/* ------------------------------------------------------------------------ */
/* MXFP4: 32 values share one E8M0 power-of-two scale, no tensor scale.      */
/* [G] "FP4の仕組み" (MXFP4 bullet; scale chosen so the block max is near 6) */
/* Elements: v = RN(x * 2^-e) (exact except below the normal range), then    */
/* E2M1 round to nearest even with saturation.                               */
/* ------------------------------------------------------------------------ */

static float pow2f_exact(int e) { return (float)ldexp(1.0, e); } /* e in [-149, 127] */

int orc_quantize_mxfp4(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                       unsigned layouts, int e8m0_mode, uint8_t *q_row, uint8_t *sf_row,
                       uint8_t *q_col, uint8_t *sf_col, int scale_layout) {
  if ((layouts & ORC_ROWWISE) && cols % 32 != 0) return 1;
  if ((layouts & ORC_COLWISE) && rows % 32 != 0) return 1;
  if (layouts & ORC_ROWWISE) {
#pragma omp parallel for
    for (int64_t r = 0; r < rows; ++r)
      for (int64_t b = 0; b < cols / 32; ++b) {
        float m = 0.0f;
        for (int k = 0; k < 32; ++k) {
          float a = fabsf(load_elem(x, dtype, ld, r, b * 32 + k));
          if (a > m) m = a;
        }
        int e = orc_e8m0_exponent(m, e8m0_mode);
        sf_row[orc_scale_offset(r, b, rows, cols / 32, scale_layout)] = (uint8_t)(e + 127);
        float inv = pow2f_exact(-e);
        for (int k = 0; k < 32; ++k) {
          int64_t c = b * 32 + k;
          put_nibble(q_row, r * (cols / 2) + c / 2, (int)(c & 1),
                     orc_e2m1_rne(load_elem(x, dtype, ld, r, c) * inv));
        }
      }
  }
  if (layouts & ORC_COLWISE) {
#pragma omp parallel for
    for (int64_t c = 0; c < cols; ++c)
      for (int64_t b = 0; b < rows / 32; ++b) {
        float m = 0.0f;
        for (int k = 0; k < 32; ++k) {
          float a = fabsf(load_elem(x, dtype, ld, b * 32 + k, c));
          if (a > m) m = a;
        }
        int e = orc_e8m0_exponent(m, e8m0_mode);
        sf_col[orc_scale_offset(c, b, cols, rows / 32, scale_layout)] = (uint8_t)(e + 127);
        float inv = pow2f_exact(-e);
        for (int k = 0; k < 32; ++k) {
          int64_t r = b * 32 + k;
          put_nibble(q_col, c * (rows / 2) + r / 2, (int)(r & 1),
                     orc_e2m1_rne(load_elem(x, dtype, ld, r, c) * inv));
        }
      }
  }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* NVFP4 with 16x16 2D block scaling for weights  [Q] "2D scaling":          */
/* one scale per 16x16 square tile, so quantizing W and quantizing W^T give  */
/* the same numbers: q(W) = q(W^T)^T.                                         */
/* Outputs: q_w [rows, cols/2], q_wt [cols, rows/2] (the same nibbles,       */
/* transposed), tile scales [rows/16, cols/16] (always linear), and          */
/* optionally the tile scale replicated into 1x16-block form for W           */
/* ([rows, cols/16]) and for W^T ([cols, rows/16]) in scale_layout.          */
/* ------------------------------------------------------------------------ */

int orc_quantize_2d(const void *w, int dtype, int64_t rows, int64_t cols, int64_t ld,
                    const float *amax_in, float *s_dec_out, uint8_t *q_w, uint8_t *q_wt,
                    uint8_t *sf_tiles, uint8_t *sf_w_1x16, uint8_t *sf_wt_1x16,
                    int scale_layout) {
  if (rows % 16 != 0 || cols % 16 != 0) return 1;
  float amax = amax_in ? *amax_in : orc_amax(w, dtype, rows, cols, ld);
  float s_enc, s_dec;
  orc_tensor_scales(amax, &s_enc, &s_dec);
  if (s_dec_out) *s_dec_out = s_dec;
#pragma omp parallel for
  for (int64_t tr = 0; tr < rows / 16; ++tr)
    for (int64_t tc = 0; tc < cols / 16; ++tc) {
      float m = 0.0f;
      for (int i = 0; i < 16; ++i)
        for (int j = 0; j < 16; ++j) {
          float a = fabsf(load_elem(w, dtype, ld, tr * 16 + i, tc * 16 + j));
          if (a > m) m = a;
        }
      uint8_t sf = nvfp4_block_scale(m, s_enc);
      float rf = nvfp4_block_factor(sf, s_enc);
      sf_tiles[tr * (cols / 16) + tc] = sf;
      for (int i = 0; i < 16; ++i) {
        int64_t r = tr * 16 + i;
        if (sf_w_1x16) sf_w_1x16[orc_scale_offset(r, tc, rows, cols / 16, scale_layout)] = sf;
        for (int j = 0; j < 16; ++j) {
          int64_t c = tc * 16 + j;
          uint8_t code = orc_e2m1_rne(load_elem(w, dtype, ld, r, c) * rf);
          if (q_w) put_nibble(q_w, r * (cols / 2) + c / 2, (int)(c & 1), code);
          if (q_wt) put_nibble(q_wt, c * (rows / 2) + r / 2, (int)(r & 1), code);
        }
      }
      if (sf_wt_1x16)
        for (int j = 0; j < 16; ++j)
          sf_wt_1x16[orc_scale_offset(tc * 16 + j, tr, cols, rows / 16, scale_layout)] = sf;
    }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Random Hadamard transform  [Q] "ランダムアダマール変換":                   */
/*   Wgrad' = q(dY H) q(H^T x), H H^T = I, and the random version multiplies  */
/*   H by a diagonal S of random signs.                                      */
/* Per column j of dY [tokens, cols] and per group of n consecutive tokens:  */
/*   u_k = S_k * x_k;                                                        */
/*   FWHT in natural (Sylvester) order, stages h = 1, 2, 4, ..., n/2 in this */
/*   order; at each stage every pair (i, i+h) with (i & h) == 0 becomes      */
/*   (RN(u_i + u_{i+h}), RN(u_i - u_{i+h}));                                 */
/*   t_k = RN(u_k * c_n), c_n = RN(1/sqrt(n)) (0.25 for n = 16), so that the */
/*   transform is orthonormal (H H^T = I).                                   */
/* READING: the sign flip comes first (H times diag(S)); one S per call.     */
/* ------------------------------------------------------------------------ */

float orc_rht_norm(int n) { return (float)(1.0 / sqrt((double)n)); }

int orc_rht(const void *dy, int dtype, int64_t tokens, int64_t cols, int64_t ld, int n,
            uint64_t seed, float *t_out /* [tokens, cols] */) {
  if (n != 16 && n != 128) return 1;
  if (tokens % n != 0) return 1;
  float S[128];
  orc_rht_signs(seed, n, S);
  float cn = orc_rht_norm(n);
#pragma omp parallel for
  for (int64_t j = 0; j < cols; ++j)
    for (int64_t g = 0; g < tokens / n; ++g) {
      float u[128];
      for (int k = 0; k < n; ++k) u[k] = S[k] * load_elem(dy, dtype, ld, g * n + k, j);
      for (int h = 1; h < n; h *= 2)
        for (int i = 0; i < n; ++i)
          if ((i & h) == 0) {
            float a = u[i], b = u[i + h];
            u[i] = a + b;
            u[i + h] = a - b;
          }
      for (int k = 0; k < n; ++k) t_out[(g * n + k) * cols + j] = u[k] * cn;
    }
  return 0;
}

/* RHT followed by column-wise NVFP4 1x16 quantization of the transformed
 * tensor (blocks of 16 tokens; the tensor amax is taken over the transformed
 * values), written as dY^T codes [cols, tokens/2] and scales [cols, tokens/16].
 * SR bits use the flat input index token*cols + col.  [Q] "確率的丸め": SR
 * is what helps gradient quantization. */
static int quantize_rht_at(const void *dy, int dtype, int64_t tokens, int64_t cols, int64_t ld,
                           int n, int round, uint64_t seed, const float *amax_rht_in,
                           float *s_dec_out, uint8_t *q_t, uint8_t *sf_t, int scale_layout,
                           float *rht_out, int64_t token0) {
  if (n != 16 && n != 128) return 1;
  if (token0 < 0) return 1;
  if (tokens % n != 0 || tokens % 16 != 0) return 1;
  float *t = (float *)malloc(sizeof(float) * (size_t)(tokens * cols));
  if (!t) return 2;
  orc_rht(dy, dtype, tokens, cols, ld, n, seed, t);
  if (rht_out) memcpy(rht_out, t, sizeof(float) * (size_t)(tokens * cols));
  float amax = amax_rht_in ? *amax_rht_in : orc_amax(t, ORC_FP32, tokens, cols, cols);
  float s_enc, s_dec;
  orc_tensor_scales(amax, &s_enc, &s_dec);
  if (s_dec_out) *s_dec_out = s_dec;
#pragma omp parallel for
  for (int64_t c = 0; c < cols; ++c)
    for (int64_t b = 0; b < tokens / 16; ++b) {
      float m = 0.0f;
      for (int k = 0; k < 16; ++k) {
        float a = fabsf(t[(b * 16 + k) * cols + c]);
        if (a > m) m = a;
      }
      uint8_t sf = nvfp4_block_scale(m, s_enc);
      float rf = nvfp4_block_factor(sf, s_enc);
      sf_t[orc_scale_offset(c, b, cols, tokens / 16, scale_layout)] = sf;
      for (int k = 0; k < 16; ++k) {
        int64_t r = b * 16 + k;
        float v = t[r * cols + c] * rf;
        uint8_t code = encode_elem(v, round, seed, (uint64_t)((token0 + r) * cols + c));
        put_nibble(q_t, c * (tokens / 2) + r / 2, (int)(r & 1), code);
      }
    }
  free(t);
  return 0;
}

int orc_quantize_rht(const void *dy, int dtype, int64_t tokens, int64_t cols, int64_t ld,
                     int n, int round, uint64_t seed, const float *amax_rht_in,
                     float *s_dec_out, uint8_t *q_t, uint8_t *sf_t, int scale_layout,
                     float *rht_out) {
  return quantize_rht_at(dy, dtype, tokens, cols, ld, n, round, seed, amax_rht_in, s_dec_out,
                         q_t, sf_t, scale_layout, rht_out, 0);
}

/* The same for tokens token0 .. token0 + tokens - 1 of a larger gradient with */
/* cols columns, given the transform's amax: the SR bits use the whole        */
/* tensor's flat index (token0 + t) * cols + c; the transform and the blocks  */
/* are local when token0 is a multiple of n (the signs repeat per group).     */
int orc_quantize_rht_rows(const void *dy, int dtype, int64_t tokens, int64_t cols, int64_t ld,
                          int n, int round, uint64_t seed, const float *amax_rht_in,
                          float *s_dec_out, uint8_t *q_t, uint8_t *sf_t, int scale_layout,
                          float *rht_out, int64_t token0) {
  return quantize_rht_at(dy, dtype, tokens, cols, ld, n, round, seed, amax_rht_in, s_dec_out,
                         q_t, sf_t, scale_layout, rht_out, token0);
}

/* ------------------------------------------------------------------------ */
/* IF4: per 16-value block, quantize both as FP4 (E2M1) and as INT4 with the  */
/* 6/7 method, keep the one with the smaller squared error, and record the   */
/* choice in the (otherwise unused) sign bit of the E4M3 scale.              */
/* [I] section 2 "提案手法：IF4" (selection by MSE, sign-bit indicator, 6/7). */
/* Steps per block (scale S and factor r exactly as NVFP4):                   */
/*   v_i = RN(x_i * r)                                                        */
/*   FP4:  g_i = E2M1 value of e2m1_rne(v_i)                                  */
/*   INT4: k_i = clamp(rint(RN(v_i * C76)), -7, 7), h_i = RN(k_i * C67)       */
/*         with C76 = RN(7/6), C67 = RN(6/7)                                  */
/*   e_fp = sum_i (v_i - g_i)^2, e_int = sum_i (v_i - h_i)^2, each summed in  */
/*         order i = 0..15 as e = fma(d, d, e) with d = RN(v_i - q_i)         */
/*   INT4 iff e_int < e_fp (ties keep FP4).                                   */
/* READING: INT4 nibbles hold k_i in two's complement; scale bit 7 set means  */
/* INT4.  int4_mode 1 is IF4; 0 keeps FP4 everywhere (NVFP4 row-wise byte for */
/* byte); 2 keeps INT4 everywhere: NVINT4, the INT4 comparison format of [I] */
/* section 4, read as IF4's INT4 candidate (same scale S, 6/7 method) in     */
/* every block, flagged so that the IF4 dequantization decodes it.           */
/* ------------------------------------------------------------------------ */

float orc_if4_c76(void) { return 7.0f / 6.0f; }
float orc_if4_c67(void) { return 6.0f / 7.0f; }

int orc_quantize_if4(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                     const float *amax_in, float *s_dec_out, uint8_t *q, uint8_t *sf_out,
                     int scale_layout, int int4_mode) {
  if (cols % 16 != 0) return 1;
  float amax = amax_in ? *amax_in : orc_amax(x, dtype, rows, cols, ld);
  float s_enc, s_dec;
  orc_tensor_scales(amax, &s_enc, &s_dec);
  if (s_dec_out) *s_dec_out = s_dec;
  const float C76 = orc_if4_c76(), C67 = orc_if4_c67();
#pragma omp parallel for
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < cols / 16; ++b) {
      float xv[16], v[16];
      float m = 0.0f;
      for (int k = 0; k < 16; ++k) {
        xv[k] = load_elem(x, dtype, ld, r, b * 16 + k);
        if (fabsf(xv[k]) > m) m = fabsf(xv[k]);
      }
      uint8_t sf = nvfp4_block_scale(m, s_enc);
      float rf = nvfp4_block_factor(sf, s_enc);
      uint8_t fp_code[16], int_code[16];
      float e_fp = 0.0f, e_int = 0.0f;
      for (int k = 0; k < 16; ++k) {
        v[k] = xv[k] * rf;
        fp_code[k] = orc_e2m1_rne(v[k]);
        float g = orc_e2m1_value(fp_code[k]);
        float kk = rintf(v[k] * C76);
        if (kk > 7.0f) kk = 7.0f;
        if (kk < -7.0f) kk = -7.0f;
        int ki = (int)kk;
        int_code[k] = (uint8_t)(ki & 0xF);
        float h = (float)ki * C67;
        float d_fp = v[k] - g;
        float d_int = v[k] - h;
        e_fp = fmaf(d_fp, d_fp, e_fp);
        e_int = fmaf(d_int, d_int, e_int);
      }
      int use_int = int4_mode == 2 || (int4_mode == 1 && e_int < e_fp);
      sf_out[orc_scale_offset(r, b, rows, cols / 16, scale_layout)] =
          (uint8_t)(sf | (use_int ? 0x80 : 0x00));
      for (int k = 0; k < 16; ++k) {
        int64_t c = b * 16 + k;
        put_nibble(q, r * (cols / 2) + c / 2, (int)(c & 1), use_int ? int_code[k] : fp_code[k]);
      }
    }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* FP6 (OCP MX element formats)  [F] "FP6で隣り合う値の間隔を見てみる":       */
/* E2M3 = sign, 2 exponent bits (bias 1), 3 mantissa bits, largest 7.5;      */
/* E3M2 = sign, 3 exponent bits (bias 3), 2 mantissa bits, largest 28 (8, 10,*/
/* 12, 14, then 16, 20, 24, 28; spacing 0.0625 near 0); subnormals, no Inf or*/
/* NaN.  Codes are 6 bits, sign in bit 5.                                     */
/* ------------------------------------------------------------------------ */

float orc_fp6_value(uint8_t code, int fmt) {
  int m = code & 0x1F;
  int mb = (fmt == ORC_FP6_E2M3) ? 3 : 2;                /* mantissa bits */
  int bias = (fmt == ORC_FP6_E2M3) ? 1 : 3;
  int e = m >> mb, f = m & ((1 << mb) - 1);
  double v = (e == 0) ? ldexp((double)f, 1 - bias - mb)
                      : ldexp(1.0 + (double)f / (double)(1 << mb), e - bias);
  return (float)((code & 0x20) ? -v : v);
}

/* nearest FP6 magnitude (ties to the even code), saturating at the largest,
 * sign copied; v finite */
uint8_t orc_fp6_rne(float v, int fmt) {
  uint8_t sign = signbit(v) ? 0x20 : 0x00;
  double a = fabs((double)v);
  int best = 0;
  double best_d = INFINITY;
  for (int c = 0; c < 32; ++c) {
    double d = fabs(a - (double)orc_fp6_value((uint8_t)c, fmt));
    if (d < best_d || (d == best_d && (c % 2) == 0)) { best = c; best_d = d; }
  }
  if (a >= (double)orc_fp6_value(31, fmt)) best = 31;
  return (uint8_t)(best | sign);
}

/* MXFP6: 32 values share one E8M0 scale chosen as for MXFP4 with the FP6
 * format's largest magnitude (7.5 = 1.875 * 2^2 for E2M3, 28 = 1.75 * 2^4 for
 * E3M2); elements v = RN(x * 2^-e), FP6 round to nearest even with
 * saturation.  READING ([F] notes that values cross byte boundaries but fixes
 * no order): four 6-bit codes go into three bytes, code j of the group in bits
 * 6j..6j+5 of the little-endian 24-bit word.  Codes [rows, cols * 3/4] bytes,
 * scales [rows, cols/32].  Row-wise only. */
int orc_quantize_mxfp6(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld, int fmt,
                       int e8m0_mode, uint8_t *q, uint8_t *sf, int scale_layout) {
  if (cols % 32 != 0) return 1;
  float qmax = orc_fp6_value(31, fmt);
  int emax = (fmt == ORC_FP6_E2M3) ? 2 : 4;
  int64_t rb = cols * 3 / 4;                              /* code bytes per row */
#pragma omp parallel for
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < cols / 32; ++b) {
      float m = 0.0f;
      for (int k = 0; k < 32; ++k) {
        float a = fabsf(load_elem(x, dtype, ld, r, b * 32 + k));
        if (a > m) m = a;
      }
      int e = e8m0_exponent_q(m, e8m0_mode, qmax, emax);
      sf[orc_scale_offset(r, b, rows, cols / 32, scale_layout)] = (uint8_t)(e + 127);
      float inv = pow2f_exact(-e);
      for (int g = 0; g < 8; ++g) {
        uint32_t w = 0;
        for (int j = 0; j < 4; ++j) {
          int64_t c = b * 32 + g * 4 + j;
          w |= (uint32_t)orc_fp6_rne(load_elem(x, dtype, ld, r, c) * inv, fmt) << (6 * j);
        }
        uint8_t *dst = q + r * rb + (b * 8 + g) * 3;
        dst[0] = (uint8_t)(w & 0xFF);
        dst[1] = (uint8_t)((w >> 8) & 0xFF);
        dst[2] = (uint8_t)((w >> 16) & 0xFF);
      }
    }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* IF6: the IF idea at 6 bits.  [I] section 2 says the per-block FP/INT      */
/* choice applies to 6-bit (IF6) formats as well, without details.           */
/* READING (the plainest one the IF4 description supports):                 */
/*   the FP candidate is FP6 E2M3 (the finer FP6 grid, largest 7.5, [F]);    */
/*   the block scale maps the block maximum to 7.5 as NVFP4 maps it to 6:    */
/*     s_enc = RN(3360/amax), s_dec = RN(amax/3360) with 3360 = 7.5 * 448,  */
/*     S = E4M3_rne_sat(RN(RN(m * s_enc) / 7.5)), r = RN(s_enc / S),         */
/*     v_i = RN(x_i * r);                                                    */
/*   FP6:  g_i = E2M3 value of fp6_rne(v_i)                                  */
/*   INT6 (the 6/7 method with 31 and 7.5): k_i = clamp(rint(RN(v_i * CU)),  */
/*         -31, 31), h_i = RN(k_i * CD), CU = RN(31/7.5), CD = RN(7.5/31);   */
/*   errors, their order and the choice exactly as IF4 (INT6 iff strictly    */
/*   smaller); scale bit 7 set = INT6.                                       */
/* Codes are 6 bits (FP6 code with the sign in bit 5, or k_i in 6-bit two's */
/* complement), packed four per three bytes like MXFP6: codes [rows,         */
/* cols * 3/4], scales [rows, cols/16].  int6_mode 0 keeps FP6 everywhere,   */
/* 1 is IF6, 2 keeps INT6 everywhere.                                        */
/* ------------------------------------------------------------------------ */

float orc_if6_cu(void) { return 31.0f / 7.5f; }
float orc_if6_cd(void) { return 7.5f / 31.0f; }

int orc_quantize_if6(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                     const float *amax_in, float *s_dec_out, uint8_t *q, uint8_t *sf_out,
                     int scale_layout, int int6_mode) {
  if (cols % 16 != 0) return 1;
  float amax = amax_in ? *amax_in : orc_amax(x, dtype, rows, cols, ld);
  float s_enc, s_dec;
  tensor_scales_top(amax, 7.5f * 448.0f, &s_enc, &s_dec);
  if (s_dec_out) *s_dec_out = s_dec;
  const float CU = orc_if6_cu(), CD = orc_if6_cd();
  const int64_t rb = cols * 3 / 4;
#pragma omp parallel for
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < cols / 16; ++b) {
      float xv[16];
      float m = 0.0f;
      for (int k = 0; k < 16; ++k) {
        xv[k] = load_elem(x, dtype, ld, r, b * 16 + k);
        if (fabsf(xv[k]) > m) m = fabsf(xv[k]);
      }
      uint8_t sf = block_scale_q(m, s_enc, 7.5f);
      float rf = nvfp4_block_factor(sf, s_enc);
      uint8_t fp_code[16], int_code[16];
      float e_fp = 0.0f, e_int = 0.0f;
      for (int k = 0; k < 16; ++k) {
        float v = xv[k] * rf;
        fp_code[k] = orc_fp6_rne(v, ORC_FP6_E2M3);
        float g = orc_fp6_value(fp_code[k], ORC_FP6_E2M3);
        float kk = rintf(v * CU);
        if (kk > 31.0f) kk = 31.0f;
        if (kk < -31.0f) kk = -31.0f;
        int ki = (int)kk;
        int_code[k] = (uint8_t)(ki & 0x3F);
        float h = (float)ki * CD;
        float d_fp = v - g;
        float d_int = v - h;
        e_fp = fmaf(d_fp, d_fp, e_fp);
        e_int = fmaf(d_int, d_int, e_int);
      }
      int use_int = int6_mode == 2 || (int6_mode == 1 && e_int < e_fp);
      sf_out[orc_scale_offset(r, b, rows, cols / 16, scale_layout)] =
          (uint8_t)(sf | (use_int ? 0x80 : 0x00));
      for (int g4 = 0; g4 < 4; ++g4) {
        uint32_t w = 0;
        for (int j = 0; j < 4; ++j) {
          int k = g4 * 4 + j;
          w |= (uint32_t)(use_int ? int_code[k] : fp_code[k]) << (6 * j);
        }
        uint8_t *dst = q + r * rb + (b * 4 + g4) * 3;
        dst[0] = (uint8_t)(w & 0xFF);
        dst[1] = (uint8_t)((w >> 8) & 0xFF);
        dst[2] = (uint8_t)((w >> 16) & 0xFF);
      }
    }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* IF3: the IF idea at 3 bits.  [I] section 2 names IF3 beside IF6 and gives */
/* no details.  READING:                                                      */
/*   a 3-bit code is a sign and two magnitude bits.  Of the two float splits */
/*   of two bits, E1M1 has the uniform magnitudes 0, 0.5, 1, 1.5, which are  */
/*   INT3's 0..3 times 0.5: with it the FP/INT choice would have nothing to  */
/*   choose between.  So the FP candidate is FP3 E2M0 (two exponent bits,    */
/*   bias 1, no mantissa; exponent field 0 is zero, as in E2M1 with a zero   */
/*   mantissa): magnitudes 0, 1, 2, 4;                                       */
/*   the block scale maps the block maximum to 4 (as 4/6 does):             */
/*     s_enc = RN(1792/amax), s_dec = RN(amax/1792) with 1792 = 4 * 448,    */
/*     S = E4M3_rne_sat(RN(RN(m * s_enc) / 4)), r = RN(s_enc / S),           */
/*     v_i = RN(x_i * r);                                                    */
/*   FP3:  g_i = E2M0 value of the nearest magnitude (ties to the even code, */
/*         saturating at 4), sign copied;                                    */
/*   INT3 (the 6/7 method with 3 and 4): k_i = clamp(rint(RN(v_i * CU)),     */
/*         -3, 3), h_i = RN(k_i * CD), CU = RN(3/4), CD = RN(4/3);           */
/*   errors, their order and the choice exactly as IF4 (INT3 iff strictly    */
/*   smaller); scale bit 7 set = INT3.                                       */
/* Codes are 3 bits (FP3: sign in bit 2, magnitude code in bits 0-1; INT3:  */
/* k_i in 3-bit two's complement), packed eight per three bytes, code j of  */
/* the group in bits 3j..3j+2 of the little-endian 24-bit word: codes       */
/* [rows, cols * 3/8], scales [rows, cols/16].  int3_mode 0 keeps FP3       */
/* everywhere, 1 is IF3, 2 keeps INT3 everywhere.                           */
/* ------------------------------------------------------------------------ */

float orc_fp3_value(uint8_t code) {
  static const float mag[4] = {0.0f, 1.0f, 2.0f, 4.0f};
  float v = mag[code & 0x3];
  return (code & 0x4) ? -v : v;
}

/* nearest E2M0 magnitude (ties to the even code), saturating at 4, sign
 * copied; v finite */
uint8_t orc_fp3_rne(float v) {
  uint8_t sign = signbit(v) ? 0x4 : 0x0;
  double a = fabs((double)v);
  int best = 0;
  double best_d = INFINITY;
  for (int c = 0; c < 4; ++c) {
    double d = fabs(a - (double)orc_fp3_value((uint8_t)c));
    if (d < best_d || (d == best_d && (c % 2) == 0)) { best = c; best_d = d; }
  }
  if (a >= 4.0) best = 3;                  /* saturate: huge a ties every distance */
  return (uint8_t)(best | sign);
}

float orc_if3_cu(void) { return 3.0f / 4.0f; }
float orc_if3_cd(void) { return 4.0f / 3.0f; }

int orc_quantize_if3(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                     const float *amax_in, float *s_dec_out, uint8_t *q, uint8_t *sf_out,
                     int scale_layout, int int3_mode) {
  if (cols % 16 != 0) return 1;
  float amax = amax_in ? *amax_in : orc_amax(x, dtype, rows, cols, ld);
  float s_enc, s_dec;
  tensor_scales_top(amax, 4.0f * 448.0f, &s_enc, &s_dec);
  if (s_dec_out) *s_dec_out = s_dec;
  const float CU = orc_if3_cu(), CD = orc_if3_cd();
  const int64_t rb = cols * 3 / 8;
#pragma omp parallel for
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < cols / 16; ++b) {
      float xv[16];
      float m = 0.0f;
      for (int k = 0; k < 16; ++k) {
        xv[k] = load_elem(x, dtype, ld, r, b * 16 + k);
        if (fabsf(xv[k]) > m) m = fabsf(xv[k]);
      }
      uint8_t sf = block_scale_q(m, s_enc, 4.0f);
      float rf = nvfp4_block_factor(sf, s_enc);
      uint8_t fp_code[16], int_code[16];
      float e_fp = 0.0f, e_int = 0.0f;
      for (int k = 0; k < 16; ++k) {
        float v = xv[k] * rf;
        fp_code[k] = orc_fp3_rne(v);
        float g = orc_fp3_value(fp_code[k]);
        float kk = rintf(v * CU);
        if (kk > 3.0f) kk = 3.0f;
        if (kk < -3.0f) kk = -3.0f;
        int ki = (int)kk;
        int_code[k] = (uint8_t)(ki & 0x7);
        float h = (float)ki * CD;
        float d_fp = v - g;
        float d_int = v - h;
        e_fp = fmaf(d_fp, d_fp, e_fp);
        e_int = fmaf(d_int, d_int, e_int);
      }
      int use_int = int3_mode == 2 || (int3_mode == 1 && e_int < e_fp);
      sf_out[orc_scale_offset(r, b, rows, cols / 16, scale_layout)] =
          (uint8_t)(sf | (use_int ? 0x80 : 0x00));
      for (int g8 = 0; g8 < 2; ++g8) {
        uint32_t w = 0;
        for (int j = 0; j < 8; ++j) {
          int k = g8 * 8 + j;
          w |= (uint32_t)(use_int ? int_code[k] : fp_code[k]) << (3 * j);
        }
        uint8_t *dst = q + r * rb + (b * 2 + g8) * 3;
        dst[0] = (uint8_t)(w & 0xFF);
        dst[1] = (uint8_t)((w >> 8) & 0xFF);
        dst[2] = (uint8_t)((w >> 16) & 0xFF);
      }
    }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Dequantization  [G] "FP4の仕組み" (reconstruct = grid value * sign * scale)*/
/* NVFP4:  y = RN(RN(g * S) * s_dec)   (g * S is exact)                       */
/* IF4 INT4 blocks: h = RN(k * C67), y = RN(RN(h * S) * s_dec)                */
/* MXFP4:  y = RN(g * 2^e)                                                    */
/* MXFP6 (E2M3 / E3M2, codes packed 4 per 3 bytes): y = RN(value * 2^e)      */
/* IF6 / IF3: FP blocks as NVFP4 with the FP6 E2M3 / FP3 E2M0 value, INT      */
/* blocks as IF4 with CD6 = RN(7.5/31) / CD3 = RN(4/3); codes 4 / 8 per 3 B   */
/* Block shape: block_rows x block_cols (1x16, 1x32, or 16x16 for 2D tiles,  */
/* whose scales are [rows/16, cols/16] linear).  Output FP32 or BF16 (RNE of */
/* the FP32 result).                                                         */
/* ------------------------------------------------------------------------ */

int orc_dequantize(int format, const uint8_t *q, const uint8_t *sf, int scale_layout,
                   int block_rows, int block_cols, const float *s_dec_in, int64_t rows,
                   int64_t cols, void *y, int y_dtype) {
  if (cols % block_cols != 0 || rows % block_rows != 0) return 1;
  float s_dec = s_dec_in ? *s_dec_in : 1.0f;
  int64_t srows = rows / block_rows, scols = cols / block_cols;
  const float C67 = orc_if4_c67(), CD6 = orc_if6_cd(), CD3 = orc_if3_cd();
  const int fp6 = (format == ORC_FMT_MXFP6_E2M3 || format == ORC_FMT_MXFP6_E3M2);
  const int six = fp6 || format == ORC_FMT_IF6;             /* 6-bit codes, 4 per 3 bytes */
  const int three = format == ORC_FMT_IF3;                  /* 3-bit codes, 8 per 3 bytes */
#pragma omp parallel for
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      uint8_t code;
      if (three) {
        const uint8_t *g3 = q + r * (cols * 3 / 8) + (c / 8) * 3;
        uint32_t w = (uint32_t)g3[0] | ((uint32_t)g3[1] << 8) | ((uint32_t)g3[2] << 16);
        code = (uint8_t)((w >> (3 * (c % 8))) & 0x7);
      } else if (six) {
        const uint8_t *g3 = q + r * (cols * 3 / 4) + (c / 4) * 3;
        uint32_t w = (uint32_t)g3[0] | ((uint32_t)g3[1] << 8) | ((uint32_t)g3[2] << 16);
        code = (uint8_t)((w >> (6 * (c % 4))) & 0x3F);
      } else {
        uint8_t byte = q[r * (cols / 2) + c / 2];
        code = (c & 1) ? (byte >> 4) : (byte & 0xF);
      }
      int64_t sr = r / block_rows, sc = c / block_cols;
      int64_t off = (block_rows == 1) ? orc_scale_offset(sr, sc, srows, scols, scale_layout)
                                      : sr * scols + sc;
      uint8_t s = sf[off];
      float out;
      if (format == ORC_FMT_MXFP4) {
        out = orc_e2m1_value(code) * pow2f_exact((int)s - 127);
      } else if (fp6) {
        out = orc_fp6_value(code, format == ORC_FMT_MXFP6_E2M3 ? ORC_FP6_E2M3 : ORC_FP6_E3M2) *
              pow2f_exact((int)s - 127);
      } else {
        float S = orc_e4m3_value((uint8_t)(s & 0x7F));
        if (format == ORC_FMT_IF4 && (s & 0x80)) {
          int k = (code & 0x8) ? (int)code - 16 : (int)code;
          float h = (float)k * C67;
          out = (h * S) * s_dec;
        } else if (format == ORC_FMT_IF6 && (s & 0x80)) {
          int k = (code & 0x20) ? (int)code - 64 : (int)code;
          float h = (float)k * CD6;
          out = (h * S) * s_dec;
        } else if (format == ORC_FMT_IF6) {
          out = (orc_fp6_value(code, ORC_FP6_E2M3) * S) * s_dec;
        } else if (format == ORC_FMT_IF3 && (s & 0x80)) {
          int k = (code & 0x4) ? (int)code - 8 : (int)code;
          float h = (float)k * CD3;
          out = (h * S) * s_dec;
        } else if (format == ORC_FMT_IF3) {
          out = (orc_fp3_value(code) * S) * s_dec;
        } else {
          out = (orc_e2m1_value(code) * S) * s_dec;
        }
      }
      if (y_dtype == ORC_BF16) ((uint16_t *)y)[r * cols + c] = orc_f32_to_bf16(out);
      else ((float *)y)[r * cols + c] = out;
    }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Glossary mode  [G] "FP4の仕組み", the block-size worked example:           */
/* scale = amax_b / 6 in FP32 (no E4M3 rounding), v = |x| / scale per        */
/* element, nearest E2M1 magnitude with ties to the FIRST (smaller) one       */
/* (argmin), dequantized value = grid * sign(x) * scale; returns the mean     */
/* absolute error over the n values (accumulated in double).                  */
/* ------------------------------------------------------------------------ */

double orc_glossary_mae(const float *x, int64_t n, int64_t block) {
  /* [G] "FP4の仕組み": the worked example scales each block so that its
   * largest magnitude becomes 6 (an FP32 scale, not rounded to E4M3),
   * rounds every scaled magnitude to the nearest E2M1 value -- an exact tie
   * going to the smaller magnitude -- restores the sign, scales back and
   * reports the mean absolute error over the tensor. */
  double err = 0.0;
  for (int64_t b = 0; b < n / block; ++b) {
    const float *xb = x + b * block;
    float m = 0.0f;
    for (int64_t k = 0; k < block; ++k)
      if (fabsf(xb[k]) > m) m = fabsf(xb[k]);
    const float scale = m / 6.0f;
    for (int64_t k = 0; k < block; ++k) {
      int code = e2m1_nearest_magnitude((double)(fabsf(xb[k]) / scale), 0);
      if (xb[k] < 0.0f) code |= 8;
      const float back = orc_e2m1_value((uint8_t)code) * scale;
      err += fabs((double)back - (double)xb[k]);
    }
  }
  return err / (double)n;
}

/* ------------------------------------------------------------------------ */
/* Array forms of the scalar format functions (for tests over many values).  */
/* ------------------------------------------------------------------------ */

void orc_e2m1_rne_n(const float *v, uint8_t *out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_rne(v[i]);
}

void orc_e2m1_sr_n(const float *v, const uint32_t *u16, uint8_t *out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_sr(v[i], u16[i]);
}

void orc_e4m3_rne_sat_n(const float *s, uint8_t *out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_rne_sat(s[i]);
}

void orc_e8m0_exponent_n(const float *m, int mode, int32_t *out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e8m0_exponent(m[i], mode);
}

void orc_sr_bits16_n(uint64_t seed, uint64_t first_index, uint32_t *out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_sr_bits16(seed, first_index + (uint64_t)i);
}

void orc_f32_to_bf16_n(const float *v, uint16_t *out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_f32_to_bf16(v[i]);
}
