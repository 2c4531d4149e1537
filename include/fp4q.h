/*
 * fp4q.h -- C ABI of the block-scaled FP4 quantization library (libfp4q.so).
 *
 * What is computed.  Each entry point quantizes (or dequantizes) one tensor
 * into a block-scaled 4-bit format, bit for bit as the CPU oracle in this
 * repository defines it:
 *
 *   NVFP4  E2M1 codes (magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6 plus a sign bit),
 *          one E4M3 scale per 16 values and one FP32 scale per tensor.
 *          Qiita note on the NVFP4 pre-training paper (nishiha): "NVFP4データ
 *          の変換" (E2M1), "Blockwise" (16 values per 8-bit scale), "scaleの
 *          導出" (global_scale = 6*448/amax, local scale = block max / 6 as
 *          E4M3), "NVFP4の表現できる最大値" (2688 = 6 * 448).
 *   MXFP4  E2M1 codes, one E8M0 power-of-two scale per 32 values, no tensor
 *          scale.  Ultralytics glossary "FP4", section "FP4の仕組み".
 *   2D     NVFP4 with one scale per 16x16 tile, so q(W) = q(W^T)^T.
 *          Qiita note, section "2D scaling".
 *   RHT    random Hadamard transform H diag(S) along tokens ahead of the
 *          Wgrad operand, with stochastic rounding.  Qiita note, sections
 *          "ランダムアダマール変換" and "確率的丸め".
 *   IF4    per 16-value block, FP4 or INT4 (6/7 method), whichever has the
 *          smaller squared error, flagged in bit 7 of the E4M3 scale.
 *          "Adaptive Block-Scaled Data Types" explainer, section 2 (IF4).
 *
 * Arithmetic, per 16-value NVFP4 block (all binary32, RN = round to nearest
 * even, no fused operations):
 *   amax = max |x| over the tensor;  s_enc = RN(2688 / amax) (1 if amax = 0),
 *   s_dec = RN(amax / 2688) (1 if amax = 0);
 *   block scale S = E4M3_rne_sat(RN(RN(m * s_enc) / 6)), m = block max |x|;
 *   r = RN(s_enc / S) (0 if S = 0);  v = RN(x * r);  code = E2M1_rne_sat(v)
 *   (or stochastic rounding); dequant y = RN(RN(E2M1(code) * S) * s_dec).
 *
 * Conventions (all entry points):
 *   - Every pointer argument is a DEVICE pointer owned by the caller, unless
 *     stated otherwise.  The library allocates nothing and keeps no state
 *     between calls.  Inputs, outputs and workspace of one call must be on
 *     the same device; the call runs on that device, making it current while
 *     it enqueues work, and puts the caller's current device back before it
 *     returns.
 *   - Matrices are row-major.  `ld` is the input's leading dimension in
 *     elements (ld >= cols); ld * element size must be a multiple of 16 bytes
 *     and every pointer must be 16-byte aligned.
 *   - Packed codes: two 4-bit codes per byte, element 2j in the low nibble.
 *     Row-wise output of a [rows, cols] input: codes [rows, cols/2], scales
 *     [rows, cols/block].  Column-wise ("transposed") output: codes
 *     [cols, rows/2], scales [cols, rows/block] -- i.e. the row-wise layout
 *     of the transpose.
 *   - Scale layout FP4Q_SCALE_LINEAR stores scales row-major.
 *     FP4Q_SCALE_SWIZZLED_128x4 stores them in the 128 x 4 tile layout that
 *     block-scaled tensor-core GEMMs read: byte (r, c) of an [R, C] scale
 *     matrix lives at ((r/128)*(C/4) + c/4)*512 + (r%32)*16 + ((r/32)%4)*4
 *     + c%4.  It requires R % 128 == 0 and C % 4 == 0.
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and is asynchronous.  Argument errors are detected on
 *     the host and returned before anything is enqueued.  A failed launch
 *     returns FP4Q_ERR_CUDA.  No call traps on the device.
 *   - Inputs must be finite; a NaN or Inf input makes the tensor amax
 *     non-finite and the outputs unspecified.
 */
#ifndef FP4Q_H_
#define FP4Q_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FP4Q_OK = 0,
  FP4Q_ERR_INVALID_ARG = 1,        /* null pointer, bad enum, host pointer, ld < cols */
  FP4Q_ERR_UNSUPPORTED_SHAPE = 2,  /* shape not a multiple of the block / tile size */
  FP4Q_ERR_MISALIGNED = 3,         /* pointer or row stride not 16-byte aligned */
  FP4Q_ERR_WORKSPACE_TOO_SMALL = 4,
  FP4Q_ERR_CUDA = 5                /* a CUDA runtime call or launch failed */
} fp4q_status;

typedef enum { FP4Q_BF16 = 0, FP4Q_FP32 = 1 } fp4q_dtype;
typedef enum { FP4Q_RNE = 0, FP4Q_SR = 1 } fp4q_round;
typedef enum { FP4Q_SCALE_LINEAR = 0, FP4Q_SCALE_SWIZZLED_128x4 = 1 } fp4q_scale_layout;
typedef enum { FP4Q_E8M0_RNE = 0, FP4Q_E8M0_CEIL = 1, FP4Q_E8M0_OCP_FLOOR = 2 } fp4q_e8m0_mode;
typedef enum {
  FP4Q_FMT_NVFP4 = 0,
  FP4Q_FMT_MXFP4 = 1,
  FP4Q_FMT_IF4 = 2,
  FP4Q_FMT_MXFP6_E2M3 = 3,   /* codes packed four per three bytes */
  FP4Q_FMT_MXFP6_E3M2 = 4,
  FP4Q_FMT_IF6 = 5,          /* 6-bit codes, four per three bytes */
  FP4Q_FMT_IF3 = 6           /* 3-bit codes, eight per three bytes */
} fp4q_format;
typedef enum { FP4Q_FP6_E2M3 = 0, FP4Q_FP6_E3M2 = 1 } fp4q_fp6_format;

#define FP4Q_ROWWISE 1u
#define FP4Q_COLWISE 2u

/* Human-readable name of a status code (static string, never NULL). */
const char *fp4q_status_string(int status);

/* Library version string (static). */
const char *fp4q_version(void);

/* Bytes of device workspace the quantize calls need for a [rows, cols]
 * input when they compute the tensor amax themselves (amax argument NULL).
 * The amax takes 4 bytes at any size, so this is the same 256 bytes for
 * every valid shape; 0 for negative sizes. */
size_t fp4q_workspace_bytes(int64_t rows, int64_t cols);

/* Bytes of a scale matrix for a [rows, cols] tensor quantized in blocks of
 * `block` values along cols: [rows, cols/block] in the given layout (the
 * swizzled layout rounds rows up to 128 and cols/block up to 4).  For a
 * column-wise output pass (cols, rows, block, layout).  Returns 0 on bad
 * arguments. */
size_t fp4q_scale_bytes(int64_t rows, int64_t cols, int block, int scale_layout);

/* Tensor amax: *amax_out = max |x| over x[rows, cols] (FP32, exact).
 * Qiita note, "scaleの導出": max|x| sets the global scale.
 * amax_out: device float, overwritten.  Shape: cols % 16 == 0. */
fp4q_status fp4q_amax(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                      float *amax_out, void *stream);

/* NVFP4 1x16 quantization of an activation or gradient, row-wise and/or
 * column-wise from one read of x.  Qiita note: "Blockwise", "誤差逆伝播と
 * 転置" (backprop needs the transposed operand), "2D scaling" (activations
 * and gradients use 1x16), "確率的丸め" (round = FP4Q_SR).
 *   layouts      FP4Q_ROWWISE | FP4Q_COLWISE (at least one)
 *   round        FP4Q_RNE, or FP4Q_SR: stochastic rounding whose 16 random
 *                bits per element come from Philox4x32-10 keyed on `seed`,
 *                counter = (flat input index r*cols + c) / 8
 *   amax         device float with the tensor amax, or NULL: then it is
 *                computed first into `workspace`
 *   tensor_scale_out  device float <- s_dec (may be NULL)
 *   q_row, sf_row     row-wise codes [rows, cols/2], scales [rows, cols/16]
 *   q_col, sf_col     column-wise codes [cols, rows/2], scales [cols, rows/16]
 *                (pointers of a layout not requested may be NULL)
 *   workspace, ws_bytes  >= fp4q_workspace_bytes(rows, cols) when amax == NULL
 * Shape: cols % 16 == 0; COLWISE also needs rows % 16 == 0. */
fp4q_status fp4q_quantize_nvfp4(const void *x, int dtype, int64_t rows, int64_t cols,
                                int64_t ld, unsigned layouts, int round, uint64_t seed,
                                const float *amax, float *tensor_scale_out, uint8_t *q_row,
                                uint8_t *sf_row, uint8_t *q_col, uint8_t *sf_col,
                                int scale_layout, void *workspace, size_t ws_bytes,
                                void *stream);

/* MXFP4 1x32 quantization, row-wise and/or column-wise from one read.
 * Ultralytics glossary "FP4", "FP4の仕組み": 32 values share an 8-bit
 * power-of-two (E8M0) scale chosen so the block maximum lands near 6.
 * e8m0_mode: FP4Q_E8M0_RNE (default reading: RN(m/6) rounded to the nearest
 * power of two, exact midpoints to the even biased exponent -- the FP6 essay
 * on blog.ast.moe notes that round-to-nearest-even in the E8M0 conversion
 * matters), FP4Q_E8M0_CEIL (smallest power of two >= RN(m/6): never clips),
 * FP4Q_E8M0_OCP_FLOOR (2^(floor(log2 m) - 2), the OCP MX rule).
 * Elements: v = RN(x * 2^-e), E2M1 round to nearest even with saturation.
 * Scale byte = e + 127.  Outputs as for NVFP4 with blocks of 32.
 * Shape: cols % 32 == 0; COLWISE also needs rows % 32 == 0. */
fp4q_status fp4q_quantize_mxfp4(const void *x, int dtype, int64_t rows, int64_t cols,
                                int64_t ld, unsigned layouts, int e8m0_mode, uint8_t *q_row,
                                uint8_t *sf_row, uint8_t *q_col, uint8_t *sf_col,
                                int scale_layout, void *stream);

/* NVFP4 with 16x16 2D block scaling of a weight (Qiita note, "2D scaling":
 * square 16x16 tiles make q(W) = q(W^T)^T), emitting W and W^T codes from
 * the same scales in one pass.
 *   q_w   [rows, cols/2]   codes of W      (may be NULL)
 *   q_wt  [cols, rows/2]   codes of W^T    (may be NULL)
 *   sf_tiles [rows/16, cols/16]  one E4M3 scale per tile, linear (required)
 *   sf_w_1x16  [rows, cols/16] (nullable)  the tile scale repeated for each
 *   sf_wt_1x16 [cols, rows/16] (nullable)  1x16 block of W / W^T, in
 *              scale_layout -- the form a 1x16 block-scaled GEMM reads
 *   amax, tensor_scale_out, workspace as for fp4q_quantize_nvfp4.
 * Shape: rows % 16 == 0, cols % 16 == 0. */
fp4q_status fp4q_quantize_2d(const void *w, int dtype, int64_t rows, int64_t cols, int64_t ld,
                             const float *amax, float *tensor_scale_out, uint8_t *q_w,
                             uint8_t *q_wt, uint8_t *sf_tiles, uint8_t *sf_w_1x16,
                             uint8_t *sf_wt_1x16, int scale_layout, void *workspace,
                             size_t ws_bytes, void *stream);

/* amax of the random-Hadamard-transformed gradient (see below), the tensor
 * amax that fp4q_quantize_rht_sr needs.  amax_out: device float, overwritten. */
fp4q_status fp4q_rht_amax(const void *dy, int dtype, int64_t tokens, int64_t cols, int64_t ld,
                          int hadamard_n, uint64_t seed, float *amax_out, void *stream);

/* Random Hadamard transform of a gradient dY [tokens, cols] along tokens,
 * fused with column-wise NVFP4 1x16 quantization (blocks of 16 tokens) of
 * the transformed values, written as the Wgrad operand dY^T.
 * Qiita note, "ランダムアダマール変換": Wgrad' = q(dY H) q(H^T x), with H a
 * Hadamard matrix (H H^T = I) times a random +-1 diagonal S; "確率的丸め":
 * stochastic rounding helps gradient quantization.
 * Per column and per group of n = hadamard_n (16 or 128) tokens:
 *   u = S * x (signs from Philox4x32-10(counter (0,0,1,0), key seed), bit k
 *   of the 128-bit output -> S_k = -1), a natural-order fast Walsh-Hadamard
 *   transform with stages h = 1, 2, ..., n/2 in that order (each butterfly
 *   (a, b) -> (RN(a+b), RN(a-b))), then t = RN(u * RN(1/sqrt(n))).
 *   round  FP4Q_SR (bits keyed on seed and the input index token*cols+col)
 *          or FP4Q_RNE
 *   amax_rht  device float: amax of t (from fp4q_rht_amax), or NULL: then
 *          it is computed first into `workspace`
 *   q_t [cols, tokens/2], sf_t [cols, tokens/16] (scale_layout)
 *   rht_debug_out  nullable device float [tokens, cols] <- t itself
 * Shape: tokens % hadamard_n == 0, cols % 8 == 0. */
fp4q_status fp4q_quantize_rht_sr(const void *dy, int dtype, int64_t tokens, int64_t cols,
                                 int64_t ld, int hadamard_n, int round, uint64_t seed,
                                 const float *amax_rht, float *tensor_scale_out, uint8_t *q_t,
                                 uint8_t *sf_t, int scale_layout, float *rht_debug_out,
                                 void *workspace, size_t ws_bytes, void *stream);

/* Both quantized operands of dY for the backward pass from ONE read of dY.
 * Qiita note, "誤差逆伝播と転置": Dgrad uses dY as is, Wgrad the transposed
 * dY^T; "ランダムアダマール変換": the transform is applied to the Wgrad
 * operands only.  The outputs are byte for byte those of
 *   fp4q_quantize_nvfp4(dy, FP4Q_ROWWISE, round, seed_row, amax_row)
 *       -> s_dec_row_out, q_row [tokens, cols/2], sf_row [tokens, cols/16]
 *   fp4q_quantize_rht_sr(dy, hadamard_n, round, seed_col, amax_rht)
 *       -> s_dec_col_out, q_t [cols, tokens/2], sf_t [cols, tokens/16]
 * with separate seeds, so the two operands draw independent random bits.
 * The random signs S depend only on seed_col: quantizing the activation X
 * with fp4q_quantize_rht_sr and the same seed applies the same H diag(S) to
 * the other Wgrad operand.
 *   amax_row, amax_rht  device floats (the tensor amax of dY, and that of
 *          its transform), or NULL: then computed first into the workspace
 *          (each NULL costs one extra read of dY)
 * Shape: tokens % hadamard_n == 0, cols % 16 == 0.  Both scale matrices use
 * scale_layout. */
fp4q_status fp4q_quantize_backward(const void *dy, int dtype, int64_t tokens, int64_t cols,
                                   int64_t ld, int hadamard_n, int round, uint64_t seed_row,
                                   uint64_t seed_col, const float *amax_row,
                                   const float *amax_rht, float *s_dec_row_out,
                                   float *s_dec_col_out, uint8_t *q_row, uint8_t *sf_row,
                                   uint8_t *q_t, uint8_t *sf_t, int scale_layout, void *workspace,
                                   size_t ws_bytes, void *stream);

/* IF4 adaptive quantization, row-wise 1x16 ("Adaptive Block-Scaled Data
 * Types" explainer, section 2): per block the NVFP4 scale S and factor r,
 * v = RN(x*r); FP4 candidate E2M1_rne(v); INT4 candidate
 * k = clamp(rint(RN(v * RN(7/6))), -7, 7) decoded as RN(k * RN(6/7)) (the 6/7
 * method); squared errors summed in order with fused multiply-add; INT4 iff
 * its error is strictly smaller.  INT4 nibbles hold k in two's complement;
 * bit 7 of the scale byte is set for INT4 blocks.
 *   q [rows, cols/2], sf [rows, cols/16]; amax / tensor_scale_out / workspace
 *   as for fp4q_quantize_nvfp4.   Shape: cols % 16 == 0. */
fp4q_status fp4q_quantize_if4(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                              const float *amax, float *tensor_scale_out, uint8_t *q,
                              uint8_t *sf, int scale_layout, void *workspace, size_t ws_bytes,
                              void *stream);

/* NVINT4, the INT4 comparison format of the "Adaptive Block-Scaled Data
 * Types" explainer (section 4), read as IF4's INT4 candidate in every block:
 * the NVFP4 scale S and factor r, v = RN(x*r), k = clamp(rint(RN(v * RN(7/6))),
 * -7, 7) in two's complement, and bit 7 of every scale byte set, so that
 * fp4q_dequantize(FP4Q_FMT_IF4, ...) decodes it (k * RN(6/7) * S * s_dec).
 * Arguments, layouts and errors as for fp4q_quantize_if4. */
fp4q_status fp4q_quantize_nvint4(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                                 const float *amax, float *tensor_scale_out, uint8_t *q,
                                 uint8_t *sf, int scale_layout, void *workspace,
                                 size_t ws_bytes, void *stream);

/* Four over six ("4/6"), the remedy the IF4 explainer (section 1) contrasts
 * IF4 with: every block maximum is mapped to 4 instead of 6, giving a finer
 * grid relative to the block at the cost of the codes +-6.  Read as NVFP4
 * 1x16 with 4 in place of 6: s_enc = RN(1792/amax), s_dec = RN(amax/1792)
 * (1792 = 4 * 448), S = E4M3_rne_sat(RN(RN(m * s_enc) / 4)), r = RN(s_enc/S),
 * v = RN(x * r), E2M1 round to nearest even (|v| < 5, so no code reaches 6).
 * Outputs, layouts and errors as for fp4q_quantize_nvfp4 with FP4Q_RNE;
 * fp4q_dequantize(FP4Q_FMT_NVFP4, ...) with this call's s_dec decodes it. */
fp4q_status fp4q_quantize_four_over_six(const void *x, int dtype, int64_t rows, int64_t cols,
                                        int64_t ld, unsigned layouts, const float *amax,
                                        float *tensor_scale_out, uint8_t *q_row, uint8_t *sf_row,
                                        uint8_t *q_col, uint8_t *sf_col, int scale_layout,
                                        void *workspace, size_t ws_bytes, void *stream);

/* IF6: the IF per-block choice at 6 bits.  "Adaptive Block-Scaled Data
 * Types" explainer, section 2: each block is quantized to a float grid and to
 * a scaled integer grid, the smaller squared error wins, the scale's sign bit
 * records the choice, and the idea extends to 6 bits.  The library's reading:
 * FP6 E2M3 (largest 7.5; "FP6で隣り合う値の間隔を見てみる") against INT6
 * (-31..31) rescaled by 7.5/31, with NVFP4's scaling at 7.5 in place of 6:
 *   s_enc = RN(3360/amax), s_dec = RN(amax/3360)       (3360 = 7.5 * 448)
 *   S = E4M3_rne_sat(RN(RN(m * s_enc) / 7.5)), r = RN(s_enc / S), v = RN(x*r)
 *   FP6:  E2M3 round to nearest even with saturation, sign copied
 *   INT6: k = clamp(rint(RN(v * RN(31/7.5))), -31, 31), value RN(k * RN(7.5/31))
 *   errors sum fma(d, d, e) over the block in order, d = RN(v - value);
 *   INT6 iff its error is strictly smaller; scale bit 7 set = INT6.
 *   q   [rows, cols * 3/4] bytes: four 6-bit codes per three bytes as in
 *       fp4q_quantize_mxfp6 (the E2M3 code, or k in 6-bit two's complement)
 *   sf  [rows, cols/16] flagged E4M3 scales in scale_layout
 * amax, tensor_scale_out, workspace and errors as for fp4q_quantize_if4;
 * shape cols % 16 == 0.  fp4q_dequantize(FP4Q_FMT_IF6, ..., 1, 16, s_dec, ...)
 * decodes it: y = RN(RN(value * S) * s_dec). */
fp4q_status fp4q_quantize_if6(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                              const float *amax, float *tensor_scale_out, uint8_t *q, uint8_t *sf,
                              int scale_layout, void *workspace, size_t ws_bytes, void *stream);

/* IF3: the IF per-block choice at 3 bits ("Adaptive Block-Scaled Data Types"
 * explainer, section 2, names IF3 beside IF6).  The library's reading: a
 * 3-bit code is a sign and two magnitude bits; the float split E1M1 would
 * give the uniform magnitudes 0, 0.5, 1, 1.5, which are INT3 times 0.5 and
 * leave nothing to choose, so the float grid is FP3 E2M0 (two exponent bits,
 * bias 1, no mantissa; field 0 is zero): magnitudes 0, 1, 2, 4.  Against it
 * INT3 (-3..3) rescaled by 4/3, with NVFP4's scaling at 4 in place of 6:
 *   s_enc = RN(1792/amax), s_dec = RN(amax/1792)       (1792 = 4 * 448)
 *   S = E4M3_rne_sat(RN(RN(m * s_enc) / 4)), r = RN(s_enc / S), v = RN(x*r)
 *   FP3:  nearest of 0, 1, 2, 4 to |v|, ties to the even code (0.5 -> 0,
 *         1.5 -> 2, 3 -> 2), saturating at 4, sign copied
 *   INT3: k = clamp(rint(RN(v * 0.75)), -3, 3), value RN(k * RN(4/3))
 *   errors sum fma(d, d, e) over the block in order, d = RN(v - value);
 *   INT3 iff its error is strictly smaller; scale bit 7 set = INT3.
 *   q   [rows, cols * 3/8] bytes: eight 3-bit codes per three bytes, code j
 *       of a group in bits 3j..3j+2 of the little-endian 24-bit word (FP3:
 *       sign in bit 2, the magnitude's index 0..3 in bits 0-1; INT3: k in
 *       3-bit two's complement)
 *   sf  [rows, cols/16] flagged E4M3 scales in scale_layout
 * amax, tensor_scale_out, workspace and errors as for fp4q_quantize_if4;
 * shape cols % 16 == 0.  fp4q_dequantize(FP4Q_FMT_IF3, ..., 1, 16, s_dec, ...)
 * decodes it: y = RN(RN(value * S) * s_dec). */
fp4q_status fp4q_quantize_if3(const void *x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                              const float *amax, float *tensor_scale_out, uint8_t *q, uint8_t *sf,
                              int scale_layout, void *workspace, size_t ws_bytes, void *stream);

/* MXFP6 1x32, row-wise: the OCP FP6 element formats with E8M0 block scales.
 * "FP6から考えるLLM量子化" (blog.ast.moe), "FP6で隣り合う値の間隔を見てみる":
 * E2M3 (sign, 2 exponent bits with bias 1, 3 mantissa bits; largest 7.5)
 * spends its bits on spacing, E3M2 (3 exponent bits with bias 3, 2 mantissa
 * bits; largest 28) on range; both have subnormals and no Inf/NaN.  32
 * values share one power-of-two scale as in fp4q_quantize_mxfp4, with the
 * format's largest magnitude qmax = 1.x * 2^emax in place of 6:
 *   FP4Q_E8M0_RNE        RN(m / qmax) to the nearest power of two (exact
 *                        midpoints to the even biased exponent)
 *   FP4Q_E8M0_CEIL       smallest power of two >= RN(m / qmax)
 *   FP4Q_E8M0_OCP_FLOOR  2^(floor(log2 m) - emax), emax 2 (E2M3) or 4 (E3M2)
 * Elements v = RN(x * 2^-e), FP6 round to nearest even with saturation, the
 * sign copied (a negative value that rounds to zero keeps its sign bit).
 *   fp6_format   FP4Q_FP6_E2M3 or FP4Q_FP6_E3M2
 *   q            [rows, cols * 3/4] bytes: each group of four codes c0..c3
 *                (consecutive columns) is the little-endian 24-bit word
 *                c0 | c1 << 6 | c2 << 12 | c3 << 18 (the page notes that FP6
 *                values straddle byte boundaries; this order is the
 *                library's reading)
 *   sf           [rows, cols/32] biased exponents e + 127, in scale_layout
 * Shape: cols % 32 == 0; swizzled scales need rows % 128 == 0 and
 * (cols/32) % 4 == 0.  x, q 16-byte aligned; ld * element size % 16 == 0.
 * fp4q_dequantize(FP4Q_FMT_MXFP6_E2M3 / _E3M2, ..., 1, 32, NULL, ...) decodes
 * it.  All buffers are the caller's; nothing is allocated. */
fp4q_status fp4q_quantize_mxfp6(const void *x, int dtype, int64_t rows, int64_t cols,
                                int64_t ld, int fp6_format, int e8m0_mode, uint8_t *q,
                                uint8_t *sf, int scale_layout, void *stream);

/* Block-scaled NVFP4 GEMM on the tensor cores: the consumer of the
 * quantized operands.  Qiita note on NVFP4 training ("Blockwise", "誤差逆伝播と
 * 転置"): Fprop multiplies X by W^T with both in NVFP4, Wgrad multiplies dY^T
 * by X^T from the column-wise copies; every 16-value block's E2M1 codes are
 * multiplied by its E4M3 block scale and the FP32 tensor scales multiply the
 * product.  With A = dequantize(qa, sfa) and B = dequantize(qb, sfb) taken
 * with the block scales only:
 *   C[m, n] = RN(acc[m, n] * RN(s_a * s_b)),  acc = A B^T accumulated in FP32
 * by tcgen05.mma kind::mxf4nvf4 (the order of the FP32 additions is the
 * hardware's; the result is within FP32 accumulation error of the exact
 * product, not bit-reproducible against a CPU sum).
 *   qa, sfa      A codes [M, K/2] (row-wise, K-major) and its 1x16 scales in
 *                FP4Q_SCALE_SWIZZLED_128x4, as fp4q_quantize_nvfp4 writes them
 *                (a column-wise output is the row-wise layout of the transpose)
 *   qb, sfb      B codes [N, K/2] and scales, the same way
 *   tensor_scale_a, tensor_scale_b  device floats s_dec of A and B, or NULL
 *                for 1
 *   c, c_dtype, ldc  output [M, ldc] row-major, FP32 or BF16 (RNE of the FP32
 *                value); ldc >= N
 *   status       device int or NULL: set to 1 if a wait inside the kernel ran
 *                out (about a second; the tile is then not written).  The
 *                library never clears it
 * Shape: M % 128 == 0, N % 128 == 0, K % 256 == 0 (one 128x128 output tile
 * per CTA, 256 values of K per pipeline stage).  All pointers 16-byte
 * aligned, ldc * element size % 16 == 0.  K == 0 writes zeros.  Device memory
 * is the caller's; nothing is allocated. */
fp4q_status fp4q_gemm_nvfp4(const uint8_t *qa, const uint8_t *sfa, const float *tensor_scale_a,
                            const uint8_t *qb, const uint8_t *sfb, const float *tensor_scale_b,
                            int64_t M, int64_t N, int64_t K, void *c, int c_dtype, int64_t ldc,
                            int *status, void *stream);

/* IF4 x NVFP4 GEMM on the tensor cores: the IF4 operand of the consumer GEMM.
 * "Adaptive Block-Scaled Data Types" explainer, section 2: an IF4 block is
 * FP4 (E2M1 code * S) or INT4 (k * RN(6/7) * S), flagged by the scale's sign
 * bit.  The block-scaled MMA multiplies E2M1 codes by E4M3 scales only, and
 * RN(6/7) * S is not an E4M3 value; every k in -7..7 is the sum of at most two
 * E2M1 values (5 = 4 + 1, 7 = 6 + 1), so A is split into three NVFP4 operands
 * sharing the unflagged scales (the FP4 blocks, and the two E2M1 parts of the
 * INT4 blocks), and one GEMM pass accumulates the FP4 part and both INT4
 * parts in two tensor-memory accumulators (FP32, by tcgen05.mma; B is read
 * once):
 *   C = RN(RN(acc_fp * a) + RN(acc_int * a67)),  a = RN(s_a * s_b),
 *   a67 = RN(a * RN(6/7)).
 * The result is within FP32 accumulation and rounding error of the exact
 * product of the dequantized IF4 and NVFP4 operands.
 *   qa, sfa      IF4 codes [M, K/2] and flagged scales in the 128x4 layout, as
 *                fp4q_quantize_if4 writes them with FP4Q_SCALE_SWIZZLED_128x4
 *   qb, sfb      NVFP4 codes [N, K/2] and swizzled scales
 *   c, ldc       FP32 output [M, ldc]
 *   workspace    device memory of fp4q_gemm_if4_workspace_bytes(M, K) bytes,
 *                16-byte aligned (the split operands; the caller's)
 *   tensor scales, status and shapes as for fp4q_gemm_nvfp4. */
size_t fp4q_gemm_if4_workspace_bytes(int64_t M, int64_t K);
fp4q_status fp4q_gemm_if4_nvfp4(const uint8_t *qa, const uint8_t *sfa, const float *tensor_scale_a,
                                const uint8_t *qb, const uint8_t *sfb,
                                const float *tensor_scale_b, int64_t M, int64_t N, int64_t K,
                                float *c, int64_t ldc, void *workspace, size_t ws_bytes,
                                int *status, void *stream);

/* Block-scaled MXFP4 GEMM on the tensor cores: the consumer of
 * fp4q_quantize_mxfp4's swizzled outputs.  Ultralytics glossary "FP4",
 * section "FP4の仕組み" (MXFP4: 32 E2M1 values share one power-of-two E8M0
 * scale, no tensor scale); the AIBR summary of Quartet (MXFP4 operands in the
 * linear layers on Blackwell).  With A = dequantize(qa, sfa) and B =
 * dequantize(qb, sfb):
 *   C[m, n] = acc[m, n],  acc = A B^T accumulated in FP32 by tcgen05.mma
 * kind::mxf4 block32 (the order of the FP32 additions is the hardware's; the
 * result is within FP32 accumulation error of the exact product).
 *   qa, sfa      A codes [M, K/2] (K-major) and its 1x32 E8M0 scales in
 *                FP4Q_SCALE_SWIZZLED_128x4, as fp4q_quantize_mxfp4 writes them
 *                (a column-wise output is the row-wise layout of the transpose)
 *   qb, sfb      B codes [N, K/2] and scales, the same way
 *   c, c_dtype, ldc, status  as for fp4q_gemm_nvfp4
 * Shape: M % 128 == 0, N % 128 == 0, K % 256 == 0; alignment as for
 * fp4q_gemm_nvfp4.  K == 0 writes zeros.  Nothing is allocated. */
fp4q_status fp4q_gemm_mxfp4(const uint8_t *qa, const uint8_t *sfa, const uint8_t *qb,
                            const uint8_t *sfb, int64_t M, int64_t N, int64_t K, void *c,
                            int c_dtype, int64_t ldc, int *status, void *stream);

/* ---- TEST-ONLY ENTRY POINT: not part of the supported interface ----------
 * Exported so that the failure-detection test can reach it through the C
 * ABI; production code has no reason to call it.
 *
 * Failure-detection test hook for fp4q_gemm_nvfp4: the same call, but the
 * kernel's loader issues no operand loads, so that the tensor-core thread's
 * bounded wait runs out (after about a second).  No tensor-core work is ever
 * issued; the kernel sets *status to 1, writes unspecified values to C, frees
 * its tensor memory and returns, and the CUDA context stays usable.
 * Arguments as for fp4q_gemm_nvfp4; status must be non-NULL and K > 0.  For
 * tests only. */
fp4q_status fp4q_gemm_nvfp4_withhold_loads(const uint8_t *qa, const uint8_t *sfa,
                                           const float *tensor_scale_a, const uint8_t *qb,
                                           const uint8_t *sfb, const float *tensor_scale_b,
                                           int64_t M, int64_t N, int64_t K, void *c, int c_dtype,
                                           int64_t ldc, int *status, void *stream);

/* Dequantization of packed codes [rows, cols/2] back to y [rows, cols]
 * (FP32 or BF16 = RNE of the FP32 value), Ultralytics glossary "FP4の仕組み"
 * (grid value * sign * scale):
 *   NVFP4  y = RN(RN(g * S) * s_dec)           block 1x16 or 16x16
 *   IF4    INT4 blocks (scale bit 7): y = RN(RN(RN(k * RN(6/7)) * S) * s_dec)
 *   MXFP4  y = g * 2^(scale - 127)             block 1x32
 *   MXFP6  y = RN(g * 2^(scale - 127))         block 1x32; q is [rows,
 *          cols * 3/4] bytes packed as fp4q_quantize_mxfp6 writes them
 *   IF6    y = RN(RN(value * S) * s_dec)        block 1x16, 6-bit codes as
 *          fp4q_quantize_if6 writes them (INT6 blocks: value = RN(k * RN(7.5/31)))
 *   IF3    y = RN(RN(value * S) * s_dec)        block 1x16, 3-bit codes as
 *          fp4q_quantize_if3 writes them (INT3 blocks: value = RN(k * RN(4/3)))
 *   block_rows x block_cols: 1x16 (NVFP4, IF4, IF6, IF3), 16x16 (NVFP4 2D tiles; then
 *   sf is the linear [rows/16, cols/16] tile matrix), 1x32 (MXFP4, MXFP6).
 *   tensor_scale: device float s_dec (NVFP4 / IF4 / IF6 / IF3), ignored for
 *   MXFP4/6.
 *   Column-wise outputs are dequantized as the [cols, rows] matrices they are.
 * Shape: cols % block_cols == 0, rows % block_rows == 0. */
fp4q_status fp4q_dequantize(int format, const uint8_t *q, const uint8_t *sf, int scale_layout,
                            int block_rows, int block_cols, const float *tensor_scale,
                            int64_t rows, int64_t cols, void *y, int y_dtype, void *stream);

/* fp4q_quantize_nvfp4 without a workspace argument, for callers that cannot
 * allocate device memory: code inside a host application or framework that
 * owns every device buffer, or that must not call cudaMalloc once set-up is
 * over.  The pages have no counterpart; this is a library convenience.
 * The arguments, outputs and error codes are those of fp4q_quantize_nvfp4.
 * The one difference is where the amax goes when amax == NULL. It is
 * computed into a 256-byte array that the library keeps in device memory:
 *   - Every GPU that loads the library holds that array until the process
 *     exits. The array's size is the most workspace this call can use.
 *     The call returns FP4Q_ERR_WORKSPACE_TOO_SMALL if
 *     fp4q_workspace_bytes(rows, cols) ever exceeded it.
 *     The amax needs 4 bytes at any tensor size, so no shape is refused for
 *     scratch.
 *   - The first call on a device with amax == NULL looks the array's device
 *     address up (cudaGetSymbolAddress, with that device made current).
 *     Make that first call before any stream capture begins.  The address
 *     is kept per device and per context: after a cudaDeviceReset the next
 *     call looks it up again, so make that call outside capture too.
 *   - Arguments are checked exactly as fp4q_quantize_nvfp4 checks them, and
 *     a rejected call returns that status before touching any device.
 *   - All calls on one device share the array. The amax pre-pass clears it
 *     before use, and the array keeps the last call's amax afterwards.
 *     Calls with amax == NULL that can overlap on the GPU (different streams,
 *     no ordering between them) race on it. Order them, or pass amax.
 * This call allocates nothing: no cudaMalloc, no cudaFree, no library
 * allocator. */
fp4q_status fp4q_quantize_nvfp4_noalloc(const void *x, int dtype, int64_t rows, int64_t cols,
                                        int64_t ld, unsigned layouts, int round, uint64_t seed,
                                        const float *amax, float *tensor_scale_out,
                                        uint8_t *q_row, uint8_t *sf_row, uint8_t *q_col,
                                        uint8_t *sf_col, int scale_layout, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* FP4Q_H_ */
