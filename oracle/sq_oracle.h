/*
 * sq_oracle.h -- plain CPU oracle for the SmoothQuant W8A8 linear layer.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only the tests, the smoke check in
 * __graft_entry__.py and the CPU-baseline leg of bench.py may load it. The CUDA
 * path never includes this header and this library never includes the CUDA
 * path's headers: the two share no code, constants or helpers.
 *
 * Conventions
 *   - Every floating-point step is one IEEE-754 binary32 operation rounded to
 *     nearest-even, compiled with -ffp-contract=off (no fused multiply-add),
 *     except where a function says it works in binary64.
 *   - Matrices are dense row-major. X is [M,K] (tokens x input channels),
 *     W is [K,N] (input channels x output channels), Y = X W is [M,N].
 *   - Quantized weights are stored transposed, Wq[n][k] ([N,K], K contiguous).
 *   - "bf16" arguments are raw bfloat16 bit patterns (uint16).
 *   - dtype codes: 0 = fp32, 1 = bf16 (raw uint16).
 *   - qtype codes: 0 = symmetric INT8 (scale amax/127, clamp to +-127),
 *                  1 = FP8 E4M3 (scale amax/448, round-to-nearest-even,
 *                      saturating to +-448).
 */
#ifndef SQ_ORACLE_H
#define SQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* bfloat16 <-> binary32 (definition of the format; widening is exact). */
float    sqo_bf16_to_f32(uint16_t h);
uint16_t sqo_f32_to_bf16_rne(float f);
void     sqo_f32_to_bf16_rne_n(const float* x, uint16_t* out, int64_t n);

/* FP8 E4M3: value of a code, and round-to-nearest-even saturating encode. */
double   sqo_e4m3_decode(uint8_t code);
uint8_t  sqo_e4m3_encode_rn_sat(float x);

/* a1/a2 calibration: out[c] = max_r |x[r*cols + c]| (per column) when
 * per_column != 0, else out[r] = max_c |x[r*cols + c]| (per row). */
void sqo_amax(const void* x, int dtype, int64_t rows, int64_t cols,
              int per_column, float* out);

/* a3 smoothing factors, computed in binary64 and rounded once to binary32:
 * s[k] = max(ax,eps)^alpha / max(aw,eps)^(1-alpha), eps = 1e-5. */
void sqo_smooth_factors(const float* amax_x, const float* amax_w, int64_t K,
                        double alpha, float* s);

/* The smoothing transform alone, before any quantization:
 * X~[m][k] = X[m][k] / s[k] and W~[k][n] = s[k] * W[k][n]. */
void sqo_smooth_act(const void* x, int dtype, int64_t M, int64_t K,
                    const float* s, float* out);
void sqo_smooth_weight(const void* w, int dtype, int64_t K, int64_t N,
                       const float* s, float* out);

/* Offline fold of the activation division into the layer that produces X:
 * its parameters for channel k of X are divided by s[k] once, so it emits
 * X~ itself and the runtime quantization runs without s.
 * p: [rows, cols] (dtype); per_column != 0: channel = column,
 * out[r][c] = p[r][c] / s[c]; else channel = row, out[r][c] = p[r][c] / s[r]. */
void sqo_fold_smoothing(const void* p, int dtype, int64_t rows, int64_t cols,
                        const float* s, int per_column, float* out);

/* a4 offline weight smoothing + per-output-channel quantization.
 * w: [K,N] (dtype), s: [K] or NULL (no smoothing).
 * wq: [N,K] int8 or E4M3 codes, sw: [N] binary32 scales. */
void sqo_quantize_weight(const void* w, int dtype, int64_t K, int64_t N,
                         const float* s, int qtype, void* wq, float* sw);

/* a5 runtime activation smoothing + per-token quantization.
 * x: [M,K] (dtype), s: [K] or NULL. xq: [M,K] codes, sx: [M] scales. */
void sqo_quantize_act(const void* x, int dtype, int64_t M, int64_t K,
                      const float* s, int qtype, void* xq, float* sx);

/* Per-tensor activation scaling ([WAQ] §4 "Per-Tensor Scaling for FP8" and
 * "FP8 vs INT8 SmoothQuant": per-tensor scaling online, or delayed scaling
 * from the previous step's max). x: [M,K] (dtype), s: [K] or NULL.
 * scale_in: the scale to use (delayed scaling), or NULL for the online scale
 * max|x/s| / Q of this tensor. xq: [M,K] codes; sx: [M] each set to the scale
 * used; *amax_out: max|x/s| over the whole tensor (the next step's max). */
void sqo_quantize_act_tensor(const void* x, int dtype, int64_t M, int64_t K,
                             const float* s, int qtype, const float* scale_in,
                             void* xq, float* sx, float* amax_out);

/* a6 INT8 x INT8 -> int32 accumulators, acc[m][n] = sum_k xq[m][k]*wq[n][k]. */
void sqo_gemm_i8(const int8_t* xq, const int8_t* wq, int64_t M, int64_t N,
                 int64_t K, int32_t* acc);

/* a7 E4M3 x E4M3 products summed exactly in binary64 (see the .c file). */
void sqo_gemm_e4m3(const uint8_t* xq, const uint8_t* wq, int64_t M, int64_t N,
                   int64_t K, double* acc);

/* Dequantization epilogue for one accumulator value (already widened to
 * binary32 by the caller's rule): t = a*sx; t = t*sw; t = t + bias. */
float sqo_dequant(float acc_f32, float sx_m, float sw_n, int has_bias,
                  uint16_t bias_bf16);

/* Full epilogue over [M,N]. acc_kind 0: int32 accumulators (acc_i32),
 * 1: binary64 accumulators (acc_f64, rounded once to binary32).
 * bias: [N] bf16 or NULL. y_f32 (may be NULL) gets the binary32 value before
 * the bf16 cast, y_bf16 (may be NULL) the bf16 result. */
void sqo_epilogue(const int32_t* acc_i32, const double* acc_f64, int acc_kind,
                  const float* sx, const float* sw, const uint16_t* bias,
                  int64_t M, int64_t N, float* y_f32, uint16_t* y_bf16);

/* One output element computed from scratch (for sampled checks at full size):
 * the dot product over K followed by the epilogue. qtype as above. */
void sqo_linear_at(const void* xq, const float* sx, const void* wq,
                   const float* sw, const uint16_t* bias, int qtype,
                   int64_t K, const int64_t* rows, const int64_t* cols,
                   int64_t count, double* acc_out, float* y_f32,
                   uint16_t* y_bf16);

/* Weight-only quantization (W8A16 / W4A16). INT4 weights: per output channel
 * sw[n] = max_k |w[k][n]| / 7, codes clamp(round-half-even(w / sw), -7, 7)
 * (0 where sw is 0), packed into wq4 [N, K/2] bytes: the codes of k = 8g ..
 * 8g+7 form the little-endian 32-bit word at byte 4g of the row, code(8g+2j)
 * in bits 4j..4j+3 and code(8g+2j+1) in bits 16+4j..16+4j+3 (two's
 * complement nibbles). K must be a multiple of 8. */
void sqo_quantize_weight_i4(const void* w, int dtype, int64_t K, int64_t N,
                            uint8_t* wq4, float* sw);
/* The codes of a packed INT4 matrix, one int8 per element: codes [N,K]. */
void sqo_unpack_i4(const uint8_t* wq4, int64_t N, int64_t K, int8_t* codes);
/* y[m][n] = sum_k x[m][k] * (q[n][k] * sw[n]) + bias[n] in binary64, with x
 * [M,K] bf16 bits, q the codes of wq (bits 8: int8 [N,K]; bits 4: packed
 * [N,K/2]), sw [N] and bias [N] bf16 or NULL. */
void sqo_gemm_weight_only(const uint16_t* x, const void* wq, int bits, const float* sw,
                          const uint16_t* bias, int64_t M, int64_t N, int64_t K,
                          double* y);

/* RMS normalization of each row of x (bf16 bits [M,K]) with the per-channel
 * gain g [K] (binary32; the smoothing factors folded in: g = gamma / s),
 * fused with per-token quantization (qtype 0 INT8, 1 E4M3). Per row:
 *   ss  = sum of x_k^2 over the k with e_k >= e_max - 48 (e: the bf16
 *         exponent of x_k, e_max the largest in the row), exactly, then
 *         rounded once to binary64;
 *   r   = binary32( binary64( 1 / sqrt( ss / K + eps ) ) ), each binary64
 *         operation rounded once (eps > 0, as binary64);
 *   xn_k = (x_k * r) * g_k in binary32, each product rounded once;
 *   then sqo_quantize_act of xn without smoothing.
 * rinv [M] (r) and xn [M,K] are written when non-NULL. */
void sqo_rmsnorm_quantize_act(const uint16_t* x, int64_t M, int64_t K, const float* g,
                              float eps, int qtype, void* xq, float* sx, float* rinv,
                              float* xn);

/* Threads OpenMP will use (1 when built without OpenMP). */
int sqo_num_threads(void);

#ifdef __cplusplus
}
#endif

#endif /* SQ_ORACLE_H */
