/*
 * sq_oracle.c -- plain, slow, obviously correct CPU oracle for the SmoothQuant
 * W8A8 linear layer Y = X W = (X diag(s)^-1)(diag(s) W).
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only tests/, __graft_entry__.smoke()
 * and the cpu_baseline / reference leg of bench.py may load it. It shares no
 * code with the CUDA path.
 *
 * Sources (web pages on W8A8 / SmoothQuant):
 *   [WAQ]  "Weight-Activation Quantization" (infra.bea.ai inference guide)
 *          §2 "The Problem: Activation Outliers" (per-tensor scale max|x|/127),
 *          §3 "SmoothQuant: The Smoothing Trick" (Y = (X S^-1)(S W), the worked
 *             example, the two-step pipeline, "Choosing the Smoothing Factor"),
 *          §4 "FP8 W8A8 (Native on Hopper+)", "Per-Tensor Scaling for FP8"
 *             (q = cast_fp8(x/s), s = max|x|/448, range [-448, 448]).
 *   [ACT]  "Define activation quantization and explain how W8A8 differs from
 *          weight only quant" (zenaique flashcard): per-token / per-channel
 *          scaling, calibration on a small held-out corpus.
 *   [LES]  grasp.study lesson on W8A16 vs W8A8, §2 "The Challenge of
 *          Activation Quantization: SmoothQuant" (the transform is offline).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - s_j indexes input channel j; max|X_j| runs over calibration tokens and
 *     max|W_j| over the output channels of row j of W.
 *   - activation smoothing is an IEEE binary32 division x / s_j (the pages say
 *     "divide each activation channel by s_j"); weight smoothing is the
 *     binary32 product s_j * W[j][n].
 *   - both amaxes are clamped to >= 1e-5 before the powers; s is computed in
 *     binary64 and rounded once to binary32.
 *   - scales: scale = amax / 127 (INT8) or amax / 448 (E4M3), one binary32
 *     division; per token for X, per output channel for W.
 *   - INT8 code: clamp(round-half-even(v / scale), -127, 127); E4M3 code:
 *     round-to-nearest-even with saturation to +-448.
 *   - a row / column whose scale is 0 (amax 0, or amax so small that amax/127
 *     underflows to 0) is stored with scale 0 and all codes 0.
 *   - dequant epilogue: t = float(acc); t = t*sx[m]; t = t*sw[n];
 *     t = t + float(bias[n]); y = bf16(t) (round-half-even), each step a
 *     separately rounded binary32 operation.
 *   - E4M3 dot products are summed exactly in binary64: every product of two
 *     E4M3 values is a multiple of 2^-18 below 2^18, so a sum of up to 2^14
 *     of them stays below 2^32 and needs at most 50 significant bits.
 *
 * Inputs must be finite; behaviour on NaN / Inf inputs is not specified.
 */
#include "sq_oracle.h"

#include <math.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Number formats                                                           */
/* ------------------------------------------------------------------------ */

static uint32_t f32_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float bits_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* bfloat16 is the top half of a binary32 word, so widening is exact. */
float sqo_bf16_to_f32(uint16_t h) { return bits_f32((uint32_t)h << 16); }

/* Round a binary32 to bfloat16, nearest-even: keep the top 16 bits, then
 * increment the magnitude when the dropped 16 bits exceed half an ulp, or
 * equal half an ulp and the kept part is odd. An increment that carries into
 * the exponent field is the correct next value (up to infinity). */
uint16_t sqo_f32_to_bf16_rne(float f) {
    uint32_t u = f32_bits(f);
    if (isnan(f)) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t kept = u >> 16;
    uint32_t dropped = u & 0xFFFFu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) kept += 1u;
    return (uint16_t)kept;
}

/* The same rounding over an array (a loop over sqo_f32_to_bf16_rne). */
void sqo_f32_to_bf16_rne_n(const float* x, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = sqo_f32_to_bf16_rne(x[i]);
}

/* E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits, no infinity,
 * S.1111.111 is NaN, largest finite value 1.75 * 2^8 = 448 ([WAQ] §4 gives
 * the range [-448, 448]). Normal: (1 + m/8) 2^(e-7) = (8+m) 2^(e-10).
 * Subnormal (e = 0): (m/8) 2^-6 = m 2^-9. */
double sqo_e4m3_decode(uint8_t code) {
    int sign = code >> 7, e = (code >> 3) & 0xF, m = code & 0x7;
    if (e == 15 && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
    return sign ? -v : v;
}

/* Round-to-nearest-even into E4M3 with saturation: magnitudes at or above the
 * largest finite value give 448. Codes 0x00..0x7E are the non-negative finite
 * values in increasing order, so a binary search brackets |x| between two
 * neighbouring codes; the midpoint of two E4M3 values is exact in binary64,
 * so the comparison with it is exact. A tie goes to the even code. */
uint8_t sqo_e4m3_encode_rn_sat(float x) {
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    int lo = 0, hi = 0x7E;              /* invariant: v(lo) <= a < v(hi) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (sqo_e4m3_decode((uint8_t)mid) <= a) lo = mid; else hi = mid;
    }
    double vlo = sqo_e4m3_decode((uint8_t)lo), vhi = sqo_e4m3_decode((uint8_t)hi);
    double midpoint = 0.5 * (vlo + vhi);
    int code;
    if (a < midpoint) code = lo;
    else if (a > midpoint) code = hi;
    else code = (lo % 2 == 0) ? lo : hi;
    return (uint8_t)(sign | code);
}

/* ------------------------------------------------------------------------ */
/* Element access                                                           */
/* ------------------------------------------------------------------------ */

static float load_elem(const void* p, int dtype, int64_t i) {
    if (dtype == 1) return sqo_bf16_to_f32(((const uint16_t*)p)[i]);
    return ((const float*)p)[i];
}

/* INT8 code of v at scale `scale` (scale > 0): round-half-even of the binary32
 * quotient, clamped to the symmetric range +-127 ([WAQ] §2 maps values by
 * max|x|/127; the pages leave the rounding rule open and round-half-even with
 * a symmetric clamp is the reading taken, so -128 is never produced). */
static int8_t quant_i8(float v, float scale) {
    float r = nearbyintf(v / scale);
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    return (int8_t)r;
}

/* [WAQ] §3: "divide each activation channel by s_j" / "multiply the
 * corresponding weight channel by s_j". */
static float smooth_x(float v, float s_k) { return v / s_k; }
static float smooth_w(float v, float s_k) { return s_k * v; }

void sqo_smooth_act(const void* x, int dtype, int64_t M, int64_t K,
                    const float* s, float* out) {
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k)
            out[m * K + k] = smooth_x(load_elem(x, dtype, m * K + k), s[k]);
}

void sqo_smooth_weight(const void* w, int dtype, int64_t K, int64_t N,
                       const float* s, float* out) {
    for (int64_t k = 0; k < K; ++k)
        for (int64_t n = 0; n < N; ++n)
            out[k * N + n] = smooth_w(load_elem(w, dtype, k * N + n), s[k]);
}

/* The smoothing is offline ([LES] §2: the transform happens during model
 * preparation, with no runtime overhead; [WAQ] §3 Step 1 lists X~ = X
 * diag(1/s) under offline preparation). Reading taken: the op that produces
 * X carries one parameter, or one row / column of a weight, per channel k of
 * X, and dividing those by s_k -- the same binary32 division smooth_x applies
 * to x -- makes it emit X~. */
void sqo_fold_smoothing(const void* p, int dtype, int64_t rows, int64_t cols,
                        const float* s, int per_column, float* out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            out[r * cols + c] = smooth_x(load_elem(p, dtype, r * cols + c),
                                         per_column ? s[c] : s[r]);
}

/* ------------------------------------------------------------------------ */
/* The producer of X with the smoothing folded in ([LES] §2: the transform   */
/* is applied offline, no runtime overhead; [WAQ] §3 "Step 1": X~ = X        */
/* diag(1/s) prepared before inference). The pages name no producer; the     */
/* transformer models they quantize (Llama) feed each linear layer from an   */
/* RMS normalization, so that is the producer taken: xn = x / rms(x) * g,    */
/* g = gamma / s folded offline, then per-token quantization of xn.          */
/* ------------------------------------------------------------------------ */

/* bf16 magnitude bits h (sign cleared, h != 0) as N * 2^(e - 7): N = 1.f in
 * 8 bits for normal numbers (128..255), 0.f for subnormals (1..127). */
static void bf16_int_exp(uint16_t h, int* N, int* e) {
    const int be = (h >> 7) & 0xFF, f = h & 0x7F;
    if (be == 0) { *N = f; *e = -126; }
    else { *N = 128 + f; *e = be - 127; }
}

/* one normalized element: the bf16 value times 1/rms, then times the gain,
 * each product a rounded binary32 operation */
static float rms_apply(uint16_t xk, float r, float gk) {
    const float a = sqo_bf16_to_f32(xk) * r;
    return a * gk;
}

void sqo_rmsnorm_quantize_act(const uint16_t* x, int64_t M, int64_t K, const float* g,
                              float eps, int qtype, void* xq, float* sx, float* rinv,
                              float* xn) {
    const float qmax = (qtype == 1) ? 448.0f : 127.0f;
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* row = x + m * K;
        /* the exact sum of squares: each x^2 = N^2 * 2^(2e - 14) is an
         * integer multiple of 2^(2 e_max - 110) when e >= e_max - 48 */
        int emax = -1000;
        for (int64_t k = 0; k < K; ++k) {
            const uint16_t h = row[k] & 0x7FFF;
            if (h == 0) continue;
            int N, e;
            bf16_int_exp(h, &N, &e);
            if (e > emax) emax = e;
        }
        unsigned __int128 S = 0;
        if (emax > -1000) {
            for (int64_t k = 0; k < K; ++k) {
                const uint16_t h = row[k] & 0x7FFF;
                if (h == 0) continue;
                int N, e;
                bf16_int_exp(h, &N, &e);
                if (e < emax - 48) continue;
                S += (unsigned __int128)(uint32_t)(N * N) << (2 * (e - emax) + 96);
            }
        }
        const double ss = (emax > -1000) ? ldexp((double)S, 2 * emax - 110) : 0.0;
        const double mean = ss / (double)K;
        const double v = mean + (double)eps;
        const double t = sqrt(v);
        const float r = (float)(1.0 / t);
        if (rinv) rinv[m] = r;
        /* xn_k = (x_k * r) * g_k, then the row's scale and codes */
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            const float y = rms_apply(row[k], r, g[k]);
            if (xn) xn[m * K + k] = y;
            const float ay = fabsf(y);
            if (ay > amax) amax = ay;
        }
        const float row_scale = amax / qmax;
        sx[m] = row_scale;
        for (int64_t k = 0; k < K; ++k) {
            const float y = rms_apply(row[k], r, g[k]);
            if (qtype == 1)
                ((uint8_t*)xq)[m * K + k] =
                    (row_scale == 0.0f) ? 0 : sqo_e4m3_encode_rn_sat(y / row_scale);
            else
                ((int8_t*)xq)[m * K + k] = (row_scale == 0.0f) ? 0 : quant_i8(y, row_scale);
        }
    }
}

int sqo_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* a1 / a2: calibration amax ([WAQ] §3 "Choosing the Smoothing Factor":     */
/* max|X_j| and max|W_j|; [ACT]: calibration on a held-out corpus).         */
/* ------------------------------------------------------------------------ */

void sqo_amax(const void* x, int dtype, int64_t rows, int64_t cols,
              int per_column, float* out) {
    if (per_column) {
        for (int64_t c = 0; c < cols; ++c) out[c] = 0.0f;
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t c = 0; c < cols; ++c) {
                float a = fabsf(load_elem(x, dtype, r * cols + c));
                if (a > out[c]) out[c] = a;
            }
    } else {
        #pragma omp parallel for schedule(static)
        for (int64_t r = 0; r < rows; ++r) {
            float m = 0.0f;
            for (int64_t c = 0; c < cols; ++c) {
                float a = fabsf(load_elem(x, dtype, r * cols + c));
                if (a > m) m = a;
            }
            out[r] = m;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* a3: s_j = max|X_j|^alpha / max|W_j|^(1-alpha)                            */
/* ([WAQ] §3 "Choosing the Smoothing Factor", alpha in [0,1]).              */
/* ------------------------------------------------------------------------ */

void sqo_smooth_factors(const float* amax_x, const float* amax_w, int64_t K,
                        double alpha, float* s) {
    const double eps = 1e-5;
    for (int64_t k = 0; k < K; ++k) {
        double ax = (double)amax_x[k] > eps ? (double)amax_x[k] : eps;
        double aw = (double)amax_w[k] > eps ? (double)amax_w[k] : eps;
        s[k] = (float)(pow(ax, alpha) / pow(aw, 1.0 - alpha));
    }
}

/* ------------------------------------------------------------------------ */
/* a4: W~ = diag(s) W, then per-output-channel quantization, stored [N,K]   */
/* ([WAQ] §3 "Step 1" / "Step 2": W_tilde = diag(s) @ W, W_int8 =           */
/* quantize(W_tilde); [ACT]: per-channel scaling for weights).              */
/* ------------------------------------------------------------------------ */

void sqo_quantize_weight(const void* w, int dtype, int64_t K, int64_t N,
                         const float* s, int qtype, void* wq, float* sw) {
    const float qmax = (qtype == 1) ? 448.0f : 127.0f;
    /* Each thread owns a block of output channels (columns of W) and walks
     * the rows of W in order; every element's value is computed exactly as
     * written in the page: wt = s_k * w[k][n]. */
    #pragma omp parallel
    {
#ifdef _OPENMP
        int nt = omp_get_num_threads(), t = omp_get_thread_num();
#else
        int nt = 1, t = 0;
#endif
        int64_t n0 = N * t / nt, n1 = N * (t + 1) / nt;
        /* pass 1: amax of column n of W~ */
        for (int64_t n = n0; n < n1; ++n) sw[n] = 0.0f;
        for (int64_t k = 0; k < K; ++k)
            for (int64_t n = n0; n < n1; ++n) {
                float v = load_elem(w, dtype, k * N + n);
                float wt = s ? smooth_w(v, s[k]) : v;
                float a = fabsf(wt);
                if (a > sw[n]) sw[n] = a;
            }
        /* scale = amax / Q */
        for (int64_t n = n0; n < n1; ++n) sw[n] = sw[n] / qmax;
        /* pass 2: codes, stored transposed as wq[n][k] */
        for (int64_t k = 0; k < K; ++k)
            for (int64_t n = n0; n < n1; ++n) {
                float v = load_elem(w, dtype, k * N + n);
                float wt = s ? smooth_w(v, s[k]) : v;
                float scale = sw[n];
                if (qtype == 1) {
                    ((uint8_t*)wq)[n * K + k] =
                        (scale == 0.0f) ? 0 : sqo_e4m3_encode_rn_sat(wt / scale);
                } else {
                    ((int8_t*)wq)[n * K + k] =
                        (scale == 0.0f) ? 0 : quant_i8(wt, scale);
                }
            }
    }
}

/* ------------------------------------------------------------------------ */
/* a5: X~ = X diag(s)^-1, then per-token quantization                       */
/* ([WAQ] §3: "divide each activation channel by s_j", X_int8 =             */
/* quantize(X_tilde) at inference time; [WAQ] §2 scale = max|x|/127;        */
/* [WAQ] §4 q = cast_fp8(x/s), s = max|x|/448; [ACT] per-token scaling).    */
/* ------------------------------------------------------------------------ */

void sqo_quantize_act(const void* x, int dtype, int64_t M, int64_t K,
                      const float* s, int qtype, void* xq, float* sx) {
    const float qmax = (qtype == 1) ? 448.0f : 127.0f;
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float v = load_elem(x, dtype, m * K + k);
            float xs = s ? smooth_x(v, s[k]) : v;
            float a = fabsf(xs);
            if (a > amax) amax = a;
        }
        float scale = amax / qmax;
        sx[m] = scale;
        for (int64_t k = 0; k < K; ++k) {
            float v = load_elem(x, dtype, m * K + k);
            float xs = s ? smooth_x(v, s[k]) : v;
            if (qtype == 1) {
                ((uint8_t*)xq)[m * K + k] =
                    (scale == 0.0f) ? 0 : sqo_e4m3_encode_rn_sat(xs / scale);
            } else {
                ((int8_t*)xq)[m * K + k] =
                    (scale == 0.0f) ? 0 : quant_i8(xs, scale);
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* a6 / a7: the 8-bit matrix product ([WAQ] §3 "Step 2":                    */
/* Y = dequantize(X_int8 @ W_int8); [WAQ] §1 INT8 x INT8 / FP8 x FP8).      */
/* ------------------------------------------------------------------------ */

/* |acc| <= K * 127 * 127, which stays below 2^31 for K < 133144. */
/* Per-tensor scaling of the (smoothed) activations, [WAQ] §4: one scale for
 * the whole tensor, q = cast(x/s / scale). Online: scale = max|x/s| / Q over
 * the tensor. Delayed: the given scale (the previous step's max / Q); values
 * beyond it saturate (INT8 clamps to +-127, E4M3 to +-448). A zero scale
 * gives all-zero codes, as for a zero row in per-token scaling. */
void sqo_quantize_act_tensor(const void* x, int dtype, int64_t M, int64_t K,
                             const float* s, int qtype, const float* scale_in,
                             void* xq, float* sx, float* amax_out) {
    const float qmax = (qtype == 1) ? 448.0f : 127.0f;
    float amax = 0.0f;
    for (int64_t i = 0; i < M * K; ++i) {
        float v = load_elem(x, dtype, i);
        float xs = s ? smooth_x(v, s[i % K]) : v;
        float a = fabsf(xs);
        if (a > amax) amax = a;
    }
    *amax_out = amax;
    const float scale = scale_in ? *scale_in : amax / qmax;
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        sx[m] = scale;
        for (int64_t k = 0; k < K; ++k) {
            float v = load_elem(x, dtype, m * K + k);
            float xs = s ? smooth_x(v, s[k]) : v;
            if (qtype == 1) {
                ((uint8_t*)xq)[m * K + k] =
                    (scale == 0.0f) ? 0 : sqo_e4m3_encode_rn_sat(xs / scale);
            } else {
                ((int8_t*)xq)[m * K + k] =
                    (scale == 0.0f) ? 0 : quant_i8(xs, scale);
            }
        }
    }
}

void sqo_gemm_i8(const int8_t* xq, const int8_t* wq, int64_t M, int64_t N,
                 int64_t K, int32_t* acc) {
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int32_t a = 0;
            for (int64_t k = 0; k < K; ++k)
                a += (int32_t)xq[m * K + k] * (int32_t)wq[n * K + k];
            acc[m * N + n] = a;
        }
}

void sqo_gemm_e4m3(const uint8_t* xq, const uint8_t* wq, int64_t M, int64_t N,
                   int64_t K, double* acc) {
    double table[256];
    for (int c = 0; c < 256; ++c) table[c] = sqo_e4m3_decode((uint8_t)c);
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double a = 0.0;
            for (int64_t k = 0; k < K; ++k)
                a += table[xq[m * K + k]] * table[wq[n * K + k]];
            acc[m * N + n] = a;
        }
}

/* Dequantize one accumulator: per-token scale, then per-channel scale, then
 * the optional bias, each a separately rounded binary32 operation. */
float sqo_dequant(float acc_f32, float sx_m, float sw_n, int has_bias,
                  uint16_t bias_bf16) {
    float t = acc_f32 * sx_m;
    t = t * sw_n;
    if (has_bias) t = t + sqo_bf16_to_f32(bias_bf16);
    return t;
}

void sqo_epilogue(const int32_t* acc_i32, const double* acc_f64, int acc_kind,
                  const float* sx, const float* sw, const uint16_t* bias,
                  int64_t M, int64_t N, float* y_f32, uint16_t* y_bf16) {
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            float a = acc_kind == 0 ? (float)acc_i32[m * N + n]
                                    : (float)acc_f64[m * N + n];
            float t = sqo_dequant(a, sx[m], sw[n], bias != 0, bias ? bias[n] : 0);
            if (y_f32) y_f32[m * N + n] = t;
            if (y_bf16) y_bf16[m * N + n] = sqo_f32_to_bf16_rne(t);
        }
}

void sqo_linear_at(const void* xq, const float* sx, const void* wq,
                   const float* sw, const uint16_t* bias, int qtype,
                   int64_t K, const int64_t* rows, const int64_t* cols,
                   int64_t count, double* acc_out, float* y_f32,
                   uint16_t* y_bf16) {
    double table[256];
    for (int c = 0; c < 256; ++c) table[c] = sqo_e4m3_decode((uint8_t)c);
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = rows[i], n = cols[i];
        float a;
        double exact;
        if (qtype == 1) {
            const uint8_t* xr = (const uint8_t*)xq + m * K;
            const uint8_t* wr = (const uint8_t*)wq + n * K;
            double d = 0.0;
            for (int64_t k = 0; k < K; ++k) d += table[xr[k]] * table[wr[k]];
            exact = d;
            a = (float)d;
        } else {
            const int8_t* xr = (const int8_t*)xq + m * K;
            const int8_t* wr = (const int8_t*)wq + n * K;
            int32_t d = 0;
            for (int64_t k = 0; k < K; ++k) d += (int32_t)xr[k] * (int32_t)wr[k];
            exact = (double)d;
            a = (float)d;
        }
        float t = sqo_dequant(a, sx[m], sw[n], bias != 0, bias ? bias[n] : 0);
        if (acc_out) acc_out[i] = exact;
        if (y_f32) y_f32[i] = t;
        if (y_bf16) y_bf16[i] = sqo_f32_to_bf16_rne(t);
    }
}

/* ------------------------------------------------------------------------ */
/* Weight-only quantization, the comparison the pages draw for decode       */
/* ([WAQ] §1 table, W4A16 row: "INT4 -> dequant to FP16, then FP16 x FP16";  */
/* [ACT]: the runtime dequantizes the weights on the fly to multiply them    */
/* against the BF16 activations; [LES] §1 and §3: W8A16, 8-bit weights       */
/* de-quantized back to 16-bit and multiplied with 16-bit activations; the   */
/* zenaique page "W8A8 vs W4A16": W4A16 reads 4x fewer weight bytes, which   */
/* is what bandwidth-bound decode needs).                                   */
/*                                                                          */
/* Readings: the weights are quantized per output channel, symmetric, with  */
/* the same rule as the W8A8 weights (the pages' per-channel scaling), for  */
/* INT4 with Q = 7 (codes -7..7; group-wise scales belong to the AWQ / GPTQ  */
/* methods, which are not built). The dequantized weight is the real value  */
/* q[n][k] * sw[n]; the activations are bf16, used as they are (no          */
/* smoothing: no activation is quantized). The product is taken in binary64: */
/* y[m][n] = sum_k x[m][k] * (q[n][k] * sw[n]) + bias[n]. Every product is   */
/* exact in binary64 (8 x 8 x 24 significant bits); only the sum rounds, so  */
/* the result is within a few binary64 ulps of the real value.              */
/* ------------------------------------------------------------------------ */

/* INT4 code of v at scale `scale` (scale > 0): round-half-even of the binary32
 * quotient, clamped to +-7. */
static int8_t quant_i4(float v, float scale) {
    float c = nearbyintf(v / scale);
    if (c > 7.0f) c = 7.0f;
    if (c < -7.0f) c = -7.0f;
    return (int8_t)c;
}

/* The two's-complement nibble of a code in -8..7, and back. */
static uint8_t nibble_of(int8_t q) { return (uint8_t)q & 0x0Fu; }
static int8_t code_of_nibble(uint8_t nb) { return (int8_t)((nb & 0x08u) ? (int)nb - 16 : (int)nb); }

/* Packed INT4 layout (the pages fix none; this is the library's format): the
 * codes of k = 8g .. 8g+7 form the little-endian 32-bit word at byte 4g of
 * the row, code(8g + 2j) in bits 4j..4j+3 and code(8g + 2j + 1) in bits
 * 16+4j..16+4j+3, j = 0..3 (the even codes in the low half-word, the odd ones
 * in the high half-word). */
static int nibble_shift(int64_t k) { return (int)((k & 1) ? 16 + 4 * ((k & 7) >> 1) : 4 * ((k & 7) >> 1)); }

static int8_t unpack_code(const uint8_t* row, int64_t k) {
    const uint8_t* wb = row + 4 * (k / 8);
    uint32_t word = (uint32_t)wb[0] | ((uint32_t)wb[1] << 8) | ((uint32_t)wb[2] << 16) |
                    ((uint32_t)wb[3] << 24);
    return code_of_nibble((uint8_t)((word >> nibble_shift(k)) & 0x0Fu));
}

void sqo_quantize_weight_i4(const void* w, int dtype, int64_t K, int64_t N,
                            uint8_t* wq4, float* sw) {
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(load_elem(w, dtype, k * N + n));
            if (a > amax) amax = a;
        }
        float scale = amax / 7.0f;
        sw[n] = scale;
        uint8_t* row = wq4 + n * (K / 2);
        for (int64_t g = 0; g < K / 8; ++g) {
            uint32_t word = 0;
            for (int64_t k = 8 * g; k < 8 * g + 8; ++k) {
                int8_t q = (scale == 0.0f) ? 0 : quant_i4(load_elem(w, dtype, k * N + n), scale);
                word |= (uint32_t)nibble_of(q) << nibble_shift(k);
            }
            for (int b = 0; b < 4; ++b) row[4 * g + b] = (uint8_t)(word >> (8 * b));
        }
    }
}

void sqo_unpack_i4(const uint8_t* wq4, int64_t N, int64_t K, int8_t* codes) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) codes[n * K + k] = unpack_code(wq4 + n * (K / 2), k);
}

void sqo_gemm_weight_only(const uint16_t* x, const void* wq, int bits, const float* sw,
                          const uint16_t* bias, int64_t M, int64_t N, int64_t K,
                          double* y) {
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                int8_t q;
                if (bits == 4) {
                    q = unpack_code((const uint8_t*)wq + n * (K / 2), k);
                } else {
                    q = ((const int8_t*)wq)[n * K + k];
                }
                double w_deq = (double)q * (double)sw[n];
                acc += (double)sqo_bf16_to_f32(x[m * K + k]) * w_deq;
            }
            if (bias) acc += (double)sqo_bf16_to_f32(bias[n]);
            y[m * N + n] = acc;
        }
}
