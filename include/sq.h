/*
 * sq.h -- C ABI of libsq.so, the B200 (sm_100a) SmoothQuant W8A8 linear layer
 *
 *     Y = X W = (X diag(s)^-1) (diag(s) W)
 *
 * as described by "Weight-Activation Quantization" (infra.bea.ai), §3
 * "SmoothQuant: The Smoothing Trick" (equivalence, two-step pipeline,
 * "Choosing the Smoothing Factor") and §4 "FP8 W8A8 (Native on Hopper+)".
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Matrices are dense and row-major. X is [M,K] (M tokens, K input
 *    channels), W is [K,N] (N output channels), Y is [M,N]. Quantized weights
 *    are stored transposed as Wq [N,K] (K contiguous); quantized activations
 *    as Xq [M,K]. Both 8-bit operands are therefore "K-major".
 *  - Every pointer argument is a DEVICE pointer owned by the caller (the
 *    library never frees or keeps it). Large tensors (x, w, xq, wq, y, acc)
 *    and the per-channel vectors of the GEMMs (sw, bias) must be 16-byte
 *    aligned, as must s in sq_quantize_act; other vectors (s elsewhere, sx,
 *    amax) 4-byte aligned. Inputs and outputs must not alias.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream). Every call is asynchronous on that stream: argument checks run
 *    synchronously on the host and launch nothing when they fail; a failed
 *    launch returns SQ_ERR_CUDA. A device-side wait that gives up (see
 *    sq_get_device_status) is reported through the device status word.
 *    The many-row activation kernel and the GEMMs are launched with
 *    programmatic dependent launch: each may be scheduled while the kernel
 *    before it in the stream finishes, and waits for that kernel to
 *    complete before touching global memory, so stream order is kept
 *    (set the environment variable SQ_PDL=0 to launch them plainly).
 *  - K must be a positive multiple of 16 (16-byte rows of 8-bit data for the
 *    tensor-memory-accelerator copies); N a positive multiple of 8 (16-byte
 *    rows of bf16 output). M may be any value >= 0; M == 0 is a no-op that
 *    returns SQ_OK after the size checks (the M-sized pointers may then be
 *    NULL, as they are for empty torch tensors).
 *  - Floating-point arithmetic is IEEE binary32 with round-to-nearest-even
 *    and no contraction into fused multiply-adds, so results are
 *    reproducible bit for bit against a plain CPU implementation (see
 *    each function for the exact operation order).
 *  - The library allocates no device memory of its own except a 4-byte
 *    device status word, the 8-byte counter of sq_selftest_fast_division and
 *    the fixed scratch array of sq_gemm_w8a8_noalloc (module data). Scratch
 *    memory for the other GEMM calls is passed in by the caller (see
 *    sq_gemm_workspace_bytes).
 */
#ifndef SQ_H
#define SQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SQ_ABI_VERSION 8

/*
 * Flags of the activation passes (sq_quantize_act, sq_rmsnorm_quantize_act).
 *
 * SQ_OVERLAP_PREVIOUS: the caller guarantees that no kernel still running when
 * the pass starts writes x (and s, s_inv, g) or reads or writes xq, sx -- in
 * practice that the kernel issued just before it on the stream does not, e.g.
 * the previous batch's GEMM with xq / sx in a second buffer. The pass may then
 * run while that kernel finishes, in the SMs it leaves idle; it still
 * completes only after that kernel has completed, so everything issued after
 * the pass sees the same stream order as without the flag. This library's
 * GEMMs let the next kernel start only once their own inputs are complete, so
 * with one of them just before the pass, every kernel before that GEMM has
 * completed when the pass starts. Results are the same with or without the
 * flag; the library may ignore it (forms launched without programmatic
 * dependence always start after the previous kernel).
 */
#define SQ_OVERLAP_PREVIOUS 1u

typedef enum {
    SQ_OK = 0,
    SQ_ERR_INVALID_ARG = 1,  /* null pointer, bad size, bad alpha, bad enum   */
    SQ_ERR_MISALIGNED = 2,   /* pointer or leading dimension misaligned       */
    SQ_ERR_UNSUPPORTED = 3,  /* valid but not implemented combination         */
    SQ_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed           */
    SQ_ERR_TIMEOUT = 5,      /* a bounded device-side wait gave up             */
    SQ_ERR_SCRATCH_TOO_SMALL = 6  /* sq_gemm_w8a8_noalloc: fixed scratch too small */
} sq_status;

typedef enum {
    SQ_F32 = 0,   /* IEEE binary32                                           */
    SQ_BF16 = 1,  /* bfloat16 (raw 16-bit patterns)                          */
    SQ_I8 = 2,    /* signed 8-bit integer code                               */
    SQ_E4M3 = 3,  /* FP8 E4M3 code: bias 7, no infinity, max finite 448      */
    SQ_I32 = 4,   /* signed 32-bit integer                                   */
    SQ_I4 = 5     /* signed 4-bit code (-7..7), packed 8 per 32-bit word       */
} sq_dtype;

typedef enum {
    SQ_AMAX_PER_COLUMN = 0,  /* amax[c] = max_r |x[r,c]|  (reduce over rows)  */
    SQ_AMAX_PER_ROW = 1      /* amax[r] = max_c |x[r,c]|  (reduce over cols)  */
} sq_axis;

/* Human-readable name of a status code (static string, never NULL). */
const char* sq_status_string(sq_status st);

/* SQ_ABI_VERSION of the loaded library. */
int sq_abi_version(void);

/*
 * Synchronizes `stream`, then reads and clears the device status word.
 * Returns SQ_OK if no kernel reported a problem since the last call, or
 * SQ_ERR_TIMEOUT if a bounded wait inside a kernel gave up (the kernel then
 * skipped the rest of its work and released its tensor memory, so the
 * context stays usable but its outputs are undefined). SQ_ERR_CUDA if the
 * synchronization itself failed.
 */
sq_status sq_get_device_status(void* stream);

/*
 * a1 / a2 -- calibration amax.
 * Source: "Weight-Activation Quantization" §3 "Choosing the Smoothing
 * Factor" (max|X_j| and max|W_j|); the zenaique flashcard "Define activation
 * quantization ..." (calibration on a small held-out corpus).
 *   x      : [rows, cols] row-major, dtype xt (SQ_F32 or SQ_BF16)
 *   axis   : SQ_AMAX_PER_COLUMN -> amax has `cols` entries (calibration of
 *            activations: one value per input channel over the tokens);
 *            SQ_AMAX_PER_ROW    -> amax has `rows` entries (weights W [K,N]:
 *            one value per input channel over the output channels).
 *   accumulate : 0 -> amax is overwritten; 1 -> amax = max(amax, new), so a
 *            calibration corpus can be streamed batch by batch.
 *   cols must be a multiple of 8; rows >= 1.
 */
sq_status sq_calibrate_amax(const void* x, sq_dtype xt, int64_t rows,
                            int64_t cols, sq_axis axis, float* amax,
                            int accumulate, void* stream);

/*
 * a3 -- smoothing factors, "Choosing the Smoothing Factor":
 *   s[k] = max(amax_x[k], 1e-5)^alpha / max(amax_w[k], 1e-5)^(1-alpha)
 * evaluated in binary64 and rounded once to binary32. 0 <= alpha <= 1
 * (SQ_ERR_INVALID_ARG otherwise). K >= 1.
 *   s_inv : [K] or NULL. When given, also receives the reciprocals the
 *           runtime kernel uses to divide by s quickly ("X_tilde = X @
 *           diag(1/s)", §3 Step 1): s_inv[k] = RN(1/s[k]) when
 *           2^-20 <= s[k] <= 2^20, NaN otherwise (NaN sends that channel to
 *           the exact division path). Pass it to sq_quantize_act/sq_linear.
 */
sq_status sq_smooth_factors(const float* amax_x, const float* amax_w,
                            int64_t K, double alpha, float* s, float* s_inv,
                            void* stream);

/*
 * a4 -- offline weight smoothing and per-output-channel quantization.
 * Source: §3 "Step 1" (W_tilde = diag(s) W) and "Step 2" (W_int8 =
 * quantize(W_tilde)); §4 "Per-Tensor Scaling for FP8" for qt = SQ_E4M3.
 *   w  : [K,N] row-major, dtype wt (SQ_F32 or SQ_BF16)
 *   s  : [K] smoothing factors, or NULL for no smoothing
 *   qt : SQ_I8, SQ_E4M3 or SQ_I4 (below)
 *   wq : [N,K] output codes (transposed, K contiguous)
 *   sw : [N] output scales
 * For each n: wt[k] = s[k]*w[k,n]; sw[n] = max_k|wt[k]| / Q (Q = 127 for
 * INT8, 448 for E4M3); wq[n,k] = clamp(rne(wt[k]/sw[n]), -127, 127) for INT8,
 * or the E4M3 code of wt[k]/sw[n] (nearest-even, saturating to +-448). A
 * column with sw[n] == 0 gets all-zero codes.
 * qt = SQ_I4 (weight-only W4A16, see sq_gemm_weight_only): s must be NULL
 * (SQ_ERR_UNSUPPORTED otherwise) and K a multiple of 32; sw[n] = max_k|w[k,n]|
 * / 7, codes clamp(rne(w[k,n]/sw[n]), -7, 7), stored packed as wq [N, K/2]
 * bytes: the codes of k = 8g .. 8g+7 form the little-endian 32-bit word at
 * byte 4g of row n, code(8g+2j) in bits 4j..4j+3 and code(8g+2j+1) in bits
 * 16+4j..16+4j+3 (two's-complement nibbles; the pages fix no packing, and
 * this one lets the GEMM widen two codes with two masks and one subtraction).
 */
sq_status sq_quantize_weight(const void* w, sq_dtype wt, int64_t K, int64_t N,
                             const float* s, sq_dtype qt, void* wq, float* sw,
                             void* stream);

/*
 * a5 -- fused runtime activation smoothing + per-token quantization (one
 * kernel, one read of X). Source: §3 "divide each activation channel by
 * s_j" and "Step 2" (X_int8 = quantize(X_tilde) at inference time); §2
 * scale = max|x|/127; §4 q = cast_fp8(x/s) with s = max|x|/448.
 *   x  : [M,K] row-major, SQ_F32 or SQ_BF16
 *   s  : [K] smoothing factors, or NULL for no smoothing
 *   qt : SQ_I8 or SQ_E4M3
 *   xq : [M,K] output codes; sx : [M] output per-token scales
 * For each row m: xs[k] = x[m,k] / s[k] (IEEE division); sx[m] =
 * max_k|xs[k]| / Q; codes as in sq_quantize_weight with xs and sx[m].
 * Rows with sx[m] == 0 get all-zero codes. K <= 65536.
 *   s_inv : [K] or NULL (16-byte aligned) -- the reciprocals written by
 *           sq_smooth_factors for this s. They only speed the kernel up: the
 *           result is the IEEE quotient x/s either way (bf16 input divides
 *           by a reciprocal product with one exact correction step and falls
 *           back to the IEEE division wherever that is not provably exact).
 *           Results are undefined if s_inv does not come from s.
 *   flags : 0 or SQ_OVERLAP_PREVIOUS (other bits: SQ_ERR_INVALID_ARG)
 */
sq_status sq_quantize_act(const void* x, sq_dtype xt, int64_t M, int64_t K,
                          const float* s, const float* s_inv, sq_dtype qt,
                          void* xq, float* sx, uint32_t flags, void* stream);

/*
 * Activation smoothing + PER-TENSOR quantization: one scale for the whole
 * smoothed tensor instead of one per token. Source: "Weight-Activation
 * Quantization" (infra.bea.ai) §4 "Per-Tensor Scaling for FP8" (q =
 * cast_fp8(x/s), s = max|x|/448) and its comparison table (per-tensor scaling
 * online; "delayed scaling uses previous step's max"). The pages have no API
 * for it; this entry point is this library's.
 *   x, xt, M, K, s, s_inv, qt, xq : as sq_quantize_act.
 *   amax_prev : device float[1] holding the previous step's max|x/s|
 *               (delayed scaling, one pass over x), or NULL for the online
 *               scale of this tensor (two passes: its max, then the codes).
 *               The scale is RN(amax / Q), Q = 127 (INT8) or 448 (E4M3).
 *   sx        : [M], every entry receives the scale used, so the GEMMs take
 *               it as they take per-token scales.
 *   amax_out  : device float[1], required, 4-byte aligned, not aliasing
 *               amax_prev: receives max|x/s| of this tensor (NaN ignored) --
 *               the next step's amax_prev. M == 0 sets it to 0.
 * Codes: INT8 clamp(rne(xs / scale), -127, 127), E4M3 round-to-nearest-even
 * saturating to +-448 (values beyond a delayed scale saturate); a zero scale
 * gives all-zero codes. Bit-exact against the IEEE definitions.
 */
sq_status sq_quantize_act_tensor(const void* x, sq_dtype xt, int64_t M, int64_t K,
                                 const float* s, const float* s_inv, sq_dtype qt,
                                 const float* amax_prev, void* xq, float* sx,
                                 float* amax_out, void* stream);

/*
 * Offline fold of the activation smoothing into the layer that produces X.
 * Source: "Weight-Activation Quantization" (infra.bea.ai) §3, the two-step
 * pipeline (X_tilde = X diag(1/s) is part of offline model preparation), and
 * the grasp.study lesson on W8A16 vs W8A8, §2 (the transform happens offline,
 * with no runtime overhead). The pages name no producer; this library takes
 * it to carry one parameter, or one row or column of a weight, per channel k
 * of X (a normalization's gain, a preceding linear layer's weight and bias).
 * Dividing those by s_k once makes the producer emit X_tilde, and this
 * layer's activations are then quantized with s = NULL.
 *   p    : [rows, cols] row-major, SQ_F32 or SQ_BF16, aligned to its element
 *   s    : the smoothing factors (sq_smooth_factors), one per channel
 *   axis : SQ_AMAX_PER_COLUMN -> channel = column: out[r,c] = p[r,c] / s[c]
 *          (s has `cols` entries; a gain vector as [1,K], or a producer
 *          weight [R,K] in this library's [in,out] layout);
 *          SQ_AMAX_PER_ROW    -> channel = row: out[r,c] = p[r,c] / s[r]
 *          (s has `rows` entries; a producer weight stored [K,R]).
 *   out  : [rows, cols] binary32, not aliasing p (SQ_ERR_INVALID_ARG if
 *          out == p).
 * Each element is one IEEE binary32 division, the operation the runtime
 * kernels apply to x, so the result is bit-exact against it. rows or cols
 * == 0 is a no-op.
 */
sq_status sq_fold_smoothing(const void* p, sq_dtype pt, int64_t rows, int64_t cols,
                            const float* s, sq_axis axis, float* out, void* stream);

/*
 * The producer of X with the smoothing folded in: RMS normalization fused with
 * per-token quantization. Source: "Weight-Activation Quantization"
 * (infra.bea.ai) §3 "Step 1" (X_tilde = X diag(1/s) prepared before
 * inference) and the grasp.study lesson on W8A16 vs W8A8, §2 (the transform
 * is applied offline, with no runtime overhead). The pages name no producer
 * of X; the models they quantize feed each linear layer from an RMS
 * normalization with a per-channel gain, and g = gamma / s (from
 * sq_fold_smoothing) makes it emit X_tilde itself, so this call replaces the
 * normalization and sq_quantize_act(.., s = NULL, ..) with one pass.
 *   x   : [M,K] bf16, the normalization's input (16-byte aligned)
 *   g   : [K] binary32 gain with 1/s folded in (16-byte aligned)
 *   eps : > 0, finite
 *   qt  : SQ_I8 or SQ_E4M3;  xq : [M,K] codes (16-byte aligned);  sx : [M]
 *   xn  : [M,K] binary32 or NULL (16-byte aligned): when given, the
 *         normalization's output xn below is written too, for the offline
 *         calibration of the smoothing factors (run it with g = gamma)
 *   flags : 0 or SQ_OVERLAP_PREVIOUS (other bits: SQ_ERR_INVALID_ARG)
 * Per row: ss = the sum of x_k^2 over the k whose bf16 exponent is within 48
 * of the row's largest, exactly, rounded once to binary64 (the others are
 * below 2^-94 of the largest square); r = binary32(1 / sqrt(ss / K + eps))
 * with each of the four binary64 operations rounded once; xn_k = (x_k * r) *
 * g_k in binary32; then sx and the codes of xn exactly as sq_quantize_act
 * with s = NULL. K a multiple of 8, at most 16384 (SQ_ERR_UNSUPPORTED
 * beyond). xq, sx and xn may overlap neither each other nor x or g
 * (SQ_ERR_INVALID_ARG). M == 0 is a no-op that accepts NULL pointers.
 * The kernels reach the r of the exact sum by a binary64 sum of the squares
 * (each square exact, the sum within 2^-36 of the exact one) whenever both
 * ends of that interval give the same binary32 r, and by the exact integer
 * sum otherwise; setting SQ_NORM_EXACT_SUM=1 in the environment takes the
 * exact sum for every row. Results are the same either way.
 */
sq_status sq_rmsnorm_quantize_act(const void* x, const float* g, float eps, int64_t M,
                                  int64_t K, sq_dtype qt, void* xq, float* sx, float* xn,
                                  uint32_t flags, void* stream);

/*
 * Size in bytes of the GEMM workspace for the current device (its SM count
 * sets the size; the same workspace serves calls of every shape). The
 * workspace lets the last, partial wave of output tiles be split along K
 * across all SMs ("stream-K"): SMs that finish part of a tile leave its raw
 * partial accumulators there, and the SM that owns the tile adds them (in a
 * fixed order; exact for INT8) before the epilogue. Contract: 256-byte
 * aligned, zero-filled by the caller before its first use (the GEMMs leave
 * it zeroed again), not shared by GEMMs that may run concurrently, and
 * re-zeroed by the caller after a call reported SQ_ERR_TIMEOUT. Passing NULL
 * (or fewer bytes) is always valid and only disables the split.
 */
size_t sq_gemm_workspace_bytes(void);

/*
 * a6 -- INT8 x INT8 tensor-core GEMM with int32 accumulation and a fused
 * dequantization epilogue. Source: §3 "Step 2" (Y = dequantize(X_int8 @
 * W_int8), "INT8 Tensor Core GEMM"); §1 table (INT8 x INT8 row).
 *   xq : [M,K] int8, sx : [M];  wq : [N,K] int8, sw : [N]
 *   bias : [N] bf16 or NULL
 *   y  : [M,N], yt = SQ_BF16 or SQ_F32
 *   acc: [M,N] int32 accumulators or NULL (written when non-NULL)
 *   workspace, workspace_bytes: see sq_gemm_workspace_bytes (NULL, 0 allowed)
 * acc[m,n] = sum_k xq[m,k]*wq[n,k] (exact in int32 for K < 133144);
 * t = float(acc) (nearest-even); t = t*sx[m]; t = t*sw[n]; t = t + bias[n];
 * y = t (SQ_F32) or bf16(t) rounded to nearest-even (SQ_BF16).
 * Kernels: M <= 16 runs a weight-streaming kernel (the weight rows are the
 * 128-row tensor-core operand, the tokens a 16-column one; no workspace),
 * every other M the tiled kernel. Results are the same either way. Setting
 * SQ_GEMM_NO_SKINNY or SQ_GEMM_TILE in the environment keeps the tiled
 * kernel for every M.
 */
sq_status sq_gemm_w8a8(const int8_t* xq, const float* sx, const int8_t* wq,
                       const float* sw, const uint16_t* bias, int64_t M,
                       int64_t N, int64_t K, void* y, sq_dtype yt,
                       int32_t* acc, void* workspace, size_t workspace_bytes,
                       void* stream);

/*
 * a7 -- FP8 E4M3 x E4M3 tensor-core GEMM, binary32 accumulation in tensor
 * memory, same epilogue. Source: §4 "FP8 W8A8 (Native on Hopper+)"; §1
 * table (FP8 x FP8 row). xq / wq hold E4M3 codes; other arguments as in
 * sq_gemm_w8a8. The tensor cores' summation order is not specified, so the
 * result differs from an exact sum by accumulated binary32 rounding.
 */
sq_status sq_gemm_fp8(const uint8_t* xq, const float* sx, const uint8_t* wq,
                      const float* sw, const uint16_t* bias, int64_t M,
                      int64_t N, int64_t K, void* y, sq_dtype yt,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * Weight-only quantized linear layer for few tokens (decode): W8A16 and
 * W4A16, the schemes the pages set against W8A8. Source: "Weight-Activation
 * Quantization" (infra.bea.ai) §1 table (W4A16: INT4 weights dequantized,
 * then a 16-bit multiply); the zenaique flashcard on activation quantization
 * (the weights are dequantized on the fly to multiply the BF16
 * activations); the grasp.study lesson on W8A16 vs W8A8, §1 and §3; the
 * zenaique page "W8A8 vs W4A16" (decode is bound by the weight read; 4-bit
 * weights halve it again).
 *   x   : [M,K] bf16 activations (not quantized, not smoothed)
 *   wq  : per-output-channel weight codes from sq_quantize_weight with s =
 *         NULL: wqt = SQ_I8 -> int8 [N,K]; wqt = SQ_I4 -> packed [N,K/2] (the
 *         layout sq_quantize_weight documents)
 *   sw  : [N] channel scales (4-byte aligned); bias : [N] bf16 or NULL
 *   y   : [M,N], yt = SQ_BF16 or SQ_F32
 * y[m,n] = bf16( RN(sum_k x[m,k] * q[n,k]) * sw[n] + bias[n] ): the codes are
 * widened exactly to bf16 and multiplied by x on the tensor cores with
 * binary32 accumulation (order unspecified); the channel scale multiplies
 * the sum, then the bias is added, each step rounded in binary32. The result
 * differs from the exact sum_k x * (q * sw) only by that accumulation.
 * K must be a multiple of 16 (SQ_I8) or 32 (SQ_I4); N a multiple of 8. Built
 * for M <= 16 (one pass over the weights); larger M runs one pass per 16
 * tokens.
 */
sq_status sq_gemm_weight_only(const void* x, const void* wq, sq_dtype wqt, const float* sw,
                              const uint16_t* bias, int64_t M, int64_t N, int64_t K, void* y,
                              sq_dtype yt, void* stream);

/*
 * Runtime forward of one SmoothQuant linear layer: sq_quantize_act followed
 * by sq_gemm_w8a8 (qt = SQ_I8) or sq_gemm_fp8 (qt = SQ_E4M3) on the same
 * stream. xq_buf [M,K] (8-bit codes) and sx_buf [M] are caller-owned
 * buffers that receive the quantized activations; s_inv as in
 * sq_quantize_act.
 */
sq_status sq_linear(const void* x, sq_dtype xt, const float* s,
                    const float* s_inv, const void* wq, const float* sw, const uint16_t* bias,
                    sq_dtype qt, int64_t M, int64_t N, int64_t K,
                    void* xq_buf, float* sx_buf, void* y, sq_dtype yt,
                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * Allocation-free variant of sq_gemm_w8a8 (no counterpart in the pages: it
 * exists for callers, not for the method). Some callers cannot allocate
 * device memory while they run -- for example an inference runtime that
 * reserves all device memory up front for its own pool, so a foreign
 * cudaMalloc would fail or fragment it, or latency-critical code that cannot
 * afford the device-wide synchronization cudaMalloc / cudaFree may imply --
 * and so cannot provide the workspace the split-tile GEMM needs. This entry
 * point takes the same inputs and outputs as sq_gemm_w8a8 (without acc and
 * without a workspace) and uses a fixed array inside the library's device
 * image as its scratch instead: 20 MiB + 4 KiB, the split-tile workspace of
 * a GPU with up to 160 SMs. It calls no cudaMalloc / cudaFree or other
 * allocating routine.
 *  - Limit: the scratch this call needs (see sq_gemm_workspace_bytes; it
 *    depends on the GPU's SM count, not on M, N, K) must fit the array, so
 *    GPUs with more than 160 SMs get SQ_ERR_SCRATCH_TOO_SMALL and nothing is
 *    launched. Every GPU that loads the library holds the array until the
 *    process exits.
 *  - Set-up: the first call on each device looks up the array's device
 *    address (cudaGetSymbolAddress) with that device current and caches it;
 *    make that first call before any stream capture. The cached address is
 *    not valid after cudaDeviceReset: do not call this entry point on a
 *    device after resetting it.
 *  - Every call shares the one array, which keeps the last call's contents;
 *    each call first clears the part that must start at zero (an async
 *    memset on `stream`). Calls that overlap on the GPU (different streams,
 *    or the same device from several host threads without ordering) race on
 *    the array and may produce wrong results.
 * Results are identical to sq_gemm_w8a8 with a workspace (INT8 sums exact).
 */
sq_status sq_gemm_w8a8_noalloc(const int8_t* xq, const float* sx,
                               const int8_t* wq, const float* sw,
                               const uint16_t* bias, int64_t M, int64_t N,
                               int64_t K, void* y, sq_dtype yt, void* stream);

/*
 * Self-test of the division shortcuts used by sq_quantize_act for bf16 input
 * (an IEEE division computed as a reciprocal product corrected with one
 * fused multiply-add residual, after Markstein): runs every bf16 significand
 * of x against every binary32 significand of s_k (2^30 pairs, both signs),
 * every binary32 significand of a row maximum divided by 127 and by 448 with
 * their constant reciprocals, and checks that the refined approximate
 * reciprocal of every binary32 significand is within one unit in the last
 * place of the IEEE reciprocal. Synchronous (waits for `stream`).
 * *mismatches receives the number of failures; 0 means the shortcuts are
 * exact (or, for the reciprocal, within its bound) wherever sq_quantize_act
 * uses them.
 */
sq_status sq_selftest_fast_division(int64_t* mismatches, void* stream);

/*
 * Diagnostic: launches one block whose single thread waits on a shared-memory
 * barrier that nothing ever completes, through the same bounded wait the GEMM
 * kernels use, with a limit of `timeout_ns` nanoseconds (1e6 .. 1e10). The
 * wait gives up, the kernel records SQ_ERR_TIMEOUT in the device status word
 * and returns; sq_get_device_status then reports it. Used to test the
 * failure path without faulting or hanging the GPU.
 */
sq_status sq_probe_wait_timeout(int64_t timeout_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SQ_H */
