// sq_norm.cu -- the producer of X with the smoothing folded in: RMS
// normalization fused with per-token quantization, so that the layer's
// activation pass reads the normalization's input once and writes only the
// 8-bit codes.
//
// "Weight-Activation Quantization" (infra.bea.ai) §3 "Step 1" (X_tilde =
// X diag(1/s) is prepared before inference) and the grasp.study lesson on
// W8A16 vs W8A8, §2 (the transform is applied offline, with no runtime
// overhead). The pages name no producer of X; the transformer models they
// quantize (Llama) feed each linear layer from an RMS normalization with a
// per-channel gain gamma, and g = gamma / s (sq_fold_smoothing) makes that
// normalization emit X_tilde itself. Per row of x (bf16, K elements):
//   ss   = sum of x_k^2 over the k whose bf16 exponent is within 48 of the
//          row's largest, exactly (every such square is an integer multiple
//          of 2^(2 e_max - 110), and the sum fits 128 bits), then rounded once
//          to binary64 (the others are below 2^-94 of the largest square);
//   r    = binary32( 1 / sqrt( ss / K + eps ) ), the division by K, the
//          addition, the square root and the reciprocal each an IEEE binary64
//          operation;
//   xn_k = (x_k * r) * g_k, two binary32 products;
//   then the per-token quantization of xn (no smoothing): sx = max|xn| / Q,
//   codes of xn / sx (INT8: round-half-even, clamped to +-127; E4M3:
//   round-to-nearest-even, saturating), all-zero codes where sx is 0.
// xn itself is written too when asked for (binary32; the calibration of the
// smoothing factors runs on it offline).
//
// Three kernels give the same results bit for bit:
//  * rmsnorm_quant_kernel, the plain form (and the only one that also writes
//    xn): one CTA per row, the row staged in shared memory, four passes over
//    it (the largest exponent, the exact sum of squares, the largest |xn|,
//    the codes) with IEEE divisions, each closed by a block reduction;
//  * rmsnorm_quant_warp_kernel, for many rows of at most 8192 elements: one
//    warp per row, with its own row slot and barrier, no block barrier on a
//    row's path;
//  * rmsnorm_quant_stream_kernel, for the other shapes: persistent CTAs with
//    the next rows in flight (bulk copies into a shared-memory ring), each
//    thread's part of the row in registers, three block barriers per row.
// The last two sum the squares in binary64 (each square exact there) and
// check that both ends of an interval around that sum, far wider than its
// rounding error, give the same binary32 r -- then it is the r of the exact
// sum; the rows where they do not take the exact integer sum. They work on
// packed binary32 pairs and use no division instruction on rows whose
// largest |xn| is in [2^-60, 2^100].
// HBM-bound in principle: 2 bytes read and 1 written per element.
#include <cstdint>
#include <cstdlib>
#include <cuda_runtime.h>

#include "sq_common.cuh"
#include "sq_internal.h"

namespace sqk {

constexpr int kNormThreads = 256;
constexpr int kNormMaxK = 16384;  // the staged row: at most 32 KB of shared memory

struct U128 {
  uint64_t lo, hi;
};

__device__ __forceinline__ void u128_add(U128& a, uint64_t lo, uint64_t hi) {
  const uint64_t s = a.lo + lo;
  a.hi += hi + (s < lo ? 1u : 0u);
  a.lo = s;
}

// bf16 magnitude bits h != 0 as N * 2^(e - 7): N = 1.f in 8 bits for normal
// numbers (128..255), 0.f for subnormals (1..127).
__device__ __forceinline__ void bf16_int_exp(uint32_t h, uint32_t& n, int& e) {
  const int be = int(h >> 7) & 0xFF;
  const uint32_t f = h & 0x7Fu;
  n = be ? 128u + f : f;
  e = be ? be - 127 : -126;
}

// The exact 128-bit integer S rounded once to binary64, times 2^shift
// (shift keeps the result in the normal range here).
__device__ __forceinline__ double u128_to_double_scaled(U128 s, int shift) {
  if (s.hi == 0) return __dmul_rn(__ull2double_rn(s.lo), __longlong_as_double(int64_t(1023 + shift) << 52));
  const int lz = __clzll(int64_t(s.hi));
  // the top 64 bits, with every bit below them folded into the last one: the
  // nearest binary64 of the 64-bit value is then that of the 128-bit value
  uint64_t top = lz ? (s.hi << lz) | (s.lo >> (64 - lz)) : s.hi;
  const uint64_t rest = s.lo << lz;
  if (rest != 0) top |= 1u;
  const int sh = shift + 64 - lz;
  return __dmul_rn(__ull2double_rn(top), __longlong_as_double(int64_t(1023 + sh) << 52));
}

template <bool E4M3>
__global__ void __launch_bounds__(kNormThreads)
    rmsnorm_quant_kernel(const uint16_t* __restrict__ x, const float* __restrict__ g,
                         float eps, int64_t M, int K, uint8_t* __restrict__ xq,
                         float* __restrict__ sx, float* __restrict__ xn, int late_wait) {
  extern __shared__ __align__(16) uint16_t row[];  // K entries
  __shared__ int red_i[kNormThreads / 32];
  __shared__ unsigned long long red_lo[kNormThreads / 32], red_hi[kNormThreads / 32];
  __shared__ float red_f[kNormThreads / 32];
  __shared__ float bcast[2];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int W = kNormThreads / 32;
  const int nchunk = K >> 3;
  // the row may come from the kernel before this one, unless the caller has
  // ruled that out (late_wait: then this grid only completes after it)
  pdl_launch_dependents();
  if (!late_wait) pdl_wait();
#pragma unroll 1
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    const uint16_t* xr = x + m * K;
    // pass 1: stage the row, the largest bf16 exponent of its nonzero entries
    int emax = -1000;
    for (int c = threadIdx.x; c < nchunk; c += kNormThreads) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(xr) + c);
      reinterpret_cast<uint4*>(row)[c] = u;
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const uint32_t h = (w[i] >> (16 * h2)) & 0x7FFFu;
          if (h != 0) {
            uint32_t n;
            int e;
            bf16_int_exp(h, n, e);
            emax = max(emax, e);
          }
        }
      }
    }
    emax = __reduce_max_sync(0xFFFFFFFFu, emax);
    if (lane == 0) red_i[warp] = emax;
    __syncthreads();
    emax = red_i[0];
#pragma unroll
    for (int i = 1; i < W; ++i) emax = max(emax, red_i[i]);
    // pass 2: the exact sum of squares, in units of 2^(2 e_max - 110)
    U128 acc = {0, 0};
    if (emax > -1000) {
      for (int c = threadIdx.x; c < nchunk; c += kNormThreads) {
        const uint4 u = reinterpret_cast<const uint4*>(row)[c];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const uint32_t h = (w[i] >> (16 * h2)) & 0x7FFFu;
            if (h == 0) continue;
            uint32_t n;
            int e;
            bf16_int_exp(h, n, e);
            if (e < emax - 48) continue;
            const uint64_t v = uint64_t(n * n);          // < 2^16
            const int sh = 2 * (e - emax) + 96;         // 0 .. 96
            if (sh < 64) u128_add(acc, v << sh, sh ? v >> (64 - sh) : 0);
            else u128_add(acc, 0, v << (sh - 64));
          }
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const uint64_t lo = __shfl_down_sync(0xFFFFFFFFu, acc.lo, off);
      const uint64_t hi = __shfl_down_sync(0xFFFFFFFFu, acc.hi, off);
      u128_add(acc, lo, hi);
    }
    if (lane == 0) {
      red_lo[warp] = acc.lo;
      red_hi[warp] = acc.hi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      U128 s = {0, 0};
      for (int i = 0; i < W; ++i) u128_add(s, red_lo[i], red_hi[i]);
      const double ss = emax > -1000 ? u128_to_double_scaled(s, 2 * emax - 110) : 0.0;
      const double mean = __ddiv_rn(ss, double(K));
      const double v = __dadd_rn(mean, double(eps));
      const double t = __dsqrt_rn(v);
      bcast[0] = __double2float_rn(__ddiv_rn(1.0, t));
    }
    __syncthreads();
    const float r = bcast[0];
    // pass 3: xn = (x * r) * g, the row's largest |xn|
    float amax = 0.0f;
    for (int c = threadIdx.x; c < nchunk; c += kNormThreads) {
      const uint4 u = reinterpret_cast<const uint4*>(row)[c];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      const float4 g0 = __ldg(reinterpret_cast<const float4*>(g) + 2 * c);
      const float4 g1 = __ldg(reinterpret_cast<const float4*>(g) + 2 * c + 1);
      const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      float y[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float xv = (i & 1) ? bf16_hi(w[i >> 1]) : bf16_lo(w[i >> 1]);
        y[i] = __fmul_rn(__fmul_rn(xv, r), gv[i]);
        amax = fmaxf(amax, fabsf(y[i]));
      }
      if (xn) {  // the normalization's output itself (offline calibration)
        float4* o = reinterpret_cast<float4*>(xn + m * K) + 2 * c;
        o[0] = make_float4(y[0], y[1], y[2], y[3]);
        o[1] = make_float4(y[4], y[5], y[6], y[7]);
      }
    }
    amax = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(amax)));
    if (lane == 0) red_f[warp] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
      float a = red_f[0];
      for (int i = 1; i < W; ++i) a = fmaxf(a, red_f[i]);
      const float scale = __fdiv_rn(a, E4M3 ? 448.0f : 127.0f);
      bcast[1] = scale;
      sx[m] = scale;
    }
    __syncthreads();
    const float scale = bcast[1];
    // pass 4: the codes
    for (int c = threadIdx.x; c < nchunk; c += kNormThreads) {
      const uint4 u = reinterpret_cast<const uint4*>(row)[c];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      const float4 g0 = __ldg(reinterpret_cast<const float4*>(g) + 2 * c);
      const float4 g1 = __ldg(reinterpret_cast<const float4*>(g) + 2 * c + 1);
      const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      float q[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float xv = (i & 1) ? bf16_hi(w[i >> 1]) : bf16_lo(w[i >> 1]);
        const float y = __fmul_rn(__fmul_rn(xv, r), gv[i]);
        q[i] = scale == 0.0f ? 0.0f : __fdiv_rn(y, scale);
      }
      uint2 o;
      if constexpr (E4M3) {
        o.x = pack_e4m3x2(q[0], q[1]) | (pack_e4m3x2(q[2], q[3]) << 16);
        o.y = pack_e4m3x2(q[4], q[5]) | (pack_e4m3x2(q[6], q[7]) << 16);
        if (scale == 0.0f) o = make_uint2(0u, 0u);
      } else {
        uint32_t b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int v = max(-127, min(127, __float2int_rn(q[i])));
          b[i] = uint32_t(v) & 0xFFu;
        }
        o.x = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
        o.y = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
      }
      reinterpret_cast<uint2*>(xq + m * K)[c] = o;
    }
    // the staged row and the reduction slots are reused by the next row
    __syncthreads();
  }
  if (late_wait) pdl_wait();
}

// ----------------------------------------------------------------------------
// The streaming form. Per row, with every thread holding its V 8-element
// chunks c = threadIdx.x + j * blockDim.x of the row (bf16):
//  1. the largest magnitude bit pattern (bf16 magnitudes order like their
//     15-bit patterns, so its exponent field is e_max's) -- barrier 1, after
//     which thread 0 refills the ring slot with the row SLOTS ahead;
//  2. the exact sum of squares in three parts: the squares of normal
//     elements within 16 binades of the largest (band A) and those 17 to 32
//     binades below it (band B) as a^2 with a = n * 2^(e - e_max + 16) < 2^24
//     (band B: n * 2^(e - e_max + 32) < 2^23), one 32 x 32 -> 64-bit
//     multiply-add each, in two 64-bit sums (units 2^(2 e_max - 46) and
//     2^(2 e_max - 78); at most 2^14 terms, so no overflow); the rest
//     (smaller, subnormal; rare) go to a 128-bit shared accumulator in units
//     of 2^(2 e_max - 110) by 64-bit shared atomics (the carry of the low
//     word added to the high one) -- barrier 2; every warp then combines the
//     three (2^64 and 2^32 apart) and takes r in the same binary64 steps as
//     the plain form;
//  3. y = (x * r) * g in packed pairs, kept in registers, and their largest
//     magnitude -- barrier 3;
//  4. sx = RN(amax / Q) and the codes of RN(y / sx): for amax in
//     [2^-60, 2^100] without a division instruction -- the scale by the
//     exact constant-divisor correction, the quotients by two corrections of
//     the reciprocal product (P. Markstein, "IA-64 and Elementary Functions",
//     2000), the INT8 code as the low byte of RN(q + 1.5 * 2^23), the E4M3
//     code by cvt.rn.satfinite with the sign bit of y (quotients too small
//     for an E4M3 subnormal keep their exact quotient's sign); other rows
//     (all zeros, extreme magnitudes) by IEEE divisions, as the plain form.
// The inputs must be finite (Inf and NaN give unspecified codes).
// ----------------------------------------------------------------------------

// Per-halfword unsigned max / min of two packed pairs.
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t min_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// RN(a / Q) for Q = 127 or 448, exact for every a whose quotient and
// residual stay normal: q0 = RN(a c) with c = RN(1/Q), one correction from
// the exact residual a - Q q0.
template <bool E4M3>
__device__ __forceinline__ float norm_div_by_qmax(float a) {
  constexpr float kQ = E4M3 ? 448.0f : 127.0f;
  constexpr float kC = 1.0f / kQ;
  const float q0 = __fmul_rn(a, kC);
  return __fmaf_rn(__fmaf_rn(-kQ, q0, a), kC, q0);
}

// One square of a bf16 magnitude h != 0 outside the fast band, added to the
// 128-bit accumulator in units of 2^(2 e_max - 110) (dropped below e_max - 48).
__device__ __forceinline__ void norm_slow_square(uint32_t h, int emax, U128& acc) {
  uint32_t n;
  int e;
  bf16_int_exp(h, n, e);
  if (e < emax - 48) return;
  const uint64_t v = uint64_t(n * n);
  const int sh = 2 * (e - emax) + 96;
  if (sh < 64) u128_add(acc, v << sh, sh ? v >> (64 - sh) : 0);
  else u128_add(acc, 0, v << (sh - 64));
}

// The two bands' sums of squares of one 8-element chunk (bf16 pairs in u),
// sh0 = 16 - efmax as an unsigned offset. Band A: the shift e - e_max + 16
// in [0, 16], clamped at 32 (a = 0) below the band, negative offsets
// included; band B: 16 more, kept only when below 16 (one unsigned comparison
// excludes both band A and everything below band B).
__device__ __forceinline__ void norm_band_squares(const uint4& u, uint32_t sh0, uint64_t& accA,
                                                  uint64_t& accB) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t h = (i & 1) ? (w[i >> 1] >> 16) : (w[i >> 1] & 0xFFFFu);
    const uint32_t n = 0x80u | (h & 0x7Fu);
    const uint32_t shA = ((h >> 7) & 0xFFu) + sh0;
    const uint32_t shB = shA + 16u;
    const uint32_t aA = __funnelshift_lc(0u, n, shA);
    const uint32_t aB = shB < 16u ? n << shB : 0u;
    accA += uint64_t(aA) * aA;
    accB += uint64_t(aB) * aB;
  }
}

// The squares of one chunk's elements below both bands (nonzero, exponent
// field < lo_ef) into the 128-bit remainder.
__device__ __forceinline__ void norm_slow_chunk(const uint4& u, int lo_ef, int emax, U128& acc) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t h = ((i & 1) ? (w[i >> 1] >> 16) : w[i >> 1]) & 0x7FFFu;
    if (h != 0u && int(h >> 7) < lo_ef) norm_slow_square(h, emax, acc);
  }
}

// binary32(1 / sqrt(ss / K + eps)) with each binary64 step rounded once (the
// chain the oracle takes from its exact sum, here from a given binary64 ss).
__device__ __forceinline__ float norm_chain(double ss, int K, float eps) {
  const double mean = __ddiv_rn(ss, double(K));
  const double t = __dsqrt_rn(__dadd_rn(mean, double(eps)));
  return __double2float_rn(__ddiv_rn(1.0, t));
}

// r = binary32(1 / sqrt(ss / K + eps)) from the exact sum: the remainder in
// units of 2^(2 e_max - 110), band A's sum 2^64 and band B's 2^32 of them.
__device__ __forceinline__ float norm_rinv(U128 rest, uint64_t totA, uint64_t totB, uint32_t hmax,
                                           int emax, int K, float eps) {
  u128_add(rest, totB << 32, (totB >> 32) + totA);
  const double ss = hmax ? u128_to_double_scaled(rest, 2 * emax - 110) : 0.0;
  const double mean = __ddiv_rn(ss, double(K));
  const double t = __dsqrt_rn(__dadd_rn(mean, double(eps)));
  return __double2float_rn(__ddiv_rn(1.0, t));
}

// The 8 gains of one chunk as four packed pairs (loads only).
__device__ __forceinline__ void norm_gains(const float* g8, uint64_t (&g2)[4]) {
  const ulonglong2 ga = __ldg(reinterpret_cast<const ulonglong2*>(g8));
  const ulonglong2 gb = __ldg(reinterpret_cast<const ulonglong2*>(g8) + 1);
  g2[0] = ga.x, g2[1] = ga.y, g2[2] = gb.x, g2[3] = gb.y;
}

// The same from the CTA's table of gains in shared memory.
__device__ __forceinline__ void norm_gains_smem(const float* g8, uint64_t (&g2)[4]) {
  const ulonglong2 ga = *reinterpret_cast<const ulonglong2*>(g8);
  const ulonglong2 gb = *(reinterpret_cast<const ulonglong2*>(g8) + 1);
  g2[0] = ga.x, g2[1] = ga.y, g2[2] = gb.x, g2[3] = gb.y;
}

// y = (x * r) * g for one chunk from its gains g2 (packed pairs).
__device__ __forceinline__ void norm_apply_g(const uint4& u, uint64_t r2, const uint64_t (&g2)[4],
                                             uint64_t (&y2)[4]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int t = 0; t < 4; ++t)
    y2[t] = f2_mul(f2_mul(f2_make(bf16_lo(w[t]), bf16_hi(w[t])), r2), g2[t]);
}

// y = (x * r) * g for one chunk, as four packed pairs; g8 = the chunk's 8 gains.
__device__ __forceinline__ void norm_apply(const uint4& u, uint64_t r2, const float* g8,
                                           uint64_t (&y2)[4]) {
  const ulonglong2 ga = __ldg(reinterpret_cast<const ulonglong2*>(g8));
  const ulonglong2 gb = __ldg(reinterpret_cast<const ulonglong2*>(g8) + 1);
  const uint64_t g2[4] = {ga.x, ga.y, gb.x, gb.y};
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int t = 0; t < 4; ++t)
    y2[t] = f2_mul(f2_mul(f2_make(bf16_lo(w[t]), bf16_hi(w[t])), r2), g2[t]);
}

// The codes of one chunk for a row whose largest |y| is in [2^-60, 2^100]:
// q = RN(y / sx) by two corrections of the reciprocal product (rs2 = RN(1/sx),
// nsc2 = -sx, as pairs); INT8: the low byte of RN(q + 1.5 * 2^23), i.e.
// rne(q) (|q| <= 127.00001); E4M3: cvt.rn.satfinite with the sign bit of y.
template <bool E4M3>
__device__ __forceinline__ uint2 norm_codes_fast(const uint64_t (&y2)[4], uint64_t rs2,
                                                 uint64_t nsc2) {
  uint64_t qq[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint64_t a2 = y2[t];
    uint64_t q = f2_mul(a2, rs2);
    q = f2_fma(f2_fma(nsc2, q, a2), rs2, q);
    qq[t] = f2_fma(f2_fma(nsc2, q, a2), rs2, q);
  }
  uint2 o;
  if constexpr (E4M3) {
    uint32_t cd[4], sg[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      float lo, hi;
      f2_split(qq[t], lo, hi);
      cd[t] = pack_e4m3x2(lo, hi);
      float ylo, yhi;
      f2_split(y2[t], ylo, yhi);
      // the signs of y, as the sign bits of two code bytes
      sg[t] = __byte_perm(__float_as_uint(ylo), __float_as_uint(yhi), 0x0073) & 0x8080u;
    }
    o.x = ((cd[0] | (cd[1] << 16)) & 0x7F7F7F7Fu) | sg[0] | (sg[1] << 16);
    o.y = ((cd[2] | (cd[3] << 16)) & 0x7F7F7F7Fu) | sg[2] | (sg[3] << 16);
  } else {
    const uint64_t mg2 = f2_make(12582912.0f, 12582912.0f);
    uint32_t tb[8];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      float lo, hi;
      f2_split(f2_add(qq[t], mg2), lo, hi);
      tb[2 * t] = __float_as_uint(lo);
      tb[2 * t + 1] = __float_as_uint(hi);
    }
    o.x = __byte_perm(__byte_perm(tb[0], tb[1], 0x0040), __byte_perm(tb[2], tb[3], 0x0040), 0x5410);
    o.y = __byte_perm(__byte_perm(tb[4], tb[5], 0x0040), __byte_perm(tb[6], tb[7], 0x0040), 0x5410);
  }
  return o;
}

// The codes of one chunk by IEEE divisions (rows outside that window; scale
// 0 gives zero codes), as the plain form.
template <bool E4M3>
__device__ __forceinline__ uint2 norm_codes_exact(const uint64_t (&y2)[4], float scale) {
  float q[8];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    float lo, hi;
    f2_split(y2[t], lo, hi);
    q[2 * t] = scale == 0.0f ? 0.0f : __fdiv_rn(lo, scale);
    q[2 * t + 1] = scale == 0.0f ? 0.0f : __fdiv_rn(hi, scale);
  }
  uint2 o;
  if constexpr (E4M3) {
    o.x = pack_e4m3x2(q[0], q[1]) | (pack_e4m3x2(q[2], q[3]) << 16);
    o.y = pack_e4m3x2(q[4], q[5]) | (pack_e4m3x2(q[6], q[7]) << 16);
    if (scale == 0.0f) o = make_uint2(0u, 0u);
  } else {
    uint32_t b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) b[i] = uint32_t(max(-127, min(127, __float2int_rn(q[i])))) & 0xFFu;
    o.x = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
    o.y = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
  }
  return o;
}

template <int V, bool E4M3, int SLOTS, int MAXT>
__global__ void __launch_bounds__(MAXT, 512 / MAXT)
    rmsnorm_quant_stream_kernel(const uint16_t* __restrict__ x, const float* __restrict__ g,
                                float eps, int64_t M, int K, uint8_t* __restrict__ xq,
                                float* __restrict__ sx, int* status, int late_wait,
                                int force_exact) {
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint32_t red_mx[2][32];
  __shared__ unsigned long long red_sum[2][2][32];
  __shared__ double red_dbl[2][32];
  __shared__ uint32_t red_am[2][32];
  __shared__ unsigned long long slow_lo[2], slow_hi[2];
  __shared__ __align__(8) uint64_t bars[SLOTS];
  const uint32_t row_bytes = uint32_t(K) * 2;
  const int nchunk = K >> 3;
  const int nthreads = blockDim.x, nwarps = nthreads >> 5;
  const int64_t stride = gridDim.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < SLOTS; ++i) mbar_init(smem_u32(&bars[i]), 1);
    fence_barrier_init();
    slow_lo[0] = slow_lo[1] = slow_hi[0] = slow_hi[1] = 0ull;
  }
  // x and g may come from the kernel before this one, which may still read
  // xq / sx -- unless the caller has ruled both out (late_wait: then this
  // grid waits for that kernel only at its end)
  if (!late_wait) pdl_wait();
  if (threadIdx.x == 0) {
    for (int i = 0; i < SLOTS; ++i) {
      const int64_t m = blockIdx.x + i * stride;
      if (m < M) {
        mbar_arrive_expect_tx(smem_u32(&bars[i]), row_bytes);
        bulk_load(smem_u32(ring + size_t(i) * row_bytes), x + m * K, row_bytes,
                  smem_u32(&bars[i]));
      }
    }
  }
  __syncthreads();
  int slot = 0, sel = 0;
  uint32_t phase = 0;
#pragma unroll 1
  for (int64_t m = blockIdx.x; m < M; m += stride) {
    const bool timed_out = !mbar_wait(smem_u32(&bars[slot]), phase);
    const uint8_t* row = ring + size_t(slot) * row_bytes;
    // 1. this thread's chunks, the largest magnitude pattern
    uint4 raw[V];
    uint32_t mx2 = 0, mn2 = 0xFFFFFFFFu;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int c = threadIdx.x + j * nthreads;
      raw[j] = c < nchunk ? *reinterpret_cast<const uint4*>(row + size_t(c) * 16)
                          : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t w[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint32_t wm = w[t] & 0x7FFF7FFFu;
        mx2 = max_u16x2(mx2, wm);
        mn2 = min_u16x2(mn2, wm);
      }
    }
    const uint32_t wmx = __reduce_max_sync(0xFFFFFFFFu, max(mx2 & 0xFFFFu, mx2 >> 16));
    if (lane == 0) red_mx[sel][warp] = wmx;
    if (__syncthreads_or(timed_out)) {
      if (threadIdx.x == 0) {
        record_status(status, kStatusTimeout);
        // let the copies still in flight land before the CTA exits
        for (int k = 0; k < SLOTS; ++k) {
          if (m + k * stride < M) {
            const int sk = (slot + k) % SLOTS;
            (void)mbar_wait(smem_u32(&bars[sk]), phase ^ uint32_t(slot + k >= SLOTS));
          }
        }
      }
      break;
    }
    if (threadIdx.x == 0) {
      // every thread has read this slot: refill it with the row SLOTS ahead,
      // and clear the slow accumulator of the next row (its last readers,
      // two rows back, are past barrier 3 of the previous row)
      const int64_t mn = m + SLOTS * stride;
      if (mn < M) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(smem_u32(&bars[slot]), row_bytes);
        bulk_load(smem_u32(ring + size_t(slot) * row_bytes), x + mn * K, row_bytes,
                  smem_u32(&bars[slot]));
      }
      slow_lo[sel ^ 1] = 0ull;
      slow_hi[sel ^ 1] = 0ull;
    }
    const uint32_t hmax =
        __reduce_max_sync(0xFFFFFFFFu, red_mx[sel][lane < nwarps ? lane : 0]);
    const int efmax = int(hmax >> 7);                 // 0 when the largest is subnormal
    const int emax = efmax ? efmax - 127 : -126;
    // 2. the sum of squares in binary64 with the interval check of the warp
    // form (the per-warp sums added in warp order, the same order in every
    // thread, so that all of them hold the same ss); the exact sum below only
    // for the rows whose r that cannot settle (a block-uniform branch)
    float r = 0.0f;
    bool exact = force_exact != 0;
    if (!exact) {
      double dacc = 0.0;
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const uint32_t w[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const double dl = double(bf16_lo(w[t])), dh = double(bf16_hi(w[t]));
          dacc = __fma_rn(dl, dl, dacc);
          dacc = __fma_rn(dh, dh, dacc);
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        dacc = __dadd_rn(dacc, __shfl_down_sync(0xFFFFFFFFu, dacc, off));
      if (lane == 0) red_dbl[sel][warp] = dacc;
      __syncthreads();
      double ss = 0.0;
      for (int i = 0; i < nwarps; ++i) ss = __dadd_rn(ss, red_dbl[sel][i]);
      const float r_lo = norm_chain(__dmul_ru(ss, 1.0 + 0x1p-36), K, eps);
      const float r_hi = norm_chain(__dmul_rd(ss, 1.0 - 0x1p-36), K, eps);
      exact = r_lo != r_hi;
      r = r_lo;
    }
    if (exact) {
    // bands A and B: normal elements with exponent field >= efmax - 32 (none
    // when the largest is below 2^-94: the whole row takes the slow path)
    const int lo_ef = efmax > 32 ? efmax - 32 : 256;
    // the exact sum of squares. Band A: the shift e - e_max + 16 in
    // [0, 16], clamped at 32 (a = 0) below the band, negative offsets
    // included; band B: 16 more, kept only when below 16 (one unsigned
    // comparison excludes both band A and everything below band B)
    uint64_t accA = 0, accB = 0;
    if (efmax > 32) {
      const uint32_t sh0 = uint32_t(16 - efmax);
#pragma unroll
      for (int j = 0; j < V; ++j) norm_band_squares(raw[j], sh0, accA, accB);
    }
    // some element of this thread below band B (zeros included: the slow
    // loop skips them)
    const bool slow = min(mn2 & 0xFFFFu, mn2 >> 16) < (uint32_t(lo_ef) << 7);
    if (slow) {  // rare: this thread's small and subnormal elements (rolled
                 // loops: the row goes through local memory here only)
      U128 s128 = {0, 0};
#pragma unroll 1
      for (int j = 0; j < V; ++j) norm_slow_chunk(raw[j], lo_ef, emax, s128);
      const unsigned long long old = atomicAdd(&slow_lo[sel], s128.lo);
      const unsigned long long carry = old + s128.lo < old ? 1ull : 0ull;
      if (s128.hi + carry) atomicAdd(&slow_hi[sel], s128.hi + carry);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      accA += __shfl_xor_sync(0xFFFFFFFFu, accA, off);
      accB += __shfl_xor_sync(0xFFFFFFFFu, accB, off);
    }
    if (lane == 0) {
      red_sum[sel][0][warp] = accA;
      red_sum[sel][1][warp] = accB;
    }
    __syncthreads();
    uint64_t totA = lane < nwarps ? red_sum[sel][0][lane] : 0ull;
    uint64_t totB = lane < nwarps ? red_sum[sel][1][lane] : 0ull;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      totA += __shfl_xor_sync(0xFFFFFFFFu, totA, off);
      totB += __shfl_xor_sync(0xFFFFFFFFu, totB, off);
    }
    r = norm_rinv(U128{slow_lo[sel], slow_hi[sel]}, totA, totB, hmax, emax, K, eps);
    }
    // 3. y = (x * r) * g, the largest |y|
    const uint64_t r2 = f2_make(r, r);
    uint64_t y2[V][4];
    float am0 = 0.0f, am1 = 0.0f;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int c = threadIdx.x + j * nthreads;
      // the gains from L1 (the same K floats for every row); none past the row
      if (c < nchunk) {
        norm_apply(raw[j], r2, g + size_t(c) * 8, y2[j]);
      } else {
#pragma unroll
        for (int t2 = 0; t2 < 4; ++t2) y2[j][t2] = 0ull;
      }
#pragma unroll
      for (int t2 = 0; t2 < 4; ++t2) {
        float a, b;
        f2_split(y2[j][t2], a, b);
        if (t2 & 1) am1 = max3_nan(am1, fabsf(a), fabsf(b));
        else am0 = max3_nan(am0, fabsf(a), fabsf(b));
      }
    }
    const uint32_t wam = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(fmaxf(am0, am1)));
    if (lane == 0) red_am[sel][warp] = wam;
    __syncthreads();
    const float amax = __uint_as_float(
        __reduce_max_sync(0xFFFFFFFFu, red_am[sel][lane < nwarps ? lane : 0]));
    uint8_t* out = xq + m * K;
    // 4. the scale and the codes
    if (amax >= 0x1p-60f && amax <= 0x1p100f) {
      const float scale = norm_div_by_qmax<E4M3>(amax);
      if (threadIdx.x == 0) sx[m] = scale;
      const float rs = __frcp_rn(scale);
      const uint64_t rs2 = f2_make(rs, rs), nsc2 = f2_make(-scale, -scale);
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const int c = threadIdx.x + j * nthreads;
        if (c < nchunk)
          *reinterpret_cast<uint2*>(out + size_t(c) * 8) = norm_codes_fast<E4M3>(y2[j], rs2, nsc2);
      }
    } else {
      const float scale = __fdiv_rn(amax, E4M3 ? 448.0f : 127.0f);
      if (threadIdx.x == 0) sx[m] = scale;
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const int c = threadIdx.x + j * nthreads;
        if (c < nchunk)
          *reinterpret_cast<uint2*>(out + size_t(c) * 8) = norm_codes_exact<E4M3>(y2[j], scale);
      }
    }
    sel ^= 1;
    if (++slot == SLOTS) {
      slot = 0;
      phase ^= 1u;
    }
  }
  if (late_wait) pdl_wait();
}

// ----------------------------------------------------------------------------
// The warp form (many rows of at most 8192 elements): every warp normalizes
// and quantizes whole rows by itself -- rows w, w + W, ... for the grid's W
// warps -- with its own SLOTS-row ring of bulk copies in shared memory and
// its own barriers, so no block barrier and no cross-warp reduction is on a
// row's path. Each lane takes the chunks c = lane + 32 j and re-reads them
// from shared memory in every pass; the arithmetic is that of the streaming
// form, chunk by chunk (the 128-bit remainder reduced by shuffles instead of
// shared atomics).
// ----------------------------------------------------------------------------
constexpr int kNormWarpMaxK = 8192;
constexpr int kNormWarpSlots = 1;

// GS: the gains in shared memory, loaded once per CTA (rows of up to 4096
// elements), instead of from L1 in every pass
template <bool E4M3, bool GS>
__global__ void __launch_bounds__(256)
    rmsnorm_quant_warp_kernel(const uint16_t* __restrict__ x, const float* __restrict__ g,
                              float eps, int64_t M, int K, uint8_t* __restrict__ xq,
                              float* __restrict__ sx, int* status, int late_wait,
                              int force_exact) {
  constexpr int SLOTS = kNormWarpSlots;
  // [K] binary32 gains (GS), then [warps][SLOTS][K] bf16 rows
  extern __shared__ __align__(128) uint8_t smem_dyn[];
  float* gtab = reinterpret_cast<float*>(smem_dyn);
  uint8_t* ring = smem_dyn + (GS ? size_t(K) * 4 : 0);
  __shared__ __align__(8) uint64_t bars[8][SLOTS];
  const uint32_t row_bytes = uint32_t(K) * 2;
  const int nchunk = K >> 3;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t nw = blockDim.x >> 5;
  const int64_t w0 = int64_t(blockIdx.x) * nw + warp, stride = int64_t(gridDim.x) * nw;
  uint8_t* my_ring = ring + size_t(warp) * SLOTS * row_bytes;
  pdl_launch_dependents();
  if (lane == 0) {
    for (int i = 0; i < SLOTS; ++i) mbar_init(smem_u32(&bars[warp][i]), 1);
    fence_barrier_init();
  }
  __syncwarp();
  // x and g may come from the kernel before this one, which may still read
  // xq / sx -- unless the caller has ruled both out (late_wait)
  if (!late_wait) pdl_wait();
  if constexpr (GS) {
    for (int i = threadIdx.x; i < K / 4; i += blockDim.x)
      reinterpret_cast<float4*>(gtab)[i] = __ldg(reinterpret_cast<const float4*>(g) + i);
    __syncthreads();
  }
  if (lane == 0) {
    for (int i = 0; i < SLOTS; ++i) {
      const int64_t m = w0 + i * stride;
      if (m < M) {
        mbar_arrive_expect_tx(smem_u32(&bars[warp][i]), row_bytes);
        bulk_load(smem_u32(my_ring + size_t(i) * row_bytes), x + m * K, row_bytes,
                  smem_u32(&bars[warp][i]));
      }
    }
  }
  int slot = 0;
  uint32_t phase = 0;
#pragma unroll 1
  for (int64_t m = w0; m < M; m += stride) {
    if (__any_sync(0xFFFFFFFFu, !mbar_wait(smem_u32(&bars[warp][slot]), phase))) {
      if (lane == 0) {
        record_status(status, kStatusTimeout);
        // let the copies still in flight land before the warp leaves
        for (int k = 0; k < SLOTS; ++k) {
          if (m + k * stride < M) {
            const int sk = (slot + k) % SLOTS;
            (void)mbar_wait(smem_u32(&bars[warp][sk]), phase ^ uint32_t(slot + k >= SLOTS));
          }
        }
      }
      __syncwarp();
      break;
    }
    const uint4* row = reinterpret_cast<const uint4*>(my_ring + size_t(slot) * row_bytes);
    // 0. the sum of squares in binary64: every square of a bf16 value is exact
    // there, so the computed sum lies within (n - 1) * 2^-53 of the exact one
    // (n <= 16384 terms, all non-negative; whatever the order), far inside
    // the 2^-36 used below, and the elements the exact sum leaves out (more
    // than 48 binades below the largest) change it by less than 2^-80. The
    // chain to r is monotone in ss, so if both ends of [ss (1 - 2^-36),
    // ss (1 + 2^-36)] give the same binary32 r, that is the r of the exact
    // sum; otherwise (about one row in 2^11) the exact sum is taken below.
    float r = 0.0f;
    bool exact = force_exact != 0;
    if (!exact) {
      double acc = 0.0;
#pragma unroll 4
      for (int c = lane; c < nchunk; c += 32) {
        const uint4 u = row[c];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const double dl = double(bf16_lo(w[t])), dh = double(bf16_hi(w[t]));
          acc = __fma_rn(dl, dl, acc);
          acc = __fma_rn(dh, dh, acc);
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc = __dadd_rn(acc, __shfl_down_sync(0xFFFFFFFFu, acc, off));
      acc = __shfl_sync(0xFFFFFFFFu, acc, 0);  // one value for every lane
      const float r_lo = norm_chain(__dmul_ru(acc, 1.0 + 0x1p-36), K, eps);
      const float r_hi = norm_chain(__dmul_rd(acc, 1.0 - 0x1p-36), K, eps);
      exact = r_lo != r_hi;
      r = r_lo;
    }
    if (exact) {
    // 1. the largest and smallest magnitude patterns
    uint32_t mx2 = 0, mn2 = 0xFFFFFFFFu;
#pragma unroll 4
    for (int c = lane; c < nchunk; c += 32) {
      const uint4 u = row[c];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint32_t wm = w[t] & 0x7FFF7FFFu;
        mx2 = max_u16x2(mx2, wm);
        mn2 = min_u16x2(mn2, wm);
      }
    }
    const uint32_t hmax = __reduce_max_sync(0xFFFFFFFFu, max(mx2 & 0xFFFFu, mx2 >> 16));
    const int efmax = int(hmax >> 7);
    const int emax = efmax ? efmax - 127 : -126;
    const int lo_ef = efmax > 32 ? efmax - 32 : 256;
    // 2. the exact sum of squares
    uint64_t accA = 0, accB = 0;
    if (efmax > 32) {
      const uint32_t sh0 = uint32_t(16 - efmax);
#pragma unroll 4
      for (int c = lane; c < nchunk; c += 32) norm_band_squares(row[c], sh0, accA, accB);
    }
    U128 rest = {0, 0};
    if (min(mn2 & 0xFFFFu, mn2 >> 16) < (uint32_t(lo_ef) << 7)) {
#pragma unroll 1
      for (int c = lane; c < nchunk; c += 32) norm_slow_chunk(row[c], lo_ef, emax, rest);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      accA += __shfl_xor_sync(0xFFFFFFFFu, accA, off);
      accB += __shfl_xor_sync(0xFFFFFFFFu, accB, off);
    }
    if (__any_sync(0xFFFFFFFFu, (rest.lo | rest.hi) != 0ull)) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const uint64_t lo = __shfl_xor_sync(0xFFFFFFFFu, rest.lo, off);
        const uint64_t hi = __shfl_xor_sync(0xFFFFFFFFu, rest.hi, off);
        u128_add(rest, lo, hi);
      }
    }
    r = norm_rinv(rest, accA, accB, hmax, emax, K, eps);
    }
    const uint64_t r2 = f2_make(r, r);
    // 3. the largest |y|, y = (x * r) * g. Two chunks per step, every load
    // of the step (row from shared memory, gains from L1) issued first.
    float am0 = 0.0f, am1 = 0.0f;
#pragma unroll 2
    for (int c = lane; c < nchunk; c += 64) {
      const bool two = c + 32 < nchunk;
      const uint4 u0 = row[c];
      const uint4 u1 = two ? row[c + 32] : make_uint4(0u, 0u, 0u, 0u);
      uint64_t g0[4], g1[4] = {0ull, 0ull, 0ull, 0ull};
      if constexpr (GS) {
        norm_gains_smem(gtab + size_t(c) * 8, g0);
        if (two) norm_gains_smem(gtab + size_t(c + 32) * 8, g1);
      } else {
        norm_gains(g + size_t(c) * 8, g0);
        if (two) norm_gains(g + size_t(c + 32) * 8, g1);
      }
      uint64_t y0[4], y1[4];
      norm_apply_g(u0, r2, g0, y0);
      norm_apply_g(u1, r2, g1, y1);
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        float a, b, a1, b1;
        f2_split(y0[t], a, b);
        f2_split(y1[t], a1, b1);
        am0 = max3_nan(am0, fabsf(a), fabsf(b));
        am1 = max3_nan(am1, fabsf(a1), fabsf(b1));
      }
    }
    const float amax =
        __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(fmaxf(am0, am1))));
    // 4. the scale and the codes (y recomputed, bit for bit the same)
    uint2* out = reinterpret_cast<uint2*>(xq + m * K);
    if (amax >= 0x1p-60f && amax <= 0x1p100f) {
      const float scale = norm_div_by_qmax<E4M3>(amax);
      if (lane == 0) sx[m] = scale;
      const float rs = __frcp_rn(scale);
      const uint64_t rs2 = f2_make(rs, rs), nsc2 = f2_make(-scale, -scale);
#pragma unroll 2
      for (int c = lane; c < nchunk; c += 64) {
        const bool two = c + 32 < nchunk;
        const uint4 u0 = row[c];
        const uint4 u1 = two ? row[c + 32] : make_uint4(0u, 0u, 0u, 0u);
        uint64_t g0[4], g1[4] = {0ull, 0ull, 0ull, 0ull};
        if constexpr (GS) {
          norm_gains_smem(gtab + size_t(c) * 8, g0);
          if (two) norm_gains_smem(gtab + size_t(c + 32) * 8, g1);
        } else {
          norm_gains(g + size_t(c) * 8, g0);
          if (two) norm_gains(g + size_t(c + 32) * 8, g1);
        }
        uint64_t y0[4], y1[4];
        norm_apply_g(u0, r2, g0, y0);
        norm_apply_g(u1, r2, g1, y1);
        out[c] = norm_codes_fast<E4M3>(y0, rs2, nsc2);
        if (two) out[c + 32] = norm_codes_fast<E4M3>(y1, rs2, nsc2);
      }
    } else {
      const float scale = __fdiv_rn(amax, E4M3 ? 448.0f : 127.0f);
      if (lane == 0) sx[m] = scale;
#pragma unroll 1
      for (int c = lane; c < nchunk; c += 32) {
        uint64_t y2[4];
        norm_apply(row[c], r2, g + size_t(c) * 8, y2);
        out[c] = norm_codes_exact<E4M3>(y2, scale);
      }
    }
    // every lane has read this slot: refill it with the row SLOTS ahead
    __syncwarp();
    if (lane == 0) {
      const int64_t mn = m + SLOTS * stride;
      if (mn < M) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(smem_u32(&bars[warp][slot]), row_bytes);
        bulk_load(smem_u32(my_ring + size_t(slot) * row_bytes), x + mn * K, row_bytes,
                  smem_u32(&bars[warp][slot]));
      }
    }
    if (++slot == SLOTS) {
      slot = 0;
      phase ^= 1u;
    }
  }
  if (late_wait) pdl_wait();
}

}  // namespace sqk

namespace sqh {

using namespace sqk;

int rmsnorm_quant_max_k() { return kNormMaxK; }

// SQ_NORM_EXACT_SUM=1 takes the exact integer sum of squares for every row
// (the path the binary64 sum falls back to), so that tests can cover it at will.
static int norm_force_exact() {
  const char* e = std::getenv("SQ_NORM_EXACT_SUM");
  return e && e[0] == '1';
}

static int norm_sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

// The streaming form: V = 4 chunks per thread, the CTA as wide as the row
// needs (a multiple of 32 threads, at most MAXT), SLOTS rows in flight, as
// many CTAs as fit on the SMs at once (no more than there are rows).
template <int MAXT>
static cudaError_t launch_norm_stream(const uint16_t* x, const float* g, float eps, int64_t M,
                                      int K, bool e4m3, uint8_t* xq, float* sx, bool overlap,
                                      cudaStream_t st) {
  constexpr int V = 4, SLOTS = 4;
  const int nchunk = K >> 3;
  const int threads = ((nchunk + V - 1) / V + 31) / 32 * 32;
  const size_t smem = size_t(SLOTS) * size_t(K) * 2;
  int* status = status_ptr();
  auto kern = e4m3 ? rmsnorm_quant_stream_kernel<V, true, SLOTS, MAXT>
                   : rmsnorm_quant_stream_kernel<V, false, SLOTS, MAXT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) !=
          cudaSuccess || per_sm < 1)
    per_sm = 1;
  int64_t grid = int64_t(per_sm) * norm_sm_count();
  if (grid > M) grid = M;
  return launch_pdl(kern, unsigned(grid), threads, smem, st, x, g, eps, M, K, xq, sx, status,
                    int(overlap), norm_force_exact());
}

cudaError_t launch_rmsnorm_quant(const uint16_t* x, const float* g, float eps, int64_t M,
                                 int64_t K, bool e4m3, void* xq, float* sx, float* xn,
                                 bool overlap, cudaStream_t st) {
  if (!xn && K <= kNormWarpMaxK && M >= 4LL * norm_sm_count()) {
    // the warp form: up to 8 warps per CTA, each with SLOTS rows in flight;
    // rows of up to 4096 elements with the gains in shared memory, at most
    // 72 KB per CTA (three CTAs per SM), longer ones with the gains from L1
    // and about 96 KB of ring per CTA; as many CTAs as fit, no more than the
    // rows need
    const bool gs = K <= 4096;
    const int per_row = int(K) * 2 * kNormWarpSlots;
    const int table = gs ? int(K) * 4 : 0;
    const int warps = max(1, min(8, ((gs ? 73728 : 98304) - table) / per_row));
    const size_t smem = size_t(table) + size_t(warps) * per_row;
    auto kern = e4m3 ? (gs ? rmsnorm_quant_warp_kernel<true, true>
                           : rmsnorm_quant_warp_kernel<true, false>)
                     : (gs ? rmsnorm_quant_warp_kernel<false, true>
                           : rmsnorm_quant_warp_kernel<false, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(smem));
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, warps * 32, smem) !=
            cudaSuccess || per_sm < 1)
      per_sm = 1;
    int64_t grid = int64_t(per_sm) * norm_sm_count();
    grid = min(grid, (M + warps - 1) / warps);
    return launch_pdl(kern, unsigned(grid), warps * 32, smem, st, x, g, eps, M, int(K),
                      static_cast<uint8_t*>(xq), sx, status_ptr(), int(overlap),
                      norm_force_exact());
  }
  if (!xn) {
    const int nchunk = int(K >> 3);  // <= 2048
    uint8_t* q = static_cast<uint8_t*>(xq);
    if (nchunk <= 4 * 128)
      return launch_norm_stream<128>(x, g, eps, M, int(K), e4m3, q, sx, overlap, st);
    if (nchunk <= 4 * 256)
      return launch_norm_stream<256>(x, g, eps, M, int(K), e4m3, q, sx, overlap, st);
    return launch_norm_stream<512>(x, g, eps, M, int(K), e4m3, q, sx, overlap, st);
  }
  // the plain form: one CTA per row, at most a few waves' worth resident:
  // rows beyond the grid are taken in turn
  const int64_t grid = M < 148 * 16 ? M : 148 * 16;
  const size_t smem = size_t(K) * 2;  // the staged row (at most 32 KB: no opt-in needed)
  if (e4m3)
    return launch_pdl(rmsnorm_quant_kernel<true>, unsigned(grid), kNormThreads, smem, st, x, g,
                      eps, M, int(K), static_cast<uint8_t*>(xq), sx, xn, int(overlap));
  return launch_pdl(rmsnorm_quant_kernel<false>, unsigned(grid), kNormThreads, smem, st, x, g,
                    eps, M, int(K), static_cast<uint8_t*>(xq), sx, xn, int(overlap));
}

}  // namespace sqh
