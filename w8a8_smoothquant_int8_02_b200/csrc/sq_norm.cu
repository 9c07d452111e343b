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
// One CTA per row: the row is staged in shared memory, then four passes over
// it (the largest exponent, the exact sum of squares, the largest |xn|, the
// codes), each closed by a block reduction. HBM-bound in principle (2 bytes
// read and 1 written per element).
#include <cstdint>

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
                         float* __restrict__ sx, float* __restrict__ xn) {
  extern __shared__ __align__(16) uint16_t row[];  // K entries
  __shared__ int red_i[kNormThreads / 32];
  __shared__ unsigned long long red_lo[kNormThreads / 32], red_hi[kNormThreads / 32];
  __shared__ float red_f[kNormThreads / 32];
  __shared__ float bcast[2];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int W = kNormThreads / 32;
  const int nchunk = K >> 3;
  // the row may come from the kernel before this one
  pdl_launch_dependents();
  pdl_wait();
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
}

}  // namespace sqk

namespace sqh {

using namespace sqk;

int rmsnorm_quant_max_k() { return kNormMaxK; }

cudaError_t launch_rmsnorm_quant(const uint16_t* x, const float* g, float eps, int64_t M,
                                 int64_t K, bool e4m3, void* xq, float* sx, float* xn,
                                 cudaStream_t st) {
  // one CTA per row, at most a few waves' worth resident: rows beyond the
  // grid are taken in turn
  const int64_t grid = M < 148 * 16 ? M : 148 * 16;
  const size_t smem = size_t(K) * 2;  // the staged row (at most 32 KB: no opt-in needed)
  if (e4m3)
    return launch_pdl(rmsnorm_quant_kernel<true>, unsigned(grid), kNormThreads, smem, st, x, g,
                      eps, M, int(K), static_cast<uint8_t*>(xq), sx, xn);
  return launch_pdl(rmsnorm_quant_kernel<false>, unsigned(grid), kNormThreads, smem, st, x, g,
                    eps, M, int(K), static_cast<uint8_t*>(xq), sx, xn);
}

}  // namespace sqh
