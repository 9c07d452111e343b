// sq_gemm.cu -- 8-bit tensor-core GEMM with fused dequantization epilogue
// for sm_100a (tcgen05 + TMA + tensor memory).
//
//   acc[m,n] = sum_k Xq[m,k] * Wq[n,k]          (INT8: exact int32;
//                                                 E4M3: binary32 in TMEM)
//   y[m,n]   = bf16( ((float(acc) * sx[m]) * sw[n]) + bias[n] )
//
// Source: "Weight-Activation Quantization" (infra.bea.ai) §3 "Step 2"
// (Y = dequantize(X_int8 @ W_int8) on INT8 tensor cores), §1 table
// (INT8 x INT8 and FP8 x FP8 GEMM rows), §4 (FP8 E4M3 operands).
//
// Kernel structure (one CTA computes one BM x BN output tile, BM = 128):
//   warp 0      : TMA producer -- streams 128-byte-wide K slices of the Xq
//                 and Wq tiles into a STAGES-deep shared-memory ring
//                 (128-byte swizzle), one mbarrier pair per slot.
//   warp 1      : allocates the tensor-memory accumulator, and one elected
//                 thread issues tcgen05.mma (M=128, N=BN, K=32 per
//                 instruction) and frees ring slots with tcgen05.commit.
//   warps 2..5  : epilogue -- tcgen05.ld the accumulator rows (warp w reads
//                 TMEM lanes 32*(w%4)..+31), dequantize with per-token and
//                 per-channel scales (+bias), round to bf16, store.
// Every barrier wait is bounded (sq_common.cuh); a wait that gives up sets
// the status word, skips the remaining work and still frees tensor memory.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "sq_common.cuh"
#include "sq_internal.h"

namespace sqk {

constexpr int kBM = 128;
constexpr int kBK = 128;  // bytes of K per pipeline stage (one swizzle row)
constexpr int kThreads = 192;

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr uint32_t kABytes = kBM * kBK;
  static constexpr uint32_t kBBytes = BN * kBK;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kRing = STAGES * kStageBytes;
  // barriers: full[STAGES], empty[STAGES], tmem_full
  static constexpr uint32_t kBarOff = kRing;
  static constexpr uint32_t kMiscOff = kBarOff + (2 * STAGES + 1) * 8;  // tmem slot, abort
  static constexpr uint32_t kScaleOff = (kMiscOff + 16 + 15) & ~15u;    // sw[BN], bias[BN]
  static constexpr uint32_t kTotal = kScaleOff + 2 * BN * 4;
  static constexpr uint32_t kDynamic = kTotal + 1024;  // slack for 1024-B alignment
  static constexpr uint32_t kTmemCols = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
};

template <int BN, int STAGES, bool E4M3, bool OUT_BF16, bool HAS_BIAS, bool WRITE_ACC>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_w8a8_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const float* __restrict__ sx, const float* __restrict__ sw,
                     const uint16_t* __restrict__ bias, void* __restrict__ y,
                     int32_t* __restrict__ acc_out, int M, int N, int K, int* status) {
  using L = GemmSmem<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_a = s_base;
  const uint32_t s_b = s_base + STAGES * L::kABytes;
  const uint32_t bar_full = s_base + L::kBarOff;
  const uint32_t bar_empty = bar_full + STAGES * 8;
  const uint32_t bar_tmem_full = bar_empty + STAGES * 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  float* s_sw = reinterpret_cast<float*>(smem + L::kScaleOff);
  float* s_bias = s_sw + BN;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * kBM, n0 = blockIdx.x * BN;
  const int nk = (K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, 1);
    }
    mbar_init(bar_tmem_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_map(&tm_a);
    tma_prefetch_map(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
#pragma unroll 1
      for (int kb = 0; kb < nk; ++kb) {
        const int st = kb % STAGES;
        const uint32_t ph = (kb / STAGES) & 1;
        if (!mbar_wait(bar_empty + 8 * st, ph ^ 1)) {
          record_status(status, kStatusTimeout);
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        mbar_arrive_expect_tx(bar_full + 8 * st, L::kStageBytes);
        tma_load_2d(s_a + st * L::kABytes, &tm_a, bar_full + 8 * st, kb * kBK, m0);
        tma_load_2d(s_b + st * L::kBBytes, &tm_b, bar_full + 8 * st, kb * kBK, n0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = E4M3 ? idesc_e4m3_f32(kBM, BN) : idesc_s8_s32(kBM, BN);
      bool ok = true;
#pragma unroll 1
      for (int kb = 0; kb < nk; ++kb) {
        const int st = kb % STAGES;
        const uint32_t ph = (kb / STAGES) & 1;
        if (!mbar_wait(bar_full + 8 * st, ph)) {
          record_status(status, kStatusTimeout);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = s_a + st * L::kABytes;
        const uint32_t b_addr = s_b + st * L::kBBytes;
#pragma unroll
        for (int kk = 0; kk < kBK / 32; ++kk) {
          const uint64_t ad = sw128_desc(a_addr + kk * 32);
          const uint64_t bd = sw128_desc(b_addr + kk * 32);
          const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
          if constexpr (E4M3) mma_f8(tmem_base, ad, bd, idesc, accum);
          else mma_i8(tmem_base, ad, bd, idesc, accum);
        }
        tc_commit(bar_empty + 8 * st);
      }
      // Signals the epilogue even after an abort so that it does not wait
      // for the full timeout a second time (the abort flag tells it to skip).
      tc_commit(bar_tmem_full);
      // After an abort nobody else consumes that signal: wait here (bounded)
      // for the MMAs already issued, so tensor memory is idle when freed.
      if (!ok) (void)mbar_wait(bar_tmem_full, 0);
    }
  } else {
    // ---------------------------------------------------------- epilogue --
    const int et = threadIdx.x - 64;  // 0..127
    for (int j = et; j < BN; j += 128) {
      const int n = n0 + j;
      s_sw[j] = n < N ? __ldg(sw + n) : 0.0f;
      if constexpr (HAS_BIAS) s_bias[j] = n < N ? __uint_as_float(uint32_t(__ldg(bias + n)) << 16) : 0.0f;
    }
    named_barrier_sync(1, 128);
    const bool ready = mbar_wait(bar_tmem_full, 0);
    if (!ready) {
      record_status(status, kStatusTimeout);
      *abort_flag = 1;
    }
    tc_fence_after();
    if (ready && !*abort_flag) {
      const int sub = warp & 3;
      const int row = sub * 32 + lane;
      const int m = m0 + row;
      const float sxm = m < M ? __ldg(sx + m) : 0.0f;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem_base + (uint32_t(sub * 32) << 16) + uint32_t(c0), r);
        tmem_wait_ld(r);
        if (m < M) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int n = n0 + c0 + g * 8;
            if (n < N) {
              float t[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const uint32_t raw = r[g * 8 + i];
                float a = E4M3 ? __uint_as_float(raw) : __int2float_rn(int32_t(raw));
                a = __fmul_rn(a, sxm);
                a = __fmul_rn(a, s_sw[c0 + g * 8 + i]);
                if constexpr (HAS_BIAS) a = __fadd_rn(a, s_bias[c0 + g * 8 + i]);
                t[i] = a;
              }
              const int64_t off = int64_t(m) * N + n;
              if constexpr (OUT_BF16) {
                uint4 u;
                u.x = pack_bf16x2(t[0], t[1]);
                u.y = pack_bf16x2(t[2], t[3]);
                u.z = pack_bf16x2(t[4], t[5]);
                u.w = pack_bf16x2(t[6], t[7]);
                *reinterpret_cast<uint4*>(static_cast<uint16_t*>(y) + off) = u;
              } else {
                float4* p = reinterpret_cast<float4*>(static_cast<float*>(y) + off);
                p[0] = make_float4(t[0], t[1], t[2], t[3]);
                p[1] = make_float4(t[4], t[5], t[6], t[7]);
              }
              if constexpr (WRITE_ACC) {
                int4* q = reinterpret_cast<int4*>(acc_out + off);
                q[0] = make_int4(int(r[g * 8 + 0]), int(r[g * 8 + 1]), int(r[g * 8 + 2]), int(r[g * 8 + 3]));
                q[1] = make_int4(int(r[g * 8 + 4]), int(r[g * 8 + 5]), int(r[g * 8 + 6]), int(r[g * 8 + 7]));
              }
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

}  // namespace sqk

namespace sqh {

using namespace sqk;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Tensor map of a row-major [rows, K] 8-bit matrix, box = box_rows x 128 B,
// 128-byte swizzle, out-of-bounds elements read as zero.
static bool make_map_k_major(CUtensorMap* map, const void* base, int64_t rows, int64_t K,
                             int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cuuint64_t(K), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(K)};
  cuuint32_t box[2] = {cuuint32_t(kBK), cuuint32_t(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int STAGES, bool E4M3, bool OUT_BF16, bool HAS_BIAS, bool WRITE_ACC>
static cudaError_t run_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const float* sx,
                            const float* sw, const uint16_t* bias, void* y, int32_t* acc, int M,
                            int N, int K, cudaStream_t st) {
  using L = GemmSmem<BN, STAGES>;
  auto kern = gemm_w8a8_kernel<BN, STAGES, E4M3, OUT_BF16, HAS_BIAS, WRITE_ACC>;
  static uint64_t attr_set_mask = 0;  // one bit per device ordinal
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64 || !((attr_set_mask >> dev) & 1u)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(L::kDynamic));
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set_mask |= uint64_t(1) << dev;
  }
  dim3 grid(unsigned((N + BN - 1) / BN), unsigned((M + kBM - 1) / kBM));
  kern<<<grid, kThreads, L::kDynamic, st>>>(ta, tb, sx, sw, bias, y, acc, M, N, K, status_ptr());
  return cudaGetLastError();
}

template <int BN, int STAGES, bool E4M3>
static cudaError_t dispatch_epilogue(const CUtensorMap& ta, const CUtensorMap& tb, const float* sx,
                                     const float* sw, const uint16_t* bias, void* y, OutKind yk,
                                     int32_t* acc, int M, int N, int K, cudaStream_t st) {
  const bool bf = yk == OutKind::BF16, hb = bias != nullptr, wa = acc != nullptr;
  const int key = (bf ? 4 : 0) | (hb ? 2 : 0) | (wa ? 1 : 0);
  switch (key) {
    case 0: return run_gemm<BN, STAGES, E4M3, false, false, false>(ta, tb, sx, sw, bias, y, acc, M, N, K, st);
    case 1: return run_gemm<BN, STAGES, E4M3, false, false, true>(ta, tb, sx, sw, bias, y, acc, M, N, K, st);
    case 2: return run_gemm<BN, STAGES, E4M3, false, true, false>(ta, tb, sx, sw, bias, y, acc, M, N, K, st);
    case 3: return run_gemm<BN, STAGES, E4M3, false, true, true>(ta, tb, sx, sw, bias, y, acc, M, N, K, st);
    case 4: return run_gemm<BN, STAGES, E4M3, true, false, false>(ta, tb, sx, sw, bias, y, acc, M, N, K, st);
    case 5: return run_gemm<BN, STAGES, E4M3, true, false, true>(ta, tb, sx, sw, bias, y, acc, M, N, K, st);
    case 6: return run_gemm<BN, STAGES, E4M3, true, true, false>(ta, tb, sx, sw, bias, y, acc, M, N, K, st);
    default: return run_gemm<BN, STAGES, E4M3, true, true, true>(ta, tb, sx, sw, bias, y, acc, M, N, K, st);
  }
}

cudaError_t launch_gemm(bool e4m3, const uint8_t* xq, const float* sx, const uint8_t* wq,
                        const float* sw, const uint16_t* bias, int64_t M, int64_t N, int64_t K,
                        void* y, OutKind yk, int32_t* acc, cudaStream_t st) {
  constexpr int BN = 128, STAGES = 6;
  CUtensorMap ta, tb;
  if (!make_map_k_major(&ta, xq, M, K, kBM) || !make_map_k_major(&tb, wq, N, K, BN))
    return cudaErrorInvalidValue;
  if (e4m3)
    return dispatch_epilogue<BN, STAGES, true>(ta, tb, sx, sw, bias, y, yk, acc, int(M), int(N),
                                               int(K), st);
  return dispatch_epilogue<BN, STAGES, false>(ta, tb, sx, sw, bias, y, yk, acc, int(M), int(N),
                                              int(K), st);
}

}  // namespace sqh
