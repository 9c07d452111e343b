// sq_gemm_small.cu -- the 8-bit GEMM + dequantization epilogue for problems
// whose 128 x 128 output tiles all fit on the SMs at once (one wave, e.g.
// prefill of 512 tokens), sm_100a (tcgen05 + TMA + tensor memory).
//
//   acc[m,n] = sum_k Xq[m,k] * Wq[n,k]          (INT8: exact int32;
//                                                 E4M3: binary32 in TMEM)
//   y[m,n]   = bf16( ((float(acc) * sx[m]) * sw[n]) + bias[n] )
//
// Same operation order and, for INT8, the same results bit for bit as the
// persistent kernel in sq_gemm.cu. Source: "Weight-Activation Quantization"
// (infra.bea.ai) §3 "Step 2" and §4; the zenaique page "W8A8 vs W4A16"
// (prefill is compute-bound and runs on the 8-bit tensor cores).
//
// With one tile per SM, the tile's own MMA stream is the critical path: a
// single issuing thread waits on the order of a hundred nanoseconds per
// tcgen05.mma once commits are interleaved (measured on B200), whatever the
// tile width, while issuing threads in different warps overlap. So each CTA
// splits its tile's K loop over four issuing threads, each accumulating
// every fourth k-block into its own 128-column accumulator (all 512 columns
// of tensor memory), and the epilogue adds the four.
//   warp 0     : TMA producer -- 128-byte K slices of the Xq and Wq tiles
//                [128 rows x 128 B each] into a 6-stage ring (128-byte swizzle)
//   warps 1..4 : warp 1 allocates tensor memory; lane 0 of warp 1 + q issues
//                the MMAs of k-blocks kb = q (mod 4) (K = 32 per instruction)
//                and frees their ring slots by tcgen05.commit
//   warps 1..8 : epilogue -- two warps per TMEM lane quarter, two 32-column
//                chunks each: the four partial accumulators are added (int32,
//                exact; E4M3 binary32 in a fixed order), dequantized and
//                stored from registers
// Every barrier wait is bounded: a wait that gives up records
// SQ_ERR_TIMEOUT, the CTA skips its remaining work, waits (bounded) for its
// copies and MMAs in flight and still frees tensor memory.
#include <cstdint>
#include <cstdlib>
#include <cuda.h>
#include <cuda_runtime.h>

#include "sq_common.cuh"
#include "sq_internal.h"

namespace sqk {

constexpr int kSmBK = 128;        // bytes of K per stage
constexpr int kSmTile = 128;      // output tile: 128 x 128
constexpr int kSmIssuers = 4;
constexpr int kSmStages = 6;
constexpr int kSmThreads = 32 * 9;  // producer + 8 (issuers, then epilogue)
constexpr uint32_t kSmOpBytes = kSmTile * kSmBK;            // one operand slice
constexpr uint32_t kSmStageBytes = 2 * kSmOpBytes;
constexpr uint32_t kSmBarOff = kSmStages * kSmStageBytes;
// barriers: full[S], empty[S], tfull, drain; then the TMEM slot and abort flag
constexpr uint32_t kSmMiscOff = kSmBarOff + (2 * kSmStages + 2) * 8;
constexpr uint32_t kSmDynamic = kSmMiscOff + 16 + 1024;   // slack for 1024-B alignment
constexpr uint32_t kSmTmemCols = 512;                      // four 128-column accumulators
static_assert(kSmStageBytes % 1024 == 0, "stages must keep 1024-byte alignment");
// an issuer waits for the release of a stage's previous use before waiting
// for it to fill; that bounds the barrier to one phase behind only while the
// issuer's own previous k-block (kb - kSmIssuers) is no older than that use
static_assert(kSmStages >= kSmIssuers, "an issuer must not skip a whole ring of stages");
static_assert(kSmDynamic + 1024 > 233472 / 2, "one CTA per SM (it holds all tensor memory)");
static_assert(kSmDynamic <= 232448, "shared memory budget exceeded");

template <bool E4M3, bool OUT_BF16, bool HAS_BIAS, bool WRITE_ACC>
__global__ void __launch_bounds__(kSmThreads, 1)
    gemm_small_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                      const float* __restrict__ sx, const float* __restrict__ sw,
                      const uint16_t* __restrict__ bias, void* __restrict__ y,
                      int32_t* __restrict__ acc_out, int M, int N, int K, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t bar_full = s_base + kSmBarOff;
  const uint32_t bar_empty = bar_full + kSmStages * 8;
  const uint32_t bar_tfull = bar_empty + kSmStages * 8;
  const uint32_t bar_drain = bar_tfull + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSmMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSmMiscOff + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = (K + kSmBK - 1) / kSmBK;
  const int n_issuers = nk < kSmIssuers ? nk : kSmIssuers;  // threads with k-blocks

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSmStages; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, 1);
    }
    mbar_init(bar_tfull, uint32_t(n_issuers));
    mbar_init(bar_drain, uint32_t(kSmIssuers));
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_map(&tm_a);
    tma_prefetch_map(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kSmTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // set-up above overlaps the previous kernel; its results are read below.
  // The next kernel may start only after that wait: by then every kernel
  // before this one has completed, which lets an activation pass that
  // overlaps this grid (SQ_OVERLAP_PREVIOUS) reuse the buffers of the GEMM
  // before this one
  pdl_wait();
  pdl_launch_dependents();

  const int num_nt = (N + kSmTile - 1) / kSmTile;
  const int mt = int(blockIdx.x) / num_nt, nt = int(blockIdx.x) - mt * num_nt;
  const int m0 = mt * kSmTile, n0 = nt * kSmTile;
  auto give_up = [&]() {
    record_status(status, kStatusTimeout);
    *abort_flag = 1;
  };

  bool ok = true;
  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      int issued = 0;
#pragma unroll 1
      for (int kb = 0; kb < nk; ++kb) {
        const uint32_t st = uint32_t(kb % kSmStages), ph = uint32_t(kb / kSmStages) & 1u;
        if (*abort_flag || !mbar_wait(bar_empty + 8 * st, ph ^ 1u)) {
          give_up();
          break;
        }
        const uint32_t dst = s_base + st * kSmStageBytes;
        mbar_arrive_expect_tx(bar_full + 8 * st, kSmStageBytes);
        tma_load_2d(dst, &tm_a, bar_full + 8 * st, kb * kSmBK, m0);
        tma_load_2d(dst + kSmOpBytes, &tm_b, bar_full + 8 * st, kb * kSmBK, n0);
        ++issued;
      }
      // no copy may still be writing shared memory when the CTA exits
      const int first = issued > kSmStages ? issued - kSmStages : 0;
#pragma unroll 1
      for (int j = first; j < issued; ++j)
        (void)mbar_wait(bar_full + 8 * uint32_t(j % kSmStages), uint32_t(j / kSmStages) & 1u);
    }
  } else {
    if (warp <= kSmIssuers && lane == 0) {
      // ------------------------------------------------------------- MMA --
      const int q = warp - 1;
      constexpr uint32_t idesc =
          E4M3 ? idesc_e4m3_f32(kSmTile, kSmTile) : idesc_s8_s32(kSmTile, kSmTile);
      const uint32_t d = tmem_base + uint32_t(q) * kSmTile;
#pragma unroll 1
      for (int kb = q; kb < nk; kb += kSmIssuers) {
        const uint32_t st = uint32_t(kb % kSmStages), ph = uint32_t(kb / kSmStages) & 1u;
        // The uses of a ring slot pass from issuer to issuer (six stages,
        // four issuers), so the previous use of this one may be another
        // thread's: wait for its commit (the phase the producer waits for
        // before refilling) first. Then the full barrier cannot be two phases
        // behind this wait, where its parity would match a completed phase.
        if (kb >= kSmStages && (*abort_flag || !mbar_wait(bar_empty + 8 * st, ph ^ 1u))) {
          give_up();
          ok = false;
          break;
        }
        if (*abort_flag || !mbar_wait(bar_full + 8 * st, ph)) {
          give_up();
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = s_base + st * kSmStageBytes;
        const uint32_t b_addr = a_addr + kSmOpBytes;
#pragma unroll
        for (int kk = 0; kk < kSmBK / 32; ++kk) {
          const uint64_t ad = sw128_desc(a_addr + kk * 32);
          const uint64_t bd = sw128_desc(b_addr + kk * 32);
          const uint32_t accum = (kb > q || kk > 0) ? 1u : 0u;
          if constexpr (E4M3) mma_f8(d, ad, bd, idesc, accum);
          else mma_i8(d, ad, bd, idesc, accum);
        }
        tc_commit(bar_empty + 8 * st);
      }
      if (ok && q < n_issuers) tc_commit(bar_tfull);
      // every MMA issued has finished before tensor memory can be freed
      tc_commit(bar_drain);
      (void)mbar_wait(bar_drain, 0);
    }
    __syncwarp();
    // ------------------------------------------------------------ epilogue --
    const int quarter = warp & 3;      // TMEM lane quarter this warp may read
    const int half = (warp - 1) >> 2;  // which warp of the quarter: chunks 2*half, 2*half+1
    const int m = m0 + quarter * 32 + lane;
    const uint32_t t_lane = tmem_base + (uint32_t(quarter * 32) << 16);
    if (*abort_flag || !mbar_wait(bar_tfull, 0)) {
      give_up();
    } else if (m0 + quarter * 32 < M) {
      tc_fence_after();
      const float sxm = m < M ? __ldg(sx + m) : 0.0f;
#pragma unroll 1
      for (int c = 2 * half; c < 2 * half + 2; ++c) {
        const int nb = n0 + c * 32;
        if (nb >= N) break;
        // the partial sums of this chunk, added in the fixed order 0 + 1 + 2 + 3
        uint32_t r[32], r2[32];
        tmem_ld32(t_lane + uint32_t(c * 32), r);
        if (n_issuers > 1) {
          tmem_ld32(t_lane + uint32_t(c * 32 + kSmTile), r2);
          tmem_wait_ld2(r, r2);
        } else {
          tmem_wait_ld(r);
        }
#pragma unroll 1
        for (int q = 1; q < n_issuers; ++q) {
          if (q > 1) {
            tmem_ld32(t_lane + uint32_t(c * 32 + q * kSmTile), r2);
            tmem_wait_ld(r2);
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if constexpr (E4M3)
              r[j] = __float_as_uint(__fadd_rn(__uint_as_float(r[j]), __uint_as_float(r2[j])));
            else
              r[j] = uint32_t(int32_t(r[j]) + int32_t(r2[j]));
          }
        }
        if (m >= M) continue;
        // eight columns at a time (N is a multiple of 8)
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int n = nb + g * 8;
          if (n >= N) break;
          const float4 w0 = __ldg(reinterpret_cast<const float4*>(sw + n));
          const float4 w1 = __ldg(reinterpret_cast<const float4*>(sw + n) + 1);
          const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
          float bv[8];
          if constexpr (HAS_BIAS) {
            const uint4 b = __ldg(reinterpret_cast<const uint4*>(bias + n));
            bv[0] = bf16_lo(b.x); bv[1] = bf16_hi(b.x);
            bv[2] = bf16_lo(b.y); bv[3] = bf16_hi(b.y);
            bv[4] = bf16_lo(b.z); bv[5] = bf16_hi(b.z);
            bv[6] = bf16_lo(b.w); bv[7] = bf16_hi(b.w);
          }
          float t[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t raw = r[g * 8 + i];
            float a = E4M3 ? __uint_as_float(raw) : __int2float_rn(int32_t(raw));
            a = __fmul_rn(a, sxm);
            a = __fmul_rn(a, wv[i]);
            if constexpr (HAS_BIAS) a = __fadd_rn(a, bv[i]);
            t[i] = a;
          }
          const int64_t off = int64_t(m) * N + n;
          if constexpr (OUT_BF16) {
            *reinterpret_cast<uint4*>(static_cast<uint16_t*>(y) + off) =
                make_uint4(pack_bf16x2(t[0], t[1]), pack_bf16x2(t[2], t[3]),
                           pack_bf16x2(t[4], t[5]), pack_bf16x2(t[6], t[7]));
          } else {
            float4* p = reinterpret_cast<float4*>(static_cast<float*>(y) + off);
            p[0] = make_float4(t[0], t[1], t[2], t[3]);
            p[1] = make_float4(t[4], t[5], t[6], t[7]);
          }
          if constexpr (WRITE_ACC) {
            int4* p = reinterpret_cast<int4*>(acc_out + off);
            p[0] = make_int4(int(r[g * 8 + 0]), int(r[g * 8 + 1]), int(r[g * 8 + 2]), int(r[g * 8 + 3]));
            p[1] = make_int4(int(r[g * 8 + 4]), int(r[g * 8 + 5]), int(r[g * 8 + 6]), int(r[g * 8 + 7]));
          }
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kSmTmemCols);
  }
}

}  // namespace sqk

namespace sqh {

using namespace sqk;

typedef CUresult (*SmEncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Tensor map of a row-major [rows, K] 8-bit matrix: box = 128 rows x 128 B,
// 128-byte swizzle, out-of-range elements read as zero.
static bool sm_map(CUtensorMap* map, const void* base, int64_t rows, int64_t K) {
  static SmEncodeTiledFn enc = nullptr;
  if (!enc) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    enc = reinterpret_cast<SmEncodeTiledFn>(p);
  }
  cuuint64_t dims[2] = {cuuint64_t(K), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(K)};
  cuuint32_t box[2] = {cuuint32_t(kSmBK), cuuint32_t(kSmTile)};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int small_sms() {
  static int n[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (n[dev] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    n[dev] = v > 0 ? v : 148;
  }
  return n[dev];
}

bool gemm_small_applies(int64_t M, int64_t N, int64_t K) {
  if (getenv("SQ_GEMM_TILE") || getenv("SQ_GEMM_NO_SMALL")) return false;
  const int64_t tiles = ((M + kSmTile - 1) / kSmTile) * ((N + kSmTile - 1) / kSmTile);
  // one wave of 128 x 128 tiles, and at least two k-blocks per issuing thread
  return tiles <= small_sms() && K >= 2 * kSmIssuers * kSmBK;
}

template <bool E4M3, bool OUT_BF16, bool HAS_BIAS, bool WRITE_ACC>
static cudaError_t run_small(const void* xq, const void* wq, const float* sx, const float* sw,
                             const uint16_t* bias, void* y, int32_t* acc, int M, int N, int K,
                             cudaStream_t st) {
  auto kern = gemm_small_kernel<E4M3, OUT_BF16, HAS_BIAS, WRITE_ACC>;
  CUtensorMap ta, tb;
  if (!sm_map(&ta, xq, M, K) || !sm_map(&tb, wq, N, K)) return cudaErrorInvalidValue;
  static uint64_t attr_set = 0;  // one bit per device ordinal
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64 || !((attr_set >> dev) & 1u)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(kSmDynamic));
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set |= uint64_t(1) << dev;
  }
  const unsigned tiles = unsigned(((M + kSmTile - 1) / kSmTile) * ((N + kSmTile - 1) / kSmTile));
  return launch_pdl(kern, tiles, kSmThreads, size_t(kSmDynamic), st, ta, tb, sx, sw, bias, y, acc,
                    M, N, K, status_ptr());
}

cudaError_t launch_gemm_small(bool e4m3, const uint8_t* xq, const float* sx, const uint8_t* wq,
                              const float* sw, const uint16_t* bias, int64_t M, int64_t N,
                              int64_t K, void* y, OutKind yk, int32_t* acc, cudaStream_t st) {
  const int m = int(M), n = int(N), k = int(K);
  const int key = (e4m3 ? 8 : 0) | (yk == OutKind::BF16 ? 4 : 0) | (bias ? 2 : 0) | (acc ? 1 : 0);
#define SQ_SM(E, B, H, W) return run_small<E, B, H, W>(xq, wq, sx, sw, bias, y, acc, m, n, k, st)
  switch (key) {
    case 0: SQ_SM(false, false, false, false);
    case 1: SQ_SM(false, false, false, true);
    case 2: SQ_SM(false, false, true, false);
    case 3: SQ_SM(false, false, true, true);
    case 4: SQ_SM(false, true, false, false);
    case 5: SQ_SM(false, true, false, true);
    case 6: SQ_SM(false, true, true, false);
    case 7: SQ_SM(false, true, true, true);
    case 8: SQ_SM(true, false, false, false);
    case 9: SQ_SM(true, false, false, true);
    case 10: SQ_SM(true, false, true, false);
    case 11: SQ_SM(true, false, true, true);
    case 12: SQ_SM(true, true, false, false);
    case 13: SQ_SM(true, true, false, true);
    case 14: SQ_SM(true, true, true, false);
    default: SQ_SM(true, true, true, true);
  }
#undef SQ_SM
}

}  // namespace sqh
