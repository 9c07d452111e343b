// sq_gemm_skinny.cu -- the 8-bit GEMM + dequantization epilogue for a few
// tokens (M <= 16, the decode regime), sm_100a (tcgen05 + TMA + tensor memory).
//
//   acc[m,n] = sum_k Xq[m,k] * Wq[n,k]          (INT8: exact int32;
//                                                 E4M3: binary32 in TMEM)
//   y[m,n]   = bf16( ((float(acc) * sx[m]) * sw[n]) + bias[n] )
//
// Same results as the many-token kernel in sq_gemm.cu (bit for bit for INT8;
// the same operation order in the epilogue). Source: "Weight-Activation
// Quantization" (infra.bea.ai) §3 "Step 2" and §4; the grasp.study lesson on
// W8A16 vs W8A8 (decode with few tokens is bound by reading the weights).
//
// With 16 tokens the layer streams the whole weight once and does little
// arithmetic, so every staged byte should be a weight byte. The roles of
// the operands are swapped: 128 rows of Wq are the M = 128 operand of the
// tensor-core instruction and the (up to) 16 token rows of Xq the N = 16
// operand, so the accumulator holds D[n][m] = acc[m][n] in 128 lanes x 16
// columns of tensor memory. One CTA per 128 output channels streams its
// weight rows over all of K through a 3-stage ring; each stage holds 256
// contiguous bytes of K from each of the 128 weight rows (two 128-byte TMA
// boxes: 32 KB) and the matching token codes (4 KB). Two CTAs fit on an SM,
// so 224 CTAs at N = 28672 cover every SM with no split of K and no
// workspace. Reading 256 rather than 128 bytes of each row per stage cut the
// time by about 6 % (fewer, longer DRAM bursts per row).
//   warp 0    : TMA producer (Wq [128 rows x 2 x 128 B] + Xq [16 rows x
//               2 x 128 B], 128-byte swizzle; token rows beyond M and k
//               beyond K read as zero)
//   warps 1, 6: warp 1 allocates 64 tensor-memory columns (four accumulators
//               of 16 columns); one thread of each warp issues the MMAs of
//               alternate stages (K = 32 per instruction, eight per stage)
//               into its own two accumulators in turn, and frees ring slots
//               with tcgen05.commit. A single thread's stream of these short
//               MMAs is slow once commits are interleaved (about 200 ns per
//               instruction, measured on B200); the streams of different
//               warps overlap.
//   warps 2-5 : epilogue -- warp w reads lanes 32*(w%4)..+31 (its output
//               channels) x 16 columns (the tokens) of each accumulator, adds
//               them (int32, exact; E4M3 binary32 in a fixed order),
//               dequantizes and stores.
// Each CTA starts its k loop at a different k-block: all CTAs read the same
// token slices, which would otherwise be requested by every CTA at once.
// Every barrier wait is bounded: a wait that gives up records SQ_ERR_TIMEOUT,
// the CTA skips its remaining work, waits (bounded) for its copies and MMAs
// in flight and still frees tensor memory.
#include <cstdint>
#include <cstdlib>
#include <cuda.h>
#include <cuda_runtime.h>

#include "sq_common.cuh"
#include "sq_internal.h"

namespace sqk {

constexpr int kSkBK = 128;       // bytes of K per TMA box (one 128-byte swizzle row)
constexpr int kSkBoxes = 2;      // boxes per row per stage: 256 contiguous bytes of each weight row
constexpr int kSkMP = 16;        // token columns (N of the instruction)
constexpr int kSkStages = 3;
constexpr int kSkIssuers = 2;    // MMA-issuing threads: warps 1 and 6
constexpr int kSkMmaWarpB = 6;   // warp of the second issuer
constexpr int kSkThreads = 32 * (kSkMmaWarpB + kSkIssuers - 1);  // producer, MMA, 4 epilogue, MMA
constexpr uint32_t kSkABytes = 128 * kSkBK * kSkBoxes;     // weight slice
constexpr uint32_t kSkBBytes = kSkMP * kSkBK * kSkBoxes;   // token slice
constexpr uint32_t kSkStageBytes = kSkABytes + kSkBBytes;
constexpr uint32_t kSkBarOff = kSkStages * kSkStageBytes;
// barriers: full[S], empty[S], tfull, drain; then the TMEM slot and abort flag
constexpr uint32_t kSkMiscOff = kSkBarOff + (2 * kSkStages + 2) * 8;
constexpr uint32_t kSkDynamic = kSkMiscOff + 16 + 1024;  // slack for 1024-B alignment
constexpr int kSkNAcc = 2 * kSkIssuers;                  // two accumulators per issuer
constexpr uint32_t kSkTmemCols = kSkNAcc * 16;          // 16 columns each
static_assert(kSkTmemCols >= 32 && (kSkTmemCols & (kSkTmemCols - 1)) == 0,
              "tensor memory is allocated in powers of two of at least 32 columns");
static_assert(kSkStageBytes % 1024 == 0, "stages must keep 1024-byte alignment");
// an issuer waits for the release of a stage's previous use before waiting
// for it to fill; that bounds the barrier to one phase behind only while the
// issuer's own previous k-block (kb - kSkIssuers) is no older than that use
static_assert(kSkStages >= kSkIssuers, "an issuer must not skip a whole ring of stages");
static_assert(kSkDynamic * 2 + 2048 <= 233472, "two CTAs per SM must fit");

// 32 lanes x 16 consecutive 32-bit columns of tensor memory -> registers,
// with the wait in the same asm block so no use can be scheduled before it.
__device__ __forceinline__ void tmem_ld16_wait(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

template <bool E4M3, bool OUT_BF16, bool HAS_BIAS, bool WRITE_ACC>
__global__ void __launch_bounds__(kSkThreads, 2)
    gemm_skinny_kernel(const __grid_constant__ CUtensorMap tm_w,
                       const __grid_constant__ CUtensorMap tm_x, const float* __restrict__ sx,
                       const float* __restrict__ sw, const uint16_t* __restrict__ bias,
                       void* __restrict__ y, int32_t* __restrict__ acc_out, int M, int N, int K,
                       int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t bar_full = s_base + kSkBarOff;
  const uint32_t bar_empty = bar_full + kSkStages * 8;
  const uint32_t bar_tfull = bar_empty + kSkStages * 8;
  const uint32_t bar_drain = bar_tfull + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSkMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSkMiscOff + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = (K + kSkBK * kSkBoxes - 1) / (kSkBK * kSkBoxes);
  const int n_active = nk < kSkIssuers ? nk : kSkIssuers;  // issuers with k-blocks

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSkStages; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, 1);
    }
    mbar_init(bar_tfull, uint32_t(n_active));  // the MMA threads with k-blocks
    mbar_init(bar_drain, kSkIssuers);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_map(&tm_w);
    tma_prefetch_map(&tm_x);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kSkTmemCols);
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

  const int n0 = int(blockIdx.x) * 128;
  // every CTA reads the same token slices; starting each CTA at a different
  // k-block spreads those reads over the L2 instead of all CTAs asking for
  // the same lines at once (integer sums do not depend on the order)
  const int kb_rot = int(blockIdx.x) % nk;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      int issued = 0;
#pragma unroll 1
      for (int kb = 0; kb < nk; ++kb) {
        const uint32_t st = uint32_t(kb % kSkStages), ph = uint32_t(kb / kSkStages) & 1u;
        if (!mbar_wait(bar_empty + 8 * st, ph ^ 1u) || *abort_flag) {
          record_status(status, kStatusTimeout);
          *abort_flag = 1;
          break;
        }
        const uint32_t dst = s_base + st * kSkStageBytes;
        const int kbe = kb + kb_rot < nk ? kb + kb_rot : kb + kb_rot - nk;
        mbar_arrive_expect_tx(bar_full + 8 * st, kSkStageBytes);
#pragma unroll
        for (int b = 0; b < kSkBoxes; ++b) {
          const int kx = (kbe * kSkBoxes + b) * kSkBK;
          tma_load_2d(dst + b * 128 * kSkBK, &tm_w, bar_full + 8 * st, kx, n0);
          tma_load_2d(dst + kSkABytes + b * kSkMP * kSkBK, &tm_x, bar_full + 8 * st, kx, 0);
        }
        ++issued;
      }
      // no copy may still be writing shared memory when the CTA exits: wait
      // (bounded) for the last loads issued (already complete on the normal
      // path, where the MMA thread has consumed them)
      const int first = issued > kSkStages ? issued - kSkStages : 0;
#pragma unroll 1
      for (int j = first; j < issued; ++j)
        (void)mbar_wait(bar_full + 8 * uint32_t(j % kSkStages), uint32_t(j / kSkStages) & 1u);
    }
  } else if (warp == 1 || warp >= kSkMmaWarpB) {
    // ----------------------------------------------------------------- MMA --
    if (lane == 0) {
      constexpr uint32_t idesc = E4M3 ? idesc_e4m3_f32(128, kSkMP) : idesc_s8_s32(128, kSkMP);
      const int q = warp == 1 ? 0 : warp - kSkMmaWarpB + 1;
      bool ok = true;
      uint32_t j = 0;  // this thread's MMAs
#pragma unroll 1
      for (int kb = q; kb < nk; kb += kSkIssuers) {
        const uint32_t st = uint32_t(kb % kSkStages), ph = uint32_t(kb / kSkStages) & 1u;
        // The uses of a ring slot pass from issuer to issuer (six stages,
        // four issuers), so the previous use of this one may be another
        // thread's: wait for its commit (the phase the producer waits for
        // before refilling) first. Then the full barrier cannot be two phases
        // behind this wait, where its parity would match a completed phase.
        if (kb >= kSkStages && (!mbar_wait(bar_empty + 8 * st, ph ^ 1u) || *abort_flag)) {
          record_status(status, kStatusTimeout);
          *abort_flag = 1;
          ok = false;
          break;
        }
        if (!mbar_wait(bar_full + 8 * st, ph) || *abort_flag) {
          record_status(status, kStatusTimeout);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = s_base + st * kSkStageBytes;
        const uint32_t b_addr = a_addr + kSkABytes;
        // this thread's MMA j accumulates into accumulator 2 * q + j % 2
#pragma unroll
        for (int kk = 0; kk < kSkBoxes * kSkBK / 32; ++kk, ++j) {
          const uint64_t ad = sw128_desc(a_addr + (kk / 4) * 128 * kSkBK + (kk % 4) * 32);
          const uint64_t bd = sw128_desc(b_addr + (kk / 4) * kSkMP * kSkBK + (kk % 4) * 32);
          const uint32_t d = tmem_base + (2u * uint32_t(q) + j % 2u) * 16u;
          const uint32_t accum = j >= 2u ? 1u : 0u;
          if constexpr (E4M3) mma_f8(d, ad, bd, idesc, accum);
          else mma_i8(d, ad, bd, idesc, accum);
        }
        tc_commit(bar_empty + 8 * st);
      }
      if (ok && q < n_active) tc_commit(bar_tfull);  // the issuers with k-blocks
      // every MMA issued has finished before tensor memory can be freed
      tc_commit(bar_drain);
      (void)mbar_wait(bar_drain, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue --
    const int sub = warp & 3;  // TMEM lane quarter this warp may read
    const int n = n0 + sub * 32 + lane;
    if (!mbar_wait(bar_tfull, 0) || *abort_flag) {
      record_status(status, kStatusTimeout);
      *abort_flag = 1;
    } else {
      tc_fence_after();
      // the sum of the accumulators (exact for INT8; in a fixed order for E4M3)
      uint32_t r[16];
      tmem_ld16_wait(tmem_base + (uint32_t(sub * 32) << 16), r);
      // accumulators that received an MMA: both of every issuer with a
      // k-block (each k-block is four MMAs)
      const int n_acc = 2 * n_active;
#pragma unroll 1
      for (int c = 1; c < n_acc; ++c) {
        uint32_t r2[16];
        tmem_ld16_wait(tmem_base + (uint32_t(sub * 32) << 16) + uint32_t(c * 16), r2);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if constexpr (E4M3)
            r[j] = __float_as_uint(__fadd_rn(__uint_as_float(r[j]), __uint_as_float(r2[j])));
          else
            r[j] = uint32_t(int32_t(r[j]) + int32_t(r2[j]));
        }
      }
      if (n < N) {
        const float swn = __ldg(sw + n);
        float bn = 0.0f;
        if constexpr (HAS_BIAS) bn = __uint_as_float(uint32_t(__ldg(bias + n)) << 16);
#pragma unroll
        for (int m = 0; m < kSkMP; ++m) {
          if (m < M) {
            float a = E4M3 ? __uint_as_float(r[m]) : __int2float_rn(int32_t(r[m]));
            a = __fmul_rn(a, __ldg(sx + m));
            a = __fmul_rn(a, swn);
            if constexpr (HAS_BIAS) a = __fadd_rn(a, bn);
            const int64_t off = int64_t(m) * N + n;
            if constexpr (OUT_BF16)
              static_cast<uint16_t*>(y)[off] = uint16_t(pack_bf16x2(a, 0.0f) & 0xFFFFu);
            else
              static_cast<float*>(y)[off] = a;
            if constexpr (WRITE_ACC) acc_out[off] = int32_t(r[m]);
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
    tmem_dealloc(tmem_base, kSkTmemCols);
  }
}

}  // namespace sqk

namespace sqh {

using namespace sqk;

typedef CUresult (*SkEncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Tensor map of a row-major [rows, K] 8-bit matrix: box = box_rows x 128 B,
// 128-byte swizzle, out-of-range elements read as zero.
static bool sk_map(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int box_rows) {
  static SkEncodeTiledFn enc = nullptr;
  if (!enc) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    enc = reinterpret_cast<SkEncodeTiledFn>(p);
  }
  cuuint64_t dims[2] = {cuuint64_t(K), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(K)};
  cuuint32_t box[2] = {cuuint32_t(kSkBK), cuuint32_t(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool E4M3, bool OUT_BF16, bool HAS_BIAS, bool WRITE_ACC>
static cudaError_t run_skinny(const void* xq, const void* wq, const float* sx, const float* sw,
                              const uint16_t* bias, void* y, int32_t* acc, int M, int N, int K,
                              cudaStream_t st) {
  auto kern = gemm_skinny_kernel<E4M3, OUT_BF16, HAS_BIAS, WRITE_ACC>;
  CUtensorMap tw, tx;
  if (!sk_map(&tw, wq, N, K, 128) || !sk_map(&tx, xq, M, K, kSkMP)) return cudaErrorInvalidValue;
  static uint64_t attr_set = 0;  // one bit per device ordinal
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64 || !((attr_set >> dev) & 1u)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(kSkDynamic));
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set |= uint64_t(1) << dev;
  }
  return launch_pdl(kern, unsigned((N + 127) / 128), kSkThreads, size_t(kSkDynamic), st, tw, tx,
                    sx, sw, bias, y, acc, M, N, K, status_ptr());
}

bool gemm_skinny_applies(int64_t M) {
  return M >= 1 && M <= kSkMP && !getenv("SQ_GEMM_TILE") && !getenv("SQ_GEMM_NO_SKINNY");
}

cudaError_t launch_gemm_skinny(bool e4m3, const uint8_t* xq, const float* sx, const uint8_t* wq,
                               const float* sw, const uint16_t* bias, int64_t M, int64_t N,
                               int64_t K, void* y, OutKind yk, int32_t* acc, cudaStream_t st) {
  const int m = int(M), n = int(N), k = int(K);
  const int key = (e4m3 ? 8 : 0) | (yk == OutKind::BF16 ? 4 : 0) | (bias ? 2 : 0) | (acc ? 1 : 0);
#define SQ_SK(E, B, H, W) return run_skinny<E, B, H, W>(xq, wq, sx, sw, bias, y, acc, m, n, k, st)
  switch (key) {
    case 0: SQ_SK(false, false, false, false);
    case 1: SQ_SK(false, false, false, true);
    case 2: SQ_SK(false, false, true, false);
    case 3: SQ_SK(false, false, true, true);
    case 4: SQ_SK(false, true, false, false);
    case 5: SQ_SK(false, true, false, true);
    case 6: SQ_SK(false, true, true, false);
    case 7: SQ_SK(false, true, true, true);
    case 8: SQ_SK(true, false, false, false);
    case 9: SQ_SK(true, false, false, true);
    case 10: SQ_SK(true, false, true, false);
    case 11: SQ_SK(true, false, true, true);
    case 12: SQ_SK(true, true, false, false);
    case 13: SQ_SK(true, true, false, true);
    case 14: SQ_SK(true, true, true, false);
    default: SQ_SK(true, true, true, true);
  }
#undef SQ_SK
}

}  // namespace sqh
