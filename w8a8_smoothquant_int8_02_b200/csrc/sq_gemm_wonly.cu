// sq_gemm_wonly.cu -- weight-only quantized GEMM for few tokens (decode),
// sm_100a (tcgen05 + TMA + tensor memory): W8A16 and W4A16.
//
//   y[m,n] = bf16( float( sum_k x[m,k] * q[n,k] ) * sw[n] + bias[n] )
//
// x is bf16 [M,K]; q are the per-output-channel weight codes (INT8 [N,K], or
// INT4 [N,K/2] packed eight per 32-bit word, see sq_quantize_weight) with
// scales sw [N]. Source: the pages' weight-only schemes -- "Weight-Activation
// Quantization" (infra.bea.ai) §1 table (W4A16: INT4 weights dequantized to
// 16 bits, then a 16-bit multiply), the zenaique flashcard on activation
// quantization (the runtime dequantizes the weights on the fly against BF16
// activations), the grasp.study lesson on W8A16 vs W8A8 §1 and §3, and the
// zenaique "W8A8 vs W4A16" page (decode is bound by the weight read; 4-bit
// weights read half the bytes of 8-bit ones).
//
// Dequantization: every INT8 / INT4 code is exactly representable in bf16,
// so the codes are widened to bf16 and multiplied by the bf16 activations on
// the tensor cores (kind::f16, binary32 accumulators in tensor memory); the
// channel scale sw[n] is constant along k, so it is applied once to the sum
// in the epilogue: sum_k x * (q * sw) = sw * sum_k x * q.
//
// Roles are swapped as in the few-token W8A8 kernel: 128 weight rows are the
// M = 128 operand, the (up to) 16 token rows the N = 16 operand, D[n][m] in
// 128 lanes x 16 columns of tensor memory. One CTA per 128 output channels
// and 16 tokens (grid.y walks token tiles of larger batches); two CTAs per SM.
//   warp 0      : weight producer -- per stage one 128-byte-wide K slice of
//                 the packed weights [128 rows x 128 B] (128 k for INT8, 256
//                 for INT4) into a 5-stage ring (128-byte swizzle)
//   warp 10     : token producer -- the matching bf16 token slices [16 rows
//                 x 64 k] into a ring of their own
//   warps 2..9  : two groups of four (one warp per lane quarter) taking
//                 alternate 64-k sub-tiles of each stage: each thread loads
//                 its weight row's codes of the stage into registers and
//                 releases the weight slot at once (the weight stream never
//                 waits for the tensor cores), then widens the codes to bf16
//                 pairs and stores them to tensor memory (tcgen05.st), a
//                 6-deep ring of A sub-tiles; warps 2..5 then run the
//                 epilogue, which adds the accumulators in a fixed order
//   warps 1, 11..13: warp 1 allocates tensor memory (256 columns: four
//                 accumulators and the A ring); one thread of each warp
//                 issues the MMAs of every fourth sub-tile (A from tensor
//                 memory, B = the token slice from shared memory, K = 16 per
//                 instruction) into its own accumulator, and frees A slots
//                 and token slots by tcgen05.commit. A single thread's stream
//                 of these short instructions is slow once commits are
//                 interleaved (about 200 ns per instruction, measured on
//                 B200); the streams of different warps overlap.
// Each CTA starts its k loop at a different k-block: all CTAs read the same
// token slices, which would otherwise be requested by every CTA at once.
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

constexpr int kWoTokens = 16;                 // token columns (N of the instruction)
constexpr int kWoConvWarps = 8;               // two groups of four, alternating sub-tiles
constexpr int kWoIssuers = 4;                 // MMA-issuing threads, one accumulator each
constexpr int kWoXWarp = 2 + kWoConvWarps;     // the token-slice producer
constexpr int kWoMmaWarpB = kWoXWarp + 1;      // warps of issuers 1.. (issuer 0 is warp 1)
constexpr int kWoThreads = 32 * (kWoMmaWarpB + kWoIssuers - 1);
constexpr uint32_t kWoWBytes = 128 * 128;     // packed weight slice of one stage
constexpr uint32_t kWoXSub = kWoTokens * 128; // bf16 token sub-tile [16 x 64 k]
constexpr uint32_t kWoTmemCols = 256;         // per CTA: accumulators + A ring
constexpr int kWoNAcc = kWoIssuers;           // accumulators (16 columns each)
constexpr uint32_t kWoAColBase = kWoNAcc * 16;  // first A column
constexpr int kWoNA = 6;                      // A sub-tiles in tensor memory (32 columns each)

// Two rings: packed weight slices (released by the widening warps as soon as
// they hold their codes in registers) and the matching token slices (released
// by the MMAs that read them), so the weight stream does not wait for the
// tensor cores.
template <int BITS>
struct WoCfg {
  static constexpr int KS = BITS == 8 ? 128 : 256;   // k per weight stage (128 B per row)
  static constexpr int SUBS = KS / 64;               // 64-k sub-tiles per stage
  static constexpr int SW = 5;                       // weight ring
  static constexpr int SX = BITS == 8 ? 7 : 3;       // token ring
  static constexpr uint32_t kXBytes = SUBS * kWoXSub;
  static constexpr uint32_t kXOff = SW * kWoWBytes;
  static constexpr uint32_t kBarOff = kXOff + SX * kXBytes;
  // barriers: wfull[SW], wempty[SW], xfull[SX], xempty[SX], afull[NA],
  // aempty[NA], tfull, drain; then the TMEM slot and the abort flag
  static constexpr uint32_t kMiscOff = kBarOff + (2 * SW + 2 * SX + 2 * kWoNA + 2) * 8;
  static constexpr uint32_t kDynamic = kMiscOff + 16 + 1024;  // slack for 1024-B alignment
  static_assert(kWoWBytes % 1024 == 0 && kXBytes % 1024 == 0,
                "ring slots must keep 1024-byte alignment");
  static_assert(2 * (kDynamic + 1024) <= 233472, "two CTAs per SM must fit");
  static_assert(SUBS % 2 == 0 && kWoNA % 2 == 0,
                "each A slot must be filled by one widening group only");
  // an issuer's consecutive token stages are kWoIssuers / SUBS apart (1 when
  // it has a sub-tile in every stage); the wait for the previous use of a
  // slot bounds the barrier to one phase behind only if that gap is no
  // larger than the ring
  static_assert(SUBS >= kWoIssuers || kWoIssuers / SUBS <= SX,
                "an issuer must not skip a whole ring of token stages");
};
static_assert(kWoAColBase + kWoNA * 32 <= kWoTmemCols, "A ring must fit the allocation");
static_assert(kWoNA >= kWoIssuers, "every issuer needs an A slot of its own in flight");

// Instruction descriptor of tcgen05.mma kind::f16 with bf16 A and B and
// binary32 accumulators: bits 4-5 D format, 7-9 / 10-12 A / B formats,
// 17-22 N/8, 24-28 M/16 (A and B not transposed).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int m, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}

// D[tmem] (+)= A[tmem] * B[smem]^T, bf16 operands, binary32 accumulators: A
// is read from tensor memory (row m in lane m, two k per 32-bit column).
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// registers -> 32 lanes x 32 consecutive 32-bit columns of tensor memory
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0],"
      " {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16,"
      " %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
        "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
        "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]),
        "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// bf16x2 a - b, rounded to nearest (exact here: every result is a small integer)
__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Widening of 8-bit codes to bf16 without a conversion instruction. A code c
// is split into its low seven bits v and its sign bit s (two's complement:
// c = v - 128 s). The bf16 with bits 0x4300 | v is 128 + v (exponent 2^7,
// one unit per mantissa step) and 0x4300 | (sign bit in place) is
// 128 + 128 s; their bf16 difference is c exactly. Two codes at bit
// 0 and bit 16 of a word give two bf16 at once (the low half is the first).
__device__ __forceinline__ uint32_t codes_to_bf16x2(uint32_t w) {
  return bf16x2_sub((w & 0x007F007Fu) | 0x43004300u, (w & 0x00800080u) | 0x43004300u);
}

// The same for 4-bit codes in one logic operation: a code c in [-8, 7] is
// the nibble n = c mod 16, and n ^ 8 = c + 8. (w & 0x000F000F) ^ 0x43084308
// keeps bits 0-2 of each nibble, inverts bit 3 and sets the bits of 0x4300,
// giving the bf16 128 + (c + 8); subtracting 136 leaves c exactly.
__device__ __forceinline__ uint32_t nibbles_to_bf16x2(uint32_t w) {
  return bf16x2_sub((w & 0x000F000Fu) ^ 0x43084308u, 0x43084308u);
}

__device__ __forceinline__ uint32_t sw128_off(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

__device__ __forceinline__ void tmem_ld16_wait_wo(uint32_t taddr, uint32_t (&r)[16]) {
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

template <int BITS, bool OUT_BF16, bool HAS_BIAS>
__global__ void __launch_bounds__(kWoThreads, 2)
    gemm_wonly_kernel(const __grid_constant__ CUtensorMap tm_w,
                      const __grid_constant__ CUtensorMap tm_x, const float* __restrict__ sw,
                      const uint16_t* __restrict__ bias, void* __restrict__ y, int M, int N,
                      int K, int* status) {
  using C = WoCfg<BITS>;
  constexpr int SW = C::SW, SX = C::SX, NA = kWoNA, SUBS = C::SUBS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t bar_wfull = s_base + C::kBarOff;
  const uint32_t bar_wempty = bar_wfull + SW * 8;
  const uint32_t bar_xfull = bar_wempty + SW * 8;
  const uint32_t bar_xempty = bar_xfull + SX * 8;
  const uint32_t bar_afull = bar_xempty + SX * 8;
  const uint32_t bar_aempty = bar_afull + NA * 8;
  const uint32_t bar_tfull = bar_aempty + NA * 8;
  const uint32_t bar_drain = bar_tfull + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = (K + C::KS - 1) / C::KS;
  // issuer q takes the sub-tiles ia with ia % kWoIssuers == q: a stage holds
  // SUBS consecutive sub-tiles, so SUBS issuers (at most all) use each one
  constexpr int kStageIssuers = SUBS < kWoIssuers ? SUBS : kWoIssuers;
  static_assert(kWoIssuers % SUBS == 0 || SUBS % kWoIssuers == 0,
                "the issuers of a stage must be SUBS distinct threads");
  const int n_sub = nk * SUBS;
  const int n_active = n_sub < kWoIssuers ? n_sub : kWoIssuers;  // issuers with sub-tiles

  if (threadIdx.x == 0) {
    for (int i = 0; i < SW; ++i) {
      mbar_init(bar_wfull + 8 * i, 1);
      mbar_init(bar_wempty + 8 * i, kWoConvWarps);    // every widening warp
    }
    for (int i = 0; i < SX; ++i) {
      mbar_init(bar_xfull + 8 * i, 1);
      mbar_init(bar_xempty + 8 * i, kStageIssuers);   // the issuers with a sub-tile in it
    }
    for (int i = 0; i < NA; ++i) {
      mbar_init(bar_afull + 8 * i, 4);                 // the four warps of one group
      mbar_init(bar_aempty + 8 * i, 1);
    }
    mbar_init(bar_tfull, uint32_t(n_active));
    mbar_init(bar_drain, kWoIssuers);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_map(&tm_w);
    tma_prefetch_map(&tm_x);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kWoTmemCols);
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
  const int m0 = int(blockIdx.y) * kWoTokens;
  // every CTA reads the same token slices; starting each CTA at a different
  // k-block spreads those reads over the L2 instead of all CTAs asking for
  // the same lines at once (the sum is the same up to binary32 rounding)
  const int kb_rot = int(blockIdx.x) % nk;
  auto give_up = [&]() {
    record_status(status, kStatusTimeout);
    *abort_flag = 1;
  };

  if (warp == 0 || warp == kWoXWarp) {
    // ----------------------------------------------------------- producers --
    // warp 0 streams the packed weights, the token-slice warp the matching
    // bf16 token slices; each is the only writer of its ring
    if (lane == 0) {
      const bool is_w = warp == 0;
      const int ns = is_w ? SW : SX;
      const uint32_t full = is_w ? bar_wfull : bar_xfull;
      const uint32_t empty = is_w ? bar_wempty : bar_xempty;
      int issued = 0;
#pragma unroll 1
      for (int kb = 0; kb < nk; ++kb) {
        const uint32_t st = uint32_t(kb % ns), ph = uint32_t(kb / ns) & 1u;
        if (*abort_flag || !mbar_wait(empty + 8 * st, ph ^ 1u)) {
          give_up();
          break;
        }
        const int kbe = kb + kb_rot < nk ? kb + kb_rot : kb + kb_rot - nk;
        if (is_w) {
          mbar_arrive_expect_tx(full + 8 * st, kWoWBytes);
          tma_load_2d(s_base + st * kWoWBytes, &tm_w, full + 8 * st, kbe * 128, n0);
        } else {
          const uint32_t dst = s_base + C::kXOff + st * C::kXBytes;
          mbar_arrive_expect_tx(full + 8 * st, C::kXBytes);
#pragma unroll
          for (int t = 0; t < SUBS; ++t)
            tma_load_2d(dst + t * kWoXSub, &tm_x, full + 8 * st, kbe * C::KS + t * 64, m0);
        }
        ++issued;
      }
      // no copy may still be writing shared memory when the CTA exits
      const int first = issued > ns ? issued - ns : 0;
#pragma unroll 1
      for (int j = first; j < issued; ++j)
        (void)mbar_wait(full + 8 * uint32_t(j % ns), uint32_t(j / ns) & 1u);
    }
  } else if (warp == 1 || warp >= kWoMmaWarpB) {
    // ----------------------------------------------------------------- MMA --
    // Four issuing threads, issuer q taking the sub-tiles ia = q (mod 4),
    // each into its own accumulator: a single thread's stream of these short
    // tcgen05.mma instructions is slow once commits are interleaved, while
    // the streams of different warps overlap.
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, kWoTokens);
      const uint32_t q = warp == 1 ? 0u : uint32_t(warp - kWoMmaWarpB + 1);
      const uint32_t d = tmem_base + q * 16u;
      bool ok = true;
      uint32_t j = 0;  // this thread's MMAs so far
#pragma unroll 1
      for (int kb = 0; kb < nk && ok; ++kb) {
        // sub-tiles SUBS*kb .. SUBS*kb + SUBS-1: is one of them this thread's?
        const uint32_t ia0 = uint32_t(kb) * SUBS;
        const uint32_t t0 = (q + kWoIssuers - ia0 % kWoIssuers) % kWoIssuers;
        if (t0 >= uint32_t(SUBS)) continue;
        const uint32_t xs = uint32_t(kb % SX), ph = uint32_t(kb / SX) & 1u;
        // The issuers of a token slot change from one use of it to the next,
        // so the previous use may be other threads': wait for its release
        // (the phase the producer waits for before refilling) first. Then
        // the full barrier cannot be two phases behind this wait, where its
        // parity would match a completed phase.
        if (kb >= SX && (*abort_flag || !mbar_wait(bar_xempty + 8 * xs, ph ^ 1u))) {
          give_up();
          ok = false;
          break;
        }
        if (*abort_flag || !mbar_wait(bar_xfull + 8 * xs, ph)) {
          give_up();
          ok = false;
          break;
        }
        const uint32_t x_addr = s_base + C::kXOff + xs * C::kXBytes;
#pragma unroll 1
        for (uint32_t t = t0; t < uint32_t(SUBS); t += kWoIssuers) {
          const uint32_t ia = ia0 + t;
          const uint32_t slot = ia % NA;
          // the same for the A slots: the previous use of this slot may
          // have been another issuer's
          if (ia >= uint32_t(NA) &&
              (*abort_flag || !mbar_wait(bar_aempty + 8 * slot, ((ia / NA) & 1u) ^ 1u))) {
            give_up();
            ok = false;
            break;
          }
          if (*abort_flag || !mbar_wait(bar_afull + 8 * slot, (ia / NA) & 1u)) {
            give_up();
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_tmem = tmem_base + kWoAColBase + slot * 32u;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk, ++j) {
            const uint64_t bd = sw128_desc(x_addr + t * kWoXSub + kk * 32);
            mma_bf16_ts(d, a_tmem + uint32_t(kk * 8), bd, idesc, j > 0u ? 1u : 0u);
          }
          tc_commit(bar_aempty + 8 * slot);
        }
        if (!ok) break;
        tc_commit(bar_xempty + 8 * xs);  // this thread is done with the slot's token slices
      }
      if (ok && q < uint32_t(n_active)) tc_commit(bar_tfull);
      // every MMA issued has finished before tensor memory can be freed
      tc_commit(bar_drain);
      (void)mbar_wait(bar_drain, 0);
    }
  } else {
    // ------------------------------------------- widening, then epilogue --
    const int cw = warp - 2;                   // 0 .. kWoConvWarps - 1
    const int quarter = warp & 3;              // TMEM lane quarter this warp may access
    const int group = cw >> 2;                 // sub-tiles t of a stage with t % 2 == group
    const uint32_t row = uint32_t(quarter) * 32u + uint32_t(lane);  // weight row of the tile
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    constexpr int kChunks = BITS == 8 ? 4 : 2;  // 16-byte chunks of a row per sub-tile
    constexpr int kMySubs = SUBS / 2;           // this group's sub-tiles per stage
    bool ok = true;
#pragma unroll 1
    for (int kb = 0; kb < nk && ok; ++kb) {
      const uint32_t st = uint32_t(kb % SW), ph = uint32_t(kb / SW) & 1u;
      if (*abort_flag || !mbar_wait(bar_wfull + 8 * st, ph)) {
        give_up();
        ok = false;
        break;
      }
      // this thread's codes of the stage into registers, then the weight
      // slot is released: the producer refills it while the codes are widened
      uint4 raw[kMySubs * kChunks];
      const uint8_t* wsrc = smem + st * kWoWBytes;
#pragma unroll
      for (int u = 0; u < kMySubs; ++u)
#pragma unroll
        for (int h = 0; h < kChunks; ++h)
          raw[u * kChunks + h] = *reinterpret_cast<const uint4*>(
              wsrc + sw128_off(row, uint32_t(kChunks * (2 * u + group) + h)));
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_wempty + 8 * st);
#pragma unroll
      for (int u = 0; u < kMySubs; ++u) {
        const uint32_t ia = uint32_t(kb) * SUBS + uint32_t(2 * u + group);
        const uint32_t slot = ia % NA;  // slots of one parity belong to one group
        if (*abort_flag || !mbar_wait(bar_aempty + 8 * slot, ((ia / NA) & 1u) ^ 1u)) {
          give_up();
          ok = false;
          break;
        }
        tc_fence_after();
        // this row's 64 codes of the sub-tile -> 32 bf16 pairs (k order)
        uint32_t a[32];
        if constexpr (BITS == 8) {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const uint4 q = raw[u * kChunks + h];
            const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              // bytes (c0 c1 c2 c3) -> (c0 c2 c1 c3): c0, c1 at bits 0 / 16
              const uint32_t p = __byte_perm(qw[i], 0u, 0x3120);
              a[8 * h + 2 * i] = codes_to_bf16x2(p);
              a[8 * h + 2 * i + 1] = codes_to_bf16x2(p >> 8);
            }
          }
        } else {
          // each 32-bit word holds 8 codes: even k at bits 0,4,8,12, odd k
          // at 16,20,24,28
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint4 q = raw[u * kChunks + h];
            const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
#pragma unroll
              for (int jj = 0; jj < 4; ++jj)
                a[16 * h + 4 * i + jj] = nibbles_to_bf16x2(qw[i] >> (4 * jj));
            }
          }
        }
        tmem_st32(tmem_base + lane_off + kWoAColBase + slot * 32u, a);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_afull + 8 * slot);
      }
    }
    if (cw < 4) {
      // epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 = output channels
      const int n = n0 + quarter * 32 + lane;
      if (!ok || *abort_flag || !mbar_wait(bar_tfull, 0)) {
        give_up();
      } else {
        tc_fence_after();
        // the sum of the accumulators of the issuers that had sub-tiles, in
        // a fixed order
        uint32_t r[16];
        tmem_ld16_wait_wo(tmem_base + lane_off, r);
#pragma unroll 1
        for (int c = 1; c < n_active; ++c) {
          uint32_t r2[16];
          tmem_ld16_wait_wo(tmem_base + lane_off + uint32_t(c * 16), r2);
#pragma unroll
          for (int j = 0; j < 16; ++j)
            r[j] = __float_as_uint(__fadd_rn(__uint_as_float(r[j]), __uint_as_float(r2[j])));
        }
        if (n < N) {
          const float swn = __ldg(sw + n);
          float bn = 0.0f;
          if constexpr (HAS_BIAS) bn = __uint_as_float(uint32_t(__ldg(bias + n)) << 16);
#pragma unroll
          for (int j = 0; j < kWoTokens; ++j) {
            const int m = m0 + j;
            if (m < M) {
              float v = __fmul_rn(__uint_as_float(r[j]), swn);
              if constexpr (HAS_BIAS) v = __fadd_rn(v, bn);
              const int64_t off = int64_t(m) * N + n;
              if constexpr (OUT_BF16)
                static_cast<uint16_t*>(y)[off] = uint16_t(pack_bf16x2(v, 0.0f) & 0xFFFFu);
              else
                static_cast<float*>(y)[off] = v;
            }
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
    tmem_dealloc(tmem_base, kWoTmemCols);
  }
}

}  // namespace sqk

namespace sqh {

using namespace sqk;

typedef CUresult (*WoEncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static WoEncodeTiledFn wo_encoder() {
  static WoEncodeTiledFn enc = nullptr;
  if (!enc) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      enc = reinterpret_cast<WoEncodeTiledFn>(p);
  }
  return enc;
}

// Row-major [rows, cols] matrix of `elem` bytes per element: box = box_cols x
// box_rows (box_cols * elem = 128 bytes), 128-byte swizzle, zero fill.
static bool wo_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem,
                   int64_t rows, int64_t cols, int box_cols, int box_rows) {
  WoEncodeTiledFn enc = wo_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(cols) * cuuint64_t(elem)};
  cuuint32_t box[2] = {cuuint32_t(box_cols), cuuint32_t(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BITS, bool OUT_BF16, bool HAS_BIAS>
static cudaError_t run_wonly(const void* x, const void* wq, const float* sw, const uint16_t* bias,
                             void* y, int M, int N, int K, cudaStream_t st) {
  using C = WoCfg<BITS>;
  auto kern = gemm_wonly_kernel<BITS, OUT_BF16, HAS_BIAS>;
  CUtensorMap tw, tx;
  const int64_t wcols = BITS == 8 ? K : K / 2;  // bytes per weight row
  if (!wo_map(&tw, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, wcols, 128, 128) ||
      !wo_map(&tx, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, K, 64, kWoTokens))
    return cudaErrorInvalidValue;
  static uint64_t attr_set = 0;  // one bit per device ordinal
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64 || !((attr_set >> dev) & 1u)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(C::kDynamic));
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set |= uint64_t(1) << dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned((N + 127) / 128), unsigned((M + kWoTokens - 1) / kWoTokens), 1);
  cfg.blockDim = dim3(kWoThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kDynamic;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, tw, tx, sw, bias, y, M, N, K, status_ptr());
}

cudaError_t launch_gemm_weight_only(int bits, const uint16_t* x, const void* wq, const float* sw,
                                    const uint16_t* bias, int64_t M, int64_t N, int64_t K,
                                    void* y, OutKind yk, cudaStream_t st) {
  const int m = int(M), n = int(N), k = int(K);
  const int key = (bits == 4 ? 4 : 0) | (yk == OutKind::BF16 ? 2 : 0) | (bias ? 1 : 0);
#define SQ_WO(B, O, H) return run_wonly<B, O, H>(x, wq, sw, bias, y, m, n, k, st)
  switch (key) {
    case 0: SQ_WO(8, false, false);
    case 1: SQ_WO(8, false, true);
    case 2: SQ_WO(8, true, false);
    case 3: SQ_WO(8, true, true);
    case 4: SQ_WO(4, false, false);
    case 5: SQ_WO(4, false, true);
    case 6: SQ_WO(4, true, false);
    default: SQ_WO(4, true, true);
  }
#undef SQ_WO
}

}  // namespace sqh
