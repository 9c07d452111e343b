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
// Persistent, warp-specialized kernel. CG = 1: one CTA computes 128 x BN
// output tiles; CG = 2: a cluster of two CTAs on neighbouring SMs computes
// 256 x BN tiles with tcgen05.mma.cta_group::2 -- each CTA loads its own 128
// rows of Xq and its own BN/2 rows of Wq (no multicast), and the pair's MMA
// reads both halves, which halves the operand bytes each SM stages per MAC.
//   warp 0     : TMA producer -- 128-byte-wide K slices of the Xq / Wq tiles
//                into a STAGES-deep ring (128-byte swizzle); in a pair both
//                CTAs' copies complete on the leader CTA's "full" barrier.
//   warp 1     : allocates tensor memory (two BN-column accumulators); in the
//                leader CTA one thread issues the MMAs (K = 32 per
//                instruction) and frees ring slots / publishes finished
//                accumulators with tcgen05.commit.
//   warps 2..9 : epilogue -- two warps per TMEM lane quarter (warp w reads
//                lanes 32*(w%4)..+31, the two warps of a quarter take
//                alternate 32-column chunks): tcgen05.ld, dequantize with the
//                per-token scale and the per-channel scales / bias that the
//                producer staged in shared memory by bulk copy, bf16, store;
//                then hand the accumulator buffer back to the MMA thread. Two
//                buffers let the epilogue of tile i overlap the MMAs of i+1.
// Tiles are walked in groups of kGroupM M-tiles so that the CTAs working at
// the same time share Wq tiles in L2. Every barrier wait is bounded: a wait
// that gives up records SQ_ERR_TIMEOUT, the CTA skips its remaining work,
// drains its MMAs and still frees tensor memory.
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <cuda.h>
#include <cuda_runtime.h>

#include "sq_common.cuh"
#include "sq_internal.h"

namespace sqk {

constexpr int kBK = 128;  // bytes of K per pipeline stage (one swizzle row)
constexpr int kEpiWarps = 8;  // 4 or 8 (one or two per TMEM lane quarter)
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kGroupM = 16;

template <int CG, int BN, int MAXST, bool OUT_BF16>
struct GemmCfg {
  static constexpr int kTileM = 128 * CG;  // output rows per tile
  static constexpr int kBRows = BN / CG;   // Wq rows staged per CTA
  static constexpr uint32_t kABytes = 128 * kBK;
  static constexpr uint32_t kBBytes = kBRows * kBK;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kTxBytes = kStageBytes * CG;  // landing on one "full" barrier
  static constexpr uint32_t kAccStride = BN <= 128 ? 128 : 256;  // TMEM columns per buffer
  static constexpr uint32_t kTmemCols = 2 * kAccStride;
  // output staging: per epilogue warp two boxes of 32 rows x 32 columns,
  // written swizzled (64-byte rows for bf16, 128-byte rows for binary32) and
  // stored by TMA
  static constexpr uint32_t kOutRow = OUT_BF16 ? 64 : 128;
  static constexpr uint32_t kOutBox = 32 * kOutRow;
  static constexpr uint32_t kOutBytes = kEpiWarps * 2 * kOutBox;
  static constexpr uint32_t kFixed = kOutBytes + 2048 + 2 * (BN * 6) + 1024;
  static constexpr int kFit = int((232448 - kFixed) / kStageBytes);
  static constexpr int STAGES = kFit < MAXST ? kFit : MAXST;
  static constexpr uint32_t kRingA = 0;
  static constexpr uint32_t kRingB = STAGES * kABytes;
  static constexpr uint32_t kOutOff = STAGES * kStageBytes;  // 1024-aligned
  static constexpr uint32_t kBarOff = kOutOff + kOutBytes;
  // barriers: full[S], empty[S], tfull[2], tempty[2], sfull[2], sempty[2], drain
  static constexpr uint32_t kMiscOff = kBarOff + (2 * STAGES + 9) * 8;  // tmem slot, abort flag
  // per-tile per-channel scales (binary32) and bias (bf16), one slot per
  // accumulator buffer
  static constexpr uint32_t kScaleSlot = BN * 4 + BN * 2;
  static constexpr uint32_t kScaleOff = (kMiscOff + 16 + 127) & ~127u;
  static constexpr uint32_t kTotal = kScaleOff + 2 * kScaleSlot;
  static constexpr uint32_t kDynamic = kTotal + 1024;  // slack for 1024-B alignment
  static_assert(BN % 32 == 0 && BN <= 256, "BN must be a multiple of 32, at most 256");
  static_assert(kBRows % 8 == 0, "staged Wq rows must be whole 8-row swizzle atoms");
  static_assert(STAGES >= 3, "too few pipeline stages fit");
  static_assert(kDynamic <= 232448, "shared memory budget exceeded");
};

__device__ __forceinline__ void tile_coords(int tile, int num_mt, int num_nt, int& mt, int& nt) {
  const int per_group = kGroupM * num_nt;
  const int g = tile / per_group, r = tile - g * per_group;
  const int first = g * kGroupM;
  const int gm = min(kGroupM, num_mt - first);
  mt = first + r % gm;
  nt = r / gm;
}

// ---------------------------------------------------------------------------
// Work schedule (identical in every role of every CTA). With U units (CTAs,
// or CTA pairs), the first dp_rounds rounds are whole tiles (tile = unit +
// r*U). The remaining sk_tiles tiles form a "stream-K" region: their
// sk_tiles * nk k-blocks are cut into U contiguous ranges, one per unit, so
// the last partial wave is shared by every unit. A tile cut by range
// boundaries is finished by the unit holding its k-block 0 (the "owner",
// whose range ends there, so it waits last); the others ("contributors",
// whose ranges start there, so they contribute first) leave their raw
// accumulators in the caller's workspace. Nothing ever waits in a cycle.
// ---------------------------------------------------------------------------
struct WorkItem {
  int tile;      // tile index in the raster order
  int kb0, kb1;  // k-blocks [kb0, kb1)
  int kind;      // 0 whole tile, 1 owner of a split tile, 2 contributor
  int sk;        // index of the tile inside the stream-K region (kinds 1, 2)
};

struct Schedule {
  int unit, U, nk, dp_limit, dp_tiles, sk_tiles;
  int64_t S, it, it_end;
  int next_dp;
  __device__ void init(int unit_, int U_, int nk_, int num_tiles, int dp_rounds, int sk_tiles_) {
    unit = unit_; U = U_; nk = nk_; sk_tiles = sk_tiles_;
    dp_tiles = dp_rounds * U;
    dp_limit = min(num_tiles, dp_tiles);
    next_dp = unit;
    S = int64_t(sk_tiles) * nk;
    it = S ? int64_t(unit) * S / U : 0;
    it_end = S ? int64_t(unit + 1) * S / U : 0;
  }
  __device__ bool next(WorkItem& w) {
    if (next_dp < dp_limit) {
      w.tile = next_dp; w.kb0 = 0; w.kb1 = nk; w.kind = 0; w.sk = -1;
      next_dp += U;
      return true;
    }
    if (it < it_end) {
      const int64_t t = it / nk;
      const int kb0 = int(it - t * nk);
      const int64_t e = min((t + 1) * int64_t(nk), it_end);
      w.tile = dp_tiles + int(t); w.kb0 = kb0; w.kb1 = int(e - t * nk); w.sk = int(t);
      w.kind = (w.kb0 == 0 && w.kb1 == nk) ? 0 : (w.kb0 == 0 ? 1 : 2);
      it = e;
      return true;
    }
    return false;
  }
  // unit whose range holds stream-K iteration i
  __device__ int unit_of(int64_t i) const { return int(((i + 1) * U - 1) / S); }
  __device__ int contributors(int t) const {
    return unit_of((int64_t(t) + 1) * nk - 1) - unit_of(int64_t(t) * nk);
  }
};

// Workspace layout: arrived[kMaxSkTiles], done[kMaxSkTiles] (uint32), then
// one partial-accumulator slot per CTA (128 rows x BN x 4 bytes). The
// counters sit at fixed offsets so that calls of any shape can share one
// workspace; every call leaves them zero.
constexpr int kMaxSkTiles = 512;
__host__ __device__ inline size_t ws_slot_offset(int) { return size_t(kMaxSkTiles) * 8; }

template <int CG, int BN, int MAXST, bool E4M3, bool OUT_BF16, bool HAS_BIAS, bool WRITE_ACC>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_w8a8_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_y, const float* __restrict__ sx,
                     const float* __restrict__ sw, const uint16_t* __restrict__ bias,
                     int32_t* __restrict__ acc_out, int M, int N, int K, int dp_rounds,
                     int sk_tiles, uint8_t* __restrict__ ws, int* status) {
  using C = GemmCfg<CG, BN, MAXST, OUT_BF16>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_a = s_base + C::kRingA;
  const uint32_t s_b = s_base + C::kRingB;
  const uint32_t bar_full = s_base + C::kBarOff;
  const uint32_t bar_empty = bar_full + STAGES * 8;
  const uint32_t bar_tfull = bar_empty + STAGES * 8;
  const uint32_t bar_tempty = bar_tfull + 2 * 8;
  const uint32_t bar_sfull = bar_tempty + 2 * 8;
  const uint32_t bar_sempty = bar_sfull + 2 * 8;
  const uint32_t bar_drain = bar_sempty + 2 * 8;
  const uint32_t s_scale = s_base + C::kScaleOff;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_tfull + 8 * b, 1);
      mbar_init(bar_tempty + 8 * b, kEpiWarps * CG);
      mbar_init(bar_sfull + 8 * b, 1);
      mbar_init(bar_sempty + 8 * b, kEpiWarps);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_map(&tm_a);
    tma_prefetch_map(&tm_b);
    tma_prefetch_map(&tm_y);
  }
  if (warp == 1) {
    if constexpr (CG == 2) {
      tmem_alloc_pair(smem_u32(tmem_slot), C::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (CG == 2) cluster_sync_all(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // set-up above overlaps the previous kernel; its results are read below.
  // The next kernel may start only after that wait: by then every kernel
  // before this one has completed, which lets an activation pass that
  // overlaps this grid (SQ_OVERLAP_PREVIOUS) reuse the buffers of the GEMM
  // before this one
  pdl_wait();
  pdl_launch_dependents();

  const int num_mt = (M + C::kTileM - 1) / C::kTileM;
  const int num_nt = (N + BN - 1) / BN;
  const int num_tiles = num_mt * num_nt;
  const int unit = blockIdx.x / CG, num_units = gridDim.x / CG;
  const int nk = (K + kBK - 1) / kBK;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      uint32_t it = 0, tc = 0;
      bool ok = true;
      Schedule sch;
      sch.init(unit, num_units, nk, num_tiles, dp_rounds, sk_tiles);
      WorkItem wi;
#pragma unroll 1
      for (; ok && sch.next(wi); ++tc) {
        int mt, nt;
        tile_coords(wi.tile, num_mt, num_nt, mt, nt);
        const int a_row = mt * C::kTileM + int(rank) * 128;
        const int b_row = nt * BN + int(rank) * C::kBRows;
        {
          // stage this tile's per-channel scales (and bias) for the epilogue
          const uint32_t buf = tc & 1u;
          if (!mbar_wait(bar_sempty + 8 * buf, ((tc >> 1) & 1u) ^ 1u) || *abort_flag) {
            record_status(status, kStatusTimeout);
            *abort_flag = 1;
            ok = false;
            break;
          }
          const int n0 = nt * BN;
          const int cols = N - n0 < BN ? N - n0 : BN;
          const uint32_t sw_bytes = uint32_t(cols) * 4, b_bytes = HAS_BIAS ? uint32_t(cols) * 2 : 0;
          const uint32_t slot = s_scale + buf * C::kScaleSlot;
          mbar_arrive_expect_tx(bar_sfull + 8 * buf, sw_bytes + b_bytes);
          bulk_load(slot, sw + n0, sw_bytes, bar_sfull + 8 * buf);
          if constexpr (HAS_BIAS) bulk_load(slot + BN * 4, bias + n0, b_bytes, bar_sfull + 8 * buf);
        }
#pragma unroll 1
        for (int kb = wi.kb0; kb < wi.kb1; ++kb, ++it) {
          const uint32_t st = it % STAGES, ph = (it / STAGES) & 1u;
          if (!mbar_wait(bar_empty + 8 * st, ph ^ 1u) || *abort_flag) {
            record_status(status, kStatusTimeout);
            *abort_flag = 1;
            ok = false;
            break;
          }
          if constexpr (CG == 2) {
            if (leader) mbar_arrive_expect_tx(bar_full + 8 * st, C::kTxBytes);
            const uint32_t full_leader = map_to_rank(bar_full + 8 * st, 0);
            tma_load_2d_pair(s_a + st * C::kABytes, &tm_a, full_leader, kb * kBK, a_row);
            tma_load_2d_pair(s_b + st * C::kBBytes, &tm_b, full_leader, kb * kBK, b_row);
          } else {
            mbar_arrive_expect_tx(bar_full + 8 * st, C::kTxBytes);
            tma_load_2d(s_a + st * C::kABytes, &tm_a, bar_full + 8 * st, kb * kBK, a_row);
            tma_load_2d(s_b + st * C::kBBytes, &tm_b, bar_full + 8 * st, kb * kBK, b_row);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA --
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = E4M3 ? idesc_e4m3_f32(C::kTileM, BN) : idesc_s8_s32(C::kTileM, BN);
      uint32_t it = 0, tc = 0;
      bool ok = true;
      Schedule sch;
      sch.init(unit, num_units, nk, num_tiles, dp_rounds, sk_tiles);
      WorkItem wi;
#pragma unroll 1
      for (; ok && sch.next(wi); ++tc) {
        const uint32_t buf = tc & 1u, use = tc >> 1;
        if (!mbar_wait(bar_tempty + 8 * buf, (use & 1u) ^ 1u)) {
          record_status(status, kStatusTimeout);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + buf * C::kAccStride;
#pragma unroll 1
        for (int kb = wi.kb0; kb < wi.kb1; ++kb, ++it) {
          const uint32_t st = it % STAGES, ph = (it / STAGES) & 1u;
          if (!mbar_wait(bar_full + 8 * st, ph)) {
            record_status(status, kStatusTimeout);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = s_a + st * C::kABytes;
          const uint32_t b_addr = s_b + st * C::kBBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 32; ++kk) {
            const uint64_t ad = sw128_desc(a_addr + kk * 32);
            const uint64_t bd = sw128_desc(b_addr + kk * 32);
            const uint32_t accum = (kb > wi.kb0 || kk > 0) ? 1u : 0u;
            if constexpr (CG == 2) {
              if constexpr (E4M3) mma_f8_pair(d, ad, bd, idesc, accum);
              else mma_i8_pair(d, ad, bd, idesc, accum);
            } else {
              if constexpr (E4M3) mma_f8(d, ad, bd, idesc, accum);
              else mma_i8(d, ad, bd, idesc, accum);
            }
          }
          if constexpr (CG == 2) {
            tc_commit_pair(bar_empty + 8 * st);
            tc_commit_pair(map_to_rank(bar_empty + 8 * st, 1));
          } else {
            tc_commit(bar_empty + 8 * st);
          }
        }
        if (!ok) break;
        if constexpr (CG == 2) {
          tc_commit_pair(bar_tfull + 8 * buf);
          tc_commit_pair(map_to_rank(bar_tfull + 8 * buf, 1));
        } else {
          tc_commit(bar_tfull + 8 * buf);
        }
      }
      // Make sure every MMA issued has completed before tensor memory can be
      // freed (matters only on the abort path; normally the epilogue has
      // already observed the last accumulator).
      if constexpr (CG == 2) tc_commit_pair(bar_drain); else tc_commit(bar_drain);
      (void)mbar_wait(bar_drain, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue --
    constexpr int NCH = BN / 32;  // 32-column chunks per tile
    const int sub = warp & 3;
    constexpr int WPQ = kEpiWarps / 4;  // epilogue warps per TMEM lane quarter
    const int half = (warp - 2) >> 2;   // which warp of this lane quarter
    const int row_in_tile = int(rank) * 128 + sub * 32 + lane;
    const uint32_t tempty_leader = CG == 2 ? map_to_rank(bar_tempty, 0) : bar_tempty;
    uint32_t tc = 0;
    uint32_t emitted = 0;  // chunks this warp has handed to TMA stores
    Schedule sch;
    sch.init(unit, num_units, nk, num_tiles, dp_rounds, sk_tiles);
    WorkItem wi;
    uint32_t* arrived = reinterpret_cast<uint32_t*>(ws);
    uint32_t* done = arrived + sk_tiles;
    int32_t* slots = reinterpret_cast<int32_t*>(ws + ws_slot_offset(sk_tiles));
    constexpr int kSlotWords = 128 * BN;
    const int row_in_cta = sub * 32 + lane;
#pragma unroll 1
    for (; sch.next(wi); ++tc) {
      const uint32_t buf = tc & 1u, use = tc >> 1;
      if (!mbar_wait(bar_tfull + 8 * buf, use & 1u) || !mbar_wait(bar_sfull + 8 * buf, use & 1u) ||
          *abort_flag) {
        record_status(status, kStatusTimeout);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      int mt, nt;
      tile_coords(wi.tile, num_mt, num_nt, mt, nt);
      const int m = mt * C::kTileM + row_in_tile;
      const int n_base = nt * BN;
      const float sxm = m < M ? __ldg(sx + m) : 0.0f;
      const uint32_t t_addr = tmem_base + buf * C::kAccStride + (uint32_t(sub * 32) << 16);
      const float* s_sw = reinterpret_cast<const float*>(smem + C::kScaleOff + buf * C::kScaleSlot);
      const uint16_t* s_b = reinterpret_cast<const uint16_t*>(smem + C::kScaleOff +
                                                                buf * C::kScaleSlot + BN * 4);

      // dequantize one 32-column chunk held in r[] into a staging box and
      // store it with TMA (the box's rows / columns outside Y are clipped)
      const int e = warp - 2;
      const int box_row = mt * C::kTileM + int(rank) * 128 + sub * 32;
      auto emit = [&](const uint32_t (&r)[32], int chunk) {
        const uint32_t sbuf = s_base + C::kOutOff + uint32_t(e * 2 + (emitted & 1)) * C::kOutBox;
        if (emitted >= 2) {
          // the bulk store that last read this buffer must be done reading
          if (lane == 0) bulk_wait_read<1>();
          __syncwarp();
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int nl = chunk * 32 + g * 8;
          const float4 w0 = *reinterpret_cast<const float4*>(s_sw + nl);
          const float4 w1 = *reinterpret_cast<const float4*>(s_sw + nl + 4);
          const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
          float bv[8];
          if constexpr (HAS_BIAS) {
            const uint4 b = *reinterpret_cast<const uint4*>(s_b + nl);
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
          if constexpr (OUT_BF16) {
            // row = lane (64 B); 16-byte unit g, 64-byte swizzle
            const uint32_t unit = uint32_t(g) ^ ((uint32_t(lane) >> 1) & 3u);
            const uint32_t addr = sbuf + uint32_t(lane) * 64 + unit * 16;
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                         "r"(pack_bf16x2(t[0], t[1])), "r"(pack_bf16x2(t[2], t[3])),
                         "r"(pack_bf16x2(t[4], t[5])), "r"(pack_bf16x2(t[6], t[7]))
                         : "memory");
          } else {
            // row = lane (128 B); 16-byte units 2g, 2g+1, 128-byte swizzle
            const uint32_t u0 = (uint32_t(2 * g) ^ (uint32_t(lane) & 7u));
            const uint32_t u1 = (uint32_t(2 * g + 1) ^ (uint32_t(lane) & 7u));
            const uint32_t base = sbuf + uint32_t(lane) * 128;
            asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(base + u0 * 16),
                         "f"(t[0]), "f"(t[1]), "f"(t[2]), "f"(t[3])
                         : "memory");
            asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(base + u1 * 16),
                         "f"(t[4]), "f"(t[5]), "f"(t[6]), "f"(t[7])
                         : "memory");
          }
          if constexpr (WRITE_ACC) {
            const int n = n_base + nl;
            if (m < M && n < N) {
              int4* q = reinterpret_cast<int4*>(acc_out + int64_t(m) * N + n);
              q[0] = make_int4(int(r[g * 8 + 0]), int(r[g * 8 + 1]), int(r[g * 8 + 2]), int(r[g * 8 + 3]));
              q[1] = make_int4(int(r[g * 8 + 4]), int(r[g * 8 + 5]), int(r[g * 8 + 6]), int(r[g * 8 + 7]));
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_y, sbuf, n_base + chunk * 32, box_row);
          bulk_commit_group();
        }
        ++emitted;
      };

      // partial accumulators of a split tile: one slot per CTA, laid out
      // [chunk][column][row] (raw int32 for INT8, binary32 bits for FP8) so
      // that a warp's 32 rows of one column are one coalesced 128-byte line
      auto slot_col = [&](int u, int chunk) {
        return slots + size_t(u * CG + int(rank)) * kSlotWords + size_t(chunk) * 32 * 128 +
               size_t(sub * 32 + lane);
      };
      int n_contrib = 0;
      bool give_up = false;
      if (wi.kind == 1) {
        // owner: wait until every contributing warp has published its part
        n_contrib = sch.contributors(wi.sk);
        const uint32_t target = uint32_t(n_contrib * kEpiWarps * CG);
        if (lane == 0) {
          const uint64_t t0 = globaltimer_ns();
          uint32_t polls = 0;
          while (ld_acquire_gpu(arrived + wi.sk) < target) {
            __nanosleep(128);
            if ((++polls & 255u) == 0u && globaltimer_ns() - t0 > kWaitTimeoutNs) {
              record_status(status, kStatusTimeout);
              *abort_flag = 1;
              break;
            }
          }
          __threadfence();
        }
        __syncwarp();
        give_up = *abort_flag != 0;
      }
      const int first_contrib = wi.kind == 1 ? sch.unit_of(int64_t(wi.sk) * nk) + 1 : 0;
      // add the contributors' partial sums to this warp's accumulator chunk
      auto add_partials = [&](uint32_t (&r)[32], int chunk) {
        for (int cu = 0; cu < n_contrib; ++cu) {
          const int32_t* src = slot_col(first_contrib + cu, chunk);
          int32_t pw[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) pw[j] = __ldcg(src + j * 128);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if constexpr (E4M3)
              r[j] = __float_as_uint(__fadd_rn(__uint_as_float(r[j]), __int_as_float(pw[j])));
            else
              r[j] = uint32_t(int32_t(r[j]) + pw[j]);
          }
        }
      };
      auto publish = [&](const uint32_t (&r)[32], int chunk) {
        int32_t* dst = slot_col(unit, chunk);
#pragma unroll
        for (int j = 0; j < 32; ++j) __stcg(dst + j * 128, int32_t(r[j]));
      };

      // a warp whose 32 rows all lie beyond M (the last M-tile of a small
      // batch) has nothing to store, publish or add: it only keeps the
      // barrier and counter protocol below
      const bool slab_live = box_row < M;
      // this warp's chunks are half, half+WPQ, half+2*WPQ, ...; two loads in
      // flight at a time
#pragma unroll 1
      for (int c = half; slab_live && c < NCH && !give_up; c += 2 * WPQ) {
        uint32_t r0[32], r1[32];
        const bool two = c + WPQ < NCH;  // warp-uniform
        tmem_ld32(t_addr + uint32_t(c * 32), r0);
        if (two) {
          tmem_ld32(t_addr + uint32_t((c + WPQ) * 32), r1);
          tmem_wait_ld2(r0, r1);
        } else {
          tmem_wait_ld(r0);
        }
        if (wi.kind == 2) {
          publish(r0, c);
          if (two) publish(r1, c + WPQ);
          continue;
        }
        if (wi.kind == 1) {
          add_partials(r0, c);
          if (two) add_partials(r1, c + WPQ);
        }
        emit(r0, c);
        if (two) emit(r1, c + WPQ);
      }
      if (wi.kind == 2) {
        // contributor: make the slot visible, then count this warp in
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(arrived + wi.sk, 1u);
      } else if (wi.kind == 1 && !give_up) {
        // owner: the last of its warps to finish resets the counters, so the
        // workspace is clean for the next launch
        __syncwarp();
        if (lane == 0) {
          if (atomicAdd(done + wi.sk, 1u) == uint32_t(kEpiWarps * CG - 1)) {
            atomicExch(arrived + wi.sk, 0u);
            atomicExch(done + wi.sk, 0u);
          }
        }
      }
      // hand the accumulator buffer and the scale slot back
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (CG == 2) mbar_arrive_cluster(tempty_leader + 8 * buf);
        else mbar_arrive(bar_tempty + 8 * buf);
        mbar_arrive(bar_sempty + 8 * buf);
      }
    }
    // the staging buffers must outlive the bulk stores reading them
    if (lane == 0) bulk_wait_all<0>();
    __syncwarp();
  }
  __syncwarp();
  tc_fence_before();
  if constexpr (CG == 2) cluster_sync_all(); else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (CG == 2) tmem_dealloc_pair(tmem_base, C::kTmemCols);
    else tmem_dealloc(tmem_base, C::kTmemCols);
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

// Tensor map of the row-major [M, N] output (bf16 or binary32) for the
// epilogue's TMA stores: box = 32 rows x 32 columns, swizzled like the
// staging buffers (64-byte rows for bf16, 128-byte rows for binary32).
static bool make_map_out(CUtensorMap* map, void* y, int64_t M, int64_t N, bool bf16) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t es = bf16 ? 2 : 4;
  cuuint64_t dims[2] = {cuuint64_t(N), cuuint64_t(M)};
  cuuint64_t strides[1] = {cuuint64_t(N) * es};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, y,
             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             bf16 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int device_sms() {
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

// Whether splitting the last partial round pays: measured on B200, the split
// region costs more than it saves unless whole-tile rounds waste at least a
// tenth of the time (FP8 down 4096 x 14336 x 4096: 256 tiles on 74 SM pairs,
// 4 rounds for 3.46 rounds of work, 180 -> 170 us; MLP up: 13 rounds for
// 12.1, 163 -> 164 us; fewer tiles than units, as at 512 tokens: 22 -> 25 us).
// SQ_GEMM_FORCE_SPLIT=1 in the environment splits every partial round (used
// by the tests to reach the split path on every tile shape).
static bool split_pays(int64_t tiles, int64_t units) {
  const int64_t full = tiles / units, rem = tiles % units;
  if (rem == 0) return false;
  const char* force = getenv("SQ_GEMM_FORCE_SPLIT");
  if (force && force[0] == '1') return true;
  if (full == 0) return false;
  return double(tiles) / double(units) <= 0.9 * double(full + 1);
}

// Whole-tile rounds first; when split_pays, the last one or two rounds' worth
// of tiles become a stream-K region shared by all units (needs a workspace).
static void plan_schedule(int num_tiles, int units, bool can_split, int* dp_rounds, int* sk_tiles) {
  const int full = num_tiles / units;
  const bool split = can_split && split_pays(num_tiles, units);
  if (!split) {
    *dp_rounds = (num_tiles + units - 1) / units;
    *sk_tiles = 0;
    return;
  }
  *dp_rounds = full > 0 ? full - 1 : 0;
  *sk_tiles = num_tiles - *dp_rounds * units;
}

template <int CG, int BN, int STAGES, bool E4M3, bool OUT_BF16, bool HAS_BIAS, bool WRITE_ACC>
static cudaError_t run_gemm(const void* xq, const void* wq, const float* sx, const float* sw,
                            const uint16_t* bias, void* y, int32_t* acc, int M, int N, int K,
                            void* ws, size_t ws_bytes, cudaStream_t st) {
  using C = GemmCfg<CG, BN, STAGES, OUT_BF16>;
  auto kern = gemm_w8a8_kernel<CG, BN, STAGES, E4M3, OUT_BF16, HAS_BIAS, WRITE_ACC>;
  CUtensorMap ta, tb, ty;
  if (!make_map_k_major(&ta, xq, M, K, 128) || !make_map_k_major(&tb, wq, N, K, C::kBRows) ||
      !make_map_out(&ty, y, M, N, OUT_BF16))
    return cudaErrorInvalidValue;
  static uint64_t attr_set_mask = 0;  // one bit per device ordinal
  static int max_units[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  const bool cached = dev < 64 && ((attr_set_mask >> dev) & 1u);
  if (!cached) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(C::kDynamic));
    if (e != cudaSuccess) return e;
    int units = device_sms() / CG;
    if (CG == 2) {
      cudaLaunchConfig_t q = {};
      cudaLaunchAttribute a[1];
      a[0].id = cudaLaunchAttributeClusterDimension;
      a[0].val.clusterDim.x = 2;
      a[0].val.clusterDim.y = 1;
      a[0].val.clusterDim.z = 1;
      q.gridDim = dim3(2 * units);
      q.blockDim = dim3(kThreads);
      q.dynamicSmemBytes = C::kDynamic;
      q.attrs = a;
      q.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, kern, &q) == cudaSuccess && clusters > 0)
        units = clusters < units ? clusters : units;
      cudaGetLastError();
    }
    if (dev < 64) {
      max_units[dev] = units;
      attr_set_mask |= uint64_t(1) << dev;
    }
  }
  const int units_max = dev < 64 ? max_units[dev] : device_sms() / CG;
  const int tiles = ((M + C::kTileM - 1) / C::kTileM) * ((N + BN - 1) / BN);
  // stream-K needs every unit resident at once: units never exceeds what the
  // occupancy query says fits. With a workspace every unit gets work even
  // when there are fewer tiles than units.
  const size_t need = ws_slot_offset(0) + size_t(units_max) * CG * 128 * BN * 4;
  const bool can_split = ws != nullptr && ws_bytes >= need && !getenv("SQ_GEMM_NO_SPLIT");
  int units = tiles < units_max ? tiles : units_max;
  if (can_split && tiles > 0 && split_pays(tiles, units_max) &&
      int64_t(tiles) * ((K + kBK - 1) / kBK) >= units_max)
    units = units_max;
  int dp_rounds = 0, sk_tiles = 0;
  plan_schedule(tiles, units, can_split, &dp_rounds, &sk_tiles);
  if (sk_tiles > kMaxSkTiles) {
    dp_rounds = (tiles + units - 1) / units;
    sk_tiles = 0;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attrs[2];
  cfg.gridDim = dim3(unsigned(units * CG));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kDynamic;
  cfg.stream = st;
  unsigned na = 0;
  if (CG == 2) {
    attrs[na].id = cudaLaunchAttributeClusterDimension;
    attrs[na].val.clusterDim.x = 2;
    attrs[na].val.clusterDim.y = 1;
    attrs[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl_enabled()) {
    // may start while the kernel before it (normally the activation
    // quantization) finishes; the kernel waits before touching memory
    attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attrs;
  cfg.numAttrs = na;
  int* status = status_ptr();
  return cudaLaunchKernelEx(&cfg, kern, ta, tb, ty, sx, sw, bias, acc, M, N, K, dp_rounds,
                            sk_tiles, static_cast<uint8_t*>(ws), status);
}

template <int CG, int BN, int STAGES, bool E4M3>
static cudaError_t dispatch_epilogue(const void* xq, const void* wq, const float* sx,
                                     const float* sw, const uint16_t* bias, void* y, OutKind yk,
                                     int32_t* acc, int M, int N, int K, void* ws, size_t ws_bytes,
                                     cudaStream_t st) {
  const bool bf = yk == OutKind::BF16, hb = bias != nullptr, wa = acc != nullptr;
  const int key = (bf ? 4 : 0) | (hb ? 2 : 0) | (wa ? 1 : 0);
#define SQ_RUN(B, H, W) \
  run_gemm<CG, BN, STAGES, E4M3, B, H, W>(xq, wq, sx, sw, bias, y, acc, M, N, K, ws, ws_bytes, st)
  switch (key) {
    case 0: return SQ_RUN(false, false, false);
    case 1: return SQ_RUN(false, false, true);
    case 2: return SQ_RUN(false, true, false);
    case 3: return SQ_RUN(false, true, true);
    case 4: return SQ_RUN(true, false, false);
    case 5: return SQ_RUN(true, false, true);
    case 6: return SQ_RUN(true, true, false);
    default: return SQ_RUN(true, true, true);
  }
#undef SQ_RUN
}

// Tile shapes compiled in. Each entry: CTAs per tile (1 or 2), N per tile,
// pipeline depth.
enum class TileCfg { C1_N128, C1_N224, C1_N256, C2_N224, C2_N256 };

static TileCfg choose_tile(int64_t M, int64_t N, bool can_split) {
  // Estimated time ~ (number of rounds of tiles over the SMs) x (work per
  // tile) / (relative MAC throughput of the tile shape, measured on B200 at
  // 4096 x 4096 x 14336: 256x256 pairs 1.0, 256x224 pairs 0.89, 128x256
  // single CTAs 0.90, 128x224 single CTAs 0.85, 128x128 single CTAs 0.62).
  // For a single M-tile (decode) the work per tile is its Wq panel, so the
  // same estimate favours the tile width that spreads N over the most SMs.
  const int sms = device_sms();
  struct Cand { TileCfg c; int cg, bm, bn; double eff; };
  const Cand cands[] = {{TileCfg::C2_N256, 2, 256, 256, 1.0},
                        {TileCfg::C2_N224, 2, 256, 224, 0.89},
                        {TileCfg::C1_N256, 1, 128, 256, 0.90},
                        {TileCfg::C1_N224, 1, 128, 224, 0.85},
                        {TileCfg::C1_N128, 1, 128, 128, 0.62}};
  double best = 1e30;
  TileCfg pick = TileCfg::C1_N128;
  for (const Cand& c : cands) {
    const int64_t tiles = ((M + c.bm - 1) / c.bm) * ((N + c.bn - 1) / c.bn);
    const int64_t units = sms / c.cg;
    // with split tiles the last wave is shared (fractional rounds, plus a
    // small cost for the partial sums); without, whole rounds
    const double rounds = (can_split && split_pays(tiles, units))
                              ? double(tiles) / double(units) + 0.1
                              : double((tiles + units - 1) / units);
    const double t = rounds * double(c.bm) * double(c.bn) / (double(c.cg) * c.eff);
    if (t < best * 0.999) {
      best = t;
      pick = c.c;
    }
  }
  return pick;
}

// SQ_GEMM_TILE = c1n128 | c1n224 | c1n256 | c2n224 | c2n256 forces one tile shape
// (used to test every shape and to compare them); unset or anything else
// selects by problem size.
static bool forced_tile(TileCfg* out) {
  const char* e = getenv("SQ_GEMM_TILE");
  if (!e) return false;
  if (!strcmp(e, "c1n128")) { *out = TileCfg::C1_N128; return true; }
  if (!strcmp(e, "c1n224")) { *out = TileCfg::C1_N224; return true; }
  if (!strcmp(e, "c1n256")) { *out = TileCfg::C1_N256; return true; }
  if (!strcmp(e, "c2n224")) { *out = TileCfg::C2_N224; return true; }
  if (!strcmp(e, "c2n256")) { *out = TileCfg::C2_N256; return true; }
  return false;
}

size_t gemm_workspace_counter_bytes() { return ws_slot_offset(0); }

size_t gemm_workspace_bytes() {
  // the largest need of any tile shape: one 128 x 256 binary32 slot per SM
  return ws_slot_offset(0) + size_t(device_sms()) * 128 * 256 * 4;
}

cudaError_t launch_gemm(bool e4m3, const uint8_t* xq, const float* sx, const uint8_t* wq,
                        const float* sw, const uint16_t* bias, int64_t M, int64_t N, int64_t K,
                        void* y, OutKind yk, int32_t* acc, void* ws, size_t ws_bytes,
                        cudaStream_t st) {
  const int m = int(M), n = int(N), k = int(K);
  TileCfg c;
  if (!forced_tile(&c)) c = choose_tile(M, N, ws != nullptr && ws_bytes >= gemm_workspace_bytes());
#define SQ_CASE(CG, BN, S)                                                                     \
  return e4m3 ? dispatch_epilogue<CG, BN, S, true>(xq, wq, sx, sw, bias, y, yk, acc, m, n, k, ws, ws_bytes, st) \
              : dispatch_epilogue<CG, BN, S, false>(xq, wq, sx, sw, bias, y, yk, acc, m, n, k, ws, ws_bytes, st)
  switch (c) {
    case TileCfg::C2_N256: SQ_CASE(2, 256, 6);
    case TileCfg::C2_N224: SQ_CASE(2, 224, 7);
    case TileCfg::C1_N256: SQ_CASE(1, 256, 4);
    case TileCfg::C1_N224: SQ_CASE(1, 224, 5);
    default: SQ_CASE(1, 128, 6);
  }
#undef SQ_CASE
}

}  // namespace sqh
