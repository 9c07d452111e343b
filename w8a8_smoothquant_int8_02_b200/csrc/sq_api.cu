// sq_api.cu -- the C ABI of libsq.so (declared in include/sq.h).
//
// Argument validation happens here, synchronously, before anything is
// launched; the launchers in sq_quant.cu / sq_gemm.cu assume valid input.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cuda_runtime.h>

#include "sq.h"
#include "sq_common.cuh"
#include "sq_internal.h"

// The library's only device allocations: one status word per device that a
// kernel sets when a bounded wait gives up, and the mismatch counter of the
// arithmetic self-test.
static __device__ int g_sq_status = 0;
static __device__ unsigned long long g_sq_selftest_count = 0;

namespace sqh {

int* status_ptr() {
  // One lookup per device (the symbol has a different address per device).
  static int* ptrs[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_sq_status) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int*>(p);
  }
  return ptrs[dev];
}

}  // namespace sqh

namespace {

__global__ void probe_wait_kernel(int64_t timeout_ns, int* status) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = sqk::smem_u32(&bar);
  if (threadIdx.x == 0) {
    sqk::mbar_init(b, 1);
    sqk::fence_barrier_init();
    // Nothing ever arrives on `bar`, so phase 0 never completes.
    if (!sqk::mbar_wait(b, 0, uint64_t(timeout_ns))) sqk::record_status(status, sqk::kStatusTimeout);
  }
}

inline bool al(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
// Byte ranges [a, a+na) and [b, b+nb) share an address.
inline bool overlap(const void* a, uint64_t na, const void* b, uint64_t nb) {
  const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return pa < pb + nb && pb < pa + na;
}
inline cudaStream_t S(void* st) { return static_cast<cudaStream_t>(st); }
inline sq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SQ_OK : SQ_ERR_CUDA; }

// Common checks for the 8-bit GEMMs.
sq_status check_gemm(const void* xq, const float* sx, const void* wq, const float* sw,
                     const uint16_t* bias, int64_t M, int64_t N, int64_t K, const void* y,
                     sq_dtype yt, const int32_t* acc) {
  if (M < 0 || N <= 0 || K <= 0 || K % 16 != 0 || N % 8 != 0) return SQ_ERR_INVALID_ARG;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return SQ_ERR_INVALID_ARG;
  if (K >= 133144) return SQ_ERR_UNSUPPORTED;  // int32 accumulator bound K*127^2 < 2^31
  if (yt != SQ_BF16 && yt != SQ_F32) return SQ_ERR_INVALID_ARG;
  if (M == 0) return SQ_OK;  // empty batch: pointers may be NULL
  if (!xq || !sx || !wq || !sw || !y) return SQ_ERR_INVALID_ARG;
  if (!al(xq, 16) || !al(wq, 16) || !al(y, 16) || !al(sx, 4) || !al(sw, 16)) return SQ_ERR_MISALIGNED;
  if (bias && !al(bias, 16)) return SQ_ERR_MISALIGNED;
  if (acc && !al(acc, 16)) return SQ_ERR_MISALIGNED;
  return SQ_OK;
}

// Few tokens (M <= 16) take the weight-streaming form with the operand roles
// swapped (sq_gemm_skinny.cu); problems whose 128 x 128 tiles fit in one wave
// the four-issuer form (sq_gemm_small.cu); everything else the persistent
// tiled kernel (sq_gemm.cu). Same results (INT8 bit for bit), no workspace
// for the first two. SQ_GEMM_TILE in the environment keeps the tiled kernel
// for every shape; SQ_GEMM_NO_SKINNY / SQ_GEMM_NO_SMALL skip one form.
cudaError_t run_gemm_any(bool e4m3, const uint8_t* xq, const float* sx, const uint8_t* wq,
                         const float* sw, const uint16_t* bias, int64_t M, int64_t N, int64_t K,
                         void* y, sqh::OutKind yk, int32_t* acc, void* ws, size_t ws_bytes,
                         cudaStream_t st) {
  if (sqh::gemm_skinny_applies(M))
    return sqh::launch_gemm_skinny(e4m3, xq, sx, wq, sw, bias, M, N, K, y, yk, acc, st);
  if (sqh::gemm_small_applies(M, N, K))
    return sqh::launch_gemm_small(e4m3, xq, sx, wq, sw, bias, M, N, K, y, yk, acc, st);
  return sqh::launch_gemm(e4m3, xq, sx, wq, sw, bias, M, N, K, y, yk, acc, ws, ws_bytes, st);
}

// ---------------------------------------------------------------------------
// Scratch of the allocation-free GEMM entry point (sq_gemm_w8a8_noalloc):
// a fixed array in the library's own device image, so the call allocates
// nothing. Its size is the split-tile workspace of a GPU with kNoAllocMaxSms
// SMs: the counter block plus one 128 x 256 x 4-byte partial-sum slot per SM
// (sq_gemm_workspace_bytes on such a GPU). Every GPU that loads the library
// keeps this array until the process exits.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocMaxSms = 160;
constexpr size_t kNoAllocSlotBytes = size_t(128) * 256 * 4;
static __device__ __align__(256) unsigned char
    g_sq_noalloc_scratch[size_t(4096) + kNoAllocMaxSms * kNoAllocSlotBytes];
constexpr size_t kNoAllocScratchBytes = sizeof(g_sq_noalloc_scratch);

// Device address of the array for the current device. Host code must not use
// the array's name as a pointer (it is a host-side stand-in); the runtime
// gives the device address. It is looked up once per device with that device
// current and cached; concurrent first calls may both look it up and store
// the same value (atomic stores). After cudaDeviceReset the module is loaded
// again and the cached address is stale, so a process that resets a device
// must not call the entry point on it afterwards.
void* noalloc_scratch_ptr() {
  static std::atomic<void*> ptrs[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  void* p = ptrs[dev].load(std::memory_order_acquire);
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_sq_noalloc_scratch) != cudaSuccess || p == nullptr)
      return nullptr;
    ptrs[dev].store(p, std::memory_order_release);
  }
  return p;
}

}  // namespace

extern "C" {

const char* sq_status_string(sq_status st) {
  switch (st) {
    case SQ_OK: return "SQ_OK";
    case SQ_ERR_INVALID_ARG: return "SQ_ERR_INVALID_ARG: invalid argument";
    case SQ_ERR_MISALIGNED: return "SQ_ERR_MISALIGNED: pointer not aligned as required";
    case SQ_ERR_UNSUPPORTED: return "SQ_ERR_UNSUPPORTED: unsupported combination";
    case SQ_ERR_CUDA: return "SQ_ERR_CUDA: CUDA runtime error";
    case SQ_ERR_TIMEOUT: return "SQ_ERR_TIMEOUT: a bounded device wait gave up";
    case SQ_ERR_SCRATCH_TOO_SMALL:
      return "SQ_ERR_SCRATCH_TOO_SMALL: this call needs more scratch than the fixed array of "
             "the allocation-free entry point (sized for GPUs with up to 160 SMs)";
  }
  return "SQ_ERR_UNKNOWN";
}

int sq_abi_version(void) { return SQ_ABI_VERSION; }

sq_status sq_get_device_status(void* stream) {
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return SQ_ERR_CUDA;
  int* p = sqh::status_ptr();
  if (!p) return SQ_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SQ_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return SQ_ERR_CUDA;
  }
  return v == 0 ? SQ_OK : static_cast<sq_status>(v);
}

sq_status sq_calibrate_amax(const void* x, sq_dtype xt, int64_t rows, int64_t cols, sq_axis axis,
                            float* amax, int accumulate, void* stream) {
  if (!x || !amax) return SQ_ERR_INVALID_ARG;
  if (xt != SQ_F32 && xt != SQ_BF16) return SQ_ERR_INVALID_ARG;
  if (axis != SQ_AMAX_PER_COLUMN && axis != SQ_AMAX_PER_ROW) return SQ_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0 || cols % 8 != 0 || rows > INT32_MAX) return SQ_ERR_INVALID_ARG;
  if (!al(x, 16) || !al(amax, 4)) return SQ_ERR_MISALIGNED;
  const bool bf = xt == SQ_BF16;
  if (axis == SQ_AMAX_PER_COLUMN)
    return from_cuda(sqh::launch_amax_cols(x, bf, rows, cols, amax, accumulate != 0, S(stream)));
  return from_cuda(sqh::launch_amax_rows(x, bf, rows, cols, amax, accumulate != 0, S(stream)));
}

sq_status sq_smooth_factors(const float* amax_x, const float* amax_w, int64_t K, double alpha,
                            float* s, float* s_inv, void* stream) {
  if (!amax_x || !amax_w || !s || K <= 0) return SQ_ERR_INVALID_ARG;
  if (!(alpha >= 0.0 && alpha <= 1.0)) return SQ_ERR_INVALID_ARG;  // also rejects NaN
  if (!al(amax_x, 4) || !al(amax_w, 4) || !al(s, 4)) return SQ_ERR_MISALIGNED;
  if (s_inv && !al(s_inv, 4)) return SQ_ERR_MISALIGNED;
  return from_cuda(sqh::launch_smooth_factors(amax_x, amax_w, K, alpha, s, s_inv, S(stream)));
}

sq_status sq_quantize_weight(const void* w, sq_dtype wt, int64_t K, int64_t N, const float* s,
                             sq_dtype qt, void* wq, float* sw, void* stream) {
  if (!w || !wq || !sw) return SQ_ERR_INVALID_ARG;
  if (wt != SQ_F32 && wt != SQ_BF16) return SQ_ERR_INVALID_ARG;
  if (qt != SQ_I8 && qt != SQ_E4M3 && qt != SQ_I4) return SQ_ERR_INVALID_ARG;
  if (K <= 0 || N <= 0 || K % 16 != 0 || N % 8 != 0 || K > INT32_MAX || N > INT32_MAX)
    return SQ_ERR_INVALID_ARG;
  if (qt == SQ_I4 && K % 32 != 0) return SQ_ERR_INVALID_ARG;
  if (qt == SQ_I4 && s) return SQ_ERR_UNSUPPORTED;  // weight-only: no smoothing
  if (!al(w, 16) || !al(wq, 16) || !al(sw, 16)) return SQ_ERR_MISALIGNED;
  if (s && !al(s, 4)) return SQ_ERR_MISALIGNED;
  if (qt == SQ_I4)
    return from_cuda(sqh::launch_quantize_weight_i4(w, wt == SQ_BF16, K, N,
                                                    static_cast<uint8_t*>(wq), sw, S(stream)));
  return from_cuda(sqh::launch_quantize_weight(w, wt == SQ_BF16, K, N, s, qt == SQ_E4M3,
                                               static_cast<uint8_t*>(wq), sw, S(stream)));
}

sq_status sq_quantize_act(const void* x, sq_dtype xt, int64_t M, int64_t K, const float* s,
                          const float* s_inv, sq_dtype qt, void* xq, float* sx, uint32_t flags,
                          void* stream) {
  if (flags & ~uint32_t(SQ_OVERLAP_PREVIOUS)) return SQ_ERR_INVALID_ARG;
  if (xt != SQ_F32 && xt != SQ_BF16) return SQ_ERR_INVALID_ARG;
  if (qt != SQ_I8 && qt != SQ_E4M3) return SQ_ERR_INVALID_ARG;
  if (M < 0 || K <= 0 || K % 16 != 0 || K > 65536 || M > INT32_MAX) return SQ_ERR_INVALID_ARG;
  if (M == 0) return SQ_OK;  // empty batch: pointers may be NULL
  if (!x || !xq || !sx) return SQ_ERR_INVALID_ARG;
  if (!al(x, 16) || !al(xq, 16) || !al(sx, 4)) return SQ_ERR_MISALIGNED;
  if (s && !al(s, 16)) return SQ_ERR_MISALIGNED;
  if (s_inv && !al(s_inv, 16)) return SQ_ERR_MISALIGNED;
  return from_cuda(sqh::launch_quantize_act(x, xt == SQ_BF16, M, K, s, s ? s_inv : nullptr,
                                            qt == SQ_E4M3, static_cast<uint8_t*>(xq), sx,
                                            (flags & SQ_OVERLAP_PREVIOUS) != 0, S(stream)));
}

sq_status sq_quantize_act_tensor(const void* x, sq_dtype xt, int64_t M, int64_t K,
                                 const float* s, const float* s_inv, sq_dtype qt,
                                 const float* amax_prev, void* xq, float* sx, float* amax_out,
                                 void* stream) {
  if (xt != SQ_F32 && xt != SQ_BF16) return SQ_ERR_INVALID_ARG;
  if (qt != SQ_I8 && qt != SQ_E4M3) return SQ_ERR_INVALID_ARG;
  if (M < 0 || K <= 0 || K % 16 != 0 || K > 65536 || M > INT32_MAX) return SQ_ERR_INVALID_ARG;
  if (!amax_out || amax_out == amax_prev) return SQ_ERR_INVALID_ARG;
  if (!al(amax_out, 4) || (amax_prev && !al(amax_prev, 4))) return SQ_ERR_MISALIGNED;
  if (M == 0) {  // empty batch: the tensor max is 0
    return from_cuda(cudaMemsetAsync(amax_out, 0, sizeof(float), S(stream)));
  }
  if (!x || !xq || !sx) return SQ_ERR_INVALID_ARG;
  if (!al(x, 16) || !al(xq, 16) || !al(sx, 4)) return SQ_ERR_MISALIGNED;
  if (s && !al(s, 16)) return SQ_ERR_MISALIGNED;
  if (s_inv && !al(s_inv, 16)) return SQ_ERR_MISALIGNED;
  return from_cuda(sqh::launch_quantize_act_tensor(x, xt == SQ_BF16, M, K, s, s ? s_inv : nullptr,
                                                   qt == SQ_E4M3, amax_prev,
                                                   static_cast<uint8_t*>(xq), sx, amax_out,
                                                   S(stream)));
}

sq_status sq_fold_smoothing(const void* p, sq_dtype pt, int64_t rows, int64_t cols,
                            const float* s, sq_axis axis, float* out, void* stream) {
  if (pt != SQ_F32 && pt != SQ_BF16) return SQ_ERR_INVALID_ARG;
  if (axis != SQ_AMAX_PER_COLUMN && axis != SQ_AMAX_PER_ROW) return SQ_ERR_INVALID_ARG;
  if (rows < 0 || cols < 0) return SQ_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return SQ_OK;  // nothing to fold: pointers may be NULL
  if (rows > INT64_MAX / cols) return SQ_ERR_INVALID_ARG;
  if (!p || !s || !out || static_cast<const void*>(out) == p) return SQ_ERR_INVALID_ARG;
  if (!al(p, pt == SQ_BF16 ? 2 : 4) || !al(s, 4) || !al(out, 4)) return SQ_ERR_MISALIGNED;
  return from_cuda(sqh::launch_fold_smoothing(p, pt == SQ_BF16, rows, cols, s,
                                              axis == SQ_AMAX_PER_COLUMN, out, S(stream)));
}

size_t sq_gemm_workspace_bytes(void) { return sqh::gemm_workspace_bytes(); }

sq_status sq_gemm_w8a8(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw,
                       const uint16_t* bias, int64_t M, int64_t N, int64_t K, void* y, sq_dtype yt,
                       int32_t* acc, void* workspace, size_t workspace_bytes, void* stream) {
  sq_status c = check_gemm(xq, sx, wq, sw, bias, M, N, K, y, yt, acc);
  if (c != SQ_OK) return c;
  if (M == 0) return SQ_OK;
  if (workspace && !al(workspace, 256)) return SQ_ERR_MISALIGNED;
  return from_cuda(run_gemm_any(false, reinterpret_cast<const uint8_t*>(xq), sx,
                                    reinterpret_cast<const uint8_t*>(wq), sw, bias, M, N, K, y,
                                    yt == SQ_BF16 ? sqh::OutKind::BF16 : sqh::OutKind::F32, acc,
                                    workspace, workspace_bytes, S(stream)));
}

sq_status sq_gemm_fp8(const uint8_t* xq, const float* sx, const uint8_t* wq, const float* sw,
                      const uint16_t* bias, int64_t M, int64_t N, int64_t K, void* y, sq_dtype yt,
                      void* workspace, size_t workspace_bytes, void* stream) {
  sq_status c = check_gemm(xq, sx, wq, sw, bias, M, N, K, y, yt, nullptr);
  if (c != SQ_OK) return c;
  if (M == 0) return SQ_OK;
  if (workspace && !al(workspace, 256)) return SQ_ERR_MISALIGNED;
  return from_cuda(run_gemm_any(true, xq, sx, wq, sw, bias, M, N, K, y,
                                    yt == SQ_BF16 ? sqh::OutKind::BF16 : sqh::OutKind::F32, nullptr,
                                    workspace, workspace_bytes, S(stream)));
}

sq_status sq_linear(const void* x, sq_dtype xt, const float* s, const float* s_inv,
                    const void* wq, const float* sw,
                    const uint16_t* bias, sq_dtype qt, int64_t M, int64_t N, int64_t K,
                    void* xq_buf, float* sx_buf, void* y, sq_dtype yt, void* workspace,
                    size_t workspace_bytes, void* stream) {
  if (qt != SQ_I8 && qt != SQ_E4M3) return SQ_ERR_INVALID_ARG;
  sq_status c = check_gemm(xq_buf, sx_buf, wq, sw, bias, M, N, K, y, yt, nullptr);
  if (c != SQ_OK || M == 0) return c;
  c = sq_quantize_act(x, xt, M, K, s, s_inv, qt, xq_buf, sx_buf, 0u, stream);
  if (c != SQ_OK) return c;
  if (qt == SQ_I8)
    return sq_gemm_w8a8(static_cast<const int8_t*>(xq_buf), sx_buf, static_cast<const int8_t*>(wq),
                        sw, bias, M, N, K, y, yt, nullptr, workspace, workspace_bytes, stream);
  return sq_gemm_fp8(static_cast<const uint8_t*>(xq_buf), sx_buf, static_cast<const uint8_t*>(wq),
                     sw, bias, M, N, K, y, yt, workspace, workspace_bytes, stream);
}

sq_status sq_gemm_w8a8_noalloc(const int8_t* xq, const float* sx, const int8_t* wq,
                               const float* sw, const uint16_t* bias, int64_t M, int64_t N,
                               int64_t K, void* y, sq_dtype yt, void* stream) {
  sq_status c = check_gemm(xq, sx, wq, sw, bias, M, N, K, y, yt, nullptr);
  if (c != SQ_OK) return c;
  if (M == 0) return SQ_OK;
  if (sqh::gemm_skinny_applies(M))  // the few-token form uses no scratch
    return from_cuda(sqh::launch_gemm_skinny(false, reinterpret_cast<const uint8_t*>(xq), sx,
                                             reinterpret_cast<const uint8_t*>(wq), sw, bias, M,
                                             N, K, y,
                                             yt == SQ_BF16 ? sqh::OutKind::BF16
                                                           : sqh::OutKind::F32,
                                             nullptr, S(stream)));
  // the split-tile scratch this device needs must fit the fixed array
  if (sqh::gemm_workspace_bytes() > kNoAllocScratchBytes) return SQ_ERR_SCRATCH_TOO_SMALL;
  void* scratch = noalloc_scratch_ptr();
  if (!scratch) return SQ_ERR_CUDA;
  // the array keeps the previous call's contents: the counters the split
  // tiles synchronize on must start at zero
  if (cudaMemsetAsync(scratch, 0, sqh::gemm_workspace_counter_bytes(), S(stream)) != cudaSuccess)
    return SQ_ERR_CUDA;
  return from_cuda(run_gemm_any(false, reinterpret_cast<const uint8_t*>(xq), sx,
                                    reinterpret_cast<const uint8_t*>(wq), sw, bias, M, N, K, y,
                                    yt == SQ_BF16 ? sqh::OutKind::BF16 : sqh::OutKind::F32, nullptr,
                                    scratch, kNoAllocScratchBytes, S(stream)));
}

sq_status sq_gemm_weight_only(const void* x, const void* wq, sq_dtype wqt, const float* sw,
                              const uint16_t* bias, int64_t M, int64_t N, int64_t K, void* y,
                              sq_dtype yt, void* stream) {
  if (wqt != SQ_I8 && wqt != SQ_I4) return SQ_ERR_INVALID_ARG;
  if (M < 0 || N <= 0 || K <= 0 || N % 8 != 0) return SQ_ERR_INVALID_ARG;
  if (K % (wqt == SQ_I4 ? 32 : 16) != 0) return SQ_ERR_INVALID_ARG;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return SQ_ERR_INVALID_ARG;
  if (yt != SQ_BF16 && yt != SQ_F32) return SQ_ERR_INVALID_ARG;
  if (M == 0) return SQ_OK;  // empty batch: pointers may be NULL
  if (!x || !wq || !sw || !y) return SQ_ERR_INVALID_ARG;
  if (!al(x, 16) || !al(wq, 16) || !al(y, 16) || !al(sw, 4)) return SQ_ERR_MISALIGNED;
  if (bias && !al(bias, 2)) return SQ_ERR_MISALIGNED;
  return from_cuda(sqh::launch_gemm_weight_only(
      wqt == SQ_I4 ? 4 : 8, static_cast<const uint16_t*>(x), wq, sw, bias, M, N, K, y,
      yt == SQ_BF16 ? sqh::OutKind::BF16 : sqh::OutKind::F32, S(stream)));
}

sq_status sq_rmsnorm_quantize_act(const void* x, const float* g, float eps, int64_t M,
                                  int64_t K, sq_dtype qt, void* xq, float* sx, float* xn,
                                  uint32_t flags, void* stream) {
  if (flags & ~uint32_t(SQ_OVERLAP_PREVIOUS)) return SQ_ERR_INVALID_ARG;
  if (qt != SQ_I8 && qt != SQ_E4M3) return SQ_ERR_INVALID_ARG;
  if (M < 0 || K <= 0 || K % 8 != 0 || M > INT32_MAX) return SQ_ERR_INVALID_ARG;
  if (!(eps > 0.0f) || !std::isfinite(eps)) return SQ_ERR_INVALID_ARG;
  if (K > sqh::rmsnorm_quant_max_k()) return SQ_ERR_UNSUPPORTED;
  if (M == 0) return SQ_OK;  // empty batch: pointers may be NULL
  if (!x || !g || !xq || !sx) return SQ_ERR_INVALID_ARG;
  // Other rows' CTAs may still be reading x while this one writes: no output may alias an input.
  const uint64_t xb = uint64_t(M) * uint64_t(K) * 2, qb = uint64_t(M) * uint64_t(K);
  if (overlap(xq, qb, x, xb) || overlap(xq, qb, g, uint64_t(K) * 4) ||
      overlap(sx, uint64_t(M) * 4, x, xb) || overlap(sx, uint64_t(M) * 4, g, uint64_t(K) * 4) ||
      overlap(sx, uint64_t(M) * 4, xq, qb))
    return SQ_ERR_INVALID_ARG;
  const uint64_t nb = uint64_t(M) * uint64_t(K) * 4;
  if (xn && (overlap(xn, nb, x, xb) || overlap(xn, nb, g, uint64_t(K) * 4) ||
             overlap(xn, nb, xq, qb) || overlap(xn, nb, sx, uint64_t(M) * 4)))
    return SQ_ERR_INVALID_ARG;
  if (!al(x, 16) || !al(g, 16) || !al(xq, 16) || !al(sx, 4) || !al(xn, 16))
    return SQ_ERR_MISALIGNED;
  return from_cuda(sqh::launch_rmsnorm_quant(static_cast<const uint16_t*>(x), g, eps, M, K,
                                             qt == SQ_E4M3, xq, sx, xn,
                                             (flags & SQ_OVERLAP_PREVIOUS) != 0, S(stream)));
}

sq_status sq_selftest_fast_division(int64_t* mismatches, void* stream) {
  if (!mismatches) return SQ_ERR_INVALID_ARG;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_sq_selftest_count) != cudaSuccess) return SQ_ERR_CUDA;
  if (cudaMemsetAsync(p, 0, sizeof(unsigned long long), S(stream)) != cudaSuccess) return SQ_ERR_CUDA;
  if (sqh::launch_selftest_fast_division(static_cast<unsigned long long*>(p), S(stream)) != cudaSuccess)
    return SQ_ERR_CUDA;
  unsigned long long v = 0;
  if (cudaMemcpyAsync(&v, p, sizeof(v), cudaMemcpyDeviceToHost, S(stream)) != cudaSuccess ||
      cudaStreamSynchronize(S(stream)) != cudaSuccess)
    return SQ_ERR_CUDA;
  *mismatches = static_cast<int64_t>(v);
  return SQ_OK;
}

sq_status sq_probe_wait_timeout(int64_t timeout_ns, void* stream) {
  if (timeout_ns < 1000000 || timeout_ns > 10000000000LL) return SQ_ERR_INVALID_ARG;
  int* st = sqh::status_ptr();
  if (!st) return SQ_ERR_CUDA;
  probe_wait_kernel<<<1, 32, 0, S(stream)>>>(timeout_ns, st);
  return from_cuda(cudaGetLastError());
}

}  // extern "C"
