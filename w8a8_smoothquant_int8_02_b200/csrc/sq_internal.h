// sq_internal.h -- host-side launchers shared between the libsq translation
// units. Arguments are already validated by the C-ABI layer (sq_api.cu).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace sqh {

// Device address of the library's status word (see sq_get_device_status).
int* status_ptr();

// a1 / a2
cudaError_t launch_amax_cols(const void* x, bool bf16, int64_t rows, int64_t cols, float* amax,
                             bool accumulate, cudaStream_t st);
cudaError_t launch_amax_rows(const void* x, bool bf16, int64_t rows, int64_t cols, float* amax,
                             bool accumulate, cudaStream_t st);
// a3
cudaError_t launch_smooth_factors(const float* ax, const float* aw, int64_t K, double alpha,
                                  float* s, float* s_inv, cudaStream_t st);
// a4
cudaError_t launch_quantize_weight(const void* w, bool bf16, int64_t K, int64_t N, const float* s,
                                   bool e4m3, uint8_t* wq, float* sw, cudaStream_t st);
// a5
// overlap: the caller rules out any access of the previous kernel in the stream
// to x, s, s_inv (writes) and xq, sx; the pass may then run while that kernel
// finishes and completes after it
cudaError_t launch_quantize_act(const void* x, bool bf16, int64_t M, int64_t K, const float* s,
                                const float* s_inv, bool e4m3, uint8_t* xq, float* sx,
                                bool overlap, cudaStream_t st);
cudaError_t launch_quantize_act_tensor(const void* x, bool bf16, int64_t M, int64_t K,
                                       const float* s, const float* s_inv, bool e4m3,
                                       const float* amax_prev, uint8_t* xq, float* sx,
                                       float* amax_out, cudaStream_t st);
// RMS normalization of x with gain g (1/s folded in) fused with per-token
// quantization; K <= rmsnorm_quant_max_k(), a multiple of 8
int rmsnorm_quant_max_k();
cudaError_t launch_rmsnorm_quant(const uint16_t* x, const float* g, float eps, int64_t M,
                                 int64_t K, bool e4m3, void* xq, float* sx, float* xn,
                                 bool overlap, cudaStream_t st);
// offline fold of 1/s into the producer of X
cudaError_t launch_fold_smoothing(const void* p, bool bf16, int64_t rows, int64_t cols,
                                  const float* s, bool per_column, float* out, cudaStream_t st);
cudaError_t launch_selftest_fast_division(unsigned long long* mismatches, cudaStream_t st);
// a6 / a7
enum class OutKind { BF16, F32 };
cudaError_t launch_gemm(bool e4m3, const uint8_t* xq, const float* sx, const uint8_t* wq,
                        const float* sw, const uint16_t* bias, int64_t M, int64_t N, int64_t K,
                        void* y, OutKind yk, int32_t* acc, void* ws, size_t ws_bytes,
                        cudaStream_t st);
// a6 / a7 for M <= 16: the weight-streaming form (sq_gemm_skinny.cu)
bool gemm_skinny_applies(int64_t M);
cudaError_t launch_gemm_skinny(bool e4m3, const uint8_t* xq, const float* sx, const uint8_t* wq,
                               const float* sw, const uint16_t* bias, int64_t M, int64_t N,
                               int64_t K, void* y, OutKind yk, int32_t* acc, cudaStream_t st);
// a6 / a7 when the 128 x 128 tiles fit in one wave (sq_gemm_small.cu)
bool gemm_small_applies(int64_t M, int64_t N, int64_t K);
cudaError_t launch_gemm_small(bool e4m3, const uint8_t* xq, const float* sx, const uint8_t* wq,
                              const float* sw, const uint16_t* bias, int64_t M, int64_t N,
                              int64_t K, void* y, OutKind yk, int32_t* acc, cudaStream_t st);
// weight-only W8A16 / W4A16 GEMM for few tokens (sq_gemm_wonly.cu)
cudaError_t launch_gemm_weight_only(int bits, const uint16_t* x, const void* wq, const float* sw,
                                    const uint16_t* bias, int64_t M, int64_t N, int64_t K,
                                    void* y, OutKind yk, cudaStream_t st);
cudaError_t launch_quantize_weight_i4(const void* w, bool bf16, int64_t K, int64_t N,
                                      uint8_t* wq4, float* sw, cudaStream_t st);
size_t gemm_workspace_bytes();
size_t gemm_workspace_counter_bytes();

// Programmatic dependent launch of the streaming kernels (on unless the
// environment sets SQ_PDL=0): such a launch may start while the previous
// kernel in the stream finishes; the kernels wait (griddepcontrol.wait)
// before touching global memory.
bool pdl_enabled();

template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kern)(Params...), unsigned grid, int threads, size_t smem,
                       cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(unsigned(threads), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}


}  // namespace sqh
