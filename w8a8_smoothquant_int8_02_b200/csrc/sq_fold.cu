// sq_fold.cu -- offline fold of the activation smoothing into the layer that
// produces X.
//
// "Weight-Activation Quantization" (infra.bea.ai) §3, the two-step pipeline:
// X_tilde = X diag(1/s) belongs to offline model preparation; the grasp.study
// lesson on W8A16 vs W8A8, §2 "The Challenge of Activation Quantization:
// SmoothQuant": the transform is done offline, with no runtime overhead. The
// producer of X carries one parameter (a gain entry, or a row or column of a
// weight) per channel k of X; dividing those by s_k once makes it emit
// X_tilde itself, and this layer then quantizes its input with s = NULL.
//
//   per column: out[r,c] = p[r,c] / s[c]   (a gain vector [1,K], or a producer
//                                           weight [R,K] in the [in,out] layout)
//   per row:    out[r,c] = p[r,c] / s[r]   (a producer weight stored [K,R])
//
// One IEEE binary32 division per element, the operation the runtime kernels
// apply to x. Offline and HBM-bound (4 or 2 bytes read, 4 written per
// element): a plain coalesced loop, one row per block iteration.
#include <cstdint>

#include "sq_internal.h"

namespace {

template <bool BF16, bool PER_COLUMN>
__global__ void __launch_bounds__(256) fold_smoothing_kernel(const void* __restrict__ p,
                                                             int64_t rows, int64_t cols,
                                                             const float* __restrict__ s,
                                                             float* __restrict__ out) {
  const int64_t c0 = int64_t(blockIdx.y) * blockDim.x + threadIdx.x;
  const int64_t cstep = int64_t(gridDim.y) * blockDim.x;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const float sr = PER_COLUMN ? 1.0f : s[r];
    for (int64_t c = c0; c < cols; c += cstep) {
      const int64_t i = r * cols + c;
      float v;
      if constexpr (BF16)
        v = __uint_as_float(uint32_t(static_cast<const uint16_t*>(p)[i]) << 16);
      else
        v = static_cast<const float*>(p)[i];
      out[i] = __fdiv_rn(v, PER_COLUMN ? s[c] : sr);
    }
  }
}

template <bool BF16, bool PER_COLUMN>
void launch_fold_t(const void* p, int64_t rows, int64_t cols, const float* s, float* out,
                   cudaStream_t st) {
  const int64_t col_blocks = (cols + 255) / 256;
  const unsigned gy = unsigned(col_blocks < 64 ? col_blocks : 64);
  const int64_t want_x = (int64_t(148) * 8 + gy - 1) / gy;
  const unsigned gx = unsigned(rows < want_x ? rows : want_x);
  fold_smoothing_kernel<BF16, PER_COLUMN><<<dim3(gx, gy), 256, 0, st>>>(p, rows, cols, s, out);
}

}  // namespace

namespace sqh {

cudaError_t launch_fold_smoothing(const void* p, bool bf16, int64_t rows, int64_t cols,
                                  const float* s, bool per_column, float* out, cudaStream_t st) {
  if (bf16) {
    if (per_column) launch_fold_t<true, true>(p, rows, cols, s, out, st);
    else launch_fold_t<true, false>(p, rows, cols, s, out, st);
  } else {
    if (per_column) launch_fold_t<false, true>(p, rows, cols, s, out, st);
    else launch_fold_t<false, false>(p, rows, cols, s, out, st);
  }
  return cudaGetLastError();
}

}  // namespace sqh
