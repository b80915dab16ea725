// Device self-test of the attention softmax's exponential (see
// softmax_exp.cuh): evaluates the same device functions the attention
// kernels call, so a test can hold them to their stated error bounds.
#include <cuda_runtime.h>

#include <string>

#include "softmax_exp.cuh"
#include "stca_internal.h"

namespace stca {
namespace {

__global__ void ex2_kernel(const float* x, float* y, int64_t n, int method) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  // method 2 evaluates elements in pairs, as the softmax does
  if (method == 2) {
    const int64_t k = 2 * i;
    if (k >= n) return;
    float y0, y1;
    sx::ex2_fma2(x[k], k + 1 < n ? x[k + 1] : 0.f, y0, y1);
    y[k] = y0;
    if (k + 1 < n) y[k + 1] = y1;
    return;
  }
  if (i >= n) return;
  y[i] = method == 0 ? sx::ex2(x[i]) : sx::ex2_fma(x[i]);
}

}  // namespace
}  // namespace stca

using namespace stca;

extern "C" int stca_selftest_ex2(const float* x, float* y, int64_t n, int method, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return set_error(STCA_EINVAL, "stca_selftest_ex2: bad arguments");
  if (method < 0 || method > 2) return set_error(STCA_EINVAL, "stca_selftest_ex2: method must be 0, 1 or 2");
  if (n == 0) return STCA_OK;
  const int64_t work = method == 2 ? (n + 1) / 2 : n;
  const unsigned grid = static_cast<unsigned>((work + 255) / 256);
  ex2_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n, method);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(STCA_ECUDA, std::string("stca_selftest_ex2: ") + cudaGetErrorString(e));
  return STCA_OK;
}
