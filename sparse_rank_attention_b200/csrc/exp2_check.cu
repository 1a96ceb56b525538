// The softmax exponentials of the head-dim-128 attention kernels, run elementwise so that
// a test can hold them against exp2 in double precision (see rola_eval_exp2).
#include "rola_internal.cuh"
#include "softmax_exp.cuh"

namespace rola {
namespace {

__global__ void eval_exp2_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n, int mode) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    y[i] = mode == 0 ? ex2_approx(x[i]) : ex2_poly(x[i]);
}

}  // namespace

cudaError_t launch_eval_exp2(const float* x, float* y, int64_t n, int mode, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int64_t blocks = (n + 255) / 256;
  eval_exp2_kernel<<<(unsigned)(blocks < 4 * 148 ? blocks : 4 * 148), 256, 0, st>>>(x, y, n, mode);
  return cudaGetLastError();
}

}  // namespace rola
