// fp_selftest.cu -- device self-test of the softmax's two exp2 paths (the FMA-pipe polynomial and
// the MUFU ex2.approx instruction), so tests can bound the polynomial's error on the GPU itself.
#include "fp_dev.cuh"
#include "fp_internal.h"

namespace fp {

__global__ void exp2_selftest_kernel(const float* x, float* y_poly, float* y_mufu, long long n) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    float lo, hi;
    f2_split(exp2_poly2(f2_make(x[i], x[i])), lo, hi);
    y_poly[i] = lo;
    y_mufu[i] = ex2_approx(x[i]);
  }
}

cudaError_t launch_exp2_selftest(const float* x, float* y_poly, float* y_mufu, long long n, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const long long blocks = (n + 255) / 256;
  exp2_selftest_kernel<<<(int)(blocks < 4096 ? blocks : 4096), 256, 0, st>>>(x, y_poly, y_mufu, n);
  return cudaGetLastError();
}

}  // namespace fp
