// Test harness (not part of the library): evaluates the prefill softmax's
// polynomial exp2 on a device array so its accuracy can be checked against
// exact powers of two on the host.
#include <cstdint>
#include <cuda_runtime.h>
#include "ptx.cuh"

namespace {
__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int n_pairs) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_pairs) return;
  float r0, r1;
  swa::f2_unpack(swa::exp2_poly2(swa::f2_pack(x[2 * i], x[2 * i + 1])), r0, r1);
  y[2 * i] = r0;
  y[2 * i + 1] = r1;
}
}  // namespace

extern "C" __attribute__((visibility("default"))) int exp2_poly_eval(const float* x, float* y, int n_pairs) {
  if (n_pairs <= 0) return 0;
  exp2_poly_kernel<<<(n_pairs + 255) / 256, 256>>>(x, y, n_pairs);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  return (int)e;
}
