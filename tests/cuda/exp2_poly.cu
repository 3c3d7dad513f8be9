// Test helper: evaluates the library's FMA-pipe exp2 (exp2_poly2 in
// ab_ptx.cuh) and CUDA's exp2f on the same inputs.  Not part of the product.
#include "ab_ptx.cuh"

__global__ void eval(const float* x, float* poly, float* ref, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    float a = x[i], b = x[i + 1];
    ab::exp2_poly2(a, b);
    poly[i] = a;
    poly[i + 1] = b;
    ref[i] = exp2f(x[i]);
    ref[i + 1] = exp2f(x[i + 1]);
  }
}

extern "C" int exp2_poly_eval(const float* x, float* poly, float* ref, int n) {
  float *dx, *dp, *dr;
  if (cudaMalloc(&dx, 4 * n) || cudaMalloc(&dp, 4 * n) || cudaMalloc(&dr, 4 * n)) return 1;
  cudaMemcpy(dx, x, 4 * n, cudaMemcpyHostToDevice);
  eval<<<(n / 2 + 255) / 256, 256>>>(dx, dp, dr, n);
  cudaMemcpy(poly, dp, 4 * n, cudaMemcpyDeviceToHost);
  const cudaError_t e = cudaMemcpy(ref, dr, 4 * n, cudaMemcpyDeviceToHost);
  cudaFree(dx); cudaFree(dp); cudaFree(dr);
  return e == cudaSuccess ? 0 : 2;
}
