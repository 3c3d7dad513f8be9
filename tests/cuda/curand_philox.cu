// Test helper: evaluates cuRAND's device-side Philox4x32-10 function on given
// counters and keys, so the tests can compare the oracle's Philox (all four
// counter words) with the library routine.  Not part of the product.
#include <cstdint>
#include <curand_kernel.h>

__global__ void philox_many(const uint4* ctr, const uint2* key, uint4* out, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = curand_Philox4x32_10(ctr[i], key[i]);
}

extern "C" int curand_philox_many(const void* ctr, const void* key, void* out, int n) {
  uint4 *dc = nullptr, *dout = nullptr;
  uint2* dk = nullptr;
  if (n <= 0) return 0;
  if (cudaMalloc(&dc, sizeof(uint4) * n) != cudaSuccess) return 1;
  if (cudaMalloc(&dk, sizeof(uint2) * n) != cudaSuccess) return 1;
  if (cudaMalloc(&dout, sizeof(uint4) * n) != cudaSuccess) return 1;
  cudaMemcpy(dc, ctr, sizeof(uint4) * n, cudaMemcpyHostToDevice);
  cudaMemcpy(dk, key, sizeof(uint2) * n, cudaMemcpyHostToDevice);
  philox_many<<<(n + 255) / 256, 256>>>(dc, dk, dout, n);
  const cudaError_t e = cudaMemcpy(out, dout, sizeof(uint4) * n, cudaMemcpyDeviceToHost);
  cudaFree(dc);
  cudaFree(dk);
  cudaFree(dout);
  return e == cudaSuccess ? 0 : 2;
}
