// Test helper: the library's bounded mbarrier waits (ab_ptx.cuh) on a barrier
// that nothing ever completes.  The waits must give up after their time limit,
// record AB_ERR_TIMEOUT in the device error word and raise the CTA's abort
// flag, and a second role must then leave its own wait at once through that
// flag.  Nothing faults or hangs: every wait is bounded.  Not part of the
// product.
#include "ab_ptx.cuh"

__global__ void timeout_probe(int* out) {
  __shared__ uint64_t never;  // a phase that no thread ever completes
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ab::mbar_init(ab::smem_u32(&never), 1);
    abort_flag = 0;
    ab::fence_mbar_init();
  }
  __syncthreads();
  const unsigned long long t0 = ab::globaltimer_ns();
  bool ok = true;
  if (threadIdx.x < 32) {
    // warp 0: waits until the time limit
    ok = ab::mbar_wait(ab::smem_u32(&never), 0, &abort_flag);
  } else {
    // warp 1: starts waiting after warp 0 has given up, and must return as
    // soon as it sees the abort flag
    while (!*reinterpret_cast<volatile int*>(&abort_flag)) {
      if (ab::globaltimer_ns() - t0 > 4ull * ab::kWaitLimitNs) break;  // bounded as well
    }
    const unsigned long long t1 = ab::globaltimer_ns();
    ok = ab::mbar_wait(ab::smem_u32(&never), 0, &abort_flag);
    if (threadIdx.x == 32) out[3] = int((ab::globaltimer_ns() - t1) / 1000000ull);  // ms spent in the wait
  }
  const unsigned long long t2 = ab::globaltimer_ns();
  if (threadIdx.x == 0) {
    out[0] = ok ? 1 : 0;
    out[1] = int((t2 - t0) / 1000000ull);  // ms until warp 0 gave up
    out[2] = abort_flag;
  }
  if (threadIdx.x == 32) out[4] = ok ? 1 : 0;
  // the drain form (no abort flag) also gives up after the limit
  if (threadIdx.x == 0) out[5] = ab::mbar_wait_drain(ab::smem_u32(&never), 0) ? 1 : 0;
}

__global__ void read_error(int* out) { out[0] = ab::g_device_error; }

extern "C" int wait_timeout_probe(int* host_out) {
  int* d = nullptr;
  if (cudaMalloc(&d, 8 * sizeof(int)) != cudaSuccess) return 1;
  cudaMemset(d, 0xFF, 8 * sizeof(int));
  timeout_probe<<<1, 64>>>(d);
  read_error<<<1, 1>>>(d + 6);
  const cudaError_t e = cudaMemcpy(host_out, d, 8 * sizeof(int), cudaMemcpyDeviceToHost);
  cudaFree(d);
  return e == cudaSuccess ? 0 : 2;
}
