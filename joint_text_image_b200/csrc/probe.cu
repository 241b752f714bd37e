// probe.cu -- exercise of the bounded-wait machinery: one thread waits on an
// mbarrier that nothing arrives on; the wait expires after `timeout_ns`,
// records HIA_ERR_DEVICE_TIMEOUT in the status word and the kernel returns.
#include "kernels.h"
#include "sm100.cuh"

namespace hia {

__global__ void wait_probe_kernel(int* status, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const WaitCtx wc{&abort_flag, status, timeout_ns};
  if (threadIdx.x == 0) mbar_wait(&bar, 0, wc);
}

__global__ void exp2_probe_kernel(const float* x, float* y, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (2 * i < n) {
    const float2 r = exp2_fma2(make_float2(x[2 * i], 2 * i + 1 < n ? x[2 * i + 1] : 0.f));
    y[2 * i] = r.x;
    if (2 * i + 1 < n) y[2 * i + 1] = r.y;
  }
}

cudaError_t launch_exp2_probe(const float* x, float* y, int n, cudaStream_t st) {
  if (n > 0) exp2_probe_kernel<<<((n + 1) / 2 + 255) / 256, 256, 0, st>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_wait_probe(int* status, uint64_t timeout_ns, cudaStream_t st) {
  wait_probe_kernel<<<1, 32, 0, st>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace hia
