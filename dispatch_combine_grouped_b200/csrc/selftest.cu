// Self-test of the failure path: a bounded wait on a barrier that nothing arrives on must
// give up after the limit, report MOE_ERR_TIMEOUT through the status word and return,
// leaving the CUDA context usable.  No fault, trap or hang is involved.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

__global__ void bounded_wait_selftest_kernel(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // expects one arrival that never comes
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait_for(&bar, 0, &abort_flag, limit_ns)) report(status, MOE_ERR_TIMEOUT);
}

}  // namespace moe

extern "C" moe_status moe_selftest_bounded_wait(int32_t* dev_status, uint64_t limit_ns, moe_stream_t stream) {
  if (!dev_status || limit_ns == 0 || limit_ns > 10000000000ull) return MOE_ERR_INVALID_ARG;
  moe::bounded_wait_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(dev_status, limit_ns);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
