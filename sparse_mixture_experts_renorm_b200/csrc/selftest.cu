// selftest.cu — a diagnostic that exercises the bounded wait every kernel of
// the library uses on its mbarriers: one warp waits on a barrier phase that
// nothing completes, and the wait must give up after the limit, set
// MOE_DEV_TIMEOUT in the status word and return, leaving the context usable.
#include "common.cuh"

namespace moe {
namespace {

__global__ void wait_timeout_kernel(int32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  // no thread ever arrives on `bar`, so phase 0 never completes
  mbar_wait(&bar, 0, reinterpret_cast<volatile int*>(&abort_flag), status, limit_ns);
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_selftest_wait_timeout(int32_t* status_dev, long long limit_ns, void* stream) {
  if (!status_dev) {
    moe::set_error_detail("moe_selftest_wait_timeout: status_dev is NULL");
    return MOE_ERR_INVALID_ARG;
  }
  if (limit_ns < 1000000ll || limit_ns > 5000000000ll) {
    moe::set_error_detail("moe_selftest_wait_timeout: limit_ns must be within [1e6, 5e9] (got %lld)", limit_ns);
    return MOE_ERR_INVALID_ARG;
  }
  moe::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status_dev, (uint64_t)limit_ns);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) {
    moe::set_error_detail("moe_selftest_wait_timeout: launch failed: %s", cudaGetErrorString(err));
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
