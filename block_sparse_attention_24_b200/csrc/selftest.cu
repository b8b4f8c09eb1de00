// Diagnostic kernel for the failure path every pipeline kernel relies on: one
// thread waits, through the same bounded wait the attention and tile-map
// kernels use, on an mbarrier that nothing ever arrives on. After the limit
// the wait gives up, records VEDA_ERR_TIMEOUT in the caller's status word and
// the kernel returns normally, leaving the context usable.
#include "veda_internal.cuh"

namespace veda {
void set_last_error(const char* fmt, ...);
namespace {

__global__ void wait_timeout_kernel(int32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
}

}  // namespace
}  // namespace veda

extern "C" int veda_selftest_wait_timeout(const veda_layer* L, uint32_t limit_ms, cudaStream_t stream) {
  if (!L || !L->dev_status) {
    veda::set_last_error("layer or dev_status is NULL");
    return VEDA_ERR_INVALID_ARG;
  }
  if (limit_ms < 1 || limit_ms > 10000) {
    veda::set_last_error("limit_ms=%u outside [1, 10000]", limit_ms);
    return VEDA_ERR_INVALID_ARG;
  }
  veda::wait_timeout_kernel<<<1, 32, 0, stream>>>(L->dev_status, (uint64_t)limit_ms * 1000000ull);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    veda::set_last_error("veda_selftest_wait_timeout: %s", cudaGetErrorString(e));
    return VEDA_ERR_CUDA;
  }
  return VEDA_OK;
}
