// selftest.cu -- exercises the library's failure detection on the device: a bounded wait
// that nothing completes gives up after its limit, reports MOE_DEV_TIMEOUT through the
// status word and returns, leaving the context usable.
#include "device.cuh"
#include "internal.h"
#include "moe.h"

namespace moe {
namespace {

// One thread waits on an mbarrier whose only expected arrival never happens.
__global__ void wait_timeout_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  mbar_init(&bar, 1);
  fence_mbar_init();
  mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
}

}  // namespace
}  // namespace moe

extern "C" moe_status_t moe_selftest_wait_timeout(uint32_t* status, uint32_t limit_us,
                                                  void* stream) {
  if (!status || limit_us == 0 || limit_us > 1000000u) return MOE_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(status) % 4) return MOE_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  moe::wait_timeout_kernel<<<1, 32, 0, s>>>(status, (uint64_t)limit_us * 1000ull);
  uint32_t host = 0;
  if (cudaGetLastError() != cudaSuccess ||
      cudaMemcpyAsync(&host, status, sizeof host, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return (host & moe::MOE_DEV_TIMEOUT) ? MOE_ERR_TIMEOUT : MOE_OK;
}
