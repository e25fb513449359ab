// Failure-detection self-test. One thread waits, bounded by a short limit, on an mbarrier
// that nothing arrives at; the same bounded wait the attention kernels use gives up, records
// WAIT_SELFTEST in the device status word and the kernel returns normally. This exercises the
// timeout path end to end (device flag -> fa_last_device_status) without faulting, trapping
// or hanging the GPU.
#include "fa.h"  // include/ is on the include path
#include "kernels.h"
#include "ptx.cuh"

namespace fa {

__global__ void fa_selftest_timeout_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ AbortState ab;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    ab.flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &ab, limit_ns, WAIT_SELFTEST);
}

}  // namespace fa

extern "C" fa_status fa_selftest_wait_timeout(unsigned int limit_us, void* stream) {
  if (limit_us == 0 || limit_us > 1000000u) return FA_ERR_INVALID;
  fa::fa_selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(1000ull * limit_us);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}
