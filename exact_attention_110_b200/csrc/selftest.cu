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

// Accuracy self-test of the FMA-pipe exp2 (ex2_poly2: range reduction x = n + f, n added into
// the exponent field, 2^f by a cubic fitted for this library), a compile-time option of the
// softmax kernels that the shipped build leaves off. Evaluates it and the special-function
// unit's ex2.approx on the same inputs, two per thread (the packed form works on pairs).
__global__ void fa_selftest_ex2_kernel(const float* x, float* y_poly, float* y_sfu, int n) {
  const Ex2PolyConsts k = ex2_poly_consts();
  const int stride = 2 * gridDim.x * blockDim.x;
  for (int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x); i < n; i += stride) {
    const float a = x[i], b = i + 1 < n ? x[i + 1] : 0.f;
    float p0, p1;
    f2_unpack(ex2_poly2(f2_pack(a, b), k), p0, p1);
    y_poly[i] = p0;
    y_sfu[i] = ex2(a);
    if (i + 1 < n) {
      y_poly[i + 1] = p1;
      y_sfu[i + 1] = ex2(b);
    }
  }
}

}  // namespace fa

extern "C" fa_status fa_selftest_ex2(const float* x, float* y_poly, float* y_sfu, int n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y_poly || !y_sfu))) return FA_ERR_INVALID;
  if (n == 0) return FA_OK;
  fa::fa_selftest_ex2_kernel<<<64, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y_poly, y_sfu, n);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

extern "C" fa_status fa_selftest_wait_timeout(unsigned int limit_us, void* stream) {
  if (limit_us == 0 || limit_us > 1000000u) return FA_ERR_INVALID;
  fa::fa_selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(1000ull * limit_us);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}
