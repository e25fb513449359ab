// Combine step of the split-key forward: the key range of every query row was cut into
// `nsplit` pieces, each of which produced its own softmax-normalised output O_s and
// log-sum-exp LSE_s. The exact result follows from the online normaliser's rule for merging
// two partial softmax states ([P2] §时间复杂度, the online normaliser; [P3] §3.2, §3.4):
//   LSE = log sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) * O_s.
// A piece that saw no key has LSE_s = -inf and weight 0; a row no piece saw gets O = 0 and
// LSE = -inf, as in the unsplit forward.
//
// HBM-bound: D/4 threads per row, 16-byte fp32 loads of each piece, one 8-byte store of four
// 16-bit outputs per thread; grid-stride over rows, sized to the SM count.
#include "kernels.h"
#include "ptx.cuh"

namespace fa {

template <int D, bool F16>
__global__ void __launch_bounds__(256) fa_fwd_merge_kernel(const FwdMergeParams p) {
  constexpr int TPR = D / 4;  // threads per row, four columns each
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long nthreads = (long long)gridDim.x * blockDim.x;
  for (long long e = tid; e < p.rows * TPR; e += nthreads) {
    const long long row = e / TPR;
    const int c4 = (int)(e % TPR);
    const long long bh = row / p.N, i = row % p.N;
    const size_t base = (size_t)bh * p.nsplit * p.Np + i;  // piece s at base + s * Np
    float mx = -INFINITY;
    for (int s = 0; s < p.nsplit; ++s) mx = fmaxf(mx, p.lse_part[base + (size_t)s * p.Np]);
    float sum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (mx > -INFINITY) {
      for (int s = 0; s < p.nsplit; ++s) {
        const size_t ps = base + (size_t)s * p.Np;
        const float w = expf(p.lse_part[ps] - mx);
        const float4 o = reinterpret_cast<const float4*>(p.o_part + ps * D)[c4];
        sum += w;
        acc.x += w * o.x;
        acc.y += w * o.y;
        acc.z += w * o.z;
        acc.w += w * o.w;
      }
    }
    const float inv = sum > 0.f ? 1.f / sum : 0.f;
    uint2 out;
    out.x = pack16<F16>(acc.x * inv, acc.y * inv);
    out.y = pack16<F16>(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2*>(p.o + row * D)[c4] = out;
    if (c4 == 0) p.lse[row] = sum > 0.f ? mx + logf(sum) : -INFINITY;
  }
}

cudaError_t launch_fwd_merge(const FwdMergeParams& p, cudaStream_t stream) {
  const int grid = device_sm_count() * 8;  // 8 resident 256-thread blocks per SM
  if (p.D == 64) {
    if (p.f16)
      fa_fwd_merge_kernel<64, true><<<grid, 256, 0, stream>>>(p);
    else
      fa_fwd_merge_kernel<64, false><<<grid, 256, 0, stream>>>(p);
  } else if (p.D == 256) {
    if (p.f16)
      fa_fwd_merge_kernel<256, true><<<grid, 256, 0, stream>>>(p);
    else
      fa_fwd_merge_kernel<256, false><<<grid, 256, 0, stream>>>(p);
  } else {
    if (p.f16)
      fa_fwd_merge_kernel<128, true><<<grid, 256, 0, stream>>>(p);
    else
      fa_fwd_merge_kernel<128, false><<<grid, 256, 0, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace fa
