// Memory-bound helper kernels of the backward pass.
//
//  * bwd_pre: D_i = sum_t dO_it * O_it for every query row (the row sums the softmax
//    Jacobian produces: sum_j P_ij dP_ij = dO_i . O_i; FlashAttention V1 lecture summary,
//    spark.aweffr.cn, §4.1) and LSE_i * log2(e) for the exp2-domain recomputation of P, both
//    stored negated (the backward's inner loops then need only fused multiply-adds; the
//    exponent offset also carries log2(scale), so the recomputed P comes out as scale * P),
//    and a zero-fill of the fp32 dQ accumulator that fa_bwd_main adds into.
//  * dq_finish: dq = bf16(dq_acc), the combine step after every key block has added its dQ
//    share ("FlashAttention-2 的前世今生" overview, jishu.shishitao.com, §主要操作, backward:
//    dQ is the one quantity shared across column blocks and is combined with atomic adds).
//
// Both are pure HBM streams: 16-byte vector loads/stores, grid-stride loops sized to the SM
// count, one row handled by D/8 consecutive threads (8 bf16 = 16 bytes each).
#include "kernels.h"
#include "ptx.cuh"

// Row groups (preprocess) or elements (dQ finish) a thread has in flight per step. Measured at
// N = 4096, d = 128: preprocess 4.42 -> 4.81 TB/s, dQ finish 5.47 -> 6.14 TB/s with 2; 4 lowers
// the preprocess again (54 registers halve its occupancy).
#define FA_AUX_UNROLL 2

namespace fa {

template <int D, bool F16>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const BwdPreParams p) {
  constexpr int TPR = D / 8;  // threads per row
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long nthreads = (long long)gridDim.x * blockDim.x;
  const int lane = threadIdx.x & 31, sub = lane % TPR;
  // Rows: dot products of O and dO. A warp covers 32/TPR rows per step; the trip count is
  // warp-uniform so the full-mask shuffles below always see all 32 lanes.
  constexpr int RPW = 32 / TPR;
  const long long warp_g = tid >> 5, nwarps = nthreads >> 5;
  // U row groups per step, their loads issued before any of their reductions (more bytes in
  // flight per thread).
  constexpr int U = FA_AUX_UNROLL;
  for (long long r0 = warp_g * RPW; r0 < p.rows; r0 += nwarps * RPW * U) {
    uint4 a[U], b[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long row = r0 + (long long)u * nwarps * RPW + lane / TPR;
      a[u] = b[u] = make_uint4(0u, 0u, 0u, 0u);
      if (row < p.rows) {
        a[u] = __ldg(reinterpret_cast<const uint4*>(p.o + row * D) + sub);
        b[u] = __ldg(reinterpret_cast<const uint4*>(p.dout + row * D) + sub);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long row = r0 + (long long)u * nwarps * RPW + lane / TPR;
      float acc = unpack16_lo<F16>(a[u].x) * unpack16_lo<F16>(b[u].x) + unpack16_hi<F16>(a[u].x) * unpack16_hi<F16>(b[u].x);
      acc += unpack16_lo<F16>(a[u].y) * unpack16_lo<F16>(b[u].y) + unpack16_hi<F16>(a[u].y) * unpack16_hi<F16>(b[u].y);
      acc += unpack16_lo<F16>(a[u].z) * unpack16_lo<F16>(b[u].z) + unpack16_hi<F16>(a[u].z) * unpack16_hi<F16>(b[u].z);
      acc += unpack16_lo<F16>(a[u].w) * unpack16_lo<F16>(b[u].w) + unpack16_hi<F16>(a[u].w) * unpack16_hi<F16>(b[u].w);
#pragma unroll
      for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off, TPR);
      if (sub == 0 && row < p.rows) {
        const long long bh = row / p.N, i = row % p.N;
        const long long out = bh * p.Np + i;
        p.delta[out] = -acc;                               // stored negated: the backward adds it
        p.lse2[out] = p.log2_scale - p.lse[row] * 1.4426950408889634f;  // log2(scale) - LSE*log2(e)
      }
    }
  }
  // Rows of a partial last query tile beyond N: -inf exponent offset (P = 0 there) and D = 0.
  const long long BH = p.rows / p.N, pad = p.Np - p.N;
  for (long long e = tid; e < BH * pad; e += nthreads) {
    const long long out = (e / pad) * p.Np + p.N + e % pad;
    p.delta[out] = 0.f;
    p.lse2[out] = -INFINITY;
  }
  if (tid == 0 && p.counters != nullptr) {  // the persistent backward's work counters
    p.counters[0] = 0ull;
    p.counters[1] = 0ull;
  }
  // Zero the dQ accumulator (float4 stores).
  const long long nvec = (p.rows / p.N) * (long long)p.Np * D / 4;
  float4* acc4 = reinterpret_cast<float4*>(p.dq_acc);
  for (long long e = tid; e < nvec; e += nthreads) acc4[e] = make_float4(0.f, 0.f, 0.f, 0.f);
}

template <int D, bool F16>
__global__ void __launch_bounds__(256) fa_dq_finish_kernel(const DqFinishParams p) {
  constexpr int TPR = D / 8;
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long nthreads = (long long)gridDim.x * blockDim.x;
  const long long total = p.rows * TPR;
  constexpr int U = FA_AUX_UNROLL;  // U elements' loads in flight before their stores
  for (long long e0 = tid; e0 < total; e0 += nthreads * U) {
    float4 a[U], b[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long e = e0 + (long long)u * nthreads;
      a[u] = b[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e < total) {
        const long long row = e / TPR;
        const int sub = (int)(e % TPR);
        const long long bh = row / p.N, i = row % p.N;
        const float4* src = reinterpret_cast<const float4*>(p.dq_acc + (bh * p.Np + i) * D) + 2 * sub;
        a[u] = src[0];
        b[u] = src[1];
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long e = e0 + (long long)u * nthreads;
      if (e < total) {
        const long long row = e / TPR;
        const int sub = (int)(e % TPR);
        uint4 w;
        w.x = pack16<F16>(a[u].x * p.scale, a[u].y * p.scale);
        w.y = pack16<F16>(a[u].z * p.scale, a[u].w * p.scale);
        w.z = pack16<F16>(b[u].x * p.scale, b[u].y * p.scale);
        w.w = pack16<F16>(b[u].z * p.scale, b[u].w * p.scale);
        reinterpret_cast<uint4*>(p.dq + row * D)[sub] = w;
      }
    }
  }
}


cudaError_t launch_bwd_pre(const BwdPreParams& p, cudaStream_t stream) {
  const int grid = device_sm_count() * 8;  // 8 resident 256-thread blocks per SM
  if (p.D == 64)
    p.f16 ? fa_bwd_pre_kernel<64, true><<<grid, 256, 0, stream>>>(p) : fa_bwd_pre_kernel<64, false><<<grid, 256, 0, stream>>>(p);
  else if (p.D == 256)
    p.f16 ? fa_bwd_pre_kernel<256, true><<<grid, 256, 0, stream>>>(p)
          : fa_bwd_pre_kernel<256, false><<<grid, 256, 0, stream>>>(p);
  else
    p.f16 ? fa_bwd_pre_kernel<128, true><<<grid, 256, 0, stream>>>(p)
          : fa_bwd_pre_kernel<128, false><<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_dq_finish(const DqFinishParams& p, cudaStream_t stream) {
  const int grid = device_sm_count() * 8;
  if (p.D == 64)
    p.f16 ? fa_dq_finish_kernel<64, true><<<grid, 256, 0, stream>>>(p)
          : fa_dq_finish_kernel<64, false><<<grid, 256, 0, stream>>>(p);
  else if (p.D == 256)
    p.f16 ? fa_dq_finish_kernel<256, true><<<grid, 256, 0, stream>>>(p)
          : fa_dq_finish_kernel<256, false><<<grid, 256, 0, stream>>>(p);
  else
    p.f16 ? fa_dq_finish_kernel<128, true><<<grid, 256, 0, stream>>>(p)
          : fa_dq_finish_kernel<128, false><<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace fa
