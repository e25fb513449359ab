// Backward kernel: recompute P from the saved LSE and produce dK, dV (and dQ shares).
//
// Method (sources cited by page and section):
//   [P1] "FlashAttention-2 的前世今生" overview, jishu.shishitao.com/detail/60083.html
//   [P3] FlashAttention V1 lecture summary, spark.aweffr.cn/summary/0684ec99-...
//  * Recomputation: only O and the per-row LSE are kept from the forward; each block of S and
//    P is rebuilt on chip when the backward needs it, with the same formula as the forward
//    ([P3] §4.2; [P1] §主要操作: FA2 keeps only the log-sum-exp).
//  * Work split: one worker per K/V column block, looping over the Q row blocks; dK and dV
//    accumulate on chip; dQ is the only quantity shared by column blocks and is combined
//    with atomic adds in memory ([P1] §主要操作, backward pass).
//  * Gradients (textbook chain rule through softmax, the Jacobian [P3] §4.1 alludes to):
//      dV_j += P_ij^T dO_i,  dP_ij = dO_i V_j^T,  dS_ij = P_ij o (dP_ij - D_i),
//      dK_j += scale dS_ij^T Q_i,  dQ_i += scale dS_ij K_j,  with D_i = rowsum(dO_i o O_i).
//
// sm_100a design (ours):
//  * CTA = one 128-key tile j of one (b, h). K_j and V_j stay in shared memory; Q_i, dO_i (and
//    the 128 LSE2 / D values of tile i) stream through an NS-deep ring.
//  * Everything is computed transposed so that on-chip results are directly operands:
//      S^T = K_j Q_i^T, dP^T = V_j dO_i^T           (TMEM, one key per TMEM lane)
//      P^T = exp2(S^T * scale*log2e - LSE2_i)        (written back over S^T, bf16, in TMEM)
//      dS^T = P^T o (dP^T - D_i)                    (bf16, 128B-swizzled shared memory)
//      dV += P^T dO_i   (A = P^T from TMEM)
//      dK += dS^T Q_i   (A = dS^T, K-major)
//      dQ_i = dS K_j    (A = the same dS^T buffer read MN-major, B = K_j MN-major)
//  * Warp 0 TMA producer, warp 1 MMA issuer (single thread), warps 4-7 compute P and dS
//    (thread = key row), warps 8-11 drain dQ_i from TMEM and add it (times scale) into the
//    fp32 accumulator with 16-byte red.global.add, then write dK, dV at the end.
//  * TMEM: S^T/P^T [0,128), dP^T [128,256) (reused for dQ_i once dP^T is consumed),
//    dV [256,256+D), dK [256+D,256+2D).
#include "kernels.h"
#include "ptx.cuh"

namespace fa {

template <int D>
struct BwdCfg {
  static constexpr int THREADS = 384;
  static constexpr int NS = (D == 128) ? 2 : 3;  // Q/dO ring depth
  static constexpr int PANEL_BYTES = 128 * 128;
  static constexpr int PANELS = D / 64;
  static constexpr int TILE_BYTES = PANELS * PANEL_BYTES;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE_BYTES;
  static constexpr int OFF_Q = OFF_V + TILE_BYTES;
  static constexpr int OFF_DO = OFF_Q + NS * TILE_BYTES;
  static constexpr int OFF_DS = OFF_DO + NS * TILE_BYTES;  // 128 keys x 128 queries bf16
  static constexpr int DS_BYTES = 2 * PANEL_BYTES;
  static constexpr int OFF_LSE = OFF_DS + DS_BYTES;        // [NS][128] fp32
  static constexpr int OFF_DEL = OFF_LSE + NS * 512;       // [NS][128] fp32
  static constexpr int OFF_BAR = OFF_DEL + NS * 512;
  static constexpr int NBAR = 1 + 2 * NS + 6 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr int TMEM_COLS = 512;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

__device__ __forceinline__ bool bwd_tile_active(const BwdParams& p, int i, int j) {
  if (p.causal && i < j) return false;
  if (p.block_mask != nullptr && p.block_mask[i * p.nb + j] == 0) return false;
  return true;
}

template <int D>
__global__ void __launch_bounds__(384, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                  const BwdParams p) {
  using C = BwdCfg<D>;
  constexpr int NS = C::NS;
  extern __shared__ __align__(1024) uint8_t smem[];

  const uint32_t warp = warp_id(), lane = lane_id();
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicCAS(&g_fa_device_status, 0, WAIT_SMEM_ALIGN);
    return;
  }

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_kv = bars;               // K_j, V_j landed
  uint64_t* bar_qf = bars + 1;           // [NS] Q_i, dO_i, LSE2_i, D_i landed
  uint64_t* bar_qe = bar_qf + NS;        // [NS] stage free
  uint64_t* bar_sdp = bar_qe + NS;       // S^T_i and dP^T_i ready in TMEM
  uint64_t* bar_ds = bar_sdp + 1;        // P^T_i in TMEM, dS^T_i in smem, S/dP fully read
  uint64_t* bar_dsfree = bar_ds + 1;     // MMAs reading dS^T_i done
  uint64_t* bar_dq = bar_dsfree + 1;     // dQ_i ready in TMEM
  uint64_t* bar_dqfree = bar_dq + 1;     // dQ_i read out of TMEM
  uint64_t* bar_acc = bar_dqfree + 1;    // dK, dV final (all MMAs retired)
  uint64_t* bar_done = bar_acc + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  AbortState* ab = reinterpret_cast<AbortState*>(smem + C::OFF_MISC + 4);

  const int bh = blockIdx.y;
  const int j = blockIdx.x;  // key tile (causal: j = 0 has the most work and starts first)
  const int i_begin = p.causal ? j : 0;
  const uint64_t lim = p.timeout_ns;

  if (warp == 0 && lane == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar_qf[s], 1);
      mbar_init(&bar_qe[s], 1);
    }
    mbar_init(bar_sdp, 1);
    mbar_init(bar_ds, 4);
    mbar_init(bar_dsfree, 1);
    mbar_init(bar_dq, 1);
    mbar_init(bar_dqfree, 4);
    mbar_init(bar_acc, 1);
    mbar_init(bar_done, 1);
    ab->flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sK = smem_u32(smem + C::OFF_K), sV = smem_u32(smem + C::OFF_V);
  const uint32_t sQ = smem_u32(smem + C::OFF_Q), sdO = smem_u32(smem + C::OFF_DO);
  const uint32_t sDS = smem_u32(smem + C::OFF_DS);

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      mbar_arrive_expect_tx(bar_kv, 2 * C::TILE_BYTES);
      for (int pn = 0; pn < C::PANELS; ++pn) {
        tma_load_3d(smem + C::OFF_K + pn * C::PANEL_BYTES, &tmK, bar_kv, pn * 64, j * 128, bh);
        tma_load_3d(smem + C::OFF_V + pn * C::PANEL_BYTES, &tmV, bar_kv, pn * 64, j * 128, bh);
      }
      int it = 0;
      int issued[NS];
      for (int s = 0; s < NS; ++s) issued[s] = -1;
      bool ok = true;
      for (int i = i_begin; i < p.nb; ++i) {
        if (!bwd_tile_active(p, i, j)) continue;
        const int s = it % NS;
        const uint32_t ph = (it / NS) & 1;
        ok = mbar_wait(&bar_qe[s], ph ^ 1, ab, lim, WAIT_BWD_LOAD + 1);
        if (!ok) break;
        mbar_arrive_expect_tx(&bar_qf[s], 2 * C::TILE_BYTES + 1024);
        for (int pn = 0; pn < C::PANELS; ++pn) {
          tma_load_3d(smem + C::OFF_Q + s * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmQ, &bar_qf[s], pn * 64, i * 128,
                      bh);
          tma_load_3d(smem + C::OFF_DO + s * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmdO, &bar_qf[s], pn * 64,
                      i * 128, bh);
        }
        const size_t vec = (size_t)bh * p.Np + (size_t)i * 128;
        bulk_load(smem + C::OFF_LSE + s * 512, p.lse2 + vec, 512, &bar_qf[s]);
        bulk_load(smem + C::OFF_DEL + s * 512, p.delta + vec, 512, &bar_qf[s]);
        issued[s] = ph;
        ++it;
      }
      AbortState none{0};
      if (!ok) {
        for (int s = 0; s < NS; ++s)
          if (issued[s] >= 0) mbar_wait(&bar_qf[s], issued[s], &none, lim, WAIT_BWD_LOAD + 2);
      }
      // K/V are always consumed by someone unless the CTA aborts; make sure they landed.
      mbar_wait(bar_kv, 0, &none, lim, WAIT_BWD_LOAD + 3);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, 0, 0);  // K/V (A) and Q/dO (B), K-major
      constexpr uint32_t IDESC_KV = idesc_bf16_f32(128, D, 0, 1);   // dV, dK: B = dO / Q MN-major
      constexpr uint32_t IDESC_Q = idesc_bf16_f32(128, D, 1, 1);    // dQ: A = dS MN-major, B = K MN-major
      const uint32_t tS = tmem + 0u, tDP = tmem + 128u, tDV = tmem + 256u, tDK = tmem + 256u + D;
      bool ok = mbar_wait(bar_kv, 0, ab, lim, WAIT_BWD_MMA + 1);

      auto issue_s_dp = [&](int s, bool do_s, bool do_dp) {
        const uint32_t qb = sQ + s * C::TILE_BYTES, dob = sdO + s * C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::PANEL_BYTES + (kk & 3) * 32;
          if (do_s) umma_ss(tS, sdesc_sw128(sK + off, 16, 1024), sdesc_sw128(qb + off, 16, 1024), IDESC_S, kk > 0);
          if (do_dp)
            umma_ss(tDP, sdesc_sw128(sV + off, 16, 1024), sdesc_sw128(dob + off, 16, 1024), IDESC_S, kk > 0);
        }
      };

      // Find the first active tile.
      int i = i_begin;
      while (i < p.nb && !bwd_tile_active(p, i, j)) ++i;
      int it = 0;
      if (ok && i < p.nb) {
        ok = mbar_wait(&bar_qf[0], 0, ab, lim, WAIT_BWD_MMA + 2);
        if (ok) {
          tc_fence_after();
          issue_s_dp(0, true, true);
          umma_commit(bar_sdp);
        }
      }
      while (ok && i < p.nb) {
        const int s = it % NS;
        int inext = i + 1;
        while (inext < p.nb && !bwd_tile_active(p, inext, j)) ++inext;
        ok = mbar_wait(bar_ds, it & 1, ab, lim, WAIT_BWD_MMA + 3);
        if (!ok) break;
        tc_fence_after();
        const uint32_t qb = sQ + s * C::TILE_BYTES, dob = sdO + s * C::TILE_BYTES;
        const uint32_t acc = it > 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // reduction over the 128 queries of tile i
          // dV += P^T dO_i
          umma_ts(tDV, tS + kk * 8, sdesc_sw128(dob + kk * 2048, C::PANEL_BYTES, 1024), IDESC_KV,
                  (acc || kk > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // dK += dS^T Q_i
          const uint32_t aoff = (kk >> 2) * C::PANEL_BYTES + (kk & 3) * 32;
          umma_ss(tDK, sdesc_sw128(sDS + aoff, 16, 1024), sdesc_sw128(qb + kk * 2048, C::PANEL_BYTES, 1024),
                  IDESC_KV, (acc || kk > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // reduction over the 128 keys of tile j
          // dQ_i = dS K_j  (into the dP^T columns, already consumed)
          umma_ss(tDP, sdesc_sw128(sDS + kk * 2048, C::PANEL_BYTES, 1024),
                  sdesc_sw128(sK + kk * 2048, C::PANEL_BYTES, 1024), IDESC_Q, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar_dq);
        umma_commit(bar_dsfree);
        umma_commit(&bar_qe[s]);
        if (inext < p.nb) {
          const int sn = (it + 1) % NS;
          ok = mbar_wait(&bar_qf[sn], ((it + 1) / NS) & 1, ab, lim, WAIT_BWD_MMA + 4);
          if (!ok) break;
          tc_fence_after();
          issue_s_dp(sn, true, false);  // S^T_{next}: P^T_i was consumed by the dV MMAs above
          ok = mbar_wait(bar_dqfree, it & 1, ab, lim, WAIT_BWD_MMA + 5);
          if (!ok) break;
          tc_fence_after();
          issue_s_dp(sn, false, true);  // dP^T_{next} once dQ_i has left TMEM
          umma_commit(bar_sdp);
        }
        i = inext;
        ++it;
      }
      umma_commit(bar_acc);
      umma_commit(bar_done);
      AbortState none{0};
      mbar_wait(bar_done, 0, &none, lim, WAIT_BWD_MMA + 6);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------------ P and dS (thread = key row)
    const uint32_t wq = warp & 3;
    const int kr = wq * 32 + lane;  // key row inside tile j
    const uint32_t lane_off = (wq * 32u) << 16;
    const uint32_t tS_row = tmem + lane_off, tDP_row = tmem + lane_off + 128u;
    const float sl2 = p.scale_log2;
    bool ok = true;
    int it = 0;
    for (int i = i_begin; i < p.nb; ++i) {
      if (!bwd_tile_active(p, i, j)) continue;
      const int s = it % NS;
      ok = warp_wait(bar_sdp, it & 1, ab, lim, WAIT_BWD_COMPUTE + 1);
      if (ok && it > 0) ok = warp_wait(bar_dsfree, (it - 1) & 1, ab, lim, WAIT_BWD_COMPUTE + 2);
      if (!ok) break;
      tc_fence_after();
      const float* lse2 = reinterpret_cast<const float*>(smem + C::OFF_LSE + s * 512);
      const float* del = reinterpret_cast<const float*>(smem + C::OFF_DEL + s * 512);
      const bool diag = p.causal && i == j;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {  // 32 queries per chunk
        uint32_t su[32], du[32];
        tmem_ld32(tS_row + c * 32, su);
        tmem_ld32(tDP_row + c * 32, du);
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int q0 = c * 32 + e;
          float p0 = ex2(fmaf(__uint_as_float(su[e]), sl2, -lse2[q0]));
          float p1 = ex2(fmaf(__uint_as_float(su[e + 1]), sl2, -lse2[q0 + 1]));
          if (diag) {  // key kr is visible to query q iff kr <= q
            if (q0 < kr) p0 = 0.f;
            if (q0 + 1 < kr) p1 = 0.f;
          }
          const float ds0 = p0 * (__uint_as_float(du[e]) - del[q0]);
          const float ds1 = p1 * (__uint_as_float(du[e + 1]) - del[q0 + 1]);
          pk[e >> 1] = pack_bf16(p0, p1);
          dk[e >> 1] = pack_bf16(ds0, ds1);
        }
        // P^T chunk over S^T columns [16c, 16c+16): those scores were already read.
        tmem_st16(tS_row + c * 16, pk);
        // dS^T row kr, queries 32c..32c+31 -> panel c/2, 16-byte chunks (c%2)*4 .. +3
        const uint32_t panel = sDS + (c >> 1) * C::PANEL_BYTES;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          st_shared_v4(panel + sw128_offset(kr, (c & 1) * 4 + q), dk[4 * q], dk[4 * q + 1], dk[4 * q + 2],
                       dk[4 * q + 3]);
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_ds);
      ++it;
    }
    // -------------------------------------------------------------- epilogue: dV
    if (ok) ok = warp_wait(bar_acc, 0, ab, lim, WAIT_BWD_EPILOGUE + 1);
    uint8_t* stage = smem + C::OFF_Q;  // Q ring stage 0 is free once every MMA retired
    if (ok) {
      tc_fence_after();
      const uint32_t sst = smem_u32(stage);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        if (it > 0) {
          tmem_ld32(tmem + lane_off + 256u + c * 32, u);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) u[e] = 0u;
        }
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) w[e] = pack_bf16(__uint_as_float(u[2 * e]), __uint_as_float(u[2 * e + 1]));
        const uint32_t panel = sst + ((c * 32) >> 6) * C::PANEL_BYTES;
        const uint32_t ch0 = ((c * 32) & 63) >> 3;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          st_shared_v4(panel + sw128_offset(kr, ch0 + q), w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
      }
      fence_proxy_async_smem();
    }
    named_bar_sync(1, 128);
    if (wq == 0 && lane == 0 && *reinterpret_cast<volatile int*>(&ab->flag) == 0) {
      for (int pn = 0; pn < C::PANELS; ++pn) tma_store_3d(&tmdV, stage + pn * C::PANEL_BYTES, pn * 64, j * 128, bh);
      bulk_commit_group();
      bulk_wait_group_read0();
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------------ dQ drain (thread = query row)
    const uint32_t wq = warp & 3;
    const int qr = wq * 32 + lane;
    const uint32_t lane_off = (wq * 32u) << 16;
    const uint32_t tDQ_row = tmem + lane_off + 128u;
    const float scale = p.scale;
    bool ok = true;
    int it = 0;
    for (int i = i_begin; i < p.nb; ++i) {
      if (!bwd_tile_active(p, i, j)) continue;
      ok = warp_wait(bar_dq, it & 1, ab, lim, WAIT_BWD_DQ + 1);
      if (!ok) break;
      tc_fence_after();
      float* dst = p.dq_acc + ((size_t)bh * p.Np + (size_t)i * 128 + qr) * D;
      uint32_t u[D];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld32(tDQ_row + c * 32, *reinterpret_cast<uint32_t (*)[32]>(&u[c * 32]));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_dqfree);
#pragma unroll
      for (int e = 0; e < D; e += 4)
        red_add_v4(dst + e, __uint_as_float(u[e]) * scale, __uint_as_float(u[e + 1]) * scale,
                   __uint_as_float(u[e + 2]) * scale, __uint_as_float(u[e + 3]) * scale);
      ++it;
    }
    // -------------------------------------------------------------- epilogue: dK (times scale)
    if (ok) ok = warp_wait(bar_acc, 0, ab, lim, WAIT_BWD_EPILOGUE + 2);
    uint8_t* stage = smem + C::OFF_DO;  // dO ring stage 0, free once every MMA retired
    if (ok) {
      tc_fence_after();
      const uint32_t sst = smem_u32(stage);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        if (it > 0) {
          tmem_ld32(tmem + lane_off + 256u + D + c * 32, u);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) u[e] = 0u;
        }
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16(__uint_as_float(u[2 * e]) * scale, __uint_as_float(u[2 * e + 1]) * scale);
        const uint32_t panel = sst + ((c * 32) >> 6) * C::PANEL_BYTES;
        const uint32_t ch0 = ((c * 32) & 63) >> 3;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          st_shared_v4(panel + sw128_offset(qr, ch0 + q), w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
      }
      fence_proxy_async_smem();
    }
    named_bar_sync(2, 128);
    if (wq == 0 && lane == 0 && *reinterpret_cast<volatile int*>(&ab->flag) == 0) {
      for (int pn = 0; pn < C::PANELS; ++pn) tma_store_3d(&tmdK, stage + pn * C::PANEL_BYTES, pn * 64, j * 128, bh);
      bulk_commit_group();
      bulk_wait_group_read0();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D>
static cudaError_t launch_bwd_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const CUtensorMap& tdo, const CUtensorMap& tdk, const CUtensorMap& tdv,
                                const BwdParams& p, int BH, cudaStream_t stream) {
  using C = BwdCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(fa_bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid(p.nb, BH);
  fa_bwd_kernel<D><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, tdk, tdv, p);
  return cudaGetLastError();
}

cudaError_t launch_bwd_main(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const CUtensorMap& tdk, const CUtensorMap& tdv,
                            const BwdParams& p, int BH, cudaStream_t stream) {
  if (D == 64) return launch_bwd_t<64>(tq, tk, tv, tdo, tdk, tdv, p, BH, stream);
  return launch_bwd_t<128>(tq, tk, tv, tdo, tdk, tdv, p, BH, stream);
}

}  // namespace fa
