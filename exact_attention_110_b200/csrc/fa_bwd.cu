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
//  * CTA = one 128-key tile j of one (b, h). K_j and V_j stay in shared memory; Q_i (with the
//    128 values -LSE_i*log2e + log2(scale) and -D_i of tile i) streams through an NS-deep ring,
//    dO_i through an NS_DO-deep one.
//  * The softmax scale rides in the exponent: the recomputed probabilities are
//    P' = exp2(S * scale*log2e - LSE*log2e + log2(scale)) = scale * P, so dS' = P' o (dP - D)
//    = scale * dS already carries the factor dK and dQ need, and dV = (1/scale) sum P'^T dO is
//    corrected once in its epilogue (this needs scale > 0; the host rejects other values).
//  * Everything but dQ is computed transposed so on-chip results are directly MMA operands:
//      S^T = K_j Q_i^T, dP^T = V_j dO_i^T            (TMEM, one key per TMEM lane)
//      P'^T                                           (bf16, written back over S^T in TMEM)
//      dS'^T = P'^T o (dP^T - D_i)                    (bf16, 128B-swizzled shared memory)
//      dV += P'^T dO_i  (A = P'^T from TMEM)
//      dK += dS'^T Q_i  (A = dS'^T, K-major)
//      dQ_i = dS'_i K_j (A = dS'^T read MN-major, B = K_j MN-major; lane = query row)
//  * Roles: warp 0 TMA; warp 1 MMA issuer (one thread; descriptors precomputed, so each MMA
//    costs only an add); warps 4-7 and 8-11 compute P (P phase) then dS (dS phase) for query
//    columns 0-63 and 64-127 respectively, thread = key row; warps 12-15 drain dQ from TMEM
//    into a 128B-swizzled staging ring and add it to the fp32 accumulator with bulk tensor
//    reductions (one thread issues them; L2 performs the adds), then write dK; warps 4-11
//    write dV.
//  * MMA order per query tile i: dV_i as soon as P_i is in TMEM; S_{i+1} (the compute warps
//    start the next P phase while the tensor core still works on tile i); dQ_i; dK_i (covers
//    the dQ drain); dP_{i+1}. d = 64 issues S_{i+1} first, into the other S^T buffer.
//  * TMEM, d = 128: S^T/P^T [0,128), dP^T [128,256), dV [256,384), dK [384,512). d = 64: S^T/P^T
//    double-buffered [0,128) and [128,256) by the parity of the active tile, dP^T [256,384),
//    dV [384,448), dK [448,512). dQ reuses the dP^T columns once dP^T has been read.
//  * PERSIST (d <= 128): one CTA per SM walks several (b, h, key tile) items, its block index
//    first and then numbers taken from a counter in the workspace (bwd_item, work_item), which
//    the producer passes to the other roles through a two-slot ring in shared memory. Ring
//    counters and barrier phases run on across items, the next item's loads overlap the
//    previous item's epilogue, and three more barriers (dV / dK read out of TMEM, dV store done
//    reading its staging buffer) keep the next item's first dV / dK MMAs and dS writes behind it;
//    they are waited once per item (the issuer after the item's first S^T and dP^T), so the
//    per-tile loops carry no per-item checks.
#include "kernels.h"
#include "ptx.cuh"

// Which of the 16 score pairs of each 32-score chunk of the P phase take 2^x on the FMA pipe
// (ex2_poly2) instead of the special-function unit: bit i set = pair i emulated.
#ifndef FA_BWD_EXP_EMU_MASK
#define FA_BWD_EXP_EMU_MASK 0x0u
#endif

#ifndef FA_BWD_REGS_CTRL
#define FA_BWD_REGS_CTRL 104
#define FA_BWD_REGS_PDS 128
#define FA_BWD_REGS_DQ 152
#endif

namespace fa {

template <int D>
struct BwdCfg {
  static constexpr int THREADS = 512;
  // d = 256: two CTAs per key tile, CTA `hh` owning the 128-column half hh of d for dK, dV
  // and its dQ share (S^T and dP^T still contract over all 256 columns). Its accumulators then
  // fill TMEM exactly as at d = 128. K_j stays in shared memory; Q_i, dO_i and V_j stream as
  // 64-column panels through one FIFO ring (see the producer), since the four full 64 KB tiles
  // the two contractions read would not fit.
  static constexpr bool SPLIT = (D == 256);
  static constexpr int DH = SPLIT ? 128 : D;       // accumulator width per CTA (dK, dV, dQ share)
  static constexpr int NS = (D == 64) ? 3 : 2;     // Q ring depth (with -LSE*log2e and -D); SPLIT: vector ring
  // d = 128: dO is single-buffered to make room for the dQ staging buffer. dO_i is last read by
  // dV_i and next needed by dP_{i+1}, three MMA groups later, which covers the load.
  static constexpr int NS_DO = (D == 128) ? 1 : (SPLIT ? 0 : NS);
  static constexpr int RING = SPLIT ? 6 : 0;       // SPLIT: 64-column panel slots
  static constexpr int DQ_CHUNKS = DH / 32;        // 32-column dQ chunks per query tile
  static constexpr int DQ_SLOTS = 2;                // staging slots: one filling, one being reduced
  static constexpr int DQ_SLOT_BYTES = 128 * 32 * 4;
  static constexpr int PANEL_BYTES = 128 * 128;
  static constexpr int PANELS = D / 64;            // panels of a whole 128 x D tile
  static constexpr int PANELS_H = DH / 64;         // panels of this CTA's dK / dV columns
  static constexpr int TILE_BYTES = PANELS * PANEL_BYTES;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE_BYTES;                              // not SPLIT
  static constexpr int OFF_Q = SPLIT ? OFF_K + TILE_BYTES : OFF_V + TILE_BYTES;  // SPLIT: the panel ring
  static constexpr int OFF_DO = SPLIT ? OFF_Q + RING * PANEL_BYTES : OFF_Q + NS * TILE_BYTES;
  static constexpr int OFF_DS = OFF_DO + NS_DO * TILE_BYTES;  // 128 keys x 128 queries bf16
  static constexpr int DS_BYTES = 2 * PANEL_BYTES;
  static constexpr int OFF_DQS = OFF_DS + DS_BYTES;           // dQ staging [DQ_SLOTS][128][32] fp32
  static constexpr int DQS_BYTES = DQ_SLOTS * DQ_SLOT_BYTES;
  static constexpr int OFF_LSE = OFF_DQS + DQS_BYTES;         // [NS][128] fp32: -LSE*log2e
  static constexpr int OFF_DEL = OFF_LSE + NS * 512;          // [NS][128] fp32: -D
  static constexpr int OFF_BAR = OFF_DEL + NS * 512;
  static constexpr int NQB = SPLIT ? RING : NS;               // full/empty barrier pairs of the Q ring
  static constexpr int NBAR = 1 + 2 * NQB + 2 * NS_DO + 18;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // TMEM address, abort flag, item ring [2]
  static constexpr int SMEM_BYTES = OFF_MISC + 32;
  static constexpr int TMEM_COLS = 512;
  // SDB (d = 64): S^T/P^T double-buffered in [0,128) and [128,256) by the parity of the active
  // query tile, so S^T_{i+1} is issued before the issuer waits for P^T_i; dQ then shares the dP^T
  // columns as at d = 128 (measured +1-2 % on every d = 64 shape; d = 128 has no columns to spare).
  static constexpr bool SDB = D == 64;
  static constexpr uint32_t T_S = 0, T_DP = SDB ? 256 : 128, T_DV = SDB ? 384 : 256, T_DK = T_DV + DH;
  static constexpr bool DQ_ALIAS = (DH == 128) || SDB;   // dQ reuses the dP^T columns
  static constexpr uint32_t T_DQ = DQ_ALIAS ? T_DP : 384u;
  // setmaxnreg split of the launch allocation (512 x 128, checked by the build script):
  // control warpgroup (TMA, MMA, 2 idle warps), two P/dS warpgroups, dQ-drain warpgroup.
  static constexpr int REGS_CTRL = FA_BWD_REGS_CTRL, REGS_PDS = FA_BWD_REGS_PDS, REGS_DQ = FA_BWD_REGS_DQ;
  static_assert(128 * (REGS_CTRL + 2 * REGS_PDS + REGS_DQ) <= 512 * 128, "setmaxnreg split exceeds the launch");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  // SPLIT: the vectors of query tile i+2 land in tile i's vector slot together with Q_{i+2}'s
  // first panel, which sits 12 panels after Q_i's first dK panel in the ring order; with at
  // most 12 slots that load cannot start before dK_i, i.e. before tile i's dS phase is done.
  static_assert(RING <= 12, "vector slot reuse needs a ring of at most 12 panels");
};

// bmask: this (b, h)'s block mask (or null), [query tiles][key tiles]. Causal: key tile j is
// active for query tile i when its first key is visible to the tile's last row
// (128j <= 128i + 127 + causal_off; i >= j for the square problem).
// The fields are copied out of the kernel parameters once per thread (see fa_fwd.cu, TileTest).
struct BwdTiles {
  int nb, nbk, Nk, causal, causal_off;
  const uint8_t* bmask;
};
__device__ __forceinline__ bool bwd_tile_active(const BwdTiles& tt, int i, int j) {
  if (tt.causal && 128 * j > 128 * i + 127 + tt.causal_off) return false;
  if (tt.bmask != nullptr && tt.bmask[i * tt.nbk + j] == 0) return false;
  return true;
}

// Writes one accumulator row (D fp32 columns of TMEM lane `row`, times `mul`) as bf16 into a
// 128-row tile staged in the TMA store layout (64-column 128B-swizzled panels).
template <int D, bool F16>
__device__ __forceinline__ void stage_row16(uint32_t taddr, uint32_t sstage, int row, float mul, bool zero) {
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t u[32];
    if (!zero) {
      tmem_ld32(taddr + c * 32, u);
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) u[e] = 0u;
    }
    uint32_t w[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) w[e] = pack16<F16>(__uint_as_float(u[2 * e]) * mul, __uint_as_float(u[2 * e + 1]) * mul);
    const uint32_t panel = sstage + ((c * 32) >> 6) * (128 * 128);
    const uint32_t ch0 = ((c * 32) & 63) >> 3;
#pragma unroll
    for (int q = 0; q < 4; ++q)
      st_shared_v4(panel + sw128_offset(row, ch0 + q), w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  }
}

// Key tile j (SPLIT: item 2j + half hh of d) of work item xj of a head, and the first query
// tile whose last row sees key tile j's first key.
template <bool SPLIT>
__device__ __forceinline__ bool bwd_item_of(const BwdParams& p, int xj, int& j, int& hh, int& i_begin) {
  j = SPLIT ? (xj >> 1) : xj;
  hh = SPLIT ? (xj & 1) : 0;
  const int i_first = 128 * j - 127 - p.causal_off;
  i_begin = (p.causal && i_first > 0) ? (i_first + 127) / 128 : 0;
  return true;
}

// Work item number x of the grid order (x >= 0: the numbers persistent CTAs take from the
// work counter) or, for x < 0, this CTA's own item in a one-CTA-per-item grid: head bh, key
// tile j (SPLIT: item 2j + half hh of d; causal: j = 0 is the heaviest) and the first query tile
// whose last row sees key tile j's first key. False past the last item.
template <bool SPLIT>
__device__ __forceinline__ bool bwd_item(const BwdParams& p, long long x, int& bh, int& j, int& hh, int& i_begin) {
  const int items = p.nbk * (SPLIT ? 2 : 1);
  int xj;
  if (x < 0) {
    if (!cta_work(p.BH, items, p.order_group, bh, xj)) return false;
  } else {
    if (x >= p.BH * items) return false;
    work_item(x, p.BH, items, p.order_group, bh, xj);
  }
  return bwd_item_of<SPLIT>(p, xj, j, hh, i_begin);
}
__device__ __forceinline__ BwdTiles bwd_tiles(const BwdParams& p, int bh) {
  const uint8_t* bmask = p.block_mask == nullptr ? nullptr : p.block_mask + (size_t)bh * p.mask_stride;
  return BwdTiles{p.nb, p.nbk, p.Nk, p.causal, p.causal_off, bmask};
}

template <int D, bool F16, bool PERSIST>
__global__ void __launch_bounds__(512, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                  const __grid_constant__ CUtensorMap tmdQa, const BwdParams p) {
  using C = BwdCfg<D>;
  constexpr int NS = C::NS, NS_DO = C::NS_DO, NQB = C::NQB;
  extern __shared__ __align__(1024) uint8_t smem[];

  const uint32_t warp = warp_id(), lane = lane_id();
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicCAS(&g_fa_device_status, 0, WAIT_SMEM_ALIGN);
    return;
  }

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_kv = bars;               // K_j, V_j landed
  uint64_t* bar_qf = bars + 1;           // [NQB] Q_i, -LSE2_i, -D_i landed (SPLIT: ring slot full)
  uint64_t* bar_qe = bar_qf + NQB;       // [NQB] Q stage free after dK_i (SPLIT: ring slot free)
  uint64_t* bar_dof = bar_qe + NQB;      // [NS_DO] dO_i landed
  uint64_t* bar_doe = bar_dof + NS_DO;   // [NS_DO] dO stage free (after dV_i)
  uint64_t* bar_s = bar_doe + NS_DO;     // S^T_i ready in TMEM
  uint64_t* bar_dp = bar_s + 1;          // dP^T_i ready in TMEM
  uint64_t* bar_p = bar_dp + 1;          // P^T_i written to TMEM (S^T_i fully read)
  uint64_t* bar_ds = bar_p + 1;          // dS^T_i in smem, dP^T_i fully read
  uint64_t* bar_dsfree = bar_ds + 1;     // MMAs reading dS^T_i done
  uint64_t* bar_dq = bar_dsfree + 1;     // dQ_i ready in TMEM
  uint64_t* bar_dqfree = bar_dq + 1;     // dQ_i read out of TMEM
  uint64_t* bar_acc = bar_dqfree + 1;    // dK, dV of the item final (all its MMAs retired)
  uint64_t* bar_done = bar_acc + 1;
  uint64_t* bar_dvfree = bar_done + 1;   // dV read out of TMEM by the epilogue (the next item may overwrite)
  uint64_t* bar_dkfree = bar_dvfree + 1; // dK read out of TMEM by the epilogue
  uint64_t* bar_vst = bar_dkfree + 1;    // the dV store has read its staging area (the dS buffer)
  uint64_t* bar_itf = bar_vst + 1;       // [2] persistent: item ring slot written by the producer
  uint64_t* bar_ite = bar_itf + 2;       // [2] persistent: item ring slot read by every other role
  uint64_t* bar_s1 = bar_ite + 2;        // SDB: bar_s and bar_p of the odd active tiles (S^T buffer 1)
  uint64_t* bar_p1 = bar_s1 + 1;
  // S^T / P^T barrier of active tile number `n` and the parity of its phase
  auto bar_s_of = [&](int n) { return (C::SDB && (n & 1)) ? bar_s1 : bar_s; };
  auto bar_p_of = [&](int n) { return (C::SDB && (n & 1)) ? bar_p1 : bar_p; };
  auto sp_par = [&](int n) -> uint32_t { return (uint32_t)(C::SDB ? (n >> 1) : n) & 1u; };
  auto s_col = [&](int n) -> uint32_t { return C::SDB ? (uint32_t)(n & 1) * 128u : 0u; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  AbortState* ab = reinterpret_cast<AbortState*>(smem + C::OFF_MISC + 4);
  volatile int* item_ring = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);  // [2] {bh, item}; bh < 0: none

  if (!PERSIST) {
    int bh0, j0, hh0, ib0;
    if (!bwd_item<C::SPLIT>(p, -1, bh0, j0, hh0, ib0)) return;
  }
  const uint64_t lim = p.timeout_ns;

  if (warp == 0 && lane == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < NQB; ++s) {
      mbar_init(&bar_qf[s], 1);
      mbar_init(&bar_qe[s], 1);
    }
    for (int s = 0; s < NS_DO; ++s) {
      mbar_init(&bar_dof[s], 1);
      mbar_init(&bar_doe[s], 1);
    }
    mbar_init(bar_s, 1);
    mbar_init(bar_dp, 1);
    mbar_init(bar_p, 8);   // one arrive per P/dS warp (two warpgroups)
    mbar_init(bar_ds, 8);
    mbar_init(bar_dsfree, 1);
    mbar_init(bar_dq, 1);
    mbar_init(bar_dqfree, 4);
    mbar_init(bar_acc, 1);
    mbar_init(bar_done, 1);
    mbar_init(bar_dvfree, 8);  // one arrive per P/dS warp
    mbar_init(bar_dkfree, 4);  // one arrive per dQ-drain warp
    mbar_init(bar_vst, 1);
    mbar_init(bar_s1, 1);
    mbar_init(bar_p1, 8);
    for (int r = 0; r < 2; ++r) {
      mbar_init(&bar_itf[r], 1);
      mbar_init(&bar_ite[r], 13);  // the MMA issuer, the eight P/dS warps, the four drain warps
    }
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
  if (warp < 4) reg_dealloc<C::REGS_CTRL>();  // producer, MMA issuer and two idle warps

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      if constexpr (!C::SPLIT) {
        int it = 0;  // active query tiles loaded so far, over all items (ring position)
        int issued[NS], issued_do[NS_DO];
        for (int s = 0; s < NS; ++s) issued[s] = -1;
        for (int s = 0; s < NS_DO; ++s) issued_do[s] = -1;
        bool ok = true;
        int w = 0;
        for (; ok && (PERSIST || w == 0); ++w) {
          long long x = -1;
          if (PERSIST) {
            // Item number w of this CTA: its block index first, then from the work counter; it goes
            // to the other roles through ring slot w & 1 (n_total: no more items).
            const int rs = w & 1;
            const uint32_t use = (uint32_t)(w >> 1);
            if (use > 0 && !mbar_wait(&bar_ite[rs], (use - 1) & 1u, ab, lim, WAIT_BWD_LOAD + 7)) {
              ok = false;
              break;
            }
            x = w == 0 ? (long long)blockIdx.x : (long long)gridDim.x + (long long)atomicAdd(&p.counters[0], 1ull);
          }
          int bh, j, hh, i_begin;
          const bool have = bwd_item<C::SPLIT>(p, x, bh, j, hh, i_begin);
          if (PERSIST) {
            const int rs = w & 1;
            item_ring[2 * rs] = have ? bh : -1;
            item_ring[2 * rs + 1] = C::SPLIT ? 2 * j + hh : j;
            mbar_arrive(&bar_itf[rs]);
          }
          if (!have) break;
          const BwdTiles tt = bwd_tiles(p, bh);
          auto load_tile = [&](int i) -> bool {
            // Q_i first: its stage frees at dK_{i-NS}, before dO_i's stage frees at dV_{i-NS_DO}.
            const int s = it % NS;
            const uint32_t ph = (it / NS) & 1;
            if (!mbar_wait(&bar_qe[s], ph ^ 1, ab, lim, WAIT_BWD_LOAD + 1)) return false;
            mbar_arrive_expect_tx(&bar_qf[s], C::TILE_BYTES + 1024);
            for (int pn = 0; pn < C::PANELS; ++pn)
              tma_load_3d(smem + C::OFF_Q + s * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmQ, &bar_qf[s], pn * 64,
                          i * 128, bh);
            const size_t vec = (size_t)bh * p.Np + (size_t)i * 128;
            bulk_load(smem + C::OFF_LSE + s * 512, p.lse2 + vec, 512, &bar_qf[s]);
            bulk_load(smem + C::OFF_DEL + s * 512, p.delta + vec, 512, &bar_qf[s]);
            issued[s] = ph;
            const int sd = it % NS_DO;
            const uint32_t phd = (it / NS_DO) & 1;
            if (!mbar_wait(&bar_doe[sd], phd ^ 1, ab, lim, WAIT_BWD_LOAD + 4)) return false;
            mbar_arrive_expect_tx(&bar_dof[sd], C::TILE_BYTES);
            for (int pn = 0; pn < C::PANELS; ++pn)
              tma_load_3d(smem + C::OFF_DO + sd * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmdO, &bar_dof[sd], pn * 64,
                          i * 128, bh);
            issued_do[sd] = phd;
            ++it;
            return true;
          };
          int i = i_begin;
          while (i < tt.nb && !bwd_tile_active(tt, i, j)) ++i;
          if (w > 0) {
            // A later item of a persistent CTA: its first query tile enters the ring as soon as a
            // stage is free, while the previous item still computes; K_j and V_j once no MMA
            // reads the previous item's K and V.
            if (i < tt.nb) ok = load_tile(i++);
            if (ok) ok = mbar_wait(bar_acc, (uint32_t)(w - 1) & 1u, ab, lim, WAIT_BWD_LOAD + 6);
            if (!ok) break;
          }
          mbar_arrive_expect_tx(bar_kv, 2 * C::TILE_BYTES);
          for (int pn = 0; pn < C::PANELS; ++pn) {
            tma_load_3d(smem + C::OFF_K + pn * C::PANEL_BYTES, &tmK, bar_kv, pn * 64, j * 128, bh);
            tma_load_3d(smem + C::OFF_V + pn * C::PANEL_BYTES, &tmV, bar_kv, pn * 64, j * 128, bh);
          }
          for (; ok && i < tt.nb; ++i)
            if (bwd_tile_active(tt, i, j)) ok = load_tile(i);
        }
        AbortState none{0};
        if (!ok) {
          for (int s = 0; s < NS; ++s)
            if (issued[s] >= 0) mbar_wait(&bar_qf[s], issued[s], &none, lim, WAIT_BWD_LOAD + 2);
          for (int s = 0; s < NS_DO; ++s)
            if (issued_do[s] >= 0) mbar_wait(&bar_dof[s], issued_do[s], &none, lim, WAIT_BWD_LOAD + 5);
        }
        // K/V of the last item whose load was issued landed before the CTA can exit
        if (w > 0) mbar_wait(bar_kv, (uint32_t)(w - 1) & 1u, &none, lim, WAIT_BWD_LOAD + 3);
      } else {
        int bh, j, hh, i_begin;
        bwd_item<C::SPLIT>(p, -1, bh, j, hh, i_begin);  // d = 256 runs one item per CTA
        const BwdTiles tt = bwd_tiles(p, bh);
        // K_j (all four panels) stays; everything else streams through the panel ring in the
        // order the MMA issuer consumes it. First tile i0: Q(i0) panels 0-3 (S^T), then V and
        // dO(i0) panels p = 0-3 in pairs (dP^T). Then per tile i (next active tile i'):
        // dO(i) panels of half hh (dV), Q(i') panels 0-3 (S^T of i'), Q(i) panels of half hh
        // (dK), V / dO(i') panel pairs (dP^T of i'). Q's first panel carries the tile's -LSE2
        // and -D vectors into vector slot (active tile index) & 1.
        mbar_arrive_expect_tx(bar_kv, C::TILE_BYTES);
        for (int pn = 0; pn < C::PANELS; ++pn)
          tma_load_3d(smem + C::OFF_K + pn * C::PANEL_BYTES, &tmK, bar_kv, pn * 64, j * 128, bh);
        int issued[C::RING];
        for (int s = 0; s < C::RING; ++s) issued[s] = -1;
        int npush = 0, vit = 0;
        bool ok = true;
        auto push = [&](const CUtensorMap* map, int x, int y, int vec_tile) -> bool {
          const int s = npush % C::RING;
          const uint32_t ph = (uint32_t)(npush / C::RING) & 1u;
          if (!mbar_wait(&bar_qe[s], ph ^ 1u, ab, lim, WAIT_BWD_LOAD + 1)) return false;
          mbar_arrive_expect_tx(&bar_qf[s], C::PANEL_BYTES + (vec_tile >= 0 ? 1024 : 0));
          tma_load_3d(smem + C::OFF_Q + s * C::PANEL_BYTES, map, &bar_qf[s], x, y, bh);
          if (vec_tile >= 0) {
            const int vs = vit & 1;
            const size_t vec = (size_t)bh * p.Np + (size_t)vec_tile * 128;
            bulk_load(smem + C::OFF_LSE + vs * 512, p.lse2 + vec, 512, &bar_qf[s]);
            bulk_load(smem + C::OFF_DEL + vs * 512, p.delta + vec, 512, &bar_qf[s]);
            ++vit;
          }
          issued[s] = (int)ph;
          ++npush;
          return true;
        };
        auto push_s = [&](int i) -> bool {  // Q(i) panels 0-3, vectors with the first
          for (int pn = 0; pn < C::PANELS; ++pn)
            if (!push(&tmQ, pn * 64, i * 128, pn == 0 ? i : -1)) return false;
          return true;
        };
        auto push_dp = [&](int i) -> bool {  // V_j and dO(i) panel pairs
          for (int pn = 0; pn < C::PANELS; ++pn)
            if (!push(&tmV, pn * 64, j * 128, -1) || !push(&tmdO, pn * 64, i * 128, -1)) return false;
          return true;
        };
        int i = i_begin;
        while (i < tt.nb && !bwd_tile_active(tt, i, j)) ++i;
        if (i < tt.nb) ok = push_s(i) && push_dp(i);
        while (ok && i < tt.nb) {
          int inext = i + 1;
          while (inext < tt.nb && !bwd_tile_active(tt, inext, j)) ++inext;
          const bool has_next = inext < tt.nb;
          ok = push(&tmdO, 128 * hh, i * 128, -1) && push(&tmdO, 128 * hh + 64, i * 128, -1);
          if (ok && has_next) ok = push_s(inext);
          if (ok) ok = push(&tmQ, 128 * hh, i * 128, -1) && push(&tmQ, 128 * hh + 64, i * 128, -1);
          if (ok && has_next) ok = push_dp(inext);
          i = inext;
        }
        AbortState none{0};
        if (!ok)
          for (int s = 0; s < C::RING; ++s)
            if (issued[s] >= 0) mbar_wait(&bar_qf[s], issued[s], &none, lim, WAIT_BWD_LOAD + 2);
        mbar_wait(bar_kv, 0, &none, lim, WAIT_BWD_LOAD + 3);  // K landed before the CTA can exit
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_f32acc(128, 128, 0, 0, F16);  // K/V (A) and Q/dO (B), K-major
      constexpr uint32_t IDESC_KV = idesc_f32acc(128, C::DH, 0, 1, F16);  // dV, dK: B = dO / Q MN-major
      constexpr uint32_t IDESC_Q = idesc_f32acc(128, C::DH, 1, 1, F16);   // dQ = dS K: A = dS^T, B = K, MN-major
      constexpr uint32_t TILE16 = C::TILE_BYTES >> 4;
      const uint32_t tS = tmem + C::T_S, tDP = tmem + C::T_DP, tDV = tmem + C::T_DV, tDK = tmem + C::T_DK;
      const uint32_t tDQ = tmem + C::T_DQ;
      const uint64_t dK_k = sdesc_sw128(sK, 16, 1024);               // K as K-major A (S^T)
      const uint64_t dV_k = sdesc_sw128(sV, 16, 1024);               // V as K-major A (dP^T)
      const uint64_t dK_mn = sdesc_sw128(sK, C::PANEL_BYTES, 1024);  // K read MN-major (dQ)
      const uint64_t dQ_k = sdesc_sw128(sQ, 16, 1024);               // Q_i as K-major B (S^T)
      const uint64_t dQ_mn = sdesc_sw128(sQ, C::PANEL_BYTES, 1024);  // Q_i as MN-major B (dK)
      const uint64_t dO_k = sdesc_sw128(sdO, 16, 1024);
      const uint64_t dO_mn = sdesc_sw128(sdO, C::PANEL_BYTES, 1024);
      const uint64_t dS_k = sdesc_sw128(sDS, 16, 1024);              // dS^T as K-major A (dK)
      const uint64_t dS_mn = sdesc_sw128(sDS, C::PANEL_BYTES, 1024); // dS^T read MN-major (dQ)
      bool ok = true;

      if constexpr (!C::SPLIT) {
        auto issue_s = [&](int st, uint32_t dst) {
          const uint64_t b = dQ_k + (uint64_t)(st * TILE16);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off16 = ((kk >> 2) * C::PANEL_BYTES + (kk & 3) * 32) >> 4;
            umma_ss(dst, dK_k + off16, b + off16, IDESC_S, kk > 0 ? 1u : 0u);
          }
        };
        auto issue_dp = [&](int st) {
          const uint64_t b = dO_k + (uint64_t)(st * TILE16);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off16 = ((kk >> 2) * C::PANEL_BYTES + (kk & 3) * 32) >> 4;
            umma_ss(tDP, dV_k + off16, b + off16, IDESC_S, kk > 0 ? 1u : 0u);
          }
        };

        int it = 0;  // active query tiles so far, over all items
        for (int w = 0; ok && (PERSIST || w == 0); ++w) {
          int bh, j, hh, i_begin;
          if (PERSIST) {
            const int rs = w & 1;
            ok = mbar_wait_spin(&bar_itf[rs], (uint32_t)(w >> 1) & 1u, ab, lim, WAIT_BWD_MMA + 13);
            if (!ok) break;
            const int2 it2 = make_int2(item_ring[2 * rs], item_ring[2 * rs + 1]);
            mbar_arrive(&bar_ite[rs]);
            if (it2.x < 0) break;
            bh = it2.x;
            bwd_item_of<C::SPLIT>(p, it2.y, j, hh, i_begin);
          } else if (!bwd_item<C::SPLIT>(p, -1, bh, j, hh, i_begin)) {
            break;
          }
          const BwdTiles tt = bwd_tiles(p, bh);
          ok = mbar_wait_spin(bar_kv, (uint32_t)w & 1u, ab, lim, WAIT_BWD_MMA + 1);
          if (!ok) break;
          int i = i_begin;
          while (i < tt.nb && !bwd_tile_active(tt, i, j)) ++i;
          int ni = 0;  // this item's active query tiles so far
          if (i < tt.nb) {
            ok = mbar_wait_spin(&bar_qf[it % NS], (uint32_t)(it / NS) & 1u, ab, lim, WAIT_BWD_MMA + 2);
            if (ok) {
              tc_fence_after();
              issue_s(it % NS, tS + s_col(it));
              umma_commit(bar_s_of(it));
              // d = 128: the dP^T columns hold the previous item's last dQ until it is drained
              if (C::DQ_ALIAS && it > 0) ok = mbar_wait_spin(bar_dqfree, (uint32_t)(it - 1) & 1u, ab, lim, WAIT_BWD_MMA + 7);
            }
            if (ok) ok = mbar_wait_spin(&bar_dof[it % NS_DO], (uint32_t)(it / NS_DO) & 1u, ab, lim, WAIT_BWD_MMA + 9);
            if (ok) {
              tc_fence_after();
              issue_dp(it % NS_DO);
              umma_commit(bar_dp);
            }
          }
          if (PERSIST && ok && w > 0) {
            // This item's first dV and dK MMAs overwrite the accumulators the previous item's
            // epilogue reads out; its first S^T and dP^T above use other columns and may run
            // meanwhile. Waiting here, once per item, keeps the per-tile loop free of checks.
            ok = mbar_wait_spin(bar_dvfree, (uint32_t)(w - 1) & 1u, ab, lim, WAIT_BWD_MMA + 11);
            if (ok) ok = mbar_wait_spin(bar_dkfree, (uint32_t)(w - 1) & 1u, ab, lim, WAIT_BWD_MMA + 12);
          }
          while (ok && i < tt.nb) {
            const int s = it % NS;
            int inext = i + 1;
            while (inext < tt.nb && !bwd_tile_active(tt, inext, j)) ++inext;
            const bool has_next = inext < tt.nb;
            const int sn = (it + 1) % NS;
            const int sd = it % NS_DO, sdn = (it + 1) % NS_DO;
            const uint32_t acc = ni > 0 ? 1u : 0u;
            const uint64_t dOs = dO_mn + (uint64_t)(sd * TILE16), dQs = dQ_mn + (uint64_t)(s * TILE16);

            if (C::SDB && has_next) {
              // S^T_{i+1} into the other buffer, whose P^T_{i-1} the previous dV has read already
              ok = mbar_wait_spin(&bar_qf[sn], ((it + 1) / NS) & 1, ab, lim, WAIT_BWD_MMA + 4);
              if (!ok) break;
              tc_fence_after();
              issue_s(sn, tS + s_col(it + 1));
              umma_commit(bar_s_of(it + 1));
            }
            // dV += P^T dO_i (reduction over the 128 queries of tile i), A = P^T from TMEM
            ok = mbar_wait_spin(bar_p_of(it), sp_par(it), ab, lim, WAIT_BWD_MMA + 3);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_ts(tDV, tS + s_col(it) + (kk >> 2) * 64 + (kk & 3) * 8, dOs + (uint64_t)(kk * (2048 >> 4)),
                      IDESC_KV, kk > 0 ? 1u : acc);
            umma_commit(&bar_doe[sd]);  // dO_i read by dP_i and dV_i
            // S^T_{i+1} over P^T_i (the dV MMAs above read it first: tcgen05.mma runs in order)
            if (!C::SDB && has_next) {
              ok = mbar_wait_spin(&bar_qf[sn], ((it + 1) / NS) & 1, ab, lim, WAIT_BWD_MMA + 4);
              if (!ok) break;
              tc_fence_after();
              issue_s(sn, tS);
              umma_commit(bar_s);
            }
            ok = mbar_wait_spin(bar_ds, it & 1, ab, lim, WAIT_BWD_MMA + 5);
            if (!ok) break;
            if (!C::DQ_ALIAS && it > 0) {  // d = 64: the dQ columns must have been drained
              ok = mbar_wait_spin(bar_dqfree, (it - 1) & 1, ab, lim, WAIT_BWD_MMA + 6);
              if (!ok) break;
            }
            tc_fence_after();
            // dQ_i (d = 128: into the dP^T columns, already read by the dS phase)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {  // reduction over the 128 keys of tile j
              const uint64_t kdesc = dK_mn + (uint64_t)(kk * (2048 >> 4)), sdesc = dS_mn + (uint64_t)(kk * (2048 >> 4));
              umma_ss(tDQ, sdesc, kdesc, IDESC_Q, kk > 0 ? 1u : 0u);
            }
            umma_commit(bar_dq);
            // dK += dS^T Q_i
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t aoff16 = ((kk >> 2) * C::PANEL_BYTES + (kk & 3) * 32) >> 4;
              umma_ss(tDK, dS_k + aoff16, dQs + (uint64_t)(kk * (2048 >> 4)), IDESC_KV, kk > 0 ? 1u : acc);
            }
            umma_commit(bar_dsfree);
            umma_commit(&bar_qe[s]);
            // dP^T_{i+1}
            if (has_next) {
              if (C::DQ_ALIAS) {  // the dP^T columns hold dQ_i until the drain warps have read it
                ok = mbar_wait_spin(bar_dqfree, it & 1, ab, lim, WAIT_BWD_MMA + 7);
                if (!ok) break;
              }
              ok = mbar_wait_spin(&bar_dof[sdn], ((it + 1) / NS_DO) & 1, ab, lim, WAIT_BWD_MMA + 10);
              if (!ok) break;
              tc_fence_after();
              issue_dp(sdn);
              umma_commit(bar_dp);
            }
            i = inext;
            ++it;
            ++ni;
          }
          // (An item without query tiles -- a block mask can empty a key tile -- commits only after
          // the waits above, so the epilogue warps cannot see its accumulator phase complete
          // before they waited for the previous one.)
          if (!ok) break;
          umma_commit(bar_acc);  // this item's dK and dV are final once every MMA so far retires
        }
      } else {
        int bh, j, hh, i_begin;
        bwd_item<C::SPLIT>(p, -1, bh, j, hh, i_begin);  // d = 256 runs one item per CTA
        const BwdTiles tt = bwd_tiles(p, bh);
        ok = mbar_wait_spin(bar_kv, 0, ab, lim, WAIT_BWD_MMA + 1);
        // Panels come off the ring in the producer's order; each is released by a commit right
        // after the MMAs that read it (commits track every earlier MMA, so release is in order).
        // dV and dK take one 64-column panel of this CTA's half at a time (two N = 64 groups).
        constexpr uint32_t IDESC_H64 = idesc_f32acc(128, 64, 0, 1, F16);
        const uint64_t ring_k = sdesc_sw128(sQ, 16, 1024);               // a panel as K-major operand
        const uint64_t ring_mn = sdesc_sw128(sQ, C::PANEL_BYTES, 1024);  // a panel as MN-major B
        constexpr uint32_t P16 = C::PANEL_BYTES >> 4;
        int npop = 0;
        auto pop = [&](int where) -> int {  // next ring slot, once its panel has landed; -1: abort
          const int sl = npop % C::RING;
          const uint32_t ph = (uint32_t)(npop / C::RING) & 1u;
          ++npop;
          return mbar_wait_spin(&bar_qf[sl], ph, ab, lim, where) ? sl : -1;
        };
        auto issue_s = [&]() -> bool {  // S^T = sum over the four panels of K_j[:, p] Q_i[:, p]^T
          for (int pn = 0; pn < C::PANELS; ++pn) {
            const int sl = pop(WAIT_BWD_MMA + 2);
            if (sl < 0) return false;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_ss(tS, dK_k + (uint64_t)((pn * C::PANEL_BYTES + kk * 32) >> 4),
                      ring_k + (uint64_t)(sl * P16 + ((kk * 32) >> 4)), IDESC_S, (pn > 0 || kk > 0) ? 1u : 0u);
            umma_commit(&bar_qe[sl]);
          }
          umma_commit(bar_s);
          return true;
        };
        auto issue_dp = [&]() -> bool {  // dP^T = sum over the panels of V_j[:, p] dO_i[:, p]^T
          for (int pn = 0; pn < C::PANELS; ++pn) {
            const int sv = pop(WAIT_BWD_MMA + 9);
            const int sd = sv < 0 ? -1 : pop(WAIT_BWD_MMA + 9);
            if (sd < 0) return false;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_ss(tDP, ring_k + (uint64_t)(sv * P16 + ((kk * 32) >> 4)),
                      ring_k + (uint64_t)(sd * P16 + ((kk * 32) >> 4)), IDESC_S, (pn > 0 || kk > 0) ? 1u : 0u);
            umma_commit(&bar_qe[sv]);
            umma_commit(&bar_qe[sd]);
          }
          umma_commit(bar_dp);
          return true;
        };
        int i = i_begin;
        while (i < tt.nb && !bwd_tile_active(tt, i, j)) ++i;
        int it = 0;
        if (ok && i < tt.nb) ok = issue_s() && issue_dp();
        while (ok && i < tt.nb) {
          int inext = i + 1;
          while (inext < tt.nb && !bwd_tile_active(tt, inext, j)) ++inext;
          const bool has_next = inext < tt.nb;
          const uint32_t acc = it > 0 ? 1u : 0u;
          // dV_hh += P^T dO_i[:, half hh], A = P^T from TMEM, one 64-column panel at a time
          ok = mbar_wait_spin(bar_p, it & 1, ab, lim, WAIT_BWD_MMA + 3);
          for (int q = 0; q < 2 && ok; ++q) {
            const int sl = pop(WAIT_BWD_MMA + 4);
            if (sl < 0) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_ts(tDV + 64u * q, tS + (kk >> 2) * 64 + (kk & 3) * 8,
                      ring_mn + (uint64_t)(sl * P16 + kk * (2048 >> 4)), IDESC_H64, kk > 0 ? 1u : acc);
            umma_commit(&bar_qe[sl]);
          }
          if (!ok) break;
          // S^T_{i+1} over P^T_i (the dV MMAs above read it first: tcgen05.mma runs in order)
          if (has_next && !issue_s()) { ok = false; break; }
          ok = mbar_wait_spin(bar_ds, it & 1, ab, lim, WAIT_BWD_MMA + 5);
          if (!ok) break;
          tc_fence_after();
          // dQ_i[:, half hh] = dS_i K_j[:, half hh] into the dP^T columns (already read)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t kdesc = dK_mn + (uint64_t)(((2 * hh) * C::PANEL_BYTES) >> 4) + (uint64_t)(kk * (2048 >> 4));
            const uint64_t sdesc = dS_mn + (uint64_t)(kk * (2048 >> 4));
            umma_ss(tDQ, sdesc, kdesc, IDESC_Q, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar_dq);
          // dK_hh += dS^T Q_i[:, half hh], one panel at a time
          for (int q = 0; q < 2 && ok; ++q) {
            const int sl = pop(WAIT_BWD_MMA + 6);
            if (sl < 0) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t aoff16 = ((kk >> 2) * C::PANEL_BYTES + (kk & 3) * 32) >> 4;
              umma_ss(tDK + 64u * q, dS_k + aoff16, ring_mn + (uint64_t)(sl * P16 + kk * (2048 >> 4)), IDESC_H64,
                      kk > 0 ? 1u : acc);
            }
            umma_commit(&bar_qe[sl]);
          }
          if (!ok) break;
          umma_commit(bar_dsfree);
          // dP^T_{i+1}: the dP^T columns hold dQ_i until the drain warps have read it
          if (has_next) {
            ok = mbar_wait_spin(bar_dqfree, it & 1, ab, lim, WAIT_BWD_MMA + 7);
            if (ok) ok = issue_dp();
            if (!ok) break;
          }
          i = inext;
          ++it;
        }
        umma_commit(bar_acc);
      }
      umma_commit(bar_done);
      AbortState none{0};
      mbar_wait(bar_done, 0, &none, lim, WAIT_BWD_MMA + 8);
    }
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------------ P and dS (thread = key row)
    // Two warpgroups split the 128 queries of a tile: group h owns query columns [64h, 64h+64)
    // of S^T and dP^T, writes its P^T into S^T columns [64h, 64h+32) (already read by itself)
    // and its dS^T into shared-memory panel h. TMEM loads are issued one chunk ahead.
    reg_alloc<C::REGS_PDS>();
    const int h = (warp - 4) >> 2;
    const uint32_t wq = warp & 3;
    const int kr = wq * 32 + lane;  // key row inside tile j
    const uint32_t lane_off = (wq * 32u) << 16;
    const uint32_t tS_row = tmem + lane_off + C::T_S + 64u * h, tDP_row = tmem + lane_off + C::T_DP + 64u * h;
    const uint64_t sl2_2 = f2_pack(p.scale_log2, p.scale_log2);
    constexpr uint32_t EMU = FA_BWD_EXP_EMU_MASK;
    const Ex2PolyConsts ek = ex2_poly_consts();
    bool ok = true;
    int it = 0;  // active query tiles so far, over all items
    for (int w = 0; PERSIST || w == 0; ++w) {
      int bh = 0, j = 0, hh = 0, i_begin = 0;
      if (PERSIST) {
        const int rs = w & 1;
        bool got = warp_wait(&bar_itf[rs], (uint32_t)(w >> 1) & 1u, ab, lim, WAIT_BWD_COMPUTE + 5);
        int2 it2 = make_int2(-1, 0);
        if (got && lane == 0) it2 = make_int2(item_ring[2 * rs], item_ring[2 * rs + 1]);
        it2.x = __shfl_sync(0xffffffffu, it2.x, 0);
        it2.y = __shfl_sync(0xffffffffu, it2.y, 0);
        if (got && lane == 0) mbar_arrive(&bar_ite[rs]);
        // The previous item's dV store reads its staging area, the dS buffer, which this item's
        // first dS phase overwrites (waiting here keeps the per-tile loop free of checks).
        if (got && w > 0 && it2.x >= 0) got = warp_wait(bar_vst, (uint32_t)(w - 1) & 1u, ab, lim, WAIT_BWD_COMPUTE + 4);
        // Every warp of the two groups takes the same decision: they meet at named barriers.
        if (!named_bar_and(1, 256, got && it2.x >= 0)) {
          ok = ok && named_bar_and(1, 256, got);
          break;
        }
        bh = it2.x;
        bwd_item_of<C::SPLIT>(p, it2.y, j, hh, i_begin);
      } else if (!bwd_item<C::SPLIT>(p, -1, bh, j, hh, i_begin)) {
        break;
      }
      const BwdTiles tt = bwd_tiles(p, bh);
      int ni = 0;  // this item's active query tiles so far
      for (int i = i_begin; i < tt.nb; ++i) {
        if (!bwd_tile_active(tt, i, j)) continue;
        const int s = it % NS;
        const float* nlse2 = reinterpret_cast<const float*>(smem + C::OFF_LSE + s * 512) + 64 * h;
        const float* ndel = reinterpret_cast<const float*>(smem + C::OFF_DEL + s * 512) + 64 * h;
        // Causal band: key 128j+kr is visible to query 128i+q iff 128j+kr <= 128i+q+causal_off,
        // i.e. q >= qmin (q >= kr on the diagonal tile of the square problem).
        const bool diag = tt.causal && (128 * j + 127 > 128 * i + tt.causal_off);
        const int qmin = kr + 128 * (j - i) - tt.causal_off;
        // Keys of a partial last tile beyond N_k (zero rows from TMA) take no part: P = 0 there,
        // so nothing non-finite can reach dQ through them.
        const bool kpad = 128 * j + kr >= tt.Nk;
        // the first visible local query of this row and group (64: none, a padded key; < 0: all)
        const int qlim = kpad ? 64 : (diag ? qmin - 64 * h : -1);

        // ---- P phase: P^T = exp2(S^T * scale*log2e - LSE*log2e), back into TMEM as bf16
        ok = warp_wait(bar_s_of(it), sp_par(it), ab, lim, WAIT_BWD_COMPUTE + 1);
        if (!ok) break;
        tc_fence_after();
        float pf[64];  // P in fp32, kept for the dS phase
        {
          uint32_t sa[32], sb[32];
          tmem_ld32_async(tS_row + s_col(it), sa);
          tmem_wait_ld_tied(sa);
          tmem_ld32_async(tS_row + s_col(it) + 32, sb);  // in flight while chunk 0 is processed
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t (&su)[32] = c == 0 ? sa : sb;
            if (c == 1) tmem_wait_ld_tied(sb);
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              const int q = 32 * c + 2 * e;  // local query index of this 4-query group
              const float4 nl = *reinterpret_cast<const float4*>(&nlse2[q]);
              const uint64_t x01 = ffma2(f2_pack(__uint_as_float(su[2 * e]), __uint_as_float(su[2 * e + 1])), sl2_2,
                                         f2_pack(nl.x, nl.y));
              const uint64_t x23 = ffma2(f2_pack(__uint_as_float(su[2 * e + 2]), __uint_as_float(su[2 * e + 3])),
                                         sl2_2, f2_pack(nl.z, nl.w));
              float p0, p1, p2, p3;
              if ((EMU >> e) & 1u) {
                f2_unpack(ex2_poly2(x01, ek), p0, p1);
              } else {
                float x0, x1;
                f2_unpack(x01, x0, x1);
                p0 = ex2(x0);
                p1 = ex2(x1);
              }
              if ((EMU >> (e + 1)) & 1u) {
                f2_unpack(ex2_poly2(x23, ek), p2, p3);
              } else {
                float x2, x3;
                f2_unpack(x23, x2, x3);
                p2 = ex2(x2);
                p3 = ex2(x3);
              }
              // Local query q is visible iff q >= qlim: a compare and a select on every tile
              // rather than a separate masked path (one copy of this loop in the code; causal
              // grids ran 1.5-4 % faster with it, the instruction cache missing less).
              p0 = q >= qlim ? p0 : 0.f;
              p1 = q + 1 >= qlim ? p1 : 0.f;
              p2 = q + 2 >= qlim ? p2 : 0.f;
              p3 = q + 3 >= qlim ? p3 : 0.f;
              pf[q] = p0;
              pf[q + 1] = p1;
              pf[q + 2] = p2;
              pf[q + 3] = p3;
              pk[e] = pack16<F16>(p0, p1);
              pk[e + 1] = pack16<F16>(p2, p3);
            }
            tmem_st16(tS_row + s_col(it) + c * 16, pk);  // columns [64h + 16c, +16): scores already read
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_p_of(it));

        // ---- dS phase: dS^T = P^T o (dP^T - D) into shared-memory panel h
        ok = warp_wait(bar_dp, it & 1, ab, lim, WAIT_BWD_COMPUTE + 2);
        if (ok && it > 0) ok = warp_wait(bar_dsfree, (it - 1) & 1, ab, lim, WAIT_BWD_COMPUTE + 3);
          if (!ok) break;
        tc_fence_after();
        {
          uint32_t da[32], db[32];
          tmem_ld32_async(tDP_row, da);
          tmem_wait_ld_tied(da);
          tmem_ld32_async(tDP_row + 32, db);
          const uint32_t panel = sDS + h * C::PANEL_BYTES;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t (&du)[32] = c == 0 ? da : db;
            if (c == 1) tmem_wait_ld_tied(db);
            uint32_t dk[16];
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              const int q = 32 * c + 2 * e;
              const float4 nd = *reinterpret_cast<const float4*>(&ndel[q]);
              const uint64_t t01 = fadd2(f2_pack(__uint_as_float(du[2 * e]), __uint_as_float(du[2 * e + 1])),
                                         f2_pack(nd.x, nd.y));
              const uint64_t t23 = fadd2(f2_pack(__uint_as_float(du[2 * e + 2]), __uint_as_float(du[2 * e + 3])),
                                         f2_pack(nd.z, nd.w));
              const uint64_t ds01 = fmul2(f2_pack(pf[q], pf[q + 1]), t01);
              const uint64_t ds23 = fmul2(f2_pack(pf[q + 2], pf[q + 3]), t23);
              float d0, d1, d2, d3;
              f2_unpack(ds01, d0, d1);
              f2_unpack(ds23, d2, d3);
              dk[e] = pack16<F16>(d0, d1);
              dk[e + 1] = pack16<F16>(d2, d3);
            }
            // dS^T row kr, local queries 32c..32c+31 -> 16-byte chunks 4c .. 4c+3 of panel h
#pragma unroll
            for (int qq = 0; qq < 4; ++qq)
              st_shared_v4(panel + sw128_offset(kr, c * 4 + qq), dk[4 * qq], dk[4 * qq + 1], dk[4 * qq + 2],
                           dk[4 * qq + 3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_ds);
        ++it;
        ++ni;
      }
      // -------------------------------------------------------------- epilogue: dV (group h: panel h)
      if (ok) ok = warp_wait(bar_acc, (uint32_t)w & 1u, ab, lim, WAIT_BWD_EPILOGUE + 1);
      // Staging: one item per CTA: Q ring stage 0 (SPLIT: panels 0-1), free once every MMA retired.
      // Persistent CTAs: the dS buffer, since the ring may already hold the next item's first tile
      // (this group's next dS phase waits for the store to have read it).
      uint8_t* stage = smem + (PERSIST ? C::OFF_DS : C::OFF_Q);
      if (ok && h < C::PANELS_H) {
        tc_fence_after();
        stage_row16<64, F16>(tmem + lane_off + C::T_DV + 64u * h, smem_u32(stage + h * C::PANEL_BYTES), kr, p.inv_scale,
                           ni == 0);
        fence_proxy_async_smem();
      }
      if (PERSIST) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_dvfree);  // dV read out: the next item's first dV may overwrite it
      }
      // staged; a persistent CTA also stops every warp after a failed wait
      bool all_ok = true;
      if (PERSIST)
        all_ok = named_bar_and(1, 256, ok);
      else
        named_bar_sync(1, 256);
      if (warp == 4 && lane == 0 && *reinterpret_cast<volatile int*>(&ab->flag) == 0) {
        for (int pn = 0; pn < C::PANELS_H; ++pn)
          tma_store_3d(&tmdV, stage + pn * C::PANEL_BYTES, C::DH * hh + pn * 64, j * 128, bh);
        bulk_commit_group();
        bulk_wait_group_read0();
        if (PERSIST) mbar_arrive(bar_vst);
      }
      if (!all_ok) break;
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------------ dQ drain
    // Thread = query row of dQ_i (TMEM lane). The tile goes back to memory in 32-column
    // chunks: each chunk is staged as 128 rows of 128 bytes (the tensor map's 128-byte
    // swizzle, so the 16-byte stores of a warp are conflict-free) and added to the fp32
    // accumulator by one thread with a bulk tensor reduction performed in L2.
    reg_alloc<C::REGS_DQ>();
    const uint32_t wq = warp & 3;
    const int ln = wq * 32 + lane;
    const uint32_t lane_off = (wq * 32u) << 16;
    const uint32_t tDQ_row = tmem + lane_off + C::T_DQ;
    const uint32_t sDQS = smem_u32(smem + C::OFF_DQS);
    const bool issuer = (wq == 0 && lane == 0);  // issues the bulk reductions of the warpgroup
    if (issuer) tma_prefetch_desc(&tmdQa);
    bool ok = true;
    int it = 0;         // active query tiles so far, over all items
    uint32_t nred = 0;  // bulk reductions issued so far (staging slot = nred % DQ_SLOTS)
    for (int w = 0; PERSIST || w == 0; ++w) {
      int bh = 0, j = 0, hh = 0, i_begin = 0;
      if (PERSIST) {
        const int rs = w & 1;
        const bool got = warp_wait(&bar_itf[rs], (uint32_t)(w >> 1) & 1u, ab, lim, WAIT_BWD_DQ + 2);
        int2 it2 = make_int2(-1, 0);
        if (got && lane == 0) it2 = make_int2(item_ring[2 * rs], item_ring[2 * rs + 1]);
        it2.x = __shfl_sync(0xffffffffu, it2.x, 0);
        it2.y = __shfl_sync(0xffffffffu, it2.y, 0);
        if (got && lane == 0) mbar_arrive(&bar_ite[rs]);
        // Every warp of the group takes the same decision: they meet at named barriers.
        if (!named_bar_and(2, 128, got && it2.x >= 0)) {
          ok = ok && named_bar_and(2, 128, got);
          break;
        }
        bh = it2.x;
        bwd_item_of<C::SPLIT>(p, it2.y, j, hh, i_begin);
      } else if (!bwd_item<C::SPLIT>(p, -1, bh, j, hh, i_begin)) {
        break;
      }
      const BwdTiles tt = bwd_tiles(p, bh);
      int ni = 0;  // this item's active query tiles so far
      for (int i = i_begin; i < tt.nb; ++i) {
        if (!bwd_tile_active(tt, i, j)) continue;
        ok = warp_wait(bar_dq, it & 1, ab, lim, WAIT_BWD_DQ + 1);
        // Read the whole row and release the TMEM columns before anything else (at d = 128 the
        // next dP^T is written there). When aborting (!ok) the values are not used; the columns
        // stay allocated until every role has left.
        uint32_t u[C::DH];
        tc_fence_after();
        if constexpr (C::DH == 128) {
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32_async(tDQ_row + c * 32, *reinterpret_cast<uint32_t (*)[32]>(&u[c * 32]));
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_wait_ld_tied(*reinterpret_cast<uint32_t (*)[32]>(&u[c * 32]));
        } else {
          tmem_ld64(tDQ_row, u);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(bar_dqfree);
        // the four warps leave together: they meet at named barriers below
        if (!named_bar_and(3, 128, ok)) break;
        const int row0 = bh * p.Np + i * 128;
#pragma unroll
        for (int c = 0; c < C::DQ_CHUNKS; ++c, ++nred) {
          if (issuer && nred >= C::DQ_SLOTS) bulk_wait_group_read<C::DQ_SLOTS - 1>();
          named_bar_sync(3, 128);  // the slot's previous reduction has read it
          const uint32_t slot = sDQS + (nred % C::DQ_SLOTS) * C::DQ_SLOT_BYTES;
#pragma unroll
          for (int k = 0; k < 8; ++k)  // 16-byte chunk k of row ln: columns 32c + 4k .. +3
            st_shared_v4(slot + sw128_offset(ln, k), u[32 * c + 4 * k], u[32 * c + 4 * k + 1], u[32 * c + 4 * k + 2],
                         u[32 * c + 4 * k + 3]);
          fence_proxy_async_smem();
          named_bar_sync(3, 128);  // slot written
          if (issuer) {
            tma_reduce_add_2d(&tmdQa, slot, C::DH * hh + 32 * c, row0);
            bulk_commit_group();
          }
        }
        ++it;
        ++ni;
      }
      // -------------------------------------------------------------- epilogue: dK (dS carries the scale)
      if (ok) ok = warp_wait(bar_acc, (uint32_t)w & 1u, ab, lim, WAIT_BWD_EPILOGUE + 2);
      // Staging: one item per CTA: dO ring stage 0 (SPLIT: ring panel slots 2-3), free once every
      // MMA retired, so the last dQ reductions complete meanwhile. Persistent CTAs: the dQ slots
      // once those reductions have read them, since the dO ring may hold the next item's first tile.
      uint8_t* stage = smem + (PERSIST ? C::OFF_DQS : C::SPLIT ? C::OFF_Q + 2 * C::PANEL_BYTES : C::OFF_DO);
      if (PERSIST) {
        if (issuer) bulk_wait_group_read0();
        named_bar_sync(2, 128);
      }
      if (ok) {
        tc_fence_after();
        stage_row16<C::DH, F16>(tmem + lane_off + C::T_DK, smem_u32(stage), ln, 1.f, ni == 0);
        fence_proxy_async_smem();
      }
      if (PERSIST) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_dkfree);  // dK read out: the next item's first dK may overwrite it
      }
      bool all_ok = true;
      if (PERSIST)
        all_ok = named_bar_and(2, 128, ok);
      else
        named_bar_sync(2, 128);
      if (wq == 0 && lane == 0 && *reinterpret_cast<volatile int*>(&ab->flag) == 0) {
        for (int pn = 0; pn < C::PANELS_H; ++pn)
          tma_store_3d(&tmdK, stage + pn * C::PANEL_BYTES, C::DH * hh + pn * 64, j * 128, bh);
        bulk_commit_group();
        bulk_wait_group_read0();
      }
      if (!all_ok) break;
    }
    if (issuer) bulk_wait_group0();  // every dQ reduction and dK store complete before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (PERSIST && threadIdx.x == 0) {
    // The last CTA to finish leaves the counters zeroed for the next launch on this workspace
    // (every CTA has taken its last item number by now).
    __threadfence();
    if (atomicAdd(&p.counters[1], 1ull) == (unsigned long long)gridDim.x - 1ull) {
      p.counters[0] = 0ull;
      p.counters[1] = 0ull;
    }
  }
}

template <int D, bool F16, bool PERSIST>
static cudaError_t launch_bwd_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const CUtensorMap& tdo, const CUtensorMap& tdk, const CUtensorMap& tdv,
                                const CUtensorMap& tdqa, const BwdParams& p, long long BH, cudaStream_t stream) {
  using C = BwdCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(fa_bwd_kernel<D, F16, PERSIST>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int items = p.nbk * (C::SPLIT ? 2 : 1);  // SPLIT: two CTAs per key tile
  dim3 grid;
  if (PERSIST) {  // one persistent CTA per SM walks the items (bwd_item)
    const long long total = BH * items, sms = device_sm_count();
    grid = dim3((unsigned)(total < sms ? total : sms));
  } else {
    grid = grid_work(items, BH, p.order_group);
  }
  fa_bwd_kernel<D, F16, PERSIST><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, tdk, tdv, tdqa, p);
  return cudaGetLastError();
}

template <int D, bool F16>
static cudaError_t launch_bwd_p(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const CUtensorMap& tdo, const CUtensorMap& tdk, const CUtensorMap& tdv,
                                const CUtensorMap& tdqa, const BwdParams& p, long long BH, cudaStream_t stream) {
  if (D != 256 && p.persist > 0) return launch_bwd_t<D, F16, D != 256>(tq, tk, tv, tdo, tdk, tdv, tdqa, p, BH, stream);
  return launch_bwd_t<D, F16, false>(tq, tk, tv, tdo, tdk, tdv, tdqa, p, BH, stream);
}

cudaError_t launch_bwd_main(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const CUtensorMap& tdk, const CUtensorMap& tdv,
                            const CUtensorMap& tdqa, const BwdParams& p, long long BH, cudaStream_t stream) {
  if (p.f16) {
    if (D == 64) return launch_bwd_p<64, true>(tq, tk, tv, tdo, tdk, tdv, tdqa, p, BH, stream);
    if (D == 256) return launch_bwd_p<256, true>(tq, tk, tv, tdo, tdk, tdv, tdqa, p, BH, stream);
    return launch_bwd_p<128, true>(tq, tk, tv, tdo, tdk, tdv, tdqa, p, BH, stream);
  }
  if (D == 64) return launch_bwd_p<64, false>(tq, tk, tv, tdo, tdk, tdv, tdqa, p, BH, stream);
  if (D == 256) return launch_bwd_p<256, false>(tq, tk, tv, tdo, tdk, tdv, tdqa, p, BH, stream);
  return launch_bwd_p<128, false>(tq, tk, tv, tdo, tdk, tdv, tdqa, p, BH, stream);
}

}  // namespace fa
