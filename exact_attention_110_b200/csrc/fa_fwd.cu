// Forward kernel: exact attention with online softmax, S and P kept in tensor memory.
//
// Method (sources cited by page and section):
//   [P1] "FlashAttention-2 的前世今生" overview, jishu.shishitao.com/detail/60083.html
//   [P2] "Attention 为什么慢" explainer, ds6.com.cn/news/67428.html
//   [P3] FlashAttention V1 lecture summary, spark.aweffr.cn/summary/0684ec99-...
//  * Tiling: Q, K, V are cut into 128-row blocks; each (Q block, K/V block) pair is processed
//    on chip and S = Q K^T, P = softmax(S) never reach HBM ([P3] §3.1, §3.3; [P1] §主要操作).
//  * FA2 loop order: a thread block owns query row-blocks and loops over K/V column-blocks,
//    no communication between thread blocks ([P1] §主要操作, forward pass).
//  * Online softmax: running row max m, running sum l, output rescaled when m grows
//    ([P2] §时间复杂度, the online normaliser; [P3] §3.2 recurrence, §3.4). The output is kept
//    unnormalised and divided by l once at the end, which removes per-step non-matmul work
//    ([P1] §主要操作: "reduce non-matmul FLOPs").
//  * Saved statistic: LSE = m + ln l per row, the only value the backward needs ([P1]
//    §主要操作, backward pass).
//
// sm_100a design (ours, not the pages'):
//  * CTA = 256 query rows of one (b, h) as two 128-row tiles t = 0, 1 that ping-pong: the
//    tensor core computes S for one tile while the other tile's softmax runs.
//  * Warp 0: TMA producer. Q tiles once; K_j and V_j through separate NS-deep shared-memory
//    rings guarded by full/empty mbarriers. No cluster multicast: neighbouring CTAs that read
//    the same K/V tiles are served from L2.
//  * Warp 1: allocates 512 TMEM columns and issues every tcgen05.mma from one thread:
//    S_t = Q_t K_j^T (128x128, fp32 in TMEM), then O_t += P_t V_j with P_t read straight
//    from TMEM (the .kind::f16 "A in tensor memory" form).
//  * Warps 4-7 and 8-11: one softmax warpgroup per tile; thread r owns row r (TMEM lane r),
//    so row max and row sum need no shuffles. Scores are scaled into the log2 domain
//    (x * scale * log2 e) and exponentiated with ex2. P (bf16) is written back over S.
//  * Lazy rescale: the reference max m_ref moves only when a row's max exceeds it by more
//    than 8 (a factor 256 in P). Using a stale reference is exact in real arithmetic because
//    O and l are scaled by the same exp2(-m_ref); it keeps O rescales off the common path.
//  * Epilogue: O / l -> bf16 into the (now unused) Q tile buffer in the TMA layout, one TMA
//    store per 64-column panel; LSE = (m_ref + log2 l) * ln 2.
//
// TMEM columns: S/P tile 0 [0,128), S/P tile 1 [128,256), O tile 0 [256,256+D),
// O tile 1 [256+D, 256+2D).
#include "kernels.h"
#include "ptx.cuh"

#ifndef FA_FWD_SOLO_MAX_NB
#define FA_FWD_SOLO_MAX_NB 8
#endif
#ifndef FA_FWD_EXP_EMU_MASK
#define FA_FWD_EXP_EMU_MASK 0x0u
#endif
// K/V stages of the one-tile layout at d = 128.
#ifndef FA_FWD_ONE_TILE_STAGES_D128
#define FA_FWD_ONE_TILE_STAGES_D128 2
#endif

namespace fa {

// ONE: one query tile per CTA (see TILES). Chosen at launch: always at d = 256, and at d = 128
// for a problem with a single query tile (N_q <= 128, e.g. decoding), where the two-tile form
// would leave its second tile empty; two ping-ponged tiles otherwise (short sequences and d = 64
// single tiles run the kernel of fa_fwd_solo.cu instead).
template <int D, bool ONE>
struct FwdCfg {
  static constexpr int THREADS = 384;  // warp 0 TMA, warp 1 MMA, warps 4-11 softmax
  // setmaxnreg split of the launch allocation (384 x 168, checked by the build script):
  // the control warpgroup (TMA, MMA, 2 idle warps) keeps 88, the softmax warpgroups get 208.
  static constexpr int REGS_CTRL = 88, REGS_SOFTMAX = 208;
  static_assert(128 * REGS_CTRL + 256 * REGS_SOFTMAX <= 384 * 168, "setmaxnreg split exceeds the launch");
  // 128-row query tiles per CTA. Two that ping-pong (S_t in columns [128t, 128t+128), O_t
  // after them), or one (required at d = 256, where two tiles' S and O would need 768 TMEM
  // columns): then S is double-buffered -- S(a) of the a-th active KV tile in columns
  // [0,128) or [128,256) by the parity of a, O in [256, 256+D) -- so the tensor core computes
  // S(a+1) while the softmax works on S(a), and both softmax warpgroups share the tile, each
  // taking 64 of the 128 key columns.
  static constexpr int TILES = ONE ? 1 : 2;
  static_assert(D != 256 || TILES == 1, "d = 256 needs the one-tile layout");
  static constexpr int NS = TILES == 2 ? ((D == 128) ? 2 : 4)  // K ring and V ring depth
                                       : (D == 256 ? 1 : (D == 128 ? FA_FWD_ONE_TILE_STAGES_D128 : 4));
  static constexpr int PANEL_BYTES = 128 * 128;        // 128 rows x 64 bf16 (one swizzle panel)
  static constexpr int PANELS = D / 64;
  static constexpr int TILE_BYTES = PANELS * PANEL_BYTES;  // 128 x D bf16
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILES * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + NS * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + NS * TILE_BYTES;
  static constexpr int NBAR = 2 + 4 * NS + 2 + 4 + 2 + 1 + (TILES == 1 ? 1 : 0);
  // one tile: the two warpgroups' row maxima [2 parities][2 halves][128] (row sums at the end)
  static constexpr int OFF_XCH = OFF_BAR + NBAR * 8;
  static constexpr int XCH_BYTES = TILES == 1 ? 2 * 2 * 128 * 4 : 0;
  static constexpr int OFF_MISC = OFF_XCH + XCH_BYTES;
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr int TMEM_COLS = 512;
  // Which of the 16 score pairs of each 32-score chunk take 2^x on the FMA pipe (ex2_poly)
  // instead of the special-function unit: bit i set = pair i emulated.
  static constexpr uint32_t EXP_EMU_MASK = FA_FWD_EXP_EMU_MASK;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// What the tile test needs, copied out of the kernel parameters once per thread: the test runs
// between inline-asm statements that clobber memory (MMA issue, barrier waits), after which
// fields read straight from the parameters would be reloaded from constant space.
// bmask: this (b, h)'s block mask (or null).
struct TileTest {
  int nb, nbk, Nk, causal, causal_off;
  const uint8_t* bmask;
};
// Causal: tile j is active when the last row of tile qb sees its first key
// (128j <= 128qb + 127 + causal_off; j <= qb for the square problem).
__device__ __forceinline__ bool fwd_tile_active(const TileTest& tt, int qb, int j) {
  if (qb >= tt.nb) return false;
  if (tt.causal && 128 * j > 128 * qb + 127 + tt.causal_off) return false;
  if (tt.bmask != nullptr && tt.bmask[qb * tt.nbk + j] == 0) return false;
  return true;
}

// p = 2^(s * scale * log2e - m_ref) for one row's 128 scores; P (bf16) goes back over the
// scores it came from, 32 scores -> 16 packed columns per chunk, so chunk c only lands on
// columns already read. Pairs whose bit is set in EMU_MASK (within each chunk of 16 pairs)
// use the FMA-pipe polynomial, the rest the special-function unit; EMU = false forces the
// special-function unit everywhere (masked tiles need exact zeros for -inf scores).
// After the first two chunks (keys 0-63) the warp arrives on `half0`, so the tensor core can
// start O += P V on those keys while the second half is computed; the caller signals the
// second half. Returns the row sum of p.
template <bool F16, bool EMU, uint32_t EMU_MASK>
__device__ __forceinline__ float softmax_exp_store(const uint32_t (&su)[128], uint64_t sl2_2, uint64_t mneg_2,
                                                   uint32_t tS_row, const Ex2PolyConsts& K, uint64_t* half0) {
  uint64_t ls2[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) ls2[k] = 0ull;  // two +0.0f lanes
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint64_t s2 = f2_pack(__uint_as_float(su[32 * c + 2 * i]), __uint_as_float(su[32 * c + 2 * i + 1]));
      const uint64_t x2 = ffma2(s2, sl2_2, mneg_2);
      uint64_t p2;
      if (EMU && ((EMU_MASK >> i) & 1u)) {
        p2 = ex2_poly2(x2, K);
      } else {
        float x0, x1;
        f2_unpack(x2, x0, x1);
        p2 = f2_pack(ex2(x0), ex2(x1));
      }
      ls2[i & 3] = fadd2(ls2[i & 3], p2);
      float p0, p1;
      f2_unpack(p2, p0, p1);
      pk[i] = pack16<F16>(p0, p1);
    }
    tmem_st16(tS_row + c * 16, pk);
    if (c == 1) {
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane_id() == 0) mbar_arrive(half0);
    }
  }
  const uint64_t t2 = fadd2(fadd2(ls2[0], ls2[1]), fadd2(ls2[2], ls2[3]));
  float a, b;
  f2_unpack(t2, a, b);
  return a + b;
}

// The one-tile form of softmax_exp_store: one warpgroup's 64 scores of a row (keys 64h..64h+63)
// -> P in 32 packed columns at tP; the caller signals the half. Returns this half's row sum.
template <bool F16, bool EMU, uint32_t EMU_MASK>
__device__ __forceinline__ float softmax_exp_store64(const uint32_t (&su)[64], uint64_t sl2_2, uint64_t mneg_2,
                                                     uint32_t tP, const Ex2PolyConsts& K) {
  uint64_t ls2[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) ls2[k] = 0ull;
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint64_t s2 = f2_pack(__uint_as_float(su[32 * c + 2 * i]), __uint_as_float(su[32 * c + 2 * i + 1]));
      const uint64_t x2 = ffma2(s2, sl2_2, mneg_2);
      uint64_t p2;
      if (EMU && ((EMU_MASK >> i) & 1u)) {
        p2 = ex2_poly2(x2, K);
      } else {
        float x0, x1;
        f2_unpack(x2, x0, x1);
        p2 = f2_pack(ex2(x0), ex2(x1));
      }
      ls2[i & 3] = fadd2(ls2[i & 3], p2);
      float p0, p1;
      f2_unpack(p2, p0, p1);
      pk[i] = pack16<F16>(p0, p1);
    }
    tmem_st16(tP + c * 16, pk);
  }
  const uint64_t t2 = fadd2(fadd2(ls2[0], ls2[1]), fadd2(ls2[2], ls2[3]));
  float a, b;
  f2_unpack(t2, a, b);
  return a + b;
}

template <int D, bool F16, bool ONE>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const FwdParams p) {
  using C = FwdCfg<D, ONE>;
  constexpr int NS = C::NS;
  extern __shared__ __align__(1024) uint8_t smem[];

  const uint32_t warp = warp_id(), lane = lane_id();
  if ((smem_u32(smem) & 1023u) != 0) {  // swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicCAS(&g_fa_device_status, 0, WAIT_SMEM_ALIGN);
    return;
  }

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_q = bars;            // [2]  Q tile t landed
  uint64_t* bar_kf = bars + 2;       // [NS] K stage full
  uint64_t* bar_ke = bar_kf + NS;    // [NS] K stage free
  uint64_t* bar_vf = bar_ke + NS;    // [NS] V stage full
  uint64_t* bar_ve = bar_vf + NS;    // [NS] V stage free
  uint64_t* bar_s = bar_ve + NS;     // [2]  S_t ready in TMEM
  uint64_t* bar_p = bar_s + 2;       // [2][2] P_t keys 0-63 / 64-127 written (O_t rescaled before)
  uint64_t* bar_o = bar_p + 4;       // [2]  all MMAs of tile t complete
  uint64_t* bar_done = bar_o + 2;    // [1]  every MMA of the CTA complete
  uint64_t* bar_pv = bar_done + 1;   // [1]  (one tile only) O += P V of one more KV tile complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  AbortState* ab = reinterpret_cast<AbortState*>(smem + C::OFF_MISC + 4);

  const int npairs = (p.nb + C::TILES - 1) / C::TILES;
  int bh, xi;  // head and work item = pair index * nsplit + split; causal: the heaviest pairs first
  if (!cta_work(p.BH, npairs * p.nsplit, p.order_group, bh, xi)) return;
  const uint8_t* bmask = p.block_mask == nullptr ? nullptr : p.block_mask + (size_t)bh * p.mask_stride;
  const TileTest tt{p.nb, p.nbk, p.Nk, p.causal, p.causal_off, bmask};
  const int pi = xi / p.nsplit, split = xi - pi * p.nsplit;
  const int pair = p.causal ? npairs - 1 - pi : pi;
  const int qb0 = C::TILES * pair;  // 128-row tile index of tile 0
  // this CTA's key tiles: its split's range, cut at the last key the pair's last row sees
  const int j_begin = split * p.kv_per_split;
  int j_end = min(p.nbk, j_begin + p.kv_per_split);
  if (p.causal) {
    const int last_key = 128 * qb0 + 128 * C::TILES - 1 + p.causal_off;
    j_end = min(j_end, last_key < 0 ? 0 : last_key / 128 + 1);
  }
  const uint64_t lim = p.timeout_ns;

  if (warp == 0 && lane == 0) {
    mbar_init(&bar_q[0], 1);
    mbar_init(&bar_q[1], 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar_kf[s], 1);
      mbar_init(&bar_ke[s], 1);
      mbar_init(&bar_vf[s], 1);
      mbar_init(&bar_ve[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bar_s[t], 1);
      mbar_init(&bar_p[2 * t], 4);  // one arrive per softmax warp
      mbar_init(&bar_p[2 * t + 1], 4);
      mbar_init(&bar_o[t], 1);
    }
    mbar_init(bar_done, 1);
    if (C::TILES == 1) mbar_init(bar_pv, 1);
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

  const uint32_t sQ = smem_u32(smem + C::OFF_Q);
  const uint32_t sK = smem_u32(smem + C::OFF_K);
  const uint32_t sV = smem_u32(smem + C::OFF_V);
  if (warp < 4) reg_dealloc<C::REGS_CTRL>();  // producer, MMA issuer and two idle warps

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmO);
      for (int t = 0; t < 2; ++t) {
        if (qb0 + t < p.nb && (C::TILES == 2 || t == 0)) {
          mbar_arrive_expect_tx(&bar_q[t], C::TILE_BYTES);
          for (int pn = 0; pn < C::PANELS; ++pn)
            tma_load_3d(smem + C::OFF_Q + t * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmQ, &bar_q[t], pn * 64,
                        (qb0 + t) * 128, bh);
        }
      }
      int it = 0;
      int issued_k[NS], issued_v[NS];
      for (int s = 0; s < NS; ++s) issued_k[s] = issued_v[s] = -1;
      bool ok = true;
      if constexpr (C::TILES == 1) {
        // S(a+1) is issued before O += P(a) V(a), so K runs ahead of V: K0 V0 K1 K2 V1 K3 V2 ...
        // K(a) waits for S(a-NS) to release its stage, V(a-1) for O += P(a-1-NS) V(a-1-NS).
        int a = 0, j_prev = -1;
        auto load_v = [&](int jv, int m) -> bool {
          const int vs = m % NS;
          const uint32_t vph = (uint32_t)(m / NS) & 1u;
          if (!mbar_wait(&bar_ve[vs], vph ^ 1u, ab, lim, WAIT_FWD_LOAD + 2)) return false;
          mbar_arrive_expect_tx(&bar_vf[vs], C::TILE_BYTES);
          for (int pn = 0; pn < C::PANELS; ++pn)
            tma_load_3d(smem + C::OFF_V + vs * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmV, &bar_vf[vs], pn * 64,
                        jv * 128, bh);
          issued_v[vs] = (int)vph;
          return true;
        };
        for (int j = j_begin; j < j_end && ok; ++j) {
          if (!fwd_tile_active(tt, qb0, j)) continue;
          const int ks = a % NS;
          const uint32_t kph = (uint32_t)(a / NS) & 1u;
          ok = mbar_wait(&bar_ke[ks], kph ^ 1u, ab, lim, WAIT_FWD_LOAD + 1);
          if (!ok) break;
          mbar_arrive_expect_tx(&bar_kf[ks], C::TILE_BYTES);
          for (int pn = 0; pn < C::PANELS; ++pn)
            tma_load_3d(smem + C::OFF_K + ks * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmK, &bar_kf[ks], pn * 64,
                        j * 128, bh);
          issued_k[ks] = (int)kph;
          if (a == 0) ok = load_v(j, 0);
          else if (a >= 2) ok = load_v(j_prev, a - 1);
          j_prev = j;
          ++a;
        }
        if (ok && a >= 2) ok = load_v(j_prev, a - 1);
      }
      for (int j = j_begin; C::TILES == 2 && j < j_end && ok; ++j) {
        if (!fwd_tile_active(tt, qb0, j) && !fwd_tile_active(tt, qb0 + 1, j)) continue;
        const int s = it % NS;
        const uint32_t ph = (it / NS) & 1;
        ok = mbar_wait(&bar_ke[s], ph ^ 1, ab, lim, WAIT_FWD_LOAD + 1);
        if (!ok) break;
        mbar_arrive_expect_tx(&bar_kf[s], C::TILE_BYTES);
        for (int pn = 0; pn < C::PANELS; ++pn)
          tma_load_3d(smem + C::OFF_K + s * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmK, &bar_kf[s], pn * 64,
                      j * 128, bh);
        issued_k[s] = ph;
        ok = mbar_wait(&bar_ve[s], ph ^ 1, ab, lim, WAIT_FWD_LOAD + 2);
        if (!ok) break;
        mbar_arrive_expect_tx(&bar_vf[s], C::TILE_BYTES);
        for (int pn = 0; pn < C::PANELS; ++pn)
          tma_load_3d(smem + C::OFF_V + s * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmV, &bar_vf[s], pn * 64,
                      j * 128, bh);
        issued_v[s] = ph;
        ++it;
      }
      if (!ok) {
        // Aborting: let the copies already in flight land before the CTA's memory goes away.
        AbortState none{0};
        for (int s = 0; s < NS; ++s) {
          if (issued_k[s] >= 0) mbar_wait(&bar_kf[s], issued_k[s], &none, lim, WAIT_FWD_LOAD + 3);
          if (issued_v[s] >= 0) mbar_wait(&bar_vf[s], issued_v[s], &none, lim, WAIT_FWD_LOAD + 3);
        }
        for (int t = 0; t < 2; ++t)
          if (qb0 + t < p.nb && (C::TILES == 2 || t == 0)) mbar_wait(&bar_q[t], 0, &none, lim, WAIT_FWD_LOAD + 4);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    // One thread issues everything. Shared-memory descriptors are built once; each MMA only
    // adds a compile-time offset (the start-address field is address >> 4), so the issuing
    // thread spends a few cycles per MMA instead of a dependent chain of 64-bit ALU ops --
    // the issue rate, not the tensor core, otherwise limits M=128 x N=128 MMAs.
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_f32acc(128, 128, 0, 0, F16);  // Q, K both K-major
      constexpr uint32_t IDESC_O = idesc_f32acc(128, D, 0, 1, F16);    // P (TMEM), V MN-major
      constexpr uint32_t TILE16 = C::TILE_BYTES >> 4;
      const uint64_t dq_base = sdesc_sw128(sQ, 16, 1024);
      const uint64_t dk_base = sdesc_sw128(sK, 16, 1024);
      const uint64_t dv_base = sdesc_sw128(sV, C::PANEL_BYTES, 1024);
      bool ok = true;
      for (int t = 0; t < 2 && ok; ++t)
        if (qb0 + t < p.nb && (C::TILES == 2 || t == 0)) ok = mbar_wait_spin(&bar_q[t], 0, ab, lim, WAIT_FWD_MMA + 1);
      if constexpr (C::TILES == 1) {
        // Order S(0), S(1), PV(0), S(2), PV(1), ...: S(a) lands in buffer a & 1 right behind
        // PV(a-2), the last reader of that buffer's P (the tensor pipe runs in order).
        auto issue_pv = [&](int k) -> bool {  // O += P(k) V(k)
          const uint32_t b = (uint32_t)(k & 1), use = (uint32_t)(k >> 1) & 1u;
          const int vs = k % NS;
          if (!mbar_wait_spin(&bar_vf[vs], (uint32_t)(k / NS) & 1u, ab, lim, WAIT_FWD_MMA + 3)) return false;
          const uint64_t dv = dv_base + (uint64_t)(vs * TILE16);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {  // keys 0-63 come from softmax warpgroup 0, 64-127 from 1
            if (!mbar_wait_spin(&bar_p[2 * b + hf], use, ab, lim, WAIT_FWD_MMA + 4)) return false;
            tc_fence_after();
#pragma unroll
            for (int kk = 4 * hf; kk < 4 * hf + 4; ++kk)
              umma_ts(tmem + 256u, tmem + b * 128u + kk * 8, dv + (uint64_t)(kk * (2048 >> 4)), IDESC_O,
                      (k > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bar_ve[vs]);
          umma_commit(bar_pv);
          return true;
        };
        int a = 0;
        for (int j = j_begin; j < j_end && ok; ++j) {
          if (!fwd_tile_active(tt, qb0, j)) continue;
          if (a >= 2) ok = issue_pv(a - 2);
          const int ks = a % NS;
          if (ok) ok = mbar_wait_spin(&bar_kf[ks], (uint32_t)(a / NS) & 1u, ab, lim, WAIT_FWD_MMA + 2);
          if (!ok) break;
          tc_fence_after();
          const uint32_t b = (uint32_t)(a & 1);
          const uint64_t dk = dk_base + (uint64_t)(ks * TILE16);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {  // S(a) = Q K_j^T
            const uint32_t off16 = ((kk >> 2) * C::PANEL_BYTES + (kk & 3) * 32) >> 4;
            umma_ss(tmem + b * 128u, dq_base + off16, dk + off16, IDESC_S, kk > 0 ? 1u : 0u);
          }
          umma_commit(&bar_s[b]);
          umma_commit(&bar_ke[ks]);
          ++a;
        }
        for (int k = a >= 2 ? a - 2 : 0; k < a && ok; ++k) ok = issue_pv(k);
      }
      uint32_t p_phase[2] = {0u, 0u};
      bool o_started[2] = {false, false};
      bool prev_act[2] = {false, false};
      int prev_s = -1;
      uint32_t prev_ph = 0;
      int it = 0;

      for (int j = j_begin; C::TILES == 2 && j < j_end && ok; ++j) {
        const bool act0 = fwd_tile_active(tt, qb0, j);
        const bool act1 = fwd_tile_active(tt, qb0 + 1, j);
        if (!act0 && !act1) continue;
        const int s = it % NS;
        const uint32_t ph = (it / NS) & 1;
        ok = mbar_wait_spin(&bar_kf[s], ph, ab, lim, WAIT_FWD_MMA + 2);
        // V of the previous KV tile (used by this step's PV MMAs of both tiles): waited once
        if (ok && prev_s >= 0 && (prev_act[0] || prev_act[1])) ok = mbar_wait_spin(&bar_vf[prev_s], prev_ph, ab, lim, WAIT_FWD_MMA + 3);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dk = dk_base + (uint64_t)(s * TILE16);
        const uint64_t dv_prev = dv_base + (uint64_t)((prev_s < 0 ? 0 : prev_s) * TILE16);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (prev_act[t]) {  // O_t += P_t V_{previous}, 16 keys per MMA, in two halves of P
            const uint32_t acc0 = o_started[t] ? 1u : 0u;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              ok = mbar_wait_spin(&bar_p[2 * t + hf], p_phase[t], ab, lim, WAIT_FWD_MMA + 4);
              if (!ok) break;
              tc_fence_after();
#pragma unroll
              for (int kk = 4 * hf; kk < 4 * hf + 4; ++kk)
                umma_ts(tmem + 256u + t * D, tmem + t * 128u + kk * 8, dv_prev + (uint64_t)(kk * (2048 >> 4)),
                        IDESC_O, kk > 0 ? 1u : acc0);
            }
            if (!ok) break;
            p_phase[t] ^= 1u;
            o_started[t] = true;
          }
          if (act0 && t == 0 || act1 && t == 1) {  // S_t = Q_t K_j^T
            const uint64_t dq = dq_base + (uint64_t)(t * TILE16);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off16 = ((kk >> 2) * C::PANEL_BYTES + (kk & 3) * 32) >> 4;
              umma_ss(tmem + t * 128u, dq + off16, dk + off16, IDESC_S, kk > 0 ? 1u : 0u);
            }
            umma_commit(&bar_s[t]);
          }
        }
        if (!ok) break;
        umma_commit(&bar_ke[s]);
        if (prev_s >= 0) umma_commit(&bar_ve[prev_s]);
        prev_s = s;
        prev_ph = ph;
        prev_act[0] = act0;
        prev_act[1] = act1;
        ++it;
      }
      const uint64_t dv_last = dv_base + (uint64_t)((prev_s < 0 ? 0 : prev_s) * TILE16);
#pragma unroll
      for (int t = 0; t < 2; ++t) {  // last PV of each tile
        if (ok && prev_act[t]) {
          ok = mbar_wait_spin(&bar_vf[prev_s], prev_ph, ab, lim, WAIT_FWD_MMA + 5);
          const uint32_t acc0 = o_started[t] ? 1u : 0u;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            if (ok) ok = mbar_wait_spin(&bar_p[2 * t + hf], p_phase[t], ab, lim, WAIT_FWD_MMA + 6);
            if (ok) {
              tc_fence_after();
#pragma unroll
              for (int kk = 4 * hf; kk < 4 * hf + 4; ++kk)
                umma_ts(tmem + 256u + t * D, tmem + t * 128u + kk * 8, dv_last + (uint64_t)(kk * (2048 >> 4)),
                        IDESC_O, kk > 0 ? 1u : acc0);
            }
          }
          if (ok) {
            p_phase[t] ^= 1u;
            o_started[t] = true;
          }
        }
      }
      if (ok && prev_s >= 0) umma_commit(&bar_ve[prev_s]);
      umma_commit(&bar_o[0]);
      umma_commit(&bar_o[1]);
      umma_commit(bar_done);
      AbortState none{0};
      mbar_wait(bar_done, 0, &none, lim, WAIT_FWD_MMA + 7);  // all MMAs retired before TMEM is freed
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ softmax warpgroups
    reg_alloc<C::REGS_SOFTMAX>();
    if constexpr (C::TILES == 1) {
      // One tile: warpgroup h takes key columns [64h, 64h+64) of every row; row r is thread r
      // of each. The halves exchange their row maxima once per KV tile, so both keep the same
      // reference max; P of keys [64h, 64h+64) is the half that O += P V waits on as half h.
      const int h = (warp - 4) >> 2;
      const uint32_t wq = warp & 3;      // TMEM lane quarter this warp may touch
      const int r = wq * 32 + lane;      // row inside the tile
      const int qb = qb0;
      const bool tvalid = qb < p.nb;     // uniform over the CTA
      const uint32_t lane_off = (wq * 32u) << 16;
      const uint32_t tS_row = tmem + lane_off;  // S buffer b at column 128 b
      const uint32_t tO_row = tmem + lane_off + 256u;
      float* xch = reinterpret_cast<float*>(smem + C::OFF_XCH);  // [parity][half][row]
      const float sl2 = p.scale_log2;
      const Ex2PolyConsts ek = ex2_poly_consts();
      float m_ref = -INFINITY;  // reference max, log2 domain, scale folded in
      float l = 0.f;            // this half's running sum of exp2(x - m_ref)
      bool o_started = false;
      bool ok = true;
      int a = 0;                // active KV tiles so far

      for (int j = j_begin; tvalid && j < j_end; ++j) {
        if (!fwd_tile_active(tt, qb, j)) continue;
        const uint32_t b = (uint32_t)(a & 1);
        const uint32_t tS = tS_row + b * 128u;
        const bool diag = tt.causal && (128 * j + 127 > 128 * qb + tt.causal_off);
        const bool masked = diag || (128 * j + 128 > tt.Nk);
        uint32_t su[64];  // this row's scores of this half (fp32 bits)
        float mh = -INFINITY;
        if (ok) ok = warp_wait(&bar_s[b], (uint32_t)(a >> 1) & 1u, ab, lim, WAIT_FWD_SOFTMAX + 1);
        if (ok) {
          tc_fence_after();
          tmem_ld64(tS + 64u * h, su);
          if (masked) {  // same rule as two tiles, for key columns 64h..64h+63
            const int lim_c = min(diag ? 128 * (qb - j) + r + tt.causal_off + 1 : 128, tt.Nk - 128 * j) - 64 * h;
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (c >= lim_c) su[c] = 0xff800000u;  // -inf
          }
          float mc[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            float m = fmax3(__uint_as_float(su[k]), __uint_as_float(su[k + 4]), __uint_as_float(su[k + 8]));
#pragma unroll
            for (int c = 12; c < 60; c += 8) m = fmax3(m, __uint_as_float(su[c + k]), __uint_as_float(su[c + 4 + k]));
            mc[k] = fmaxf(m, __uint_as_float(su[60 + k]));
          }
          mh = fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3]));
          xch[(b * 2 + h) * 128 + r] = mh;
        }
        // Both halves' S columns are read before either half writes P over them (P of keys
        // 64-127 lands on S columns 32-63); a failed wait anywhere ends the loop for all.
        tc_fence_before();
        if (!named_bar_and(1, 256, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float mx = fmaxf(mh, xch[(b * 2 + (h ^ 1)) * 128 + r]);
        const float cand = mx * sl2;
        float alpha = 1.f;
        if (cand > m_ref + 8.f) {  // also taken on the first visible tile (m_ref = -inf)
          alpha = ex2(m_ref - cand);
          m_ref = cand;
        }
        if (h == 0 && o_started && __any_sync(0xffffffffu, alpha != 1.f)) {
          // S(a) was issued before O += P(a-1) V(a-1): wait for that PV, then rescale O in
          // place, all columns, before this half's P lets O += P(a) V(a) start.
          ok = warp_wait(bar_pv, (uint32_t)(a - 1) & 1u, ab, lim, WAIT_FWD_SOFTMAX + 2);
          if (ok) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t u[32];
              tmem_ld32(tO_row + c * 32, u);
#pragma unroll
              for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
              tmem_st32(tO_row + c * 32, u);
            }
          }
        }
        l *= alpha;
        if (ok) {
          const float mneg = (m_ref == -INFINITY) ? 0.f : -m_ref;
          const uint64_t sl2_2 = f2_pack(sl2, sl2), mneg_2 = f2_pack(mneg, mneg);
          const uint32_t tP = tS + 32u * h;  // keys 64h..64h+63 -> 32 packed columns
          if (masked)
            l += softmax_exp_store64<F16, false, 0u>(su, sl2_2, mneg_2, tP, ek);
          else
            l += softmax_exp_store64<F16, true, C::EXP_EMU_MASK>(su, sl2_2, mneg_2, tP, ek);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar_p[2 * b + h]);
        }
        o_started = true;
        ++a;
      }

      // ---------------------------------------------------------------- epilogue
      // Row sum of both halves, through the parity slot the last KV tile did not use (its
      // last readers passed the last exchange barrier before anyone got here).
      float* lx = xch + (a & 1) * 2 * 128;
      if (tvalid) lx[h * 128 + r] = l;
      ok = named_bar_and(1, 256, ok);
      const float l_tot = tvalid ? lx[r] + lx[128 + r] : 0.f;
      if (ok && tvalid) ok = warp_wait(&bar_o[0], 0, ab, lim, WAIT_FWD_EPILOGUE + 1);
      uint8_t* stage = smem + C::OFF_Q;  // Q is no longer read
      if (ok && tvalid) {
        tc_fence_after();
        const float inv_l = (l_tot > 0.f) ? 1.f / l_tot : 0.f;
        const uint32_t sstage = smem_u32(stage);
#pragma unroll 1
        for (int c = h * (D / 64); c < (h + 1) * (D / 64); ++c) {  // this half's D/2 output columns
          uint32_t u[32];
          if (o_started) {
            tmem_ld32(tO_row + c * 32, u);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) u[i] = 0u;
          }
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = pack16<F16>(__uint_as_float(u[2 * i]) * inv_l, __uint_as_float(u[2 * i + 1]) * inv_l);
          const int col0 = c * 32;
          const uint32_t panel = sstage + (col0 >> 6) * C::PANEL_BYTES;
          const uint32_t chunk0 = (col0 & 63) >> 3;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            st_shared_v4(panel + sw128_offset(r, chunk0 + q), w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
        fence_proxy_async_smem();
        const int row = qb * 128 + r;
        const float lse_row = (l_tot > 0.f) ? (m_ref + __log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
        if (p.nsplit > 1) {
          const size_t prow = ((size_t)bh * p.nsplit + split) * p.Np + row;
          float4* dst = reinterpret_cast<float4*>(p.o_part + prow * D);
#pragma unroll 1
          for (int c = h * (D / 64); c < (h + 1) * (D / 64); ++c) {
            uint32_t u[32];
            if (o_started) {
              tmem_ld32(tO_row + c * 32, u);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) u[i] = 0u;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[c * 8 + q] = make_float4(__uint_as_float(u[4 * q]) * inv_l, __uint_as_float(u[4 * q + 1]) * inv_l,
                                           __uint_as_float(u[4 * q + 2]) * inv_l, __uint_as_float(u[4 * q + 3]) * inv_l);
          }
          if (h == 0) p.lse_part[prow] = lse_row;
        } else if (h == 0 && row < p.N) {
          p.lse[(size_t)bh * p.N + row] = lse_row;
        }
      }
      named_bar_sync(1, 256);  // both halves of the output tile are staged
      if (tvalid && p.nsplit == 1 && h == 0 && wq == 0 && lane == 0 &&
          *reinterpret_cast<volatile int*>(&ab->flag) == 0) {
        for (int pn = 0; pn < C::PANELS; ++pn) tma_store_3d(&tmO, stage + pn * C::PANEL_BYTES, pn * 64, qb * 128, bh);
        bulk_commit_group();
        bulk_wait_group_read0();
      }
    } else {
      const int t = (warp - 4) >> 2;    // warps 4-7: tile 0, warps 8-11: tile 1
      const uint32_t wq = warp & 3;      // TMEM lane quarter this warp may touch
      const int r = wq * 32 + lane;      // row inside the tile
      const int qb = qb0 + t;
      const bool tvalid = qb < p.nb;
      const uint32_t lane_off = (wq * 32u) << 16;
      const uint32_t tS_row = tmem + lane_off + t * 128u;
      const uint32_t tO_row = tmem + lane_off + 256u + t * D;
      const float sl2 = p.scale_log2;
      const Ex2PolyConsts ek = ex2_poly_consts();
      float m_ref = -INFINITY;  // reference max, log2 domain, scale folded in
      float l = 0.f;            // running sum of exp2(x - m_ref)
      uint32_t s_phase = 0;
      bool o_started = false;
      bool ok = true;

      if (tvalid) {
        for (int j = j_begin; j < j_end; ++j) {
          if (!fwd_tile_active(tt, qb, j)) continue;
          ok = warp_wait(&bar_s[t], s_phase, ab, lim, WAIT_FWD_SOFTMAX + 1);
          if (!ok) break;
          s_phase ^= 1u;
          tc_fence_after();

          uint32_t su[128];  // this row's 128 scores (fp32 bits)
          tmem_ld128(tS_row, su);
          // Elementwise mask: on the causal diagonal band key 128j+c is visible to row 128qb+r iff
          // 128j+c <= 128qb+r+causal_off (c <= r for the square problem); in a partial last key
          // tile keys 128j+c >= Nk do not exist (TMA filled zeros).
          const bool diag = tt.causal && (128 * j + 127 > 128 * qb + tt.causal_off);
          const bool masked = diag || (128 * j + 128 > tt.Nk);
          if (masked) {
            const int lim = min(diag ? 128 * (qb - j) + r + tt.causal_off + 1 : 128, tt.Nk - 128 * j);
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (c >= lim) su[c] = 0xff800000u;  // -inf
          }
          // Row max: 8 independent chains of three-input max, then a short tree.
          float mc[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            float m = fmax3(__uint_as_float(su[k]), __uint_as_float(su[k + 8]), __uint_as_float(su[k + 16]));
#pragma unroll
            for (int c = 24; c < 120; c += 16) m = fmax3(m, __uint_as_float(su[c + k]), __uint_as_float(su[c + 8 + k]));
            mc[k] = fmaxf(m, __uint_as_float(su[120 + k]));
          }
          const float mx = fmax3(fmax3(mc[0], mc[1], mc[2]), fmax3(mc[3], mc[4], mc[5]), fmaxf(mc[6], mc[7]));
          const float cand = mx * sl2;
          float alpha = 1.f;
          if (cand > m_ref + 8.f) {  // also taken on the first visible tile (m_ref = -inf)
            alpha = ex2(m_ref - cand);
            m_ref = cand;
          }
          if (o_started && __any_sync(0xffffffffu, alpha != 1.f)) {
            // O_t already holds every earlier PV (S_t's commit retired them): rescale in place.
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t u[32];
              tmem_ld32(tO_row + c * 32, u);
#pragma unroll
              for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
              tmem_st32(tO_row + c * 32, u);
            }
          }
          l *= alpha;
          const float mneg = (m_ref == -INFINITY) ? 0.f : -m_ref;
          const uint64_t sl2_2 = f2_pack(sl2, sl2), mneg_2 = f2_pack(mneg, mneg);
          // Without FMA-pipe exponentials the masked and unmasked calls are the same code; at
          // d = 64 one call site (one inlined copy of the 128-score loop) ran 1.7-2.5 % faster,
          // at d = 128 0.5 % slower, so only d = 64 takes it.
          if constexpr (C::EXP_EMU_MASK == 0u && D == 64)
            l += softmax_exp_store<F16, false, 0u>(su, sl2_2, mneg_2, tS_row, ek, &bar_p[2 * t]);
          else if (masked)
            l += softmax_exp_store<F16, false, 0u>(su, sl2_2, mneg_2, tS_row, ek, &bar_p[2 * t]);
          else
            l += softmax_exp_store<F16, true, C::EXP_EMU_MASK>(su, sl2_2, mneg_2, tS_row, ek, &bar_p[2 * t]);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar_p[2 * t + 1]);
          o_started = true;
        }

        // ---------------------------------------------------------------- epilogue
        if (ok) ok = warp_wait(&bar_o[t], 0, ab, lim, WAIT_FWD_EPILOGUE + 1);
        uint8_t* stage = smem + C::OFF_Q + t * C::TILE_BYTES;  // Q_t is no longer read
        if (ok) {
          tc_fence_after();
          const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
          const uint32_t sstage = smem_u32(stage);
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t u[32];
            if (o_started) {
              tmem_ld32(tO_row + c * 32, u);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) u[i] = 0u;
            }
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              w[i] = pack16<F16>(__uint_as_float(u[2 * i]) * inv_l, __uint_as_float(u[2 * i + 1]) * inv_l);
            const int col0 = c * 32;                   // first column of this chunk
            const uint32_t panel = sstage + (col0 >> 6) * C::PANEL_BYTES;
            const uint32_t chunk0 = (col0 & 63) >> 3;  // 16-byte chunk inside the 128-byte row
#pragma unroll
            for (int q = 0; q < 4; ++q)
              st_shared_v4(panel + sw128_offset(r, chunk0 + q), w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
          }
          fence_proxy_async_smem();
          const int row = qb * 128 + r;
          const float lse_row = (l > 0.f) ? (m_ref + __log2f(l)) * 0.69314718055994531f : -INFINITY;
          if (p.nsplit > 1) {
            // Split of the key range: this split's O / l (fp32, re-read from TMEM) and LSE for the
            // merge kernel, every row of the tile (the buffers are padded to Np).
            const size_t prow = ((size_t)bh * p.nsplit + split) * p.Np + row;
            float4* dst = reinterpret_cast<float4*>(p.o_part + prow * D);
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t u[32];
              if (o_started) {
                tmem_ld32(tO_row + c * 32, u);
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) u[i] = 0u;
              }
#pragma unroll
              for (int q = 0; q < 8; ++q)
                dst[c * 8 + q] = make_float4(__uint_as_float(u[4 * q]) * inv_l, __uint_as_float(u[4 * q + 1]) * inv_l,
                                             __uint_as_float(u[4 * q + 2]) * inv_l, __uint_as_float(u[4 * q + 3]) * inv_l);
            }
            p.lse_part[prow] = lse_row;
          } else if (row < p.N) {  // rows of a partial last tile beyond N are not stored (the O store clips them)
            p.lse[(size_t)bh * p.N + row] = lse_row;
          }
        }
        // Every thread of the warpgroup reaches this barrier (tvalid is uniform per warpgroup).
        named_bar_sync(1 + t, 128);
        if (p.nsplit == 1 && wq == 0 && lane == 0 && *reinterpret_cast<volatile int*>(&ab->flag) == 0) {
          for (int pn = 0; pn < C::PANELS; ++pn) tma_store_3d(&tmO, stage + pn * C::PANEL_BYTES, pn * 64, qb * 128, bh);
          bulk_commit_group();
          bulk_wait_group_read0();
        }
      }
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

// The one-tile kernel (one CTA per SM) runs d = 256, and a single query tile (decode) at d = 128;
// a single tile at d = 64 goes to the two-CTAs-per-SM kernel below, whose second CTA hides
// the first one's chain (decode at Nq = 128, 16384 keys: K/V read 3.3 -> 3.7 TB/s; fewer rows
// also copy them across the lane quarters, fwd_rep).
bool fwd_one_tile(int D, int nb) { return D == 256 || (nb == 1 && D == 128); }

// Short sequences (few query tiles per head) run one query tile per CTA, two CTAs per SM
// (fa_fwd_solo.cu), so that one CTA's prologue and epilogue overlap the other's KV steps.
bool fwd_solo(int D, int nb) { return !fwd_one_tile(D, nb) && nb <= FA_FWD_SOLO_MAX_NB; }

int fwd_tiles_per_cta(int D, int nb) { return (fwd_one_tile(D, nb) || fwd_solo(D, nb)) ? 1 : 2; }

// At most 32 (64) query rows and d = 64 (decode): the tile's lane quarters hold four (two)
// copies of those rows and split each KV step's keys between them, so the softmax warps share
// the step's exponentials instead of the quarters holding the real rows doing them all.
int fwd_rep(int D, int Nq) { return D != 64 ? 1 : Nq <= 32 ? 4 : Nq <= 64 ? 2 : 1; }

template <int D, bool F16, int REP>
cudaError_t launch_fwd_solo(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& to, const FwdParams& p, long long BH, cudaStream_t stream);

template <int D, bool F16, bool ONE>
static cudaError_t launch_fwd_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const CUtensorMap& to, const FwdParams& p, long long BH, cudaStream_t stream) {
  using C = FwdCfg<D, ONE>;
  cudaError_t e =
      cudaFuncSetAttribute(fa_fwd_kernel<D, F16, ONE>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const dim3 grid = grid_work((p.nb + C::TILES - 1) / C::TILES * p.nsplit, BH, p.order_group);
  fa_fwd_kernel<D, F16, ONE><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, to, p);
  return cudaGetLastError();
}

template <bool F16>
static cudaError_t launch_fwd_dtype(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                    const CUtensorMap& to, const FwdParams& p, long long BH, cudaStream_t stream) {
  if (D == 256) return launch_fwd_t<256, F16, true>(tq, tk, tv, to, p, BH, stream);
  if (fwd_solo(D, p.nb))
    return D == 128                 ? launch_fwd_solo<128, F16, 1>(tq, tk, tv, to, p, BH, stream)
           : fwd_rep(D, p.N) == 4 ? launch_fwd_solo<64, F16, 4>(tq, tk, tv, to, p, BH, stream)
           : fwd_rep(D, p.N) == 2 ? launch_fwd_solo<64, F16, 2>(tq, tk, tv, to, p, BH, stream)
                                  : launch_fwd_solo<64, F16, 1>(tq, tk, tv, to, p, BH, stream);
  const bool one = fwd_one_tile(D, p.nb);
  if (D == 64)
    return one ? launch_fwd_t<64, F16, true>(tq, tk, tv, to, p, BH, stream)
               : launch_fwd_t<64, F16, false>(tq, tk, tv, to, p, BH, stream);
  return one ? launch_fwd_t<128, F16, true>(tq, tk, tv, to, p, BH, stream)
             : launch_fwd_t<128, F16, false>(tq, tk, tv, to, p, BH, stream);
}

cudaError_t launch_fwd(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& to, const FwdParams& p, long long BH, cudaStream_t stream) {
  return p.f16 ? launch_fwd_dtype<true>(D, tq, tk, tv, to, p, BH, stream)
               : launch_fwd_dtype<false>(D, tq, tk, tv, to, p, BH, stream);
}

}  // namespace fa
