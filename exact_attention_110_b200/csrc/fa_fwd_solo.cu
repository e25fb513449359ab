// Forward kernel for short sequences: one 128-row query tile per CTA, two CTAs per SM.
//
// Same method and per-tile data flow as the two-tile kernel in fa_fwd.cu (tiling and online
// softmax of [P3] §3.1-§3.3, FA2 loop order and deferred normalisation of [P1] §主要操作; S and
// P in tensor memory, O += P V with P read from TMEM, the lazy rescale). What differs is how
// the SM is shared. The two-tile kernel owns a whole SM (512 TMEM columns, ~192 KB of shared
// memory), so nothing overlaps its per-CTA prologue (barrier set-up, TMEM allocation, the first
// Q/K/V loads, the first S) and epilogue (O out of TMEM, the TMA store); with few KV steps per
// CTA (N of 512 to 1024) those dominate. Here a CTA needs 256 TMEM columns (S [0,128), O
// [128, 128+D)), at most ~96 KB of shared memory and 192 threads at 168 registers, so two
// CTAs are resident per SM: the tensor core and the special-function unit interleave the two
// CTAs' chains (the ping-pong of the two-tile kernel, across CTAs) and one CTA's prologue and
// epilogue overlap the other's KV steps.
// Decode form (REP = 4 or 2: d = 64, at most 32 or 64 query rows): a tile with one real row
// still costs a whole 128-row softmax per KV step, all of it in the warp that holds the row.
// Here the query tile is loaded as REP copies of its first 128 / REP rows (four copies: one
// per TMEM lane quarter), and copy c scores only keys (128 / REP) c .. of each step (P of the
// row's other keys is zero in its lanes), so the warps share the exponentials; the copies' O
// are combined at the end like the partial results of a key-range split (LSE-weighted).
// Roles (192 threads, so two CTAs keep 168 registers per thread): warps 0-3 the softmax
// (thread = row = TMEM lane), warp 4 the TMA producer, warp 5 the MMA issuer (one thread),
// which also allocates and frees the tensor memory.
#include "kernels.h"
#include "ptx.cuh"

namespace fa {

template <int D>
struct FwdSoloCfg {
  static constexpr int THREADS = 192;
  static constexpr int NS = D == 128 ? 1 : 2;  // K ring and V ring depth
  static constexpr int PANEL_BYTES = 128 * 128;
  static constexpr int PANELS = D / 64;
  static constexpr int TILE_BYTES = PANELS * PANEL_BYTES;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILE_BYTES;
  static constexpr int OFF_V = OFF_K + NS * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + NS * TILE_BYTES;
  static constexpr int NBAR = 1 + 4 * NS + 1 + 2 + 1 + 1;  // q, k/v full/empty, s, p[2], o, done
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr int TMEM_COLS = 256;
  static_assert(2 * (SMEM_BYTES + 1024) <= 233472, "two CTAs per SM");
};

template <int D, bool F16, int REP>
__global__ void __launch_bounds__(192, 2)
    fa_fwd_solo_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                       const FwdParams p) {
  using C = FwdSoloCfg<D>;
  constexpr int NS = C::NS;
  extern __shared__ __align__(1024) uint8_t smem[];

  const uint32_t warp = warp_id(), lane = lane_id();
  if ((smem_u32(smem) & 1023u) != 0) {  // swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicCAS(&g_fa_device_status, 0, WAIT_SMEM_ALIGN);
    return;
  }

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_q = bars;            // Q tile landed
  uint64_t* bar_kf = bars + 1;       // [NS] K stage full
  uint64_t* bar_ke = bar_kf + NS;    // [NS] K stage free
  uint64_t* bar_vf = bar_ke + NS;    // [NS] V stage full
  uint64_t* bar_ve = bar_vf + NS;    // [NS] V stage free
  uint64_t* bar_s = bar_ve + NS;     // S ready in TMEM
  uint64_t* bar_p = bar_s + 1;       // [2] P keys 0-63 / 64-127 written (O rescaled before)
  uint64_t* bar_o = bar_p + 2;       // all MMAs complete (epilogue)
  uint64_t* bar_done = bar_o + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  AbortState* ab = reinterpret_cast<AbortState*>(smem + C::OFF_MISC + 4);

  int bh, xi;  // head and work item = query tile * nsplit + split; causal: the heaviest tiles first
  if (!cta_work(p.BH, p.nb * p.nsplit, p.order_group, bh, xi)) return;
  const uint8_t* bmask = p.block_mask == nullptr ? nullptr : p.block_mask + (size_t)bh * p.mask_stride;
  const TileTest tt{p.nb, p.nbk, p.Nk, p.causal, p.causal_off, bmask};
  const int ti = xi / p.nsplit, split = xi - ti * p.nsplit;
  const int qb = p.causal ? p.nb - 1 - ti : ti;
  const int j_begin = split * p.kv_per_split;
  int j_end = min(p.nbk, j_begin + p.kv_per_split);
  if (p.causal) {
    const int last_key = 128 * qb + 127 + p.causal_off;
    j_end = min(j_end, last_key < 0 ? 0 : last_key / 128 + 1);
  }
  const uint64_t lim = p.timeout_ns;

  if (warp == 4 && lane == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar_kf[s], 1);
      mbar_init(&bar_ke[s], 1);
      mbar_init(&bar_vf[s], 1);
      mbar_init(&bar_ve[s], 1);
    }
    mbar_init(bar_s, 1);
    mbar_init(&bar_p[0], 4);  // one arrive per softmax warp
    mbar_init(&bar_p[1], 4);
    mbar_init(bar_o, 1);
    mbar_init(bar_done, 1);
    ab->flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
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
  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmO);
      mbar_arrive_expect_tx(bar_q, C::TILE_BYTES);
      for (int pn = 0; pn < C::PANELS; ++pn)
        for (int w = 0; w < REP; ++w)  // REP copies of the tile's first 128 / REP rows (tmQ's box height)
          tma_load_3d(smem + C::OFF_Q + pn * C::PANEL_BYTES + w * (128 / REP) * 128, &tmQ, bar_q, pn * 64, qb * 128,
                      bh);
      int it = 0;
      int issued_k[NS], issued_v[NS];
      for (int s = 0; s < NS; ++s) issued_k[s] = issued_v[s] = -1;
      bool ok = true;
      for (int j = j_begin; j < j_end && ok; ++j) {
        if (!fwd_tile_active(tt, qb, j)) continue;
        const int s = it % NS;
        const uint32_t ph = (uint32_t)(it / NS) & 1u;
        ok = mbar_wait(&bar_ke[s], ph ^ 1u, ab, lim, WAIT_FWD_LOAD + 1);
        if (!ok) break;
        mbar_arrive_expect_tx(&bar_kf[s], C::TILE_BYTES);
        for (int pn = 0; pn < C::PANELS; ++pn)
          tma_load_3d(smem + C::OFF_K + s * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmK, &bar_kf[s], pn * 64, j * 128,
                      bh);
        issued_k[s] = (int)ph;
        ok = mbar_wait(&bar_ve[s], ph ^ 1u, ab, lim, WAIT_FWD_LOAD + 2);
        if (!ok) break;
        mbar_arrive_expect_tx(&bar_vf[s], C::TILE_BYTES);
        for (int pn = 0; pn < C::PANELS; ++pn)
          tma_load_3d(smem + C::OFF_V + s * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmV, &bar_vf[s], pn * 64, j * 128,
                      bh);
        issued_v[s] = (int)ph;
        ++it;
      }
      if (!ok) {
        AbortState none{0};
        for (int s = 0; s < NS; ++s) {
          if (issued_k[s] >= 0) mbar_wait(&bar_kf[s], issued_k[s], &none, lim, WAIT_FWD_LOAD + 3);
          if (issued_v[s] >= 0) mbar_wait(&bar_vf[s], issued_v[s], &none, lim, WAIT_FWD_LOAD + 3);
        }
        mbar_wait(bar_q, 0, &none, lim, WAIT_FWD_LOAD + 4);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    // Per KV step j: O += P(j-1) V(j-1) (P read from TMEM, in two halves as the softmax writes
    // them), then S = Q K_j^T over the same columns (the tensor pipe runs in order, so the PV
    // MMAs read P before S overwrites it).
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_f32acc(128, 128, 0, 0, F16);
      constexpr uint32_t IDESC_O = idesc_f32acc(128, D, 0, 1, F16);
      constexpr uint32_t TILE16 = C::TILE_BYTES >> 4;
      const uint64_t dq = sdesc_sw128(sQ, 16, 1024);
      const uint64_t dk_base = sdesc_sw128(sK, 16, 1024);
      const uint64_t dv_base = sdesc_sw128(sV, C::PANEL_BYTES, 1024);
      bool ok = mbar_wait_spin(bar_q, 0, ab, lim, WAIT_FWD_MMA + 1);
      uint32_t p_phase = 0;
      bool o_started = false;
      int prev_s = -1;
      uint32_t prev_ph = 0;
      int it = 0;
      auto issue_pv = [&](int where) -> bool {
        if (!mbar_wait_spin(&bar_vf[prev_s], prev_ph, ab, lim, where)) return false;
        const uint64_t dv = dv_base + (uint64_t)(prev_s * TILE16);
        const uint32_t acc0 = o_started ? 1u : 0u;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          if (!mbar_wait_spin(&bar_p[hf], p_phase, ab, lim, WAIT_FWD_MMA + 4)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 4 * hf; kk < 4 * hf + 4; ++kk)
            umma_ts(tmem + 128u, tmem + kk * 8, dv + (uint64_t)(kk * (2048 >> 4)), IDESC_O, kk > 0 ? 1u : acc0);
        }
        p_phase ^= 1u;
        o_started = true;
        umma_commit(&bar_ve[prev_s]);
        return true;
      };
      for (int j = j_begin; j < j_end && ok; ++j) {
        if (!fwd_tile_active(tt, qb, j)) continue;
        const int s = it % NS;
        const uint32_t ph = (uint32_t)(it / NS) & 1u;
        ok = mbar_wait_spin(&bar_kf[s], ph, ab, lim, WAIT_FWD_MMA + 2);
        if (ok && prev_s >= 0) ok = issue_pv(WAIT_FWD_MMA + 3);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dk = dk_base + (uint64_t)(s * TILE16);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {  // S = Q K_j^T
          const uint32_t off16 = ((kk >> 2) * C::PANEL_BYTES + (kk & 3) * 32) >> 4;
          umma_ss(tmem, dq + off16, dk + off16, IDESC_S, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar_s);
        umma_commit(&bar_ke[s]);
        prev_s = s;
        prev_ph = ph;
        ++it;
      }
      if (ok && prev_s >= 0) ok = issue_pv(WAIT_FWD_MMA + 5);  // the last step's O += P V
      umma_commit(bar_o);
      umma_commit(bar_done);
      AbortState none{0};
      mbar_wait(bar_done, 0, &none, lim, WAIT_FWD_MMA + 7);  // all MMAs retired before TMEM is freed
    }
  } else {
    // ------------------------------------------------------------------ softmax warpgroup
    const uint32_t wq = warp & 3;  // TMEM lane quarter this warp may touch
    // The tile's lanes hold REP copies of its first 128 / REP rows (REP = 1: all 128 rows, thread
    // = row). Copy cp = wq / QPR scores keys W cp .. W cp + W - 1 of each step; the copies'
    // partial softmaxes are combined in the epilogue.
    constexpr int W = 128 / REP;   // keys of a step this warp scores
    constexpr int QPR = 4 / REP;   // lane quarters per copy
    const int r = (int)((wq % QPR) * 32 + lane);  // row inside the tile
    const int c0 = (int)(wq / QPR) * W;          // first of this warp's keys in a step
    const uint32_t lane_off = (wq * 32u) << 16;
    const uint32_t tS_row = tmem + lane_off;
    const uint32_t tO_row = tmem + lane_off + 128u;
    const float sl2 = p.scale_log2;
    const Ex2PolyConsts ek = ex2_poly_consts();
    float m_ref = -INFINITY;  // reference max, log2 domain, scale folded in
    float l = 0.f;            // running sum of exp2(x - m_ref)
    uint32_t s_phase = 0;
    bool o_started = false;
    bool ok = true;

    for (int j = j_begin; j < j_end; ++j) {
      if (!fwd_tile_active(tt, qb, j)) continue;
      ok = warp_wait(bar_s, s_phase, ab, lim, WAIT_FWD_SOFTMAX + 1);
      if (!ok) break;
      s_phase ^= 1u;
      tc_fence_after();
      uint32_t su[W];
      if constexpr (REP == 1)
        tmem_ld128(tS_row, su);
      else if constexpr (REP == 2)
        tmem_ld64(tS_row + c0, su);
      else
        tmem_ld32(tS_row + c0, su);
      // causal band and the keys >= Nk of a partial last key tile, as in the two-tile kernel
      const bool diag = tt.causal && (128 * j + 127 > 128 * qb + tt.causal_off);
      const bool masked = diag || (128 * j + 128 > tt.Nk);
      if (masked) {
        const int lim_c = min(diag ? 128 * (qb - j) + r + tt.causal_off + 1 - c0 : W, tt.Nk - 128 * j - c0);
#pragma unroll
        for (int c = 0; c < W; ++c)
          if (c >= lim_c) su[c] = 0xff800000u;  // -inf
      }
      float mx;
      if constexpr (REP == 1) {
        float mc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float m = fmax3(__uint_as_float(su[k]), __uint_as_float(su[k + 8]), __uint_as_float(su[k + 16]));
#pragma unroll
          for (int c = 24; c < 120; c += 16) m = fmax3(m, __uint_as_float(su[c + k]), __uint_as_float(su[c + 8 + k]));
          mc[k] = fmaxf(m, __uint_as_float(su[120 + k]));
        }
        mx = fmax3(fmax3(mc[0], mc[1], mc[2]), fmax3(mc[3], mc[4], mc[5]), fmaxf(mc[6], mc[7]));
      } else {
        float mc[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {  // four chains over k, k + 4, ..., k + W - 4
          float m = __uint_as_float(su[k]);
#pragma unroll
          for (int c = 4; c + 4 < W; c += 8) m = fmax3(m, __uint_as_float(su[c + k]), __uint_as_float(su[c + 4 + k]));
          mc[k] = fmaxf(m, __uint_as_float(su[W - 4 + k]));
        }
        mx = fmaxf(fmax3(mc[0], mc[1], mc[2]), mc[3]);
      }
      const float cand = mx * sl2;
      float alpha = 1.f;
      if (cand > m_ref + 8.f) {  // also taken on the first visible tile (m_ref = -inf)
        alpha = ex2(m_ref - cand);
        m_ref = cand;
      }
      if (o_started && __any_sync(0xffffffffu, alpha != 1.f)) {
        // O already holds every earlier PV (S's commit retired them): rescale in place.
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
      if constexpr (REP == 1) {
        l += softmax_exp_store<F16, false, 0u>(su, sl2_2, mneg_2, tS_row, ek, &bar_p[0]);
      } else {
        // P of this warp's W keys in packed columns c0 / 2 ..; the row's other keys belong to
        // the other copies, so their P columns are zero in this lane quarter.
        uint64_t ls2[2] = {0ull, 0ull};
#pragma unroll
        for (int c = 0; c < W / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint64_t s2 = f2_pack(__uint_as_float(su[32 * c + 2 * i]), __uint_as_float(su[32 * c + 2 * i + 1]));
            const uint64_t x2 = ffma2(s2, sl2_2, mneg_2);
            float x0, x1;
            f2_unpack(x2, x0, x1);
            const uint64_t p2 = f2_pack(ex2(x0), ex2(x1));
            ls2[i & 1] = fadd2(ls2[i & 1], p2);
            float p0, p1;
            f2_unpack(p2, p0, p1);
            pk[i] = pack16<F16>(p0, p1);
          }
          tmem_st16(tS_row + c0 / 2 + 16 * c, pk);
        }
        uint32_t zero[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) zero[i] = 0u;
#pragma unroll
        for (int g = 0; g < 4; ++g)
          if (g < c0 / 32 || g >= c0 / 32 + W / 32) tmem_st16(tS_row + 16 * g, zero);
        const uint64_t t2 = fadd2(ls2[0], ls2[1]);
        float a, b;
        f2_unpack(t2, a, b);
        l += a + b;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_p[0]);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_p[1]);
      o_started = true;
    }

    // ---------------------------------------------------------------- epilogue
    if (ok) ok = warp_wait(bar_o, 0, ab, lim, WAIT_FWD_EPILOGUE + 1);
    uint8_t* stage = smem + C::OFF_Q;  // Q is no longer read
    if constexpr (REP == 1) {
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
          const int col0 = c * 32;
          const uint32_t panel = sstage + (col0 >> 6) * C::PANEL_BYTES;
          const uint32_t chunk0 = (col0 & 63) >> 3;
  #pragma unroll
          for (int q = 0; q < 4; ++q)
            st_shared_v4(panel + sw128_offset(r, chunk0 + q), w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
        fence_proxy_async_smem();
        const int row = qb * 128 + r;
        const float lse_row = (l > 0.f) ? (m_ref + __log2f(l)) * 0.69314718055994531f : -INFINITY;
        if (p.nsplit > 1) {
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
        } else if (row < p.N) {
          p.lse[(size_t)bh * p.N + row] = lse_row;
        }
      }
    } else {
      // Combine the copies' partial softmaxes of each row i < 128 / REP (the same split-and-merge
      // rule as the key-range pieces): M = max_w m_w, L = sum_w 2^(m_w - M) l_w,
      // O = sum_w 2^(m_w - M) O_w / L, LSE = (M + log2 L) ln 2. The K/V ring is free once every
      // MMA has completed; it holds the copies' m, l and unnormalised O rows, entry
      // w * 128 / REP + i for copy w of row i (= the lane's TMEM row wq * 32 + lane).
      constexpr int OS = D + 4;  // padded row stride (floats) of the O scratch
      static_assert((2 * 128 + 128 * OS) * 4 <= 2 * C::NS * C::TILE_BYTES, "combine scratch fits the K/V ring");
      constexpr int RPC = 128 / REP;  // rows per copy
      float* cm = reinterpret_cast<float*>(smem + C::OFF_K);  // [REP][RPC]
      float* cl = cm + 128;                                   // [REP][RPC]
      float* co = cl + 128;                                   // [REP][RPC][OS]
      if (ok) {
        tc_fence_after();
        cm[wq * 32 + lane] = m_ref;
        cl[wq * 32 + lane] = l;
        float4* orow = reinterpret_cast<float4*>(co + (wq * 32 + lane) * OS);  // copy wq / QPR, row r
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
            orow[c * 8 + q] = make_float4(__uint_as_float(u[4 * q]), __uint_as_float(u[4 * q + 1]),
                                          __uint_as_float(u[4 * q + 2]), __uint_as_float(u[4 * q + 3]));
        }
      }
      named_bar_sync(1, 128);  // every copy's partial rows are in shared memory
      if (ok) {
        // REP threads per row, each on D / REP of its columns
        const int i = (int)threadIdx.x / REP, part = (int)threadIdx.x % REP;
        constexpr int CW = D / REP;
        const int col0 = part * CW;
        float f[REP], M = -INFINITY;
#pragma unroll
        for (int w = 0; w < REP; ++w) M = fmaxf(M, cm[w * RPC + i]);
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < REP; ++w) {
          const float mw = cm[w * RPC + i];
          f[w] = (mw == -INFINITY) ? 0.f : ex2(mw - M);
          L += f[w] * cl[w * RPC + i];
        }
        const float inv_L = (L > 0.f) ? 1.f / L : 0.f;
#pragma unroll
        for (int w = 0; w < REP; ++w) f[w] *= inv_L;
        float o[CW];
#pragma unroll
        for (int c = 0; c < CW; c += 4) {
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int w = 0; w < REP; ++w) {
            const float4 v4 = *reinterpret_cast<const float4*>(co + (w * RPC + i) * OS + col0 + c);
            acc.x += f[w] * v4.x;
            acc.y += f[w] * v4.y;
            acc.z += f[w] * v4.z;
            acc.w += f[w] * v4.w;
          }
          o[c] = acc.x;
          o[c + 1] = acc.y;
          o[c + 2] = acc.z;
          o[c + 3] = acc.w;
        }
        const int row = qb * 128 + i;
        const float lse_row = (L > 0.f) ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
        if (p.nsplit > 1) {
          const size_t prow = ((size_t)bh * p.nsplit + split) * p.Np + row;
          float4* dst = reinterpret_cast<float4*>(p.o_part + prow * D + col0);
#pragma unroll
          for (int c = 0; c < CW / 4; ++c) dst[c] = make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
          if (part == 0) p.lse_part[prow] = lse_row;
        } else {
          const uint32_t sstage = smem_u32(stage);
#pragma unroll
          for (int k = 0; k < CW / 8; ++k) {
            const int col = col0 + 8 * k;
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) w4[e] = pack16<F16>(o[8 * k + 2 * e], o[8 * k + 2 * e + 1]);
            st_shared_v4(sstage + (col >> 6) * C::PANEL_BYTES + sw128_offset(i, (col & 63) >> 3), w4[0], w4[1], w4[2],
                         w4[3]);
          }
          fence_proxy_async_smem();
          if (part == 0 && row < p.N) p.lse[(size_t)bh * p.N + row] = lse_row;
        }
      }
    }
    named_bar_sync(1, 128);  // the whole output tile is staged
    if (p.nsplit == 1 && wq == 0 && lane == 0 && *reinterpret_cast<volatile int*>(&ab->flag) == 0) {
      for (int pn = 0; pn < C::PANELS; ++pn) tma_store_3d(&tmO, stage + pn * C::PANEL_BYTES, pn * 64, qb * 128, bh);
      bulk_commit_group();
      bulk_wait_group_read0();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D, bool F16, int REP>
cudaError_t launch_fwd_solo(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& to, const FwdParams& p, long long BH, cudaStream_t stream) {
  using C = FwdSoloCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(fa_fwd_solo_kernel<D, F16, REP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const dim3 grid = grid_work(p.nb * p.nsplit, BH, p.order_group);
  fa_fwd_solo_kernel<D, F16, REP><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, to, p);
  return cudaGetLastError();
}

}  // namespace fa
