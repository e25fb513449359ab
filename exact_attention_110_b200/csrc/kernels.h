// Kernel parameter blocks and launchers shared by the host API (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

// Where a device-side bounded wait gave up (stored in the device status word).
enum WaitSite : int {
  WAIT_NONE = 0,
  WAIT_SMEM_ALIGN = 1,
  WAIT_FWD_LOAD = 0x100,
  WAIT_FWD_MMA = 0x200,
  WAIT_FWD_SOFTMAX = 0x300,
  WAIT_FWD_EPILOGUE = 0x400,
  WAIT_BWD_LOAD = 0x1100,
  WAIT_BWD_MMA = 0x1200,
  WAIT_BWD_COMPUTE = 0x1300,
  WAIT_BWD_DQ = 0x1400,
  WAIT_BWD_EPILOGUE = 0x1500,
  WAIT_SELFTEST = 0x7700,
};

// (b, h) of this CTA. Up to 65535 heads the grid's y index is the head; beyond that the
// heads are spread over y and z (grid_bh), and CTAs past the last head exit at once.
__device__ __forceinline__ long long cta_bh() { return (long long)blockIdx.z * gridDim.y + blockIdx.y; }
inline dim3 grid_bh(unsigned x, long long BH) {
  const unsigned z = (unsigned)((BH + 65534) / 65535);
  const unsigned y = (unsigned)((BH + z - 1) / z);
  return dim3(x, y, z);
}

// Work items (CTAs) of one head: `items` of them. Without a causal mask they all cost the same
// and the grid is (items, heads) as grid_bh lays it out (group = 0). With a causal mask item 0
// is the heaviest and the cost falls item by item; the block scheduler starts CTAs in grid
// order, so a head-by-head order would start the last heads' heaviest items at the very end
// and leave SMs idle in the tail. The grid is then one-dimensional: groups of `group` heads,
// and within a group every head's item 0, then every head's item 1, and so on (longest items
// first), while the CTAs in flight still read the tiles of few heads, which stay in L2.
// Returns false for a CTA past the last head.
__device__ __forceinline__ bool cta_work(long long BH, int items, int group, int& bh, int& item) {
  if (group <= 0) {
    const long long b = cta_bh();
    bh = (int)b;
    item = (int)blockIdx.x;
    return b < BH;
  }
  const long long G = group < BH ? group : BH;
  const long long x = blockIdx.x, g = x / (G * items), rem = x - g * G * items;
  const long long gsz = BH - g * G < G ? BH - g * G : G;
  item = (int)(rem / gsz);
  bh = (int)(g * G + rem % gsz);
  return true;
}
// Head and item of work-item number x in grid order (the order cta_work gives the CTAs of a
// one-CTA-per-item grid: head by head, or the causal longest-first groups), for persistent
// CTAs that take item numbers from a counter. x < BH * items.
__device__ __forceinline__ void work_item(long long x, long long BH, int items, int group, int& bh, int& item) {
  if (group <= 0) {
    const long long b = x / items;
    bh = (int)b;
    item = (int)(x - b * items);
    return;
  }
  const long long G = group < BH ? group : BH;
  const long long g = x / (G * items), rem = x - g * G * items;
  const long long gsz = BH - g * G < G ? BH - g * G : G;
  item = (int)(rem / gsz);
  bh = (int)(g * G + rem % gsz);
}
inline dim3 grid_work(int items, long long BH, int group) {
  return group > 0 ? dim3((unsigned)(items * BH)) : grid_bh((unsigned)items, BH);
}
// Heads per group for a causal grid: about two CTAs per SM per group (measured on the N = 1024 to
// 16384 sweep: +6 to +9 % on the causal forward and backward against the head-by-head order); 0
// (head by head) without the causal mask or when the one-dimensional grid would be too long.
inline int causal_group(bool causal, int items, long long BH, int sms) {
  if (!causal || (long long)items * BH > 0x7fffffffll) return 0;
  const int g = 2 * sms / (items > 0 ? items : 1);
  return g < 1 ? 1 : g;
}

struct FwdParams {
  float* lse;                  // [BH][N]
  long long BH;                // heads (B * H)
  int order_group;             // grid order: 0 = head by head, G > 0 = longest-first in groups of G heads
  const uint8_t* block_mask;   // [nb][nb] (or one per (b, h), mask_stride apart) or null
  long long mask_stride;       // elements between consecutive (b, h) masks; 0 = one shared mask
  int N;                       // query rows per head
  int nb;                      // ceil(N / 128) query tiles
  int Nk;                      // keys per head (N for the square problem)
  int nbk;                     // ceil(Nk / 128) key tiles
  int causal_off;              // causal: key j is visible to query i iff j <= i + causal_off
  int nsplit;                  // key-range splits per pair of query tiles (1: no split)
  int kv_per_split;            // key tiles per split
  int Np;                      // N rounded up to 128 (rows of the split partials)
  float* o_part;               // nsplit > 1: fp32 [BH][nsplit][Np][D], each split's O / l
  float* lse_part;             // nsplit > 1: fp32 [BH][nsplit][Np], each split's LSE
  int causal;
  float scale_log2;            // scale * log2(e)
  unsigned long long timeout_ns;
  int f16;                     // element type: fp16 if non-zero, bf16 otherwise
};

struct BwdPreParams {
  const uint16_t* o;     // bf16 [BH][N][D]
  const uint16_t* dout;  // bf16 [BH][N][D]
  const float* lse;      // [BH][N]
  float* delta;          // [BH][Np]  = -D = -rowsum(dO o O)
  float* lse2;           // [BH][Np]  = -LSE * log2(e) + log2(scale)
  float* dq_acc;         // [BH][Np][D], zeroed here
  unsigned long long* counters;  // [2] backward work-scheduling counters, zeroed here
  long long rows;        // BH * N
  int N, Np, D;
  float log2_scale;      // log2(scale), scale > 0: folds the softmax scale into P (see fa_bwd.cu)
  int f16;               // element type: fp16 if non-zero, bf16 otherwise
};

struct BwdParams {
  long long BH;          // heads (B * H)
  int order_group;       // grid order: 0 = head by head, G > 0 = longest-first in groups of G heads
  const float* delta;    // [BH][Np]  -D
  const float* lse2;     // [BH][Np]  -LSE * log2(e) + log2(scale)
  float* dq_acc;         // [BH][Np][D]
  const uint8_t* block_mask;
  long long mask_stride; // elements between consecutive (b, h) masks; 0 = one shared mask
  int N, Np, nb;         // query rows, padded to 128, query tiles
  int Nk, nbk;           // keys, key tiles (N_k = N for the square problem)
  int causal;
  int causal_off;        // causal: key j is visible to query i iff j <= i + causal_off
  float inv_scale;       // 1 / scale (dV epilogue: P carries the scale)
  float scale_log2;      // scale * log2(e)
  unsigned long long timeout_ns;
  int f16;               // element type: fp16 if non-zero, bf16 otherwise
  int persist;           // 0: one CTA per (head, key tile); > 0: persistent CTAs
  unsigned long long* counters;  // persistent: [0] items handed out after each CTA's first, [1] CTAs done
};

struct FwdMergeParams {
  const float* o_part;   // [BH][nsplit][Np][D]
  const float* lse_part; // [BH][nsplit][Np]
  uint16_t* o;           // bf16 / fp16 [BH][N][D]
  float* lse;            // [BH][N]
  long long rows;        // BH * N
  int N, Np, nsplit, D;
  int f16;
};

struct DqFinishParams {
  const float* dq_acc;   // [BH][Np][D]
  uint16_t* dq;          // bf16 [BH][N][D]
  long long rows;        // BH * N
  int N, Np, D;
  float scale;
  int f16;               // element type: fp16 if non-zero, bf16 otherwise
};

// Streaming multiprocessors of the current device (cached per device ordinal).
inline int device_sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cached[dev] <= 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 148;
  }
  return cached[dev];
}

// Launchers (return the launch error, if any).
cudaError_t launch_fwd(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& to, const FwdParams& p, long long BH, cudaStream_t stream);
cudaError_t launch_fwd_merge(const FwdMergeParams& p, cudaStream_t stream);
// Whether the forward runs one 128-row query tile per CTA (head dimension D, nb query tiles),
// and the tiles per CTA that follow (1 or 2).
bool fwd_one_tile(int D, int nb);
int fwd_tiles_per_cta(int D, int nb);
// Copies of the query rows per 128-row tile (at d = 64: 4 for at most 32 rows, 2 for at most
// 64, each copy scoring its share of every KV step's keys; else 1); the Q tensor map's box is
// 128 / that many rows high.
int fwd_rep(int D, int Nq);
cudaError_t launch_bwd_pre(const BwdPreParams& p, cudaStream_t stream);
cudaError_t launch_bwd_main(int D, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const CUtensorMap& tdk, const CUtensorMap& tdv,
                            const CUtensorMap& tdqa, const BwdParams& p, long long BH, cudaStream_t stream);
cudaError_t launch_dq_finish(const DqFinishParams& p, cudaStream_t stream);

}  // namespace fa
