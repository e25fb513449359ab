// Host side of the C ABI declared in include/fa.h: argument validation, workspace layout,
// TMA tensor-map encoding and kernel launches. No device memory is allocated here.
#include <cudaTypedefs.h>
#include <math.h>
#include <mutex>

#include "fa.h"  // include/ is on the include path
#include "kernels.h"
#include "ptx.cuh"

namespace {

constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per bounded device wait

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// [BH][N][D] bf16 (or fp16) viewed as a 3-D tensor {D, N, BH}; box 64 x rows x 1 (rows = 128,
// or 128 / k for a query tile loaded as k copies of its first 128 / k rows), 128-byte swizzle.
bool encode_bhnd(CUtensorMap* map, const void* base, long long BH, int N, int D, int f16, int rows = 128) {
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)N * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType dt = f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = g_encode(map, dt, 3, const_cast<void*>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The fp32 dQ accumulator [BH*Np][D] as a 2-D tensor {D, BH*Np}; box 32 x 128 (one 128-byte
// swizzled row per query), the unit of the backward's bulk reductions.
bool encode_dq_acc(CUtensorMap* map, float* base, long long rows, int D) {
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 4};
  cuuint32_t box[2] = {32, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool valid_dtype(int dt) { return dt == FA_DTYPE_BF16 || dt == FA_DTYPE_F16; }

// A per-(b, h) block-mask stride is 0 (one mask shared by every head) or at least one whole
// ceil(N/128)^2 mask; it is ignored without a mask.
bool mask_stride_ok(const uint8_t* mask, long long stride, int N) {
  if (mask == nullptr) return true;
  const long long nb = (N + 127) / 128;
  return stride == 0 || stride >= nb * nb;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Head dimensions: 64, 128 and 256 in every pass.
fa_status check_common(int B, int H, int N, int d, float scale) {
  if (B <= 0 || H <= 0 || N <= 0 || !isfinite(scale)) return FA_ERR_INVALID;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  if (BH > 0x7fffffffll) return FA_ERR_UNSUPPORTED;        // TMA head coordinate (int32)
  if ((long long)N * d > (1ll << 31) / 2) return FA_ERR_UNSUPPORTED;  // per-head elements
  return FA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Workspace {
  float* delta;
  float* lse2;
  float* dq_acc;
  unsigned long long* counters;
  size_t bytes;
};

Workspace layout(void* base, int B, int H, int N, int d) {
  const size_t BH = (size_t)B * H, Np = ((size_t)N + 127) / 128 * 128;
  Workspace w;
  const size_t s_vec = align256(BH * Np * sizeof(float));
  const size_t s_acc = align256(BH * Np * d * sizeof(float));
  char* p = static_cast<char*>(base);
  w.delta = reinterpret_cast<float*>(p);
  w.lse2 = reinterpret_cast<float*>(p + s_vec);
  w.dq_acc = reinterpret_cast<float*>(p + 2 * s_vec);
  w.counters = reinterpret_cast<unsigned long long*>(p + 2 * s_vec + s_acc);  // 256 bytes, two used
  w.bytes = 2 * s_vec + s_acc + 256;
  return w;
}

fa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? FA_OK : FA_ERR_CUDA; }

}  // namespace

extern "C" {

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID: return "FA_ERR_INVALID: invalid argument";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: valid but unsupported problem size";
    case FA_ERR_CUDA: return "FA_ERR_CUDA: CUDA call or kernel launch failed";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: a device-side wait gave up";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE: workspace missing or too small";
  }
  return "unknown fa_status";
}

fa_status fa_fwd_ex(int dtype, const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                    int N, int d, float scale, int causal, const uint8_t* block_mask, long long block_mask_head_stride,
                    void* stream) {
  if (!valid_dtype(dtype)) return FA_ERR_INVALID;
  if (!mask_stride_ok(block_mask, block_mask_head_stride, N)) return FA_ERR_INVALID;
  const int f16 = dtype == FA_DTYPE_F16;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_INVALID;
  fa_status st = check_common(B, H, N, d, scale);
  if (st != FA_OK) return st;
  if (!(scale > 0.f)) return FA_ERR_UNSUPPORTED;  // see check_decode
  if (!get_encoder()) return FA_ERR_CUDA;
  const long long BH = (long long)B * H;
  alignas(64) CUtensorMap tq, tk, tv, to;
  if (!encode_bhnd(&tq, q, BH, N, d, f16, 128 / fa::fwd_rep(d, N)) || !encode_bhnd(&tk, k, BH, N, d, f16) ||
      !encode_bhnd(&tv, v, BH, N, d, f16) || !encode_bhnd(&to, o, BH, N, d, f16))
    return FA_ERR_CUDA;
  fa::FwdParams p;
  p.BH = BH;
  p.lse = lse;
  p.block_mask = block_mask;
  p.mask_stride = block_mask_head_stride;
  p.N = N;
  p.nb = (N + 127) / 128;  // the last tile may be partial: TMA zero-fills rows >= N
  p.Nk = N;
  p.nbk = p.nb;
  p.causal_off = 0;
  p.nsplit = 1;
  p.kv_per_split = p.nbk;
  p.Np = p.nb * 128;
  p.o_part = nullptr;
  p.lse_part = nullptr;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = kWaitLimitNs;
  p.f16 = f16;
  const int items = (p.nb + fa::fwd_tiles_per_cta(d, p.nb) - 1) / fa::fwd_tiles_per_cta(d, p.nb);
  p.order_group = fa::causal_group(p.causal, items, BH, fa::device_sm_count());
  return from_cuda(fa::launch_fwd(d, tq, tk, tv, to, p, BH, static_cast<cudaStream_t>(stream)));
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                 float scale, int causal, const uint8_t* block_mask, void* stream) {
  return fa_fwd_ex(FA_DTYPE_BF16, q, k, v, o, lse, B, H, N, d, scale, causal, block_mask, 0, stream);
}

// ------------------------------------------------------------------------- decode-shaped forward
namespace {

// Key-range splits for the decode forward: enough thread blocks for about three quarters of
// a wave (measured: with 128 query-tile pairs one piece streams K/V faster than three, the
// partial writes and the merge cost more than the idle SMs), but at least two key tiles per
// split; an explicit request is only capped by the number of key tiles.
int decode_splits(long long BH, int Nq, int Nk, int d, int requested) {
  const int nbk = (Nk + 127) / 128;
  if (requested > 0) return requested < nbk ? requested : nbk;
  const int nb = (Nq + 127) / 128;
  const int tiles_per_cta = fa::fwd_tiles_per_cta(d, nb);  // the forward kernel's query tiles per CTA
  const long long pairs = BH * ((nb + tiles_per_cta - 1) / tiles_per_cta);
  const long long target = 3ll * fa::device_sm_count() / 4;
  long long s = (target + pairs - 1) / pairs;
  const long long cap = nbk / 2 > 1 ? nbk / 2 : 1;
  if (s > cap) s = cap;
  return s < 1 ? 1 : (int)s;
}

struct DecodeWorkspace {
  float* o_part;
  float* lse_part;
  size_t bytes;
};

DecodeWorkspace decode_layout(void* base, long long BH, int Nq, int d, int nsplit) {
  const size_t Np = ((size_t)Nq + 127) / 128 * 128;
  const size_t s_o = align256((size_t)BH * nsplit * Np * d * sizeof(float));
  const size_t s_l = align256((size_t)BH * nsplit * Np * sizeof(float));
  DecodeWorkspace w;
  char* c = static_cast<char*>(base);
  w.o_part = reinterpret_cast<float*>(c);
  w.lse_part = reinterpret_cast<float*>(c + s_o);
  w.bytes = nsplit > 1 ? s_o + s_l : 0;
  return w;
}

fa_status check_decode(int B, int H, int Nq, int Nk, int d, float scale, int nsplit) {
  if (B <= 0 || H <= 0 || Nq <= 0 || Nk <= 0 || nsplit < 0 || !isfinite(scale)) return FA_ERR_INVALID;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  // The forward's softmax takes (max of a row's raw scores) x scale as its reference max, which
  // is the row max of the scaled scores only for scale >= 0 (a negative scale would let P grow
  // to 2^(row range) and overflow), and it masks scores as -inf before scaling, which scale = 0
  // would turn into NaN. So the scale must be positive, as in the backward.
  if (!(scale > 0.f)) return FA_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  if (BH > 0x7fffffffll) return FA_ERR_UNSUPPORTED;  // TMA head coordinate (int32)
  if ((long long)Nq * d > (1ll << 31) / 2 || (long long)Nk * d > (1ll << 31) / 2) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

}  // namespace

size_t fa_fwd_decode_workspace_bytes(int B, int H, int Nq, int Nk, int d, int nsplit) {
  if (check_decode(B, H, Nq, Nk, d, 1.0f, nsplit) != FA_OK) return 0;
  const long long BH = (long long)B * H;
  return decode_layout(nullptr, BH, Nq, d, decode_splits(BH, Nq, Nk, d, nsplit)).bytes;
}

fa_status fa_fwd_decode(int dtype, const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                        int Nq, int Nk, int d, float scale, int causal, int nsplit, void* workspace,
                        size_t workspace_bytes, void* stream) {
  if (!valid_dtype(dtype)) return FA_ERR_INVALID;
  const int f16 = dtype == FA_DTYPE_F16;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_INVALID;
  fa_status st = check_decode(B, H, Nq, Nk, d, scale, nsplit);
  if (st != FA_OK) return st;
  const long long BH = (long long)B * H;
  const int ns = decode_splits(BH, Nq, Nk, d, nsplit);
  DecodeWorkspace w = decode_layout(workspace, BH, Nq, d, ns);
  if (ns > 1 && (!workspace || !aligned16(workspace) || workspace_bytes < w.bytes)) return FA_ERR_WORKSPACE;
  if (!get_encoder()) return FA_ERR_CUDA;
  alignas(64) CUtensorMap tq, tk, tv, to;
  if (!encode_bhnd(&tq, q, BH, Nq, d, f16, 128 / fa::fwd_rep(d, Nq)) || !encode_bhnd(&tk, k, BH, Nk, d, f16) ||
      !encode_bhnd(&tv, v, BH, Nk, d, f16) || !encode_bhnd(&to, o, BH, Nq, d, f16))
    return FA_ERR_CUDA;
  fa::FwdParams p;
  p.BH = BH;
  p.lse = lse;
  p.block_mask = nullptr;
  p.mask_stride = 0;
  p.N = Nq;
  p.nb = (Nq + 127) / 128;
  p.Nk = Nk;
  p.nbk = (Nk + 127) / 128;
  p.causal_off = Nk - Nq;  // bottom-right alignment: the last query sees every key
  p.nsplit = ns;
  p.kv_per_split = (p.nbk + ns - 1) / ns;
  p.Np = p.nb * 128;
  p.o_part = ns > 1 ? w.o_part : nullptr;
  p.lse_part = ns > 1 ? w.lse_part : nullptr;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = kWaitLimitNs;
  p.f16 = f16;
  const int tpc = fa::fwd_tiles_per_cta(d, p.nb);
  p.order_group = fa::causal_group(p.causal, (p.nb + tpc - 1) / tpc * ns, BH, fa::device_sm_count());
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = fa::launch_fwd(d, tq, tk, tv, to, p, BH, s);
  if (e != cudaSuccess || ns == 1) return from_cuda(e);
  fa::FwdMergeParams m;
  m.o_part = w.o_part;
  m.lse_part = w.lse_part;
  m.o = static_cast<uint16_t*>(o);
  m.lse = lse;
  m.rows = BH * Nq;
  m.N = Nq;
  m.Np = p.Np;
  m.nsplit = ns;
  m.D = d;
  m.f16 = f16;
  return from_cuda(fa::launch_fwd_merge(m, s));
}

size_t fa_bwd_workspace_bytes(int B, int H, int N, int d) {
  if (check_common(B, H, N, d, 1.0f) != FA_OK) return 0;
  return layout(nullptr, B, H, N, d).bytes;
}

}  // extern "C"

// ------------------------------------------------------------------------- backward plans
// Each stage of the backward is validated and prepared (parameter block, tensor maps) by a
// plan function that enqueues nothing; the entry points launch only after every plan they
// need has succeeded, so an argument error never leaves a stage half-run.
namespace {

// Shapes of one backward problem: N_q query rows and N_k keys per head (N_q = N_k = N for
// the square calls), causal alignment offset (key j visible to query i iff j <= i + off).
struct BwdShape {
  int B, H, Nq, Nk, d;
  int causal_off;
};

fa_status check_bwd_shape(const BwdShape& sh, float scale) {
  fa_status st = check_common(sh.B, sh.H, sh.Nq, sh.d, scale);
  if (st != FA_OK) return st;
  st = check_common(sh.B, sh.H, sh.Nk, sh.d, scale);
  if (st != FA_OK) return st;
  if (!(scale > 0.f)) return FA_ERR_UNSUPPORTED;  // the backward folds log2(scale) into P
  return FA_OK;
}

fa_status plan_bwd_pre(int dtype, const void* o, const void* dO, const float* lse, const BwdShape& sh, float scale,
                       void* workspace, size_t workspace_bytes, fa::BwdPreParams* p) {
  if (!valid_dtype(dtype)) return FA_ERR_INVALID;
  if (!o || !dO || !lse) return FA_ERR_INVALID;
  if (!aligned16(o) || !aligned16(dO) || !aligned16(lse)) return FA_ERR_INVALID;
  fa_status st = check_bwd_shape(sh, scale);
  if (st != FA_OK) return st;
  if (!workspace || !aligned16(workspace)) return FA_ERR_WORKSPACE;
  Workspace w = layout(workspace, sh.B, sh.H, sh.Nq, sh.d);
  if (workspace_bytes < w.bytes) return FA_ERR_WORKSPACE;
  p->o = static_cast<const uint16_t*>(o);
  p->dout = static_cast<const uint16_t*>(dO);
  p->lse = lse;
  p->delta = w.delta;
  p->lse2 = w.lse2;
  p->dq_acc = w.dq_acc;
  p->counters = w.counters;
  p->rows = (long long)sh.B * sh.H * sh.Nq;
  p->N = sh.Nq;
  p->Np = (sh.Nq + 127) / 128 * 128;
  p->D = sh.d;
  p->log2_scale = log2f(scale);
  p->f16 = dtype == FA_DTYPE_F16;
  return FA_OK;
}

struct BwdMainPlan {
  alignas(64) CUtensorMap tq, tk, tv, tdo, tdk, tdv, tdqa;
  fa::BwdParams p;
  long long BH;
  int d;
};

fa_status plan_bwd_main(int dtype, const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv,
                        const BwdShape& sh, float scale, int causal, const uint8_t* block_mask,
                        long long block_mask_head_stride, void* workspace, size_t workspace_bytes,
                        BwdMainPlan* m) {
  if (!valid_dtype(dtype)) return FA_ERR_INVALID;
  if (block_mask != nullptr && sh.Nq != sh.Nk) return FA_ERR_INVALID;  // masks are square
  if (!mask_stride_ok(block_mask, block_mask_head_stride, sh.Nq)) return FA_ERR_INVALID;
  const int f16 = dtype == FA_DTYPE_F16;
  if (!q || !k || !v || !dO || !dk || !dv) return FA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_INVALID;
  fa_status st = check_bwd_shape(sh, scale);
  if (st != FA_OK) return st;
  const long long BH = (long long)sh.B * sh.H;
  const int Np = (sh.Nq + 127) / 128 * 128;
  if (BH * Np > 0x7fffffffll) return FA_ERR_UNSUPPORTED;  // TMA row coordinate of the dQ accumulator
  if (!workspace || !aligned16(workspace)) return FA_ERR_WORKSPACE;
  Workspace w = layout(workspace, sh.B, sh.H, sh.Nq, sh.d);
  if (workspace_bytes < w.bytes) return FA_ERR_WORKSPACE;
  if (!get_encoder()) return FA_ERR_CUDA;
  if (!encode_bhnd(&m->tq, q, BH, sh.Nq, sh.d, f16) || !encode_bhnd(&m->tk, k, BH, sh.Nk, sh.d, f16) ||
      !encode_bhnd(&m->tv, v, BH, sh.Nk, sh.d, f16) || !encode_bhnd(&m->tdo, dO, BH, sh.Nq, sh.d, f16) ||
      !encode_bhnd(&m->tdk, dk, BH, sh.Nk, sh.d, f16) || !encode_bhnd(&m->tdv, dv, BH, sh.Nk, sh.d, f16) ||
      !encode_dq_acc(&m->tdqa, w.dq_acc, BH * Np, sh.d))
    return FA_ERR_CUDA;
  fa::BwdParams& p = m->p;
  p.BH = BH;
  p.delta = w.delta;
  p.lse2 = w.lse2;
  p.dq_acc = w.dq_acc;
  p.counters = w.counters;
  p.block_mask = block_mask;
  p.mask_stride = block_mask_head_stride;
  p.N = sh.Nq;
  p.Np = Np;
  p.nb = (sh.Nq + 127) / 128;
  p.Nk = sh.Nk;
  p.nbk = (sh.Nk + 127) / 128;
  p.causal = causal ? 1 : 0;
  p.causal_off = sh.causal_off;
  p.order_group = fa::causal_group(p.causal, p.nbk * (sh.d == 256 ? 2 : 1), BH, fa::device_sm_count());
  p.inv_scale = 1.0f / scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = kWaitLimitNs;
  p.f16 = f16;
  // Persistent CTAs (one per SM, each taking (head, key tile) items from a counter in the
  // workspace, the next item's loads overlapping the previous one's epilogue) for d <= 128 (d =
  // 256 runs two CTAs per key tile, one per half of d). Measured (backward kernel alone, against
  // one CTA per item): N = 512 d = 128 +10-11%, BERT-large shape +12%, N = 1024 d = 64 +4%, N = 2048
  // +1%, N = 4096 d = 64 +2%, N = 4096 and 16384 at d = 128 and causal N = 4096 unchanged.
  p.persist = (sh.d != 256) ? 1 : 0;
  m->BH = BH;
  m->d = sh.d;
  return FA_OK;
}

cudaError_t launch_plan(const BwdMainPlan& m, cudaStream_t s) {
  return fa::launch_bwd_main(m.d, m.tq, m.tk, m.tv, m.tdo, m.tdk, m.tdv, m.tdqa, m.p, m.BH, s);
}

fa_status plan_dq_finish(int dtype, void* dq, const BwdShape& sh, void* workspace, size_t workspace_bytes,
                         fa::DqFinishParams* p) {
  if (!valid_dtype(dtype)) return FA_ERR_INVALID;
  if (!dq || !aligned16(dq)) return FA_ERR_INVALID;
  fa_status st = check_bwd_shape(sh, 1.0f);
  if (st != FA_OK) return st;
  if (!workspace || !aligned16(workspace)) return FA_ERR_WORKSPACE;
  Workspace w = layout(workspace, sh.B, sh.H, sh.Nq, sh.d);
  if (workspace_bytes < w.bytes) return FA_ERR_WORKSPACE;
  p->dq_acc = w.dq_acc;
  p->dq = static_cast<uint16_t*>(dq);
  p->rows = (long long)sh.B * sh.H * sh.Nq;
  p->N = sh.Nq;
  p->Np = (sh.Nq + 127) / 128 * 128;
  p->D = sh.d;
  p->scale = 1.0f;  // the accumulated dQ already carries the scale (the main kernel folds it into P)
  p->f16 = dtype == FA_DTYPE_F16;
  return FA_OK;
}

// Null and alignment checks of every tensor pointer of a whole backward call (pure host
// logic, no CUDA call), so that a bad pointer of any stage is refused first.
fa_status bwd_check_pointers(const void* q, const void* k, const void* v, const void* o, const void* dO,
                             const float* lse, const void* dq, const void* dk, const void* dv) {
  const void* ptrs[9] = {q, k, v, o, dO, lse, dq, dk, dv};
  for (const void* x : ptrs)
    if (x == nullptr || !aligned16(x)) return FA_ERR_INVALID;
  return FA_OK;
}

// The whole backward: every stage planned first, then the three launches.
fa_status bwd_all(int dtype, const void* q, const void* k, const void* v, const void* o, const void* dO,
                  const float* lse, void* dq, void* dk, void* dv, const BwdShape& sh, float scale, int causal,
                  const uint8_t* block_mask, long long block_mask_head_stride, void* workspace,
                  size_t workspace_bytes, void* stream) {
  fa_status st = bwd_check_pointers(q, k, v, o, dO, lse, dq, dk, dv);
  if (st != FA_OK) return st;
  fa::BwdPreParams pre;
  st = plan_bwd_pre(dtype, o, dO, lse, sh, scale, workspace, workspace_bytes, &pre);
  if (st != FA_OK) return st;
  BwdMainPlan m;
  st = plan_bwd_main(dtype, q, k, v, dO, dk, dv, sh, scale, causal, block_mask, block_mask_head_stride, workspace,
                     workspace_bytes, &m);
  if (st != FA_OK) return st;
  fa::DqFinishParams fin;
  st = plan_dq_finish(dtype, dq, sh, workspace, workspace_bytes, &fin);
  if (st != FA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = fa::launch_bwd_pre(pre, s);
  if (e == cudaSuccess) e = launch_plan(m, s);
  if (e == cudaSuccess) e = fa::launch_dq_finish(fin, s);
  return from_cuda(e);
}

BwdShape square(int B, int H, int N, int d) { return BwdShape{B, H, N, N, d, 0}; }

}  // namespace

extern "C" {

fa_status fa_bwd_preprocess_ex(int dtype, const void* o, const void* dO, const float* lse, int B, int H, int N,
                               int d, float scale, void* workspace, size_t workspace_bytes, void* stream) {
  fa::BwdPreParams p;
  fa_status st = plan_bwd_pre(dtype, o, dO, lse, square(B, H, N, d), scale, workspace, workspace_bytes, &p);
  if (st != FA_OK) return st;
  return from_cuda(fa::launch_bwd_pre(p, static_cast<cudaStream_t>(stream)));
}

fa_status fa_bwd_preprocess(const void* o, const void* dO, const float* lse, int B, int H, int N, int d,
                            float scale, void* workspace, size_t workspace_bytes, void* stream) {
  return fa_bwd_preprocess_ex(FA_DTYPE_BF16, o, dO, lse, B, H, N, d, scale, workspace, workspace_bytes, stream);
}

fa_status fa_bwd_main_ex(int dtype, const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv,
                         int B, int H, int N, int d, float scale, int causal, const uint8_t* block_mask,
                         long long block_mask_head_stride, void* workspace, size_t workspace_bytes, void* stream) {
  BwdMainPlan m;
  fa_status st = plan_bwd_main(dtype, q, k, v, dO, dk, dv, square(B, H, N, d), scale, causal, block_mask,
                               block_mask_head_stride, workspace, workspace_bytes, &m);
  if (st != FA_OK) return st;
  return from_cuda(launch_plan(m, static_cast<cudaStream_t>(stream)));
}

fa_status fa_bwd_main(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv, int B,
                      int H, int N, int d, float scale, int causal, const uint8_t* block_mask, void* workspace,
                      size_t workspace_bytes, void* stream) {
  return fa_bwd_main_ex(FA_DTYPE_BF16, q, k, v, dO, dk, dv, B, H, N, d, scale, causal, block_mask, 0, workspace,
                        workspace_bytes, stream);
}

fa_status fa_bwd_dq_finish_ex(int dtype, void* dq, int B, int H, int N, int d, void* workspace,
                              size_t workspace_bytes, void* stream) {
  fa::DqFinishParams p;
  fa_status st = plan_dq_finish(dtype, dq, square(B, H, N, d), workspace, workspace_bytes, &p);
  if (st != FA_OK) return st;
  return from_cuda(fa::launch_dq_finish(p, static_cast<cudaStream_t>(stream)));
}

fa_status fa_bwd_dq_finish(void* dq, int B, int H, int N, int d, void* workspace, size_t workspace_bytes,
                           void* stream) {
  return fa_bwd_dq_finish_ex(FA_DTYPE_BF16, dq, B, H, N, d, workspace, workspace_bytes, stream);
}

fa_status fa_bwd_ex(int dtype, const void* q, const void* k, const void* v, const void* o, const void* dO,
                    const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale,
                    int causal, const uint8_t* block_mask, long long block_mask_head_stride, void* workspace,
                    size_t workspace_bytes, void* stream) {
  return bwd_all(dtype, q, k, v, o, dO, lse, dq, dk, dv, square(B, H, N, d), scale, causal, block_mask,
                 block_mask_head_stride, workspace, workspace_bytes, stream);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                 void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal,
                 const uint8_t* block_mask, void* workspace, size_t workspace_bytes, void* stream) {
  return fa_bwd_ex(FA_DTYPE_BF16, q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal, block_mask, 0,
                   workspace, workspace_bytes, stream);
}

fa_status fa_bwd_qk(int dtype, const void* q, const void* k, const void* v, const void* o, const void* dO,
                    const float* lse, void* dq, void* dk, void* dv, int B, int H, int Nq, int Nk, int d, float scale,
                    int causal, void* workspace, size_t workspace_bytes, void* stream) {
  const BwdShape sh{B, H, Nq, Nk, d, Nk - Nq};  // bottom-right alignment, as fa_fwd_decode
  return bwd_all(dtype, q, k, v, o, dO, lse, dq, dk, dv, sh, scale, causal, nullptr, 0, workspace, workspace_bytes,
                 stream);
}

fa_status fa_last_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return FA_ERR_CUDA;
  int word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, fa::g_fa_device_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (word != 0) {
    if (cudaMemcpyToSymbol(fa::g_fa_device_status, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
    return FA_ERR_TIMEOUT;
  }
  return FA_OK;
}

}  // extern "C"
