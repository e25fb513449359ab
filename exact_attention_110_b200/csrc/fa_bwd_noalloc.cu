// fa_bwd_noalloc: the backward pass for callers that cannot allocate device memory.
//
// fa_bwd needs a caller-provided workspace (the D vector, the scaled LSE and the fp32 dQ
// accumulator). Some callers cannot obtain one: code running inside a host framework that
// owns every device allocation and forbids allocating from its execution callbacks (plugin
// interfaces of inference runtimes, for example), and real-time loops that must not allocate
// once they have started. This entry point gives them the same computation with the
// workspace taken from a fixed array in the library's own device memory.
//
// The array is a file-scope __device__ object: every GPU that loads the library holds it
// until the process exits. Host code must never pass the array's name to a kernel -- on the
// host that name is only a stand-in symbol -- so its device address is looked up once per
// device with cudaGetSymbolAddress and cached.
#include <mutex>

#include "fa.h"  // include/ is on the include path

static __device__ __align__(256) unsigned char g_fa_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::once_flag g_scratch_once[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up on first use).
void* scratch_for_current_device(fa_status* st) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *st = FA_ERR_CUDA;
    return nullptr;
  }
  std::call_once(g_scratch_once[dev], [dev] {
    void* p = nullptr;
    g_scratch_err[dev] = cudaGetSymbolAddress(&p, g_fa_noalloc_scratch);
    if (g_scratch_err[dev] == cudaSuccess) g_scratch_addr[dev] = p;
  });
  if (g_scratch_err[dev] != cudaSuccess || g_scratch_addr[dev] == nullptr) {
    *st = FA_ERR_CUDA;
    return nullptr;
  }
  *st = FA_OK;
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                                    const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                                    float scale, int causal, const uint8_t* block_mask, void* stream) {
  // Pointer errors first, before the scratch array's address is looked up (a CUDA call).
  const fa_status pst = bwd_check_pointers(q, k, v, o, dO, lse, dq, dk, dv);
  if (pst != FA_OK) return pst;
  const size_t need = fa_bwd_workspace_bytes(B, H, N, d);
  if (need == 0) {  // sizes fa_bwd rejects: let it report the precise reason
    return fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal, block_mask, nullptr, 0, stream);
  }
  if (need > (size_t)FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_WORKSPACE;
  fa_status st;
  void* scratch = scratch_for_current_device(&st);
  if (st != FA_OK) return st;
  // fa_bwd's first kernel zeroes the dQ accumulator and overwrites the rest of the
  // workspace, so whatever an earlier call left in the array does not leak into this one.
  return fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal, block_mask, scratch,
                (size_t)FA_NOALLOC_SCRATCH_BYTES, stream);
}
