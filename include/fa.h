/*
 * fa.h -- C ABI of libfa.so: exact softmax attention on NVIDIA B200 (sm_100a).
 *
 * The library computes O = softmax(scale * Q K^T) V with the N x N score and probability
 * matrices never written to memory (tiling + online softmax), saves one log-sum-exp per
 * query row, and computes dQ, dK, dV by recomputing the probabilities from that
 * statistic.
 *
 * Sources (cited by page and section):
 *   [P1] "FlashAttention-2 的前世今生" overview, jishu.shishitao.com/detail/60083.html
 *   [P2] "Attention 为什么慢" / Flash Attention explainer, ds6.com.cn/news/67428.html
 *   [P3] FlashAttention V1 lecture summary, spark.aweffr.cn/summary/0684ec99-...
 *
 * Conventions shared by every call:
 *  - Tensors q, k, v, o, dO, dq, dk, dv are bf16, contiguous [B][H][N][d], d fastest.
 *    The problem statement of [P3] §2.1/§2.2 (Q, K, V of N x d per head), batched over B
 *    and H as in [P1] §主要操作 ("parallelise over batch and heads").
 *  - lse is fp32 [B][H][N]: LSE_i = ln sum_j exp(scale * q_i . k_j) over the allowed keys,
 *    natural log, scale included -- the single per-row statistic FA2 keeps for the
 *    backward ([P1] §主要操作, backward pass). A row with no allowed key gets -inf and O=0.
 *  - causal != 0 allows key j for query i only if j <= i (top-left aligned; [P1] benchmark
 *    setting "with or without causal mask").
 *  - block_mask (nullable) is a device array of ceil(N/128) x ceil(N/128) uint8, row-major,
 *    shared by all (b, h); block (I, J) != 0 lets queries 128I..128I+127 see keys
 *    128J..128J+127 ([P1] §Block-Sparse FlashAttention). Tiles that are off are never
 *    loaded or computed. causal and block_mask combine (AND).
 *  - All pointers are device memory owned by the caller. The library allocates no device
 *    memory apart from one static device status word and the fixed scratch array that
 *    fa_bwd_noalloc uses.
 *  - Every pointer must be 16-byte aligned. d must be 64, 128 or 256 (at 256 the forward runs
 *    one 128-row query tile per thread block and the backward two thread blocks per key tile,
 *    one per 128-column half of d, because the dK and dV accumulators of a whole tile would not
 *    fit tensor memory together). N is any positive length;
 *    a partial last 128-row tile is handled inside the kernels (rows and keys beyond N take no
 *    part and are never written).
 *  - B*H may be any positive count up to 2^31 - 1 (heads beyond 65535 are spread over two
 *    grid dimensions); the backward also needs B*H*ceil(N/128)*128 < 2^31.
 *  - stream is a cudaStream_t (NULL = legacy default stream). All calls are asynchronous
 *    on it; argument errors are reported synchronously, before anything is enqueued: a
 *    call that runs several kernels (fa_bwd and its variants) checks every argument of
 *    every stage before the first launch.
 *  - Not re-entrant on the same output buffers; distinct calls on distinct buffers may run
 *    concurrently on different streams.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID = 1,     /* null/misaligned pointer, non-positive size, non-finite scale */
  FA_ERR_UNSUPPORTED = 2, /* valid but not implemented: d not in {64,128,256}; scale <= 0 */
  FA_ERR_CUDA = 3,        /* a CUDA runtime/driver call or a kernel launch failed */
  FA_ERR_TIMEOUT = 4,     /* a device-side bounded wait gave up (see fa_last_device_status) */
  FA_ERR_WORKSPACE = 5    /* workspace pointer null or smaller than fa_bwd_workspace_bytes */
} fa_status;

/* Element type of q, k, v, o, dO, dq, dk, dv for the *_ex entry points. */
typedef enum {
  FA_DTYPE_BF16 = 0, /* bfloat16: the type of every untyped entry point */
  FA_DTYPE_F16 = 1   /* IEEE half; the kernels still compute S, P, O and gradients in fp32 */
} fa_dtype;

/*
 * Forward pass ([P3] §3.1-§3.3 tiling + online softmax; FA2 loop order of [P1] §主要操作:
 * each thread block owns query row-blocks and loops over key/value column-blocks).
 *   in : q, k, v       bf16 [B][H][N][d]
 *   out: o             bf16 [B][H][N][d]
 *        lse           fp32 [B][H][N]
 *   scale: multiplies q.k (typically 1/sqrt(d)); must be finite and > 0, else
 *          FA_ERR_UNSUPPORTED: the softmax's reference max is the largest raw score times the
 *          scale (the largest scaled score only for a positive scale), and masked scores are
 *          -inf before scaling (scale 0 would make them NaN).
 * One kernel launch.
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int N, int d, float scale, int causal, const uint8_t* block_mask, void* stream);

/*
 * Bytes of caller-provided device workspace fa_bwd needs: fp32 D [B][H][Np], fp32 scaled
 * LSE [B][H][Np] and the fp32 dQ accumulator [B][H][Np][d] (Np = N rounded up to 128),
 * each 256-byte aligned, then 256 bytes of work-scheduling counters. Returns 0 for sizes
 * fa_bwd would reject.
 */
size_t fa_bwd_workspace_bytes(int B, int H, int N, int d);

/*
 * Backward pass by recomputation ([P3] §4.2; [P1] §主要操作, backward: only the LSE is
 * kept; column-block workers; dQ combined across thread blocks).
 *   in : q, k, v, o, dO  bf16 [B][H][N][d];  lse fp32 [B][H][N] from fa_fwd
 *   out: dq, dk, dv      bf16 [B][H][N][d]
 *   workspace: device buffer of at least fa_bwd_workspace_bytes(B,H,N,d) bytes; its
 *              contents on entry are ignored and on exit unspecified.
 *   scale: as passed to fa_fwd, and > 0: the kernels fold log2(scale) into the recomputed
 *          probabilities (FA_ERR_UNSUPPORTED otherwise).
 * Equivalent to fa_bwd_preprocess + fa_bwd_main + fa_bwd_dq_finish on the same workspace.
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                 const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                 float scale, int causal, const uint8_t* block_mask, void* workspace,
                 size_t workspace_bytes, void* stream);

/*
 * The three stages of fa_bwd, exposed so each kernel can be launched (and timed) alone.
 * fa_bwd_preprocess: D_i = sum_t dO_it * O_it (the row sums of dP o P, from the softmax
 *   Jacobian [P3] §4.1), the scaled LSE, and zeroes the fp32 dQ accumulator and the
 *   scheduling counters. HBM-bound.
 * fa_bwd_main: per key tile, recompute S and P, accumulate dK and dV on chip, write dk and
 *   dv (bf16), and add each tile's dQ contribution into the fp32 accumulator.
 * fa_bwd_dq_finish: dq = bf16(accumulator).
 * They must be called in this order on one stream with the same workspace, sizes and scale.
 */
fa_status fa_bwd_preprocess(const void* o, const void* dO, const float* lse, int B, int H, int N,
                            int d, float scale, void* workspace, size_t workspace_bytes,
                            void* stream);
fa_status fa_bwd_main(const void* q, const void* k, const void* v, const void* dO, void* dk,
                      void* dv, int B, int H, int N, int d, float scale, int causal,
                      const uint8_t* block_mask, void* workspace, size_t workspace_bytes,
                      void* stream);
fa_status fa_bwd_dq_finish(void* dq, int B, int H, int N, int d, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * Backward pass without a caller workspace, for callers that cannot allocate device memory
 * (hosts that own every allocation and forbid allocating from their execution callbacks,
 * real-time loops that must not allocate once started). The source pages have no
 * counterpart: this is a deployment convenience, not part of the method.
 * Same arguments, outputs and numerics as fa_bwd, minus the workspace. The workspace comes
 * from a fixed array of FA_NOALLOC_SCRATCH_BYTES in the library's device memory, reserved
 * on every GPU that loads the library until the process exits. Problems whose
 * fa_bwd_workspace_bytes exceed it return FA_ERR_WORKSPACE (about (d+2)*4 bytes per query
 * row: B*H*N up to ~65k rows at d = 256, ~129k at d = 128, ~254k at d = 64). Allocates nothing.
 * The first call on each device looks up the array's device address (cudaGetSymbolAddress)
 * with that device current; make that first call before any stream capture. All calls share
 * the one array: calls whose kernels overlap on the GPU (different streams, no ordering)
 * race on it and give wrong results. Calls ordered on one stream are safe: each call
 * re-initialises everything it reads from the array.
 */
/*
 * Extended forms of the calls above: the 16-bit element type and per-(b, h) block masks.
 *   dtype: an fa_dtype value (anything else returns FA_ERR_INVALID); the tensor operands of
 *          one call all have that element type (lse and the workspace stay fp32).
 *   block_mask_head_stride: 0 = one ceil(N/128)^2 mask shared by every (b, h), as in the
 *          calls above; otherwise the mask of head (b, h) starts at
 *          block_mask + (b*H + h) * block_mask_head_stride (at least ceil(N/128)^2, else
 *          FA_ERR_INVALID), so B*H masks can give every head its own sparsity pattern
 *          ([P1] §Block-Sparse FlashAttention: the work scales with the blocks that are on).
 *          The forward and fa_bwd_main of one problem must see the same masks.
 * Arguments, layouts, workspace and errors are otherwise those of the plain calls.
 * The pages discuss fp16's narrow range for exp ([P2] §时间复杂度): here exponentials,
 * the softmax statistics and every accumulator are fp32 in both types, and P (bounded by
 * 2^8 by the reference-max rule) is the only 16-bit intermediate besides the inputs.
 * fa_bwd_noalloc is bf16 with a shared mask only.
 */
fa_status fa_fwd_ex(int dtype, const void* q, const void* k, const void* v, void* o, float* lse,
                    int B, int H, int N, int d, float scale, int causal,
                    const uint8_t* block_mask, long long block_mask_head_stride, void* stream);
fa_status fa_bwd_ex(int dtype, const void* q, const void* k, const void* v, const void* o,
                    const void* dO, const float* lse, void* dq, void* dk, void* dv, int B, int H,
                    int N, int d, float scale, int causal, const uint8_t* block_mask,
                    long long block_mask_head_stride, void* workspace, size_t workspace_bytes,
                    void* stream);
fa_status fa_bwd_preprocess_ex(int dtype, const void* o, const void* dO, const float* lse, int B,
                               int H, int N, int d, float scale, void* workspace,
                               size_t workspace_bytes, void* stream);
fa_status fa_bwd_main_ex(int dtype, const void* q, const void* k, const void* v, const void* dO,
                         void* dk, void* dv, int B, int H, int N, int d, float scale, int causal,
                         const uint8_t* block_mask, long long block_mask_head_stride,
                         void* workspace, size_t workspace_bytes, void* stream);
fa_status fa_bwd_dq_finish_ex(int dtype, void* dq, int B, int H, int N, int d, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * Decode-shaped forward: Nq query rows against Nk keys per head (typically few queries and a
 * long key/value history), for inference; there is no matching backward. The key range is
 * cut into `nsplit` pieces processed by separate thread blocks, each producing its own
 * normalised output and log-sum-exp, which a second kernel merges with the online
 * normaliser's combine rule ([P2] §时间复杂度; [P3] §3.2): LSE = log sum_s exp(LSE_s),
 * O = sum_s exp(LSE_s - LSE) O_s. (The pages mention inference use only in passing; the
 * split is ours.)
 *   in : q [B][H][Nq][d], k, v [B][H][Nk][d] (dtype as for fa_fwd_ex)
 *   out: o [B][H][Nq][d], lse [B][H][Nq] (natural log, scale included)
 *   causal: bottom-right alignment, the last query sees every key: key j is visible to
 *           query i iff j <= i + Nk - Nq (j <= i when Nq = Nk). Rows that see no key get
 *           O = 0 and LSE = -inf. No block mask.
 *   nsplit: key-range pieces; 0 = chosen from the problem size and SM count (about three
 *           quarters of a wave of thread blocks, at least two 128-key tiles per piece);
 *           capped at ceil(Nk / 128). With one piece the output is written directly.
 *   workspace: fa_fwd_decode_workspace_bytes(B, H, Nq, Nk, d, nsplit) bytes (0 when the
 *           problem runs as one piece; pass the same nsplit to both calls), caller-owned,
 *           contents ignored on entry.
 * Errors as for fa_fwd; a too-small workspace returns FA_ERR_WORKSPACE.
 */
size_t fa_fwd_decode_workspace_bytes(int B, int H, int Nq, int Nk, int d, int nsplit);
fa_status fa_fwd_decode(int dtype, const void* q, const void* k, const void* v, void* o,
                        float* lse, int B, int H, int Nq, int Nk, int d, float scale, int causal,
                        int nsplit, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward pass for N_q query rows against N_k keys per head: the gradient of the forward that
 * fa_fwd_decode computes (the problem statement of [P3] §2.1/§2.2 gives Q and K/V their own
 * lengths), by the same recomputation as fa_bwd ([P3] §4.2; [P1] §主要操作, backward).
 *   in : q, o, dO  [B][H][Nq][d];  k, v  [B][H][Nk][d]  (dtype as for fa_bwd_ex)
 *        lse       fp32 [B][H][Nq] from fa_fwd_decode with the same causal flag and scale
 *   out: dq [B][H][Nq][d];  dk, dv [B][H][Nk][d]
 *   causal: bottom-right alignment as in fa_fwd_decode (key j visible to query i iff
 *           j <= i + Nk - Nq). Rows that see no key (Nq > Nk) have LSE = -inf and O = 0;
 *           they contribute nothing and get dq = 0. No block mask.
 *   workspace: fa_bwd_workspace_bytes(B, H, Nq, d) bytes (it depends on the query rows only).
 * Errors as for fa_bwd. With Nq = Nk it computes exactly what fa_bwd_ex computes.
 */
fa_status fa_bwd_qk(int dtype, const void* q, const void* k, const void* v, const void* o,
                    const void* dO, const float* lse, void* dq, void* dk, void* dv, int B, int H,
                    int Nq, int Nk, int d, float scale, int causal, void* workspace,
                    size_t workspace_bytes, void* stream);

#define FA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                         const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                         float scale, int causal, const uint8_t* block_mask, void* stream);

/*
 * Synchronises `stream`, then reports and clears the device status word: FA_ERR_TIMEOUT if
 * any kernel since the last call gave up on a bounded wait (its outputs are then invalid),
 * FA_ERR_CUDA if the stream reports an error, FA_OK otherwise.
 */
fa_status fa_last_device_status(void* stream);

/*
 * Failure-detection self-test (no counterpart on the pages; it tests the library's own
 * device-side wait limits). Enqueues one tiny kernel whose single thread waits, bounded by
 * limit_us microseconds (1 .. 1,000,000), on a barrier that nothing arrives at. The wait
 * gives up exactly as a stuck attention kernel would: it records a code in the device
 * status word and returns, leaving the context usable. A following fa_last_device_status
 * reports FA_ERR_TIMEOUT. Returns FA_ERR_INVALID for an out-of-range limit.
 */
fa_status fa_selftest_wait_timeout(unsigned int limit_us, void* stream);

/*
 * Accuracy self-test of the library's own FMA-pipe exp2 (no counterpart on the pages): a
 * compile-time option of the softmax kernels, off in the shipped build, kept testable. For n
 * device fp32 inputs x, writes the packed polynomial's 2^x to y_poly and the special-function
 * unit's ex2.approx to y_sfu (device buffers of n floats). Meant for inputs in [-125, 127]
 * (softmax exponents are <= 8). Returns FA_ERR_INVALID for n < 0 or null buffers.
 */
fa_status fa_selftest_ex2(const float* x, float* y_poly, float* y_sfu, int n, void* stream);

/* Static, human-readable name of a status code. Never NULL. */
const char* fa_status_string(fa_status status);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
