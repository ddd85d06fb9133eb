/*
 * fa.h -- C ABI of libfa: exact scaled-dot-product attention on NVIDIA B200 (sm_100a),
 * forward and backward, computed tile by tile so that the N x N score matrix never reaches HBM.
 *
 * The operation ("Attention optimisation: FlashAttention and sparse attention", mdooai Ch.04,
 * sections "core formula" and "formula key points", and its sparse-masking paragraph):
 *     S_ij = scale * q_i . k_j            (scale is 1/sqrt(d) in the usual setting)
 *     S_ij = -inf for keys j outside the allowed set of row i
 *     A    = softmax of each row of S     (each row of A sums to 1)
 *     O    = A V
 * computed exactly -- not an approximation -- with the IO-aware tiling of "FlashAttention:
 * Fast and Memory-Efficient Exact Attention with IO-Awareness" (ai-paper-library summary of
 * arXiv 2205.14135): tiles of Q, K, V are staged on chip, partial softmax statistics are kept
 * on chip, and only O and the per-row log-sum-exp go back to HBM.  The backward pass
 * recomputes the scores from Q, K, V and that log-sum-exp.
 *
 * Conventions shared by every entry point
 *   Layout     q, k, v, o, dO, dq, dk, dv are contiguous [B][H][N][d] row-major (d innermost);
 *              lse is [B][H][N]. One (b, h) pair is one independent attention problem.
 *   Masks      the allowed set of row i is the AND of
 *                causal != 0        : j <= i (square self-attention, lower triangle);
 *                kv_len != NULL     : j < kv_len[b] (key padding; device int32 [B]);
 *                block_mask != NULL : block_mask[i/128][j/128] != 0 (device uint8
 *                                     [ceil(N/128)][ceil(N/128)], shared by every (b, h)).
 *              A row with no allowed key gets O = 0, lse = -inf and no gradient.
 *   lse        natural-log log-sum-exp of the scaled, masked logits of the row.
 *   Memory     every pointer is device memory owned by the caller; the library allocates
 *              nothing and keeps no pointer after the call returns.
 *   Execution  asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream); the
 *              host never waits, so results are ready once the stream reaches this point.
 *   Errors     a negative fa_status is returned without launching anything when an argument
 *              is rejected; fa_get_last_error() then describes it.  A CUDA launch failure
 *              returns FA_ERR_CUDA.  Device-side waits are bounded: a wait that gives up
 *              records a code that fa_device_status() reports (FA_ERR_TIMEOUT).
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { FA_BF16 = 0, FA_F32 = 1 } fa_dtype;

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID = -1,     /* null pointer, non-positive size, bad scale, unknown dtype   */
  FA_ERR_UNSUPPORTED = -2, /* head dimension or dtype the library has no kernel for       */
  FA_ERR_ALIGN = -3,       /* a tensor pointer is not 16-byte aligned (TMA requirement)   */
  FA_ERR_CUDA = -4,        /* a CUDA call or kernel launch failed                         */
  FA_ERR_TIMEOUT = -5,     /* a device-side bounded wait gave up (see fa_device_status)  */
  FA_ERR_WORKSPACE = -6    /* workspace missing, misaligned or smaller than required      */
} fa_status;

/*
 * fa_fwd -- forward pass: O = softmax(scale * Q K^T, masked) V and lse.
 *   dtype FA_BF16: q, k, v, o are bf16, d in {64, 128}; tensor-core (tcgen05) kernel with
 *                  TMA-fed tiles and an online softmax; fp32 accumulation.
 *   dtype FA_F32 : q, k, v, o are fp32, 1 <= d <= 128; CUDA-core fp32 kernel.
 *   scale must be finite and > 0.  N >= 1, B >= 1, H >= 1.
 *   Pointers q, k, v, o, lse must be 16-byte aligned.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
           int N, int d, float scale, int causal, const uint8_t* block_mask,
           const int32_t* kv_len, int dtype, void* stream);

/* Bytes of device workspace fa_bwd needs: log2-scaled lse and Dvec ([B][H][ceil128(N)] fp32
 * each) and the fp32 dQ accumulator ([B][H][N][d]). */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * fa_bwd -- backward pass of fa_fwd from (q, k, v, o, lse, dO), recomputing the scores:
 *   dV = A^T dO,  dS = A o (dO V^T - rowsum(dO o O)),  dQ = scale dS K,  dK = scale dS^T Q.
 *   dtype FA_BF16: d in {64, 128}; tensor-core kernel.  dq accumulates across key tiles with
 *                  fp32 reductions in L2 (atomics at d = 64, TMA reduce-adds at d = 128) whose
 *                  order varies, so its last bits may differ between runs; dk and dv are
 *                  deterministic.
 *   dtype FA_F32 : 1 <= d <= 128; CUDA-core fp32 kernels (one warp per query row for dq, one
 *                  per key row for dk and dv), exact expf, every sum in a fixed order: all
 *                  three gradients are deterministic.
 *   o and lse must be fa_fwd's outputs for the same arguments.  workspace: device memory of at
 *   least fa_bwd_workspace_size() bytes, 256-byte aligned, owned by the caller, scratch only
 *   (its contents on entry do not matter).
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d,
           float scale, int causal, const uint8_t* block_mask, const int32_t* kv_len,
           int dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_bwd_noalloc -- the backward pass of fa_bwd for callers that cannot provide or allocate
 * device memory.  The pages have no counterpart: this entry point exists for integration.
 *   Who needs it: code running inside a host framework that owns every device allocation (a
 *   plugin interface that hands over only the input and output tensors, a fixed-budget memory
 *   pool), or code that must not call cudaMalloc / cudaFree because they can synchronise the
 *   whole device.  This call allocates nothing: its scratch (log2-scaled lse, Dvec and the fp32
 *   dQ accumulator, sized as fa_bwd_workspace_size() reports) is a fixed 32 MiB array that the
 *   library keeps on every device that loads it, until the process exits.
 *   Arguments, layouts, masks and results are those of fa_bwd, without the workspace pair.
 *   Limit: problems whose fa_bwd_workspace_size(B, H, N, d) exceeds 32 MiB (33554432 bytes)
 *   are rejected with FA_ERR_WORKSPACE before anything is launched.
 *   Set-up: the array's device address is looked up with the device current and cached
 *   together with the id of the CUDA context it belongs to.  The first call on a device, and
 *   the first call after the current context changes (cudaDeviceReset, or a context the caller
 *   made current), does that look-up; later calls only compare the context id.  Make the first
 *   call in each context before any stream capture.
 *   Sharing: every call on a device uses the same scratch and leaves its contents behind; each
 *   call re-initialises everything it reads, but two calls that overlap on the GPU (different
 *   streams, no ordering between them) race on the scratch and give wrong gradients.
 */
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                   float scale, int causal, const uint8_t* block_mask, const int32_t* kv_len,
                   int dtype, void* stream);

/*
 * Grouped-query and multi-query attention (the MQA/GQA of the tcdigital FA-2 ROI article, section
 * "MQA/GQA ... との相乗効果"): H query heads share H_kv K/V heads, H a multiple of H_kv, and query
 * head h reads K/V head h / (H / H_kv) (contiguous groups; H_kv = 1 is multi-query attention).
 * q, o, dO, dq are [B][H][N][d]; k, v, dk, dv are [B][H_kv][N][d]; lse is [B][H][N].
 * Everything else -- dtypes, masks, alignment, status codes -- is as for fa_fwd / fa_bwd; the
 * workspace of fa_bwd_gqa is fa_bwd_workspace_size(B, H, N, d) (query heads).  fa_bwd_gqa
 * accumulates dK and dV of a shared head over its query heads on chip, in a fixed order, so
 * they stay deterministic.  H_kv < 1, H_kv > H or H % H_kv != 0 give FA_ERR_INVALID.
 * fa_fwd_gqa with H_kv = H is fa_fwd; fa_bwd_gqa with H_kv = H is fa_bwd.
 */
int fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int H_kv, int N, int d, float scale, int causal, const uint8_t* block_mask,
               const int32_t* kv_len, int dtype, void* stream);
int fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const float* lse,
               const void* dO, void* dq, void* dk, void* dv, int B, int H, int H_kv, int N,
               int d, float scale, int causal, const uint8_t* block_mask,
               const int32_t* kv_len, int dtype, void* workspace, size_t workspace_bytes,
               void* stream);

/*
 * fa_bwd_deterministic -- fa_bwd_gqa with bit-reproducible gradients: the same inputs give the
 * same dq, dk and dv bits on every run.  Arguments, layouts, workspace and errors are those of
 * fa_bwd_gqa (H_kv = H for ordinary attention).
 *   dtype FA_BF16: dk and dv come from the tensor-core backward without its dq part; dq comes
 *                  from a second tensor-core kernel that owns 128 query rows per CTA and walks
 *                  their KV tiles in increasing order, accumulating on chip -- no atomics.  It
 *                  recomputes S and dP, so the call does 14 d FLOP per unmasked (row, key) pair
 *                  instead of fa_bwd's 10 d.
 *   dtype FA_F32 : the fp32 backward of fa_bwd, which is deterministic already.
 */
int fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dO, void* dq, void* dk, void* dv, int B,
                         int H, int H_kv, int N, int d, float scale, int causal,
                         const uint8_t* block_mask, const int32_t* kv_len, int dtype,
                         void* workspace, size_t workspace_bytes, void* stream);

/* Options of fa_bwd_deterministic_ex (bits; 0 = the library's default). */
enum {
  FA_BWD_DKDV_PAIR = 1,   /* d = 128: dK and dV on pairs of CTAs with 2-CTA MMAs */
  FA_BWD_DKDV_SINGLE = 2  /* d = 128: dK and dV with one CTA per 128 keys (default) */
};

/*
 * fa_bwd_deterministic_ex -- fa_bwd_deterministic with a choice of dK/dV kernel at d = 128
 * (`options`, FA_BWD_DKDV_*; ignored at d = 64 and for FA_F32).  Both kernels sum every dK and
 * dV element over the same terms in the same order.
 *   FA_BWD_DKDV_PAIR: a cluster of two CTAs owns 256 keys and the even CTA issues tcgen05 MMAs
 *     with cta_group::2 (M = 256 keys, each CTA holding its 128 keys' K, V and accumulators); Q
 *     and dO are loaded in halves (query rows for the scores, head-dimension columns for the
 *     gradients), so each SM's tensor core reads half of every B operand from its own shared
 *     memory.  Every tile load is a plain TMA load of this GPU's memory (no multicast).
 *   FA_BWD_DKDV_SINGLE: one CTA per 128 keys with cta_group::1 MMAs.
 * Setting both bits, or any other bit, gives FA_ERR_INVALID.  Everything else is as for
 * fa_bwd_deterministic.
 */
int fa_bwd_deterministic_ex(const void* q, const void* k, const void* v, const void* o,
                            const float* lse, const void* dO, void* dq, void* dk, void* dv, int B,
                            int H, int H_kv, int N, int d, float scale, int causal,
                            const uint8_t* block_mask, const int32_t* kv_len, int dtype,
                            void* workspace, size_t workspace_bytes, int options, void* stream);

/* Flags of fa_fwd_tile_reference: the other two axes of the deviation study. */
enum {
  FA_TILE_REVERSE = 1,    /* visit the key tiles from the last to the first */
  FA_TILE_L_ROUNDED = 2,  /* the normaliser l sums the bf16-rounded P that enters P.V (else the
                             fp32 P before rounding) */
  FA_TILE_TENSOR_CORE = 4,/* run the tcgen05 forward itself with key tiles of bc keys (d = 64,
                             bc in {64, 128}; not with FA_TILE_REVERSE or FA_TILE_L_ROUNDED) */
  FA_TILE_O_F32 = 8       /* o receives the fp32 O/l, [B][H][N][d] float, before its bf16
                             rounding (the deviation of the arithmetic without the output cast) */
};

/*
 * fa_fwd_tile_reference -- bf16 forward on CUDA cores for the numeric-deviation study of "Is
 * Flash Attention Stable?" (aibr.jp summary, sections 3-4): the running maximum and sum are
 * rescaled after every tile of `bc` keys (bc in {32, 64, ..., 256}) and P is rounded to bf16
 * before P.V, as in a tensor-core kernel with that key-tile width.  `flags` (FA_TILE_*) picks
 * the tile order and which P the normaliser sums, or swaps in the tensor-core forward itself
 * with bc-key tiles, and whether o is written as fp32; unknown bits give FA_ERR_INVALID.  Same
 * layouts, masks and errors as fa_fwd (bf16, 1 <= d <= 128).  Not a fast path.
 */
int fa_fwd_tile_reference(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int H, int N, int d, float scale, int causal,
                          const uint8_t* block_mask, const int32_t* kv_len, int bc, int flags,
                          void* stream);

/* Bytes of workspace fa_naive_fwd needs: the materialised S / P matrix, [B][H][N][N] bf16. */
size_t fa_naive_workspace_size(int B, int H, int N);

/*
 * fa_naive_fwd -- the materialised "Baseline Attention" of "Is Flash Attention Stable?":
 * S = bf16(scale Q K^T) written to the workspace, row softmax in fp32 read from it with
 * P = bf16 written back, then O = bf16(P V) with fp32 accumulation.  bf16, 1 <= d <= 128.
 * A deviation and speed reference, not a fast path.
 */
int fa_naive_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int N, int d, float scale, int causal, const uint8_t* block_mask,
                 const int32_t* kv_len, void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_diag_exp2 -- diagnostic for the two ways the forward softmax evaluates 2^x: y_fma gets the
 * FMA-pipe evaluation (rounding reduction x = n + f, |f| <= 1/2, a cubic for 2^f with constant
 * term 1 fitted for minimal relative error, and 2^n added to the exponent bits; relative error
 * below 1.1e-4 for -125 <= x <= 126), y_mufu the hardware ex2.approx, y_ref CUDA's exp2f.
 * x, y_fma, y_mufu, y_ref: device float arrays of n elements.  Asynchronous on `stream`.
 */
int fa_diag_exp2(const float* x, float* y_fma, float* y_mufu, float* y_ref, int n, void* stream);

/*
 * fa_diag_wait_timeout -- diagnostic for the device-side failure path: launches one CTA that
 * waits, through the kernels' bounded mbarrier wait, on a barrier nothing arrives at.  After the
 * wait's time limit (about 2 s) it records `site` (1..32767) in the status word and returns;
 * fa_device_status() then reports FA_ERR_TIMEOUT with code (site << 16).  Nothing traps.
 */
int fa_diag_wait_timeout(int site, void* stream);

/*
 * Measurement diagnostics (no counterpart on the pages; they let a benchmark count and time this
 * library's own kernels from inside a timed region).
 *   fa_launch_count       -- number of kernels this library has launched in the process, over
 *                            every entry point and device (a launch the driver rejected is not
 *                            counted).
 *   fa_kernel_timing      -- enable != 0: from now on every launch of a tensor-core kernel
 *                            (fa_fwd_sm100_kernel, fa_bwd_sm100_kernel, fa_bwd_dkdv_sm100_kernel,
 *                            fa_bwd_dkdv_pair_sm100_kernel, fa_bwd_dq_sm100_kernel) is
 *                            bracketed by two CUDA events recorded on
 *                            the launch's stream; enable == 0 stops recording.  Off by default.
 *   fa_kernel_timing_read -- waits for the recorded launches of every kernel whose name contains
 *                            `name` ("" = all), stores how many there were in *launches and the
 *                            sum of their event-measured durations in *total_ms, and forgets
 *                            them.  FA_ERR_INVALID for a null pointer; FA_ERR_CUDA if an event
 *                            query fails (the counts are still stored).
 */
unsigned long long fa_launch_count(void);
int fa_kernel_timing(int enable);
int fa_kernel_timing_read(const char* name, int* launches, double* total_ms);

/* Message for the most recent non-OK status returned on this host thread. */
const char* fa_get_last_error(void);

/*
 * fa_device_status -- synchronises the current device, then returns FA_OK, or FA_ERR_TIMEOUT
 * if a kernel's bounded wait gave up since the last call (the first such event's code,
 * (site << 16) | (block index & 0xffff), is stored in *code when code != NULL), and clears it.
 * Returns FA_ERR_CUDA if the synchronisation itself reports an error.
 */
int fa_device_status(unsigned int* code);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
