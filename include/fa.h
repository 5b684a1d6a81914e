/*
 * fa.h - C ABI of the B200 (sm_100a) fused exact attention (forward and backward).
 *
 * The operation (one call):
 *   O[b,i,h,:] = sum_j softmax_j(scale * q[b,i,h,:] . k[b,j,h,:]) * v[b,j,h,:]
 *   LSE[b,h,i] = ln sum_j exp(scale * q[b,i,h,:] . k[b,j,h,:])
 * over the visible keys j (all j < N, or j <= i when causal).
 *   - The formula and its four steps (similarity, scaling, softmax, weighted
 *     sum of V): llmtrend.com, "FlashAttention ...", self-attention section.
 *   - Computed tile by tile with a running max / running sum (online
 *     softmax), Q/K/V loaded once and no N x N matrix written to memory:
 *     jsqmd.com "Flash Attention applications", core-mechanism section
 *     (kernel fusion, tiling + streaming); tuning handbook ch. 3,
 *     "engineering implementation" section (tiled routine with lse).
 *   - Causal masking skips future positions: handbook ch. 3, practical notes.
 *   - The per-row log-sum-exp output (lse of shape [B, H, N]): the handbook's
 *     tiled routine, which keeps and updates lse per query row.
 *   - API shape (q, k, v, causal): mlqm.cn FA1/FA2 comparison, section 6.1.
 *
 * Layout (all buffers device memory, owned by the caller, never retained):
 *   q, k, v, o : [B, N, H, D] contiguous, one 16-bit dtype (bf16 or fp16),
 *                element (b,n,h,d) at ((b*N + n)*H + h)*D + d.
 *   lse        : float32 [B, H, N] contiguous, natural log of the scaled logits.
 *   Base pointers must be 16-byte aligned.
 *
 * The library makes no device allocation per call; its only device-side
 * state is one status word per device (a static __device__ variable) that
 * records asynchronous faults (see fa_status_sync).
 *
 * Errors: host-detectable errors return a status WITHOUT launching anything
 * and leave o and lse untouched. A successful return means the work was
 * enqueued on `stream`; device-side timeouts are reported later through
 * fa_status_sync. No C++ exception ever crosses this boundary.
 *
 * Debugging (the pages name a debug switch for their library: FLASH_ATTN_DEBUG
 * on the jsqmd.com page, usage notes; FLASH_ATTENTION_DEBUG on the mlqm.cn
 * page, section 6.2). With FA_DEBUG (or either of those names) set to a
 * nonzero value in the environment when the library is first used, every
 * call prints its launch configuration to stderr and, after enqueueing,
 * synchronises `stream` and reads the status word itself: a device-side
 * failure is then returned by the call (FA_ERR_TIMEOUT, FA_ERR_INVALID_ARG,
 * FA_ERR_DEVICE_CHECK) instead of by a later fa_status_sync. Calls become
 * synchronous; results are unchanged.
 *
 * Checking build: libfa_b200_checks.so is the same library compiled with
 * -DFA_CHECKS. Before every global-memory store its kernels check that the
 * index lies inside the output the host described; a failed check skips the
 * store, sets the status word (FA_ERR_DEVICE_CHECK from fa_status_sync) and
 * never traps. Results of a passing run are bit-identical to the normal build.
 */
#ifndef FA_B200_FA_H_
#define FA_B200_FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same ABI as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* fa_stream_t;

typedef enum {
  FA_BF16 = 0, /* bfloat16 inputs and output */
  FA_FP16 = 1  /* IEEE binary16 inputs and output */
} fa_dtype;

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null pointer, negative size, unknown dtype, non-finite scale */
  FA_ERR_UNSUPPORTED = 2, /* D not in {64, 128}, sizes beyond the limits below, or not an sm_100 device */
  FA_ERR_MISALIGNED = 3,  /* a base pointer is not 16-byte aligned */
  FA_ERR_CUDA = 4,        /* a CUDA runtime call failed (no device, launch failure, ...) */
  FA_ERR_TIMEOUT = 5,     /* a device-side wait ran out (reported by fa_status_sync) */
  FA_ERR_DEVICE_CHECK = 6 /* checking build only: a device-side index check failed (reported by fa_status_sync) */
} fa_status;

/* Limits checked before launch: D in {64,128}; B*H*ceil(N/256) <= 2^31-1;
 * rows (B*N, or total) below 2^31 - 512; each of q/k/v/o spans < 2^40 bytes. */

/* Static, human-readable name of a status code; never NULL. */
const char* fa_status_string(fa_status status);

/* Detail of the last FA_ERR_CUDA returned on the calling thread (the failing
 * call and CUDA's message), or "" if none; owned by the library, valid until
 * the thread's next call into it. */
const char* fa_last_error(void);

/*
 * fa_fwd - fused exact-attention forward, enqueued on `stream`.
 *
 *   q, k, v : device pointers, [B, N, H, D], dtype `dtype`        (read only)
 *   o       : device pointer,  [B, N, H, D], dtype `dtype`        (written)
 *   lse     : device pointer,  float32 [B, H, N]                  (written)
 *   B, N, H : batch, sequence length (queries = keys), heads; >= 0
 *   D       : head dimension, 64 or 128
 *   scale   : multiplies q.k before the softmax (1/sqrt(D) in the pages); finite
 *   causal  : nonzero -> key j is visible to query i iff j <= i (square, top-left aligned)
 *   stream  : CUDA stream the kernel is launched on
 *
 * B*N*H == 0 is a valid no-op (FA_OK, nothing launched, pointers unchecked).
 * Results are bitwise deterministic for identical inputs on one device.
 * Returns FA_OK after enqueueing, or an error code without launching.
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t N,
                 int64_t H, int64_t D, float scale, int causal, fa_dtype dtype, fa_stream_t stream);

/*
 * fa_fwd_gqa - fa_fwd generalised to grouped-query heads and to queries and
 * keys of different lengths (cross-attention); fa_fwd(..., N, H, ...) is
 * fa_fwd_gqa(..., Nq = Nk = N, Hq = Hkv = H, ...).
 *
 *   q, o   : [B, Nq, Hq,  D] contiguous          k, v : [B, Nk, Hkv, D] contiguous
 *   lse    : float32 [B, Hq, Nq]
 *   Hq % Hkv == 0; query head h reads key/value head h / (Hq / Hkv)
 *     (grouped-query / multi-query attention: llmtrend.com FlashAttention
 *     page, Mistral case; separate query and key lengths: the same page's
 *     limitations section, cross-attention).
 *   causal : key j visible to query i iff j <= i + (Nk - Nq), i.e. the mask is
 *            aligned at the bottom-right corner (the square mask when Nq == Nk).
 *            A query with no visible key (possible when Nq > Nk) gets O = 0 and
 *            LSE = -inf; so does every query when Nk == 0.
 * Errors and asynchrony as fa_fwd; Hkv < 1 or Hq % Hkv != 0 -> FA_ERR_INVALID_ARG.
 */
fa_status fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t Nq,
                     int64_t Nk, int64_t Hq, int64_t Hkv, int64_t D, float scale, int causal, fa_dtype dtype,
                     fa_stream_t stream);

/*
 * fa_fwd_varlen - forward over B sequences of different lengths packed
 * without padding (the padding-free form of the pages' padding mask,
 * jsqmd.com page, usage notes), with grouped-query heads.
 *
 *   q, o          : [total_q, Hq,  D] contiguous; sequence b owns query rows
 *                   cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1
 *   k, v          : [total_k, Hkv, D] contiguous; key rows cu_seqlens_k[b] ..
 *   cu_seqlens_q/k: int32 DEVICE arrays of B+1 non-decreasing offsets,
 *                   cu[0] = 0, cu[B] = total_q / total_k
 *   max_seqlen_q  : >= every query length (sizes the grid)
 *   lse           : float32 [Hq, total_q]
 *   causal, GQA, empty rows: as fa_fwd_gqa, per sequence (nq, nk its lengths).
 * The offsets live in device memory and are checked by the kernel: a sequence
 * whose offsets are inconsistent (decreasing, beyond total, or longer than
 * max_seqlen_q) is skipped, its outputs are left untouched, and
 * fa_status_sync reports FA_ERR_INVALID_ARG.
 */
fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int32_t* cu_seqlens_q,
                        const int32_t* cu_seqlens_k, int64_t B, int64_t max_seqlen_q, int64_t total_q, int64_t total_k,
                        int64_t Hq, int64_t Hkv, int64_t D, float scale, int causal, fa_dtype dtype,
                        fa_stream_t stream);

/*
 * fa_fwd_splitkv - fa_fwd_gqa with the keys cut into ranges processed by
 * separate CTAs, for shapes whose query side alone cannot fill the GPU
 * (decoding: few queries per head, long key sequences). Each range writes its
 * partial O (normalised by its own sum, fp32) and LSE to `workspace`; a
 * second kernel merges them with weights exp(LSE_r - LSE). Same arguments,
 * layouts, masks and errors as fa_fwd_gqa, plus:
 *   num_splits       : 0 = choose (enough CTAs for every SM), else requested
 *                      count; capped at 64 and at the number of 128-key tiles
 *   workspace        : device memory, 256-byte aligned, owned by the caller,
 *                      at least the size fa_fwd_splitkv_plan reports; unused
 *                      (may be NULL) when the plan has one range
 *   workspace_bytes  : its size; too small -> FA_ERR_INVALID_ARG, no launch
 * Calls that share a workspace must not overlap on the GPU.
 */
fa_status fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t Nq,
                         int64_t Nk, int64_t Hq, int64_t Hkv, int64_t D, float scale, int causal, fa_dtype dtype,
                         int num_splits, void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_fwd_splitkv_plan - number of key ranges fa_fwd_splitkv will use for
 * these sizes on the current device, and the workspace it needs in bytes
 * (0 when it uses one range). Host only; launches nothing. Hkv matters:
 * when Nq * (Hq / Hkv) <= 128 and Hq / Hkv > 1 the forward packs the query
 * heads that share a key/value head into one tile (one work item per K/V head
 * instead of one per query head), and the key range count is chosen for that
 * smaller grid (each CTA then computes two ranges, one per query tile of the
 * kernel, so the plan returns twice the ranges that fill the SMs).
 */
fa_status fa_fwd_splitkv_plan(int64_t B, int64_t Nq, int64_t Nk, int64_t Hq, int64_t Hkv, int64_t D, int num_splits,
                              int* splits_out, size_t* workspace_bytes);

/*
 * fa_fwd_splitkv_noalloc - fa_fwd_splitkv without a workspace argument, for
 * callers that must not allocate device memory on the call path: for example
 * a serving loop whose GPU memory is reserved up front by another allocator,
 * or code that cannot handle an out-of-memory failure in the middle of a
 * request. The pages describe no such entry point; it has no counterpart
 * there.
 *
 *   Arguments, layouts, masks and results as fa_fwd_splitkv; the caller still
 *   provides q, k, v, o and lse.
 *   The partial results go to a scratch buffer compiled into the library:
 *   FA_NOALLOC_SCRATCH_BYTES (16 MiB) of device memory that every GPU which
 *   loads the library holds until the process exits. With num_splits = 0 the
 *   call uses the plan's range count, or the largest smaller count whose
 *   partial results fit the scratch; an explicit num_splits whose partial
 *   results would not fit (fa_fwd_splitkv_plan's workspace_bytes above that)
 *   returns FA_ERR_UNSUPPORTED without launching, with the sizes in
 *   fa_last_error().
 *   No cudaMalloc, cudaFree or other allocating call is made. The first call
 *   on each device looks up the scratch buffer's device address
 *   (cudaGetSymbolAddress) and caches it; make that first call before any
 *   stream capture on that device.
 *   Every call uses the same buffer and leaves its last contents there;
 *   nothing in it has to start at zero (each call overwrites every entry it
 *   reads). Calls that overlap on the GPU (different streams, or the same
 *   buffer used concurrently) race with each other and give wrong results.
 */
#define FA_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
fa_status fa_fwd_splitkv_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
                                 int64_t Nq, int64_t Nk, int64_t Hq, int64_t Hkv, int64_t D, float scale, int causal,
                                 fa_dtype dtype, int num_splits, fa_stream_t stream);

/*
 * fa_status_sync - synchronise `stream`, then read and clear this device's
 * status word. Returns FA_OK; FA_ERR_TIMEOUT if a kernel on this device gave
 * up on a bounded wait since the last call (its outputs are then invalid);
 * FA_ERR_INVALID_ARG if fa_fwd_varlen met inconsistent sequence offsets;
 * FA_ERR_DEVICE_CHECK if a device-side index check of the checking build
 * failed; or FA_ERR_CUDA if the synchronisation itself failed. When several
 * were recorded, the first of that list is returned (all are cleared).
 */
fa_status fa_status_sync(fa_stream_t stream);

/*
 * fa_bwd_workspace_size - bytes of device workspace fa_bwd needs for these
 * sizes: two fp32 arrays [B*H, ceil(N/128)*128], each rounded up to 256 bytes,
 * then 256 bytes for the gradient kernels' work-item counters (0 in all when
 * B or H is 0: there is nothing to do). For fa_bwd_gqa pass the query side's
 * sizes (B, Nq, Hq).
 * Returns FA_ERR_INVALID_ARG for a NULL output or a negative size.
 */
fa_status fa_bwd_workspace_size(int64_t B, int64_t N, int64_t H, size_t* workspace_bytes);

/*
 * fa_bwd - gradients of the forward above, enqueued on `stream`.
 *
 * Given dO = dL/dO, with P[i,j] = exp(scale q_i.k_j - LSE_i) over the
 * visible keys (the forward's weights, recomputed from q, k and lse rather
 * than stored: jsqmd.com "Flash Attention applications", core-mechanism
 * section, item 3 "Recomputation"), D_i = dO_i . O_i and
 * dS[i,j] = P[i,j] (dO_i . v_j - D_i):
 *   dV_j = sum_i P[i,j] dO_i,  dQ_i = scale sum_j dS[i,j] k_j,
 *   dK_j = scale sum_i dS[i,j] q_i        (per batch and head).
 * The result is deterministic: no atomics, every output element is written
 * by exactly one thread, with a fixed summation order (the deterministic
 * mode of mlqm.cn FA1/FA2 comparison, section 3.2).
 *
 *   q, k, v, o, dout : device, [B, N, H, D], dtype `dtype` (read only); o and
 *                      lse are the forward's outputs for these q, k, v, scale
 *                      and causal
 *   lse              : device, float32 [B, H, N] (read only)
 *   dq, dk, dv       : device, [B, N, H, D], dtype `dtype` (written; must not
 *                      overlap the inputs)
 *   D                : 64 or 128;  scale, causal, dtype : as in fa_fwd
 *   workspace        : device, at least fa_bwd_workspace_size(B, N, H) bytes,
 *                      256-byte aligned; owned by the caller, scratch for the
 *                      duration of the call (stream-ordered)
 * Three kernels run in stream order: D and LSE log2(e) into the workspace
 * (which also resets the work-item counters), then dQ (work items of 128
 * queries), then dK and dV (work items of 128 keys); the last two are
 * persistent, one CTA per SM taking items from its counter, and an item's
 * result does not depend on which CTA computed it. fp32 accumulation in
 * Tensor Memory; P and dS enter the tensor cores rounded to `dtype`.
 * Errors: as fa_fwd; additionally FA_ERR_INVALID_ARG for a NULL or too small
 * workspace and FA_ERR_MISALIGNED for a workspace not 256-byte aligned.
 * B, N or H == 0 returns FA_OK without launching.
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                 void* dq, void* dk, void* dv, int64_t B, int64_t N, int64_t H, int64_t D, float scale, int causal,
                 fa_dtype dtype, void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_bwd_gqa - fa_bwd generalised like fa_fwd_gqa: grouped-query heads and
 * queries and keys of different lengths (cross-attention), the gradients of
 * fa_fwd_gqa's output; fa_bwd(..., N, H, ...) is fa_bwd_gqa(..., Nq = Nk = N,
 * Hq = Hkv = H, ...).
 *
 *   q, o, dout, dq : [B, Nq, Hq,  D]        k, v, dk, dv : [B, Nk, Hkv, D]
 *   lse            : float32 [B, Hq, Nq], as fa_fwd_gqa returned it
 *   Hq % Hkv == 0; query head h reads key/value head h / (Hq / Hkv), so the
 *     gradient of a key/value head is the sum over the Hq / Hkv query heads
 *     that read it (grouped-query attention: llmtrend.com FlashAttention page,
 *     Mistral case; separate query and key lengths: the same page's
 *     limitations section, cross-attention). The sum is taken inside one CTA
 *     in a fixed order: results stay deterministic, with no atomics.
 *   causal : the bottom-right aligned mask of fa_fwd_gqa (key j visible to
 *            query i iff j <= i + Nk - Nq). A query that sees no key gets
 *            dQ = 0; a key that no query sees gets dK = dV = 0.
 *   workspace : at least fa_bwd_workspace_size(B, Nq, Hq) bytes (may be NULL
 *               when that is 0, i.e. Nq == 0).
 * Errors and asynchrony as fa_bwd; Hkv < 1 or Hq % Hkv != 0 -> FA_ERR_INVALID_ARG.
 * B == 0, Hq == 0, or Nq == Nk == 0 returns FA_OK without launching; Nq == 0
 * with Nk > 0 writes dk = dv = 0, Nk == 0 with Nq > 0 writes dq = 0.
 */
fa_status fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                     void* dq, void* dk, void* dv, int64_t B, int64_t Nq, int64_t Nk, int64_t Hq, int64_t Hkv,
                     int64_t D, float scale, int causal, fa_dtype dtype, void* workspace, size_t workspace_bytes,
                     fa_stream_t stream);

/*
 * fa_bwd_varlen - the backward of fa_fwd_varlen: B sequences of different
 * lengths packed without padding (the padding-free form of the pages'
 * padding mask, jsqmd.com page, usage notes), grouped-query heads, the
 * bottom-right causal mask per sequence.
 *
 *   q, o, dout, dq : [total_q, Hq,  D]; sequence b owns query rows
 *                    cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1
 *   k, v, dk, dv   : [total_k, Hkv, D]; key rows cu_seqlens_k[b] ..
 *   lse            : float32 [Hq, total_q], as fa_fwd_varlen returned it
 *   cu_seqlens_q/k : int32 DEVICE arrays of B+1 non-decreasing offsets
 *   max_seqlen_q/k : >= every query / key length (size the grids)
 *   workspace      : at least fa_bwd_workspace_size(B, max_seqlen_q, Hq) bytes
 * Gradients, masks, grouped heads and determinism as fa_bwd_gqa, per
 * sequence. As in fa_fwd_varlen the kernels check the offsets: a sequence
 * whose offsets are inconsistent (decreasing, beyond the totals, or longer
 * than the maxima) is skipped, its gradients are left untouched, and
 * fa_status_sync reports FA_ERR_INVALID_ARG.
 */
fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, const int32_t* cu_seqlens_q,
                        const int32_t* cu_seqlens_k, int64_t B, int64_t max_seqlen_q, int64_t max_seqlen_k,
                        int64_t total_q, int64_t total_k, int64_t Hq, int64_t Hkv, int64_t D, float scale, int causal,
                        fa_dtype dtype, void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_fwd_debug - fa_fwd with two test hooks (same arguments first).
 *   wait_limit_ns   : give-up time for every device-side wait (0 = default, about 1 s).
 *   withhold_v_load : nonzero -> the loader of the first CTA never issues the
 *                     V load of its first key tile, so that CTA's waits run
 *                     out and report FA_ERR_TIMEOUT through fa_status_sync
 *                     (the GPU stays usable). For tests of the timeout path.
 */
fa_status fa_fwd_debug(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t N,
                       int64_t H, int64_t D, float scale, int causal, fa_dtype dtype, fa_stream_t stream,
                       uint64_t wait_limit_ns, int withhold_v_load);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_FA_H_ */
