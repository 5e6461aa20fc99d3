/*
 * libmla -- MLA (Multi-head Latent Attention) prefill attention for NVIDIA
 * B200 (sm_100a).  C ABI: plain pointers and sizes, no framework types.
 *
 * What the calls compute (sources named by page and section):
 *
 *   O = softmax(Q K^T * softmax_scale [+ causal mask]) V
 *
 * the only formula the pages print ("SparseFlashMla" README, Description --
 * Formula, where K~ = V~ are the rows that take part), over ragged batches
 * given by cu_seqlens_q / cu_seqlens_k ("Sgl project Sglang FA4 Interface",
 * I/O Contract), with MLA head dims: Q/K have 128 nope + 64 rope = 192 dims,
 * V has 128 (vLLM "flash_attn.py" MLA prefill backend,
 * supports_mla_dimensions and FA4MLAPrefillKernel.dispatch), K/V already
 * expanded to every head (same file, module comment: qhead_per_kvhead = 1).
 *
 * Conventions shared by every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library allocates no device memory and keeps no pointer after return.
 *   - Every call only enqueues work on `stream` (NULL = legacy default
 *     stream) and returns; there is no host synchronisation and no
 *     device-to-host copy.  Outputs are valid once the stream reaches the
 *     point after the call.
 *   - bf16 tensors are packed and row-major exactly as described per call;
 *     tensors read by TMA (q, k, v, kv_latent) need 16-byte aligned bases.
 *   - Errors: the return value is an mla_status.  Host-checkable problems
 *     (null or misaligned pointers, bad sizes, unsupported GPU) are reported
 *     before anything is launched.  Device-resident metadata (cu_seqlens
 *     values, index values) is not validated; out-of-range sparse indices
 *     are treated as padding by the kernel.  Kernel waits are bounded: a
 *     wait that gives up sets a bit in the device status word (see
 *     mla_device_status) instead of hanging.
 *   - LSE ("log-sum-exp", float32 per the FA4 interface I/O Contract) is the
 *     natural log of sum_j exp(softmax_scale * q.k_j), laid out [heads,
 *     tokens]; a row that sees no key gets O = 0 and LSE = -inf.
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle (cudaStream_t / CUstream); NULL = default stream. */
typedef struct CUstream_st* mla_stream_t;

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or value  */
  MLA_ERR_UNSUPPORTED = 2, /* not an sm_100 GPU, or an unsupported shape   */
  MLA_ERR_CUDA = 3,        /* a CUDA runtime/driver call or launch failed  */
  MLA_ERR_SCRATCH_TOO_SMALL = 4 /* call too large for mla_prefill_fwd_noalloc */
} mla_status;

/* Bits of the device status word. */
#define MLA_DEVSTAT_WAIT_TIMEOUT_LOAD 0x1u    /* load warp gave up waiting    */
#define MLA_DEVSTAT_WAIT_TIMEOUT_MMA 0x2u     /* MMA warp gave up waiting     */
#define MLA_DEVSTAT_WAIT_TIMEOUT_SOFTMAX 0x4u /* softmax warps gave up waiting */
#define MLA_DEVSTAT_PLAN_OVERFLOW 0x10u       /* cu_seqlens_q[batch] > total_q */
#define MLA_DEVSTAT_WAIT_TIMEOUT_TEST 0x100u  /* mla_debug_wait_timeout probe  */

/* Human-readable text for an mla_status value (static storage). */
const char* mla_status_string(int status);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int mla_version(void);

/*
 * Bytes of device workspace mla_prefill_fwd needs for a call with these
 * sizes: a small header plus one 8-byte entry per (sequence, 512-row query
 * block), at most ceil(total_q / 512) + batch of them.  Returns 0 for
 * invalid sizes.
 */
size_t mla_prefill_workspace_size(int batch, int total_q);

/*
 * Dense varlen MLA prefill forward.
 *
 * Computes, for every sequence b, head h and query row i of b,
 *   O[i,h,:]  = sum_j softmax_j(softmax_scale * q[i,h,:].k[j,h,:]) v[j,h,:]
 *   lse[h,i]  = ln sum_j exp(softmax_scale * q[i,h,:].k[j,h,:])
 * over the keys j of sequence b that row i may see: all Lk keys when
 * causal == 0; keys j <= i + (Lk - Lq) when causal != 0 (bottom-right
 * aligned; equal to j <= i when Lq == Lk, the new-token case of the vLLM
 * backend's run_prefill_new_tokens; causal == 0 with a separate key set is
 * its run_prefill_context_chunk).
 *
 * Two kernels are enqueued: a one-CTA planner that orders the work (longest
 * first) into `workspace`, and a persistent attention kernel (one CTA per
 * SM) that consumes it.
 *
 * Arguments:
 *   q            bf16 [total_q, num_heads, 192], contiguous, 16-B aligned.
 *   k            bf16 [total_k, num_heads, 192], contiguous, 16-B aligned.
 *   v            bf16 [total_k, num_heads, 128], contiguous, 16-B aligned.
 *   cu_seqlens_q int32 [batch+1] on the device: cu[0] = 0, non-decreasing,
 *                cu[batch] = total_q.  Sequence b owns query rows
 *                [cu_q[b], cu_q[b+1]).
 *   cu_seqlens_k int32 [batch+1] on the device, same rules for keys.
 *   max_seqlen_q, max_seqlen_k  informational upper bounds (>= 0); the
 *                kernels take the lengths from cu_seqlens.
 *   softmax_scale finite, > 0; multiplies q.k (1/sqrt(192) for MLA).
 *   causal       0 or 1.
 *   out          bf16 [total_q, num_heads, 128], 16-B aligned; fully written.
 *   lse          float32 [num_heads, total_q] or NULL (not returned).
 *   stream       stream to enqueue on.
 *   batch, num_heads, total_q, total_k: sizes (total_* >= 0, batch >= 1,
 *                1 <= num_heads <= 65535).
 *   workspace    device memory of at least mla_prefill_workspace_size(batch,
 *                total_q) bytes, 16-B aligned, owned by the caller; its
 *                contents need no initialisation.  Calls that may run at the
 *                same time (different streams) need separate workspaces.
 *   workspace_bytes  its size (MLA_ERR_INVALID_ARG if too small).
 * Returns MLA_OK or an error; on error nothing was launched.
 */
int mla_prefill_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                    const int32_t* cu_seqlens_k, int max_seqlen_q, int max_seqlen_k,
                    float softmax_scale, int causal, void* out, float* lse, mla_stream_t stream,
                    int batch, int num_heads, int total_q, int total_k, void* workspace,
                    size_t workspace_bytes);

/*
 * mla_prefill_fwd over strided q, k and v (for example V as a view into a
 * buffer that interleaves k_nope and v per head, the layout of vLLM's MLA
 * prefill backend, "Vllm project Vllm FlashAttention MLA Prefill", where v
 * is a slice with row stride num_heads * (nope + v) and head stride nope + v).
 *
 * Element (row r, head h, dim d) of x is at x + r * x_row_stride +
 * h * x_head_stride + d (bf16 elements; the dim is contiguous).  Each stride
 * must be positive, a multiple of 8 elements (16 bytes) and below 2^39; the
 * base pointers stay 16-B aligned.  Rows of different heads may overlap in
 * memory (the call only reads q, k and v).  All other arguments are those of
 * mla_prefill_fwd, which is this call with the packed strides
 * (num_heads * 192, 192) for q and k and (num_heads * 128, 128) for v.
 * Returns MLA_ERR_INVALID_ARG for a stride the tensor-map encoder refuses.
 */
int mla_prefill_fwd_strided(const void* q, int64_t q_row_stride, int64_t q_head_stride,
                            const void* k, int64_t k_row_stride, int64_t k_head_stride,
                            const void* v, int64_t v_row_stride, int64_t v_head_stride,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                            int max_seqlen_q, int max_seqlen_k, float softmax_scale, int causal,
                            void* out, float* lse, mla_stream_t stream, int batch, int num_heads,
                            int total_q, int total_k, void* workspace, size_t workspace_bytes);

/*
 * Chunked prefill in one pass.  For each sequence b, the queries attend to
 * every key of its context (k_ctx / v_ctx rows [cu_seqlens_ctx[b],
 * cu_seqlens_ctx[b+1]), no mask) and to its own keys (k / v rows
 * [cu_seqlens_k[b], cu_seqlens_k[b+1]), with the causal mask of
 * mla_prefill_fwd when causal == 1), under one softmax.  The result (out,
 * and the LSE over both key sets) is what mla_attn_merge gives for a
 * context pass (mla_prefill_fwd over the context, causal = 0, LSE
 * returned) and a pass over the sequence's own keys -- the two passes of
 * vLLM's MLA prefill backend ("flash_attn.py", run_prefill_context_chunk:
 * unmasked, LSE returned; run_prefill_new_tokens: causal), merged by their
 * LSEs -- without the partial outputs, the merge launch or their trip
 * through HBM.  The kernel visits a tile's context blocks first, then its
 * own visible blocks.
 *   k_ctx        bf16 [total_ctx, num_heads, 192], packed, 16-B aligned.
 *   v_ctx        bf16 [total_ctx, num_heads, 128], packed, 16-B aligned.
 *   cu_seqlens_ctx int32 [batch + 1] on the device: cu[0] = 0,
 *                non-decreasing, cu[batch] = total_ctx; a sequence may have
 *                an empty context (the call is then mla_prefill_fwd for it).
 *   max_seqlen_ctx, total_ctx  sizes (>= 0).
 * Every other argument is that of mla_prefill_fwd (packed q, k, v; the same
 * workspace size).  Returns MLA_OK or an error; on error nothing was
 * launched.
 */
int mla_prefill_fwd_context(const void* q, const void* k, const void* v,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                            const void* k_ctx, const void* v_ctx, const int32_t* cu_seqlens_ctx,
                            int max_seqlen_q, int max_seqlen_k, int max_seqlen_ctx,
                            float softmax_scale, int causal, void* out, float* lse,
                            mla_stream_t stream, int batch, int num_heads, int total_q,
                            int total_k, int total_ctx, void* workspace, size_t workspace_bytes);

/*
 * mla_prefill_fwd with two options: attention sinks (the "Sgl project
 * Sglang FA4 Interface" page, Description: learnable sink tokens; the
 * SparseFlashMla README's `sinks` parameter; the Mojo sparse branch's
 * attn_sink_ptr) and a static FP8 output scale (vLLM "flash_attn.py",
 * supports_quant_output: kFp8StaticTensorSym, output_scale).
 *   sinks         float [num_heads] device array, or NULL.  Head h's sink
 *                 logit s_h (in the units of softmax_scale * q.k) joins
 *                 every row's softmax with a zero value:
 *                 O = sum_j e^x_j v_j / (e^s_h + sum_j e^x_j),
 *                 LSE = ln(e^s_h + sum_j e^x_j); a row that sees no key gets
 *                 O = 0 and LSE = s_h.  (The pages name the input, not its
 *                 arithmetic; this is the plain reading of a sink token.)
 *   output_scale  float device scalar, or NULL.  When set, `out` is e4m3
 *                 (1 byte per element, [total_q, num_heads, 128], 16-B
 *                 aligned) holding O / *output_scale rounded to nearest even
 *                 and saturated at +-448; otherwise `out` is bf16 as in
 *                 mla_prefill_fwd.
 * Every other argument is that of mla_prefill_fwd (packed q, k, v).  With
 * both options NULL the result is bit for bit that of mla_prefill_fwd.
 */
int mla_prefill_fwd_ex(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                       const int32_t* cu_seqlens_k, int max_seqlen_q, int max_seqlen_k,
                       float softmax_scale, int causal, const float* sinks,
                       const float* output_scale, void* out, float* lse, mla_stream_t stream,
                       int batch, int num_heads, int total_q, int total_k, void* workspace,
                       size_t workspace_bytes);

/*
 * Split-KV (the split-KV path of the "Sgl project Sglang FA4 Interface"
 * page, Description: num_splits_heuristic and the FlashAttentionForwardCombine
 * kernel; vLLM's warmup probes of shapes with max_seqlen_q = 1 and long
 * keys).  When a call has fewer (sequence, 512-row block, head) tiles than
 * the GPU has CTA pairs, most of them idle; split-KV cuts each tile's KV
 * blocks into num_splits ranges, computes a partial result (O normalised
 * over its range, and its LSE) per range into the workspace, and combines
 * the partials by their LSEs (the N-way form of mla_attn_merge).  The
 * result equals mla_prefill_fwd's up to floating-point rounding; the split
 * boundaries depend only on each tile and num_splits, so a call is
 * deterministic, but its result depends on num_splits (pass 1 where
 * results must not depend on the batch).
 */
#define MLA_MAX_SPLITS 64

/* Workspace bytes of mla_prefill_fwd_splitkv (0 for invalid sizes):
 * mla_prefill_workspace_size plus num_splits x total_q x num_heads x
 * (128 + 1) floats of partials.  num_splits == 1 needs no partials. */
size_t mla_prefill_splitkv_workspace_size(int batch, int total_q, int num_heads, int num_splits);

/* A number of splits for a call of these sizes on the current device (1 when
 * the call already has a tile for every CTA pair): the fewest splits that
 * minimise (waves of split tiles over the CTA pairs) x (128-key blocks of a
 * split + 2), with at least two blocks a split and at most MLA_MAX_SPLITS. */
int mla_prefill_num_splits(int batch, int total_q, int num_heads, int max_seqlen_q,
                           int max_seqlen_k);

/* mla_prefill_fwd with num_splits (1 .. MLA_MAX_SPLITS) KV splits per tile
 * and a workspace of mla_prefill_splitkv_workspace_size bytes.  Enqueues
 * the planner, the attention kernel and (num_splits > 1) the combine
 * kernel.  Every other argument is that of mla_prefill_fwd (packed q, k, v).
 * num_splits == 1 is bit for bit mla_prefill_fwd. */
int mla_prefill_fwd_splitkv(const void* q, const void* k, const void* v,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                            int max_seqlen_q, int max_seqlen_k, float softmax_scale, int causal,
                            int num_splits, void* out, float* lse, mla_stream_t stream, int batch,
                            int num_heads, int total_q, int total_k, void* workspace,
                            size_t workspace_bytes);

/*
 * mla_prefill_fwd for the other MLA head geometries of vLLM's MLA prefill
 * backend ("flash_attn.py", supports_mla_dimensions: (qk_nope, qk_rope, v)
 * = (128, 64, 128), (192, 64, 256), (64, 64, 128) and (256, 0, 256)):
 * qk_dim = qk_nope + qk_rope in {128, 192, 256}, v_dim in {128, 256}.
 *   q [total_q, H, qk_dim], k [total_k, H, qk_dim], v [total_k, H, v_dim],
 *   out [total_q, H, v_dim] (bf16, packed, 16-B aligned); lse as in
 *   mla_prefill_fwd.
 * The kernel computes 128 value dims per pass: v_dim = 256 runs two passes
 * over the halves of V (strided views), each recomputing the scores, and
 * writes the LSE in the first.  (qk_dim, v_dim) = (192, 128) is
 * mla_prefill_fwd.  Same workspace as mla_prefill_fwd.
 */
int mla_prefill_fwd_dims(const void* q, const void* k, const void* v,
                         const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                         int max_seqlen_q, int max_seqlen_k, float softmax_scale, int causal,
                         void* out, float* lse, mla_stream_t stream, int batch, int num_heads,
                         int total_q, int total_k, int qk_dim, int v_dim, void* workspace,
                         size_t workspace_bytes);

/*
 * mla_prefill_fwd for callers that cannot allocate device memory.
 *
 * (The pages have no counterpart to this entry point; it is a convenience of
 * this library.)  Some callers have no way to obtain the workspace that
 * mla_prefill_fwd needs: code that must not call cudaMalloc at all (for
 * example inside a runtime that owns every device allocation and hands out
 * none), or a plain C caller with no allocator of its own.  This
 * variant takes the same arguments minus the workspace and runs the same
 * kernels with their work list in a fixed scratch array that is part of the
 * library itself (MLA_NOALLOC_SCRATCH_BYTES of device memory, reserved on
 * every GPU that loads the library until the process exits).  It calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *
 *   - Size limit: mla_prefill_workspace_size(batch, total_q) must not exceed
 *     MLA_NOALLOC_SCRATCH_BYTES, i.e. ceil(total_q / 512) + batch <= 8160;
 *     larger calls return MLA_ERR_SCRATCH_TOO_SMALL and launch nothing.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and keeps it for
 *     that device's CUDA context; a context created anew (for example
 *     after cudaDeviceReset) gets the lookup again on its first call.
 *   - All calls share the one array.  The kernels rewrite everything they
 *     read from it, so nothing needs clearing between calls, but two calls
 *     whose kernels can overlap on the GPU (different streams without an
 *     ordering between them) race on it.
 * Returns the same codes as mla_prefill_fwd, plus MLA_ERR_SCRATCH_TOO_SMALL.
 */
#define MLA_NOALLOC_SCRATCH_BYTES 65536u
int mla_prefill_fwd_noalloc(const void* q, const void* k, const void* v,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                            int max_seqlen_q, int max_seqlen_k, float softmax_scale, int causal,
                            void* out, float* lse, mla_stream_t stream, int batch, int num_heads,
                            int total_q, int total_k);

/*
 * Merge two partial attention results over disjoint key sets A and B into
 * the result over A u B (the context-chunk + new-token combination of the
 * vLLM MLA prefill backend; the same log-sum-exp identity as the split-KV
 * combine kernels named on the FA4 interface page and the Mojo mla module):
 *   lse  = m + ln(exp(lse_a - m) + exp(lse_b - m)),  m = max(lse_a, lse_b)
 *   out  = exp(lse_a - lse) * o_a + exp(lse_b - lse) * o_b
 * A side with lse = -inf has weight 0; if both are -inf, out = 0 and
 * lse = -inf.
 *
 *   o_a, o_b, out     bf16 [num_tokens, num_heads, head_dim], 16-B aligned;
 *                     out may be the same pointer as o_a or o_b.
 *   lse_a, lse_b      float32 [num_heads, num_tokens].
 *   lse_out           float32 [num_heads, num_tokens] or NULL; must not
 *                     overlap lse_a or lse_b (MLA_ERR_INVALID_ARG if it is
 *                     the same pointer).
 *   head_dim          a positive multiple of 8.
 */
int mla_attn_merge(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b,
                   void* out, float* lse_out, int num_tokens, int num_heads, int head_dim,
                   mla_stream_t stream);

/*
 * Absorbed top-k sparse MLA prefill forward ("SparseFlashMla" README,
 * Formula with K~ = V~; Parameters: index -1 = invalid or padded slot;
 * Constraints: indices [Q_T, KV_N = 1, K], one list per token shared by all
 * heads; Mojo "mla_prefill_branch_sparse_fp8": the absorbed sparse prefill
 * over the BF16 latent cache with indices already mapped to physical rows).
 *
 * For token t and head h, with R(t) = { r : 0 <= indices[t,r] < num_kv_rows }:
 *   s_r       = softmax_scale * q[t,h,:] . kv_latent[indices[t,r], :]  (576 dims)
 *   out[t,h,:] = sum_{r in R(t)} softmax_r(s) kv_latent[indices[t,r], 0:512]
 *   lse[h,t]  = ln sum_{r in R(t)} exp(s_r)
 *
 *   q          bf16 [num_tokens, num_heads, 576] (512 latent + 64 rope).
 *   kv_latent  bf16 [num_kv_rows, 576]; V is its first 512 dims.
 *   indices    int32 [num_tokens, topk]; any value < 0 or >= num_kv_rows is
 *              padding and is skipped.
 *   out        bf16 [num_tokens, num_heads, 512].
 *   lse        float32 [num_heads, num_tokens] or NULL.
 *   softmax_scale finite, > 0 (1/sqrt(576) for the absorbed shape).
 *   num_heads  1..128.
 *   num_tokens 0 <= num_tokens < 2^30 and num_tokens * num_heads < 2^31
 *              (otherwise MLA_ERR_INVALID_ARG, nothing launched).
 */
int mla_sparse_prefill_fwd(const void* q, const void* kv_latent, const int32_t* indices,
                           int topk, float softmax_scale, void* out, float* lse,
                           mla_stream_t stream, int num_tokens, int num_heads, int num_kv_rows);

/*
 * Read (and optionally clear) the device status word of the current device:
 * the OR of MLA_DEVSTAT_* bits set by kernels whose bounded waits gave up.
 * This call synchronises the device.  0 means no kernel gave up.
 */
int mla_device_status(unsigned int* status, int reset);

/*
 * Test hook for the bounded-wait machinery: launches one CTA that waits on
 * an mbarrier nothing will ever arrive on, with a time limit of
 * `timeout_us` microseconds (1..10,000,000).  The kernel gives up, sets
 * MLA_DEVSTAT_WAIT_TIMEOUT_TEST in the status word and returns normally.
 */
int mla_debug_wait_timeout(int timeout_us, mla_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_H_ */
