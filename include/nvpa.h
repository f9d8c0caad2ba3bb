/*
 * nvpa.h -- paged-KV attention on NVIDIA B200 (sm_100a): the C ABI.
 *
 * Three operations make up the attention data plane of a vLLM-style engine:
 *
 *   nvpa_store_kvcache             write each new token's K and V rows into the
 *                                  block-paged cache at the slot its slot_mapping gives;
 *   nvpa_paged_decode_attention    one query token per sequence attends to its cached
 *                                  keys/values, read through its block table;
 *   nvpa_varlen_prefill_attention  causal attention for a batch of variable-length
 *                                  prompts given by cumulative lengths, reading keys and
 *                                  values (cached prefix plus new suffix) through the
 *                                  block tables.
 *
 * Sources, by page title and section:
 *   [P1] Neutree AI, "Nano-vLLM part 1" (Chinese translation, blog.itpub.net):
 *        section 4.1 "From Sequences to Blocks" (fixed-size blocks, 256 tokens by
 *        default; tokens of different sequences never share a block), section 4.2
 *        "Prefix caching through hashing" (a block with the same content is reused by
 *        raising its refcount), section 4.3 (a freed block is not cleared), section 5.2
 *        (prefill gets cumulative sequence lengths; decode gets one token per sequence
 *        with its position and slot mapping), section 5.3 (decode runs as CUDA graphs
 *        captured for batch sizes 1, 2, 4, 8, 16 ... 512).
 *   [P3] "Nano-vLLM inference engine architecture" (blog.hotdry.top): section
 *        "PagedAttention's lightweight implementation" (slot_mapping maps each
 *        position to its cache slot; the cache is laid out flat as
 *        [total_slots, head_dim]; store_kvcache_kernel writes K and V there) and
 *        section "Low-level performance details" (prefill uses a varlen attention
 *        over cumulative lengths, decode an attention over the cached K/V).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer is DEVICE memory owned by the caller, unless stated otherwise.
 *    The library never allocates, frees or retains memory, never synchronises the
 *    host with the device, and returns as soon as its kernels are enqueued on
 *    `stream` (0 = the legacy default stream).
 *  - bf16 tensors are passed as `const void*`/`void*` and hold IEEE bfloat16 values.
 *    Pointers to bf16 data and all token strides must be 16-byte aligned (strides a
 *    multiple of 8 elements).  Index tensors are int32.
 *  - KV cache layout: k_cache and v_cache are two separate pools, each
 *    [num_blocks, block_size, num_kv_heads, head_dim] bf16, contiguous.  Slot
 *    s = block * block_size + row names one token row; this is [P3]'s flat
 *    [total_slots, num_kv_heads * head_dim] view of the same memory.
 *  - Supported shapes: head_dim in {64, 128}; block_size in {16, 32, 64, 128, 256};
 *    num_q_heads a multiple of num_kv_heads with a group num_q_heads/num_kv_heads
 *    of at most 8.  Other values return NVPA_ERR_UNSUPPORTED.
 *  - Grouped-query attention: query head h reads KV head h / (num_q_heads /
 *    num_kv_heads).
 *  - Host-side checks return a status before anything is launched.  Values that only
 *    the device can see (slots, block ids, lengths) are checked by the kernels: a bad
 *    value is never dereferenced, the affected row is skipped (treated as absent) and
 *    a bit is OR-ed into *err_flag (a device int32 the caller zeroes; may be NULL).
 *    Kernels never trap.
 *  - A status other than NVPA_OK leaves outputs unspecified; nvpa_last_error() then
 *    returns a message (thread-local, valid until the next call on that thread).
 */
#ifndef NVPA_H
#define NVPA_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum nvpa_status {
    NVPA_OK = 0,
    NVPA_ERR_INVALID_ARG = 1,          /* null pointer, negative size, misalignment ... */
    NVPA_ERR_UNSUPPORTED = 2,          /* valid but not implemented shape                */
    NVPA_ERR_CUDA = 3,                 /* a CUDA runtime call or launch failed           */
    NVPA_ERR_WORKSPACE_TOO_SMALL = 4   /* workspace_bytes below the size query's answer  */
} nvpa_status_t;

/* Bits OR-ed into *err_flag by the kernels. */
#define NVPA_FLAG_BAD_SLOT     1  /* slot < -1 or >= num_blocks*block_size: row not written  */
#define NVPA_FLAG_BAD_BLOCK_ID 2  /* a block-table entry that had to be read is outside
                                     [0, num_blocks): its rows are treated as absent        */
#define NVPA_FLAG_BAD_LENGTH   4  /* a context length / cumulative length outside the bounds
                                     declared by the call: clamped to those bounds          */
#define NVPA_FLAG_TIMEOUT      8  /* a tensor-core kernel stopped early: an internal wait
                                     exceeded its time limit (2 s); outputs are incomplete;
                                     never expected in correct operation                    */

/* Library version, as 10000*major + 100*minor + patch. */
int nvpa_version(void);

/* Human-readable name of a status code. */
const char* nvpa_status_string(int status);

/* Detail of the last non-OK status returned on the calling thread ("" if none). */
const char* nvpa_last_error(void);

/* Number of kernels this library has enqueued in this process so far (all devices,
 * all threads).  Lets a caller count the library's launches in a region of its own. */
uint64_t nvpa_kernel_launch_count(void);

/*
 * nvpa_store_kvcache -- [P3] "PagedAttention's lightweight implementation": for each
 * token t with s = slot_mapping[t] != -1, copy k[t] to the cache row with slot s and
 * v[t] likewise.  Slot -1 marks a padding token (a padded CUDA-graph batch, [P1] 5.3)
 * and is skipped.  The copy is bit-exact.
 *
 *   k, v            bf16 [num_tokens, num_kv_heads, head_dim]; token t starts at
 *                   element t * k_token_stride (resp. v_token_stride); heads and dims
 *                   inside a token are contiguous.  Strides >= num_kv_heads*head_dim.
 *   k_cache,v_cache bf16 pools as described above (written).
 *   slot_mapping    int32 [num_tokens].  Two tokens with the same slot: undefined which
 *                   one lands (the engine never produces that).
 *   num_tokens      >= 0 (0 is a no-op).
 *   head_dim        any multiple of 8 (the copy does not depend on the attention
 *                   kernels' head_dim set).
 * Errors: NVPA_ERR_INVALID_ARG for null pointers, negative sizes, unaligned pointers or
 * strides; slots outside [-1, num_blocks*block_size) set NVPA_FLAG_BAD_SLOT.
 */
nvpa_status_t nvpa_store_kvcache(const void* k, const void* v,
                                 int64_t k_token_stride, int64_t v_token_stride,
                                 void* k_cache, void* v_cache,
                                 const int32_t* slot_mapping, int num_tokens,
                                 int num_kv_heads, int head_dim,
                                 int num_blocks, int block_size,
                                 int32_t* err_flag, cudaStream_t stream);

/*
 * Workspace for nvpa_paged_decode_attention, in bytes, for the same arguments.  It
 * depends only on host-side values (never on the device-side context lengths), so a
 * buffer sized once serves every call with the same batch and bounds.
 */
size_t nvpa_paged_decode_workspace_size(int batch, int num_q_heads, int num_kv_heads,
                                        int head_dim, int max_context_len,
                                        int block_size, int num_splits);

/*
 * nvpa_paged_decode_attention -- [P1] 5.2 decode preparation and [P3] "Low-level
 * performance details": sequence b has one query token q[b] and context_lens[b] cached
 * tokens (counting the token stored by this step, which the caller writes first with
 * nvpa_store_kvcache).  For every query head h:
 *     s_j   = softmax_scale * <q[b,h], K_j>      for keys j < context_lens[b]
 *     out   = sum_j softmax(s)_j * V_j,   lse = log sum_j exp(s_j)
 * where key j of sequence b is row j % block_size of physical block
 * block_tables[b, j / block_size] on KV head h / (num_q_heads / num_kv_heads).
 * Long contexts are cut into partitions processed in parallel and merged with their
 * log-sum-exp weights; the result does not depend on the partition count beyond
 * floating-point rounding.
 *
 *   out             bf16 [batch, num_q_heads, head_dim] (written).
 *   lse_out         float32 [batch, num_q_heads] natural-log sum-exp (written), or NULL.
 *                   A sequence with context length 0 gets out = 0 and lse = -inf.
 *   q               bf16 [batch, num_q_heads, head_dim], contiguous.
 *   block_tables    int32 [batch, max_blocks_per_seq]; only the first
 *                   ceil(context_lens[b] / block_size) entries of row b are read.
 *   context_lens    int32 [batch], each in [0, max_context_len] and at most
 *                   max_blocks_per_seq * block_size (else clamped, NVPA_FLAG_BAD_LENGTH).
 *   max_context_len host-side upper bound of context_lens (sizes the partitioning).
 *   num_splits      0 = automatic: partitions sized from batch, num_kv_heads and
 *                   max_context_len (counting full-length contexts) against the 1776
 *                   resident worker warps of a 148-SM B200: small batches get at least
 *                   one item per warp (partitions of 64 keys or more), many sequences
 *                   352-key partitions, a few long sequences about two rounds of items
 *                   (128 to 1024 keys, at most 32 cache blocks); n > 0 = cut the longest
 *                   possible context into at most n partitions (rounded to the library's
 *                   tile size).
 *   workspace       device scratch of at least nvpa_paged_decode_workspace_size(...)
 *                   bytes, 256-byte aligned; contents need no initialisation and are
 *                   overwritten.  Calls that share a workspace must not overlap.
 * The launch configuration depends only on host-side arguments and the device, never
 * on device data.
 * Errors: NVPA_ERR_INVALID_ARG, NVPA_ERR_UNSUPPORTED (shapes above),
 * NVPA_ERR_WORKSPACE_TOO_SMALL, NVPA_ERR_CUDA.
 */
nvpa_status_t nvpa_paged_decode_attention(void* out, float* lse_out, const void* q,
                                          const void* k_cache, const void* v_cache,
                                          const int32_t* block_tables, int max_blocks_per_seq,
                                          const int32_t* context_lens,
                                          int batch, int num_q_heads, int num_kv_heads,
                                          int head_dim, int num_blocks, int block_size,
                                          int max_context_len, float softmax_scale,
                                          int num_splits,
                                          void* workspace, size_t workspace_bytes,
                                          int32_t* err_flag, cudaStream_t stream);

/*
 * nvpa_decode_step -- one decode step in one call: store each sequence's new key/value
 * row and attend over the context that includes it ([P1] 5.2: decode prepares one token
 * per sequence with its slot mapping; [P3] store_kvcache then flash_attn_with_kvcache).
 * Equivalent to nvpa_store_kvcache(k_new, v_new, ..., slot_mapping, batch) followed by
 * nvpa_paged_decode_attention(...), under the decode contract that sequence b's new
 * token is its key at position context_lens[b] - 1 and slot_mapping[b] is that
 * position's cache slot (-1: not stored, e.g. a padded batch entry).  The attention reads
 * the new row from k_new/v_new directly and the row is written to the cache from the
 * kernel that consumes it, so there is no separate store launch and no read-after-write
 * through the cache.
 *
 *   k_new, v_new    bf16 [batch, num_kv_heads, head_dim] with token strides as in
 *                   nvpa_store_kvcache.
 *   slot_mapping    int32 [batch].  Out-of-range slots other than -1 set
 *                   NVPA_FLAG_BAD_SLOT and are not written.
 *   other arguments as for nvpa_paged_decode_attention (same workspace size).
 */
nvpa_status_t nvpa_decode_step(void* out, float* lse_out, const void* q,
                               const void* k_new, const void* v_new,
                               int64_t k_token_stride, int64_t v_token_stride,
                               void* k_cache, void* v_cache, const int32_t* slot_mapping,
                               const int32_t* block_tables, int max_blocks_per_seq,
                               const int32_t* context_lens, int batch, int num_q_heads,
                               int num_kv_heads, int head_dim, int num_blocks, int block_size,
                               int max_context_len, float softmax_scale, int num_splits,
                               void* workspace, size_t workspace_bytes, int32_t* err_flag,
                               cudaStream_t stream);

/*
 * Workspace for nvpa_decode_step_shared_prefix, in bytes, for the same arguments
 * (host-side values only; 0 for invalid arguments).
 */
size_t nvpa_decode_shared_prefix_workspace_size(int batch, int num_q_heads, int num_kv_heads,
                                                int head_dim, int max_context_len,
                                                int block_size, int num_splits,
                                                int min_group_size);

/*
 * nvpa_decode_step_shared_prefix -- the decode step of nvpa_decode_step (or, with
 * k_new = v_new = slot_mapping = NULL, the attention of nvpa_paged_decode_attention) for
 * batches in which many sequences share a cached prefix.  [P1] 4.2: prefix caching hands
 * the blocks of an already cached prompt to every sequence that starts with it, raising
 * the blocks' refcount, so those sequences' block tables begin with the same physical
 * block ids.  The result is the same attention as nvpa_paged_decode_attention (up to
 * floating-point rounding); only the schedule differs:
 *  - sequences whose block_tables[b, 0] agree form a bucket; a bucket of at least
 *    min_group_size sequences is a group.  The group's prefix is the longest run of
 *    leading blocks that all members' tables hold, counting only blocks that lie
 *    wholly before each member's newest key (position context_lens[b] - 1);
 *  - each group's prefix keys are attended once for all its members on the tensor
 *    cores (every member's query rows against the same K/V tiles), in partitions;
 *  - the worker reads only each member's remaining keys; the combine merges the
 *    prefix and private partitions with their log-sum-exp weights.
 * Sequences in no group are decoded exactly as by nvpa_decode_step.  A batch above
 * 2048 sequences, or below min_group_size (no group can form), is decoded without
 * groups, as by nvpa_decode_step.  The fused store writes only position
 * context_lens[b] - 1, which is never inside a group's prefix.
 *
 *   k_new, v_new,   as for nvpa_decode_step, or all three NULL (no store).
 *   slot_mapping
 *   min_group_size  smallest group (0 = the library default, 8; values below 2 act as 2).
 *   workspace       at least nvpa_decode_shared_prefix_workspace_size(...) bytes,
 *                   256-byte aligned.  After the call its first 256 bytes hold int32
 *                   counters the plan wrote: [2] groups found, [3] sequences in them,
 *                   [4] prefix work units, each a pair of 128-row query tiles
 *                   against one key partition (diagnostics; read after the stream syncs).
 *   other arguments as for nvpa_decode_step.
 * Errors: as nvpa_decode_step; a mix of NULL and non-NULL k_new/v_new/slot_mapping is
 * NVPA_ERR_INVALID_ARG.
 */
nvpa_status_t nvpa_decode_step_shared_prefix(
    void* out, float* lse_out, const void* q, const void* k_new, const void* v_new,
    int64_t k_token_stride, int64_t v_token_stride, void* k_cache, void* v_cache,
    const int32_t* slot_mapping, const int32_t* block_tables, int max_blocks_per_seq,
    const int32_t* context_lens, int batch, int num_q_heads, int num_kv_heads, int head_dim,
    int num_blocks, int block_size, int max_context_len, float softmax_scale, int num_splits,
    int min_group_size, void* workspace, size_t workspace_bytes, int32_t* err_flag,
    cudaStream_t stream);

/*
 * nvpa_paged_decode_attention_static_scratch -- the same decode attention for callers
 * that cannot allocate device memory: a plugin inside a host runtime whose memory
 * manager owns all device memory and offers no allocation hook, or code running where an
 * allocation is not allowed (a cudaMalloc there fails, or synchronises the device and
 * stalls queued work).  No page describes this: it is an interface addition with no
 * counterpart in the method.
 *
 * Arguments and results are those of nvpa_paged_decode_attention without
 * workspace/workspace_bytes.  The scratch the decode needs (partition plan and split
 * partials) lives in a fixed 64 MiB array compiled into the library; every GPU that
 * loads the library holds those 64 MiB until the process exits.  The call allocates
 * nothing (no cudaMalloc, no cudaFree, no allocating library routine).
 *  - The first call on a device resolves the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call before any
 *    stream capture.  Only a successful resolution is kept: if it fails, the call returns
 *    NVPA_ERR_CUDA and the next call tries again.  cudaDeviceReset unloads the library's
 *    device image and makes the kept address stale: do not call this entry point on a
 *    device again after resetting it in the same process.
 *  - A call whose scratch need (nvpa_paged_decode_workspace_size with the same
 *    arguments) exceeds 64 MiB returns NVPA_ERR_WORKSPACE_TOO_SMALL with a message;
 *    lowering num_splits lowers the need (batch 1024 at max_context_len 4096 with 16
 *    query heads of dim 128 needs 97 MiB with automatic partitioning and fits with
 *    num_splits <= 7).
 *  - All calls share the one array, which keeps the last call's contents.  Nothing in it
 *    has to start at zero.  Calls whose kernels can overlap on the GPU (different streams
 *    or threads) race on the array: serialise them.
 */
nvpa_status_t nvpa_paged_decode_attention_static_scratch(
    void* out, float* lse_out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
    int batch, int num_q_heads, int num_kv_heads, int head_dim, int num_blocks,
    int block_size, int max_context_len, float softmax_scale, int num_splits,
    int32_t* err_flag, cudaStream_t stream);

/*
 * nvpa_paged_decode_partial -- the decode attention of nvpa_paged_decode_attention over the
 * keys this call sees, returned as a partial (fp32 output and log-sum-exp) for a later
 * log-sum-exp merge: for long contexts whose keys are spread over several devices, each device runs
 * this over its own key range (its own block tables and context lengths) and
 * nvpa_lse_combine merges the parts (the split-KV combine of [P1] 5.2 decode, across
 * devices; the exchange of the parts between devices is the caller's collective).
 *
 *   o_part          float32 [batch, num_q_heads, head_dim] (written): this call's output
 *                   normalised over its own keys; all zeros for a sequence with no keys.
 *   lse_part        float32 [batch, num_q_heads] (written): natural-log sum-exp of the
 *                   scaled scores over this call's keys, -inf with no keys.  Required.
 *   other arguments and the workspace as for nvpa_paged_decode_attention.
 */
nvpa_status_t nvpa_paged_decode_partial(float* o_part, float* lse_part, const void* q,
                                        const void* k_cache, const void* v_cache,
                                        const int32_t* block_tables, int max_blocks_per_seq,
                                        const int32_t* context_lens, int batch, int num_q_heads,
                                        int num_kv_heads, int head_dim, int num_blocks,
                                        int block_size, int max_context_len, float softmax_scale,
                                        int num_splits, void* workspace, size_t workspace_bytes,
                                        int32_t* err_flag, cudaStream_t stream);

/*
 * nvpa_lse_combine -- merge num_parts partials of the same queries over disjoint key sets:
 *     lse = log sum_r exp(lse_r),   out = sum_r exp(lse_r - lse) * o_r.
 * A part with lse_r = -inf weighs 0; a row whose parts are all -inf gets out = 0 and
 * lse = -inf.  The result equals attention over the union of the parts' keys up to
 * floating-point rounding.
 *
 *   out             bf16 [batch, num_q_heads, head_dim] (written).
 *   lse_out         float32 [batch, num_q_heads] (written) or NULL.
 *   o_parts         float32 [num_parts, batch, num_q_heads, head_dim], 16-byte aligned.
 *   lse_parts       float32 [num_parts, batch, num_q_heads].
 *   head_dim        64 or 128.
 * Errors: NVPA_ERR_INVALID_ARG (null, num_parts < 1, misaligned), NVPA_ERR_UNSUPPORTED.
 */
nvpa_status_t nvpa_lse_combine(void* out, float* lse_out, const float* o_parts,
                               const float* lse_parts, int num_parts, int batch, int num_q_heads,
                               int head_dim, cudaStream_t stream);

/*
 * Workspace for nvpa_varlen_prefill_attention, in bytes (the query-tile schedule), for a
 * call with `batch` sequences and `total_q` query rows.  Host-side values only.
 */
size_t nvpa_varlen_prefill_workspace_size(int batch, int total_q);

/*
 * nvpa_varlen_prefill_attention -- [P1] 5.2 prefill preparation (cumulative sequence
 * lengths) and [P3] "Low-level performance details" (varlen attention in prefill),
 * with prefix caching ([P1] 4.2): sequence i owns query rows
 * cu_seqlens_q[i] .. cu_seqlens_q[i+1]-1 (its uncached suffix, Lq tokens) and keys
 * 0 .. Lk-1, Lk = cu_seqlens_k[i+1] - cu_seqlens_k[i] (cached prefix plus the suffix,
 * which the caller stores first), all read through block_tables[i].  With causal = 1
 * the mask is bottom-right aligned: query r (0-based inside the sequence) is at
 * position Lk - Lq + r and sees keys 0 .. Lk - Lq + r.  With causal = 0 every query
 * sees all Lk keys.
 *
 *   out             bf16 [total_q, num_q_heads, head_dim] (written).
 *   lse_out         float32 [total_q, num_q_heads] (written) or NULL.
 *   q               bf16 [total_q, num_q_heads, head_dim], contiguous.
 *   cu_seqlens_q/k  int32 [batch + 1], non-decreasing, starting at 0, with
 *                   0 <= Lq <= Lk per sequence, Lq <= max_seqlen_q, Lk <= max_seqlen_k,
 *                   Lk <= max_blocks_per_seq*block_size, cu_seqlens_q[batch] = total_q.
 *                   A violation is flagged (NVPA_FLAG_BAD_LENGTH) and that sequence's
 *                   rows are left unwritten.
 *   workspace       device scratch of at least nvpa_varlen_prefill_workspace_size(batch,
 *                   total_q) bytes, 256-byte aligned, no initialisation needed; calls that
 *                   share a workspace must not overlap.
 * A block-table entry outside [0, num_blocks) is flagged (NVPA_FLAG_BAD_BLOCK_ID), its
 * rows are not read (zeros stand in for them), and that sequence's output is unspecified
 * but finite.
 * QK^T and PV run on the tensor cores (tcgen05, bf16 inputs, fp32 accumulation in TMEM);
 * P is rounded to bf16 before the PV product.
 * Errors: as for decode.
 */
nvpa_status_t nvpa_varlen_prefill_attention(void* out, float* lse_out, const void* q,
                                            const void* k_cache, const void* v_cache,
                                            const int32_t* block_tables, int max_blocks_per_seq,
                                            const int32_t* cu_seqlens_q,
                                            const int32_t* cu_seqlens_k,
                                            int batch, int total_q,
                                            int max_seqlen_q, int max_seqlen_k,
                                            int num_q_heads, int num_kv_heads, int head_dim,
                                            int num_blocks, int block_size,
                                            float softmax_scale, int causal,
                                            void* workspace, size_t workspace_bytes,
                                            int32_t* err_flag, cudaStream_t stream);

/*
 * nvpa_gather_kv -- copy the paged rows of each sequence into a contiguous array,
 * bit-exact: dst[cu_seqlens_k[i] + j] = cache row j of sequence i (block
 * block_tables[i, j / block_size], row j % block_size), for j < Lk.  This is the
 * addressing the attention kernels use, exposed so that it can be checked on its own
 * ([P1] 4.1: a sequence spans several blocks, the last one partly filled).
 *
 *   dst             bf16 [total_k, num_kv_heads, head_dim] (written), total_k =
 *                   cu_seqlens_k[batch].
 *   cache           one pool (K or V).
 * Rows whose block id is out of range are written as zeros and flagged.
 */
nvpa_status_t nvpa_gather_kv(void* dst, const void* cache,
                             const int32_t* block_tables, int max_blocks_per_seq,
                             const int32_t* cu_seqlens_k, int batch, int total_k,
                             int num_kv_heads, int head_dim, int num_blocks, int block_size,
                             int32_t* err_flag, cudaStream_t stream);

/*
 * nvpa_check_bounded_wait -- test helper for the tensor-core kernels' time-bounded waits:
 * one warp waits, with the same wait those kernels use, on a shared-memory barrier that
 * nothing arrives at.  After 2 s the wait gives up, NVPA_FLAG_TIMEOUT is OR-ed into
 * *err_flag and the kernel returns; the context stays usable.  (No page defines this: it
 * shows on the device that a wait which cannot complete ends in a status, not a hang.)
 *
 *   err_flag        device int32, required (not null).
 * Errors: NVPA_ERR_INVALID_ARG for a null err_flag; NVPA_ERR_CUDA if the launch fails.
 */
nvpa_status_t nvpa_check_bounded_wait(int32_t* err_flag, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* NVPA_H */
