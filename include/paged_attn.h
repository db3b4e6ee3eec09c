/*
 * paged_attn.h -- C ABI of libpagedattn.so: exact attention over a paged KV
 * cache on NVIDIA B200 (sm_100a).
 *
 * The method: softmax(Q K^T * scale) V computed tile by tile with an online
 * softmax (running max m, running sum l), so the score matrix never reaches
 * HBM ("大模型推理加速技术全景", iopencloud, sections 2.1-2.2), over a
 * PagedAttention cache: K/V live in fixed 16-token blocks of a global pool,
 * each sequence reaches its blocks through a block table (same page, section
 * 3.2 and its page-table figure; the zhihu roofline page, "显存管理", gives
 * 16 tokens as the default and adds refcounted copy-on-write blocks).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every pointer argument is a DEVICE pointer owned by the caller unless its
 *   comment says otherwise.  Nothing is retained after the call returns and
 *   nothing is freed.  The library allocates no device memory.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   Every call only enqueues work on it and never synchronises.
 * - Element type: pa_dtype, PA_F16 (IEEE binary16) or PA_BF16 (bfloat16), for
 *   Q, O and the caches alike.  Accumulation and softmax are fp32.
 * - Layouts (dense, row-major, no padding):
 *     q, out              [T][H_q][d]        token-major; sequence b owns rows
 *                                            cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1
 *     k_new, v_new        [T][H_kv][d]
 *     key_cache,
 *     value_cache         [num_blocks][H_kv][16][d]   one (block, head) = 16*d contiguous
 *     block_tables        int32 [B][max_blocks_per_seq]; page p of sequence b is
 *                         block block_tables[b][p]; entries past the last page
 *                         are never read
 *     cu_seqlens_q        int32 [B+1], cu_seqlens_q[0] = 0, non-decreasing
 *     context_lens        int32 [B], keys of sequence b INCLUDING its q_b new tokens
 * - Positions: query i (0 <= i < q_b) of sequence b sits at absolute position
 *   ctx_b - q_b + i and attends to keys 0 .. ctx_b - q_b + i (causal,
 *   bottom-right aligned).  Keys past ctx_b in the last block are never used,
 *   whatever they hold (NaN included).
 * - GQA: H_q % H_kv == 0 and query head h reads KV head h / (H_q / H_kv).
 * - Supported head sizes: d = 64 or 128.  All pointers 16-byte aligned.
 * - Return value: PA_OK (0) or a negative pa_status.  Host-detectable argument
 *   errors return at once and launch nothing.  Errors that only the device can
 *   see (a block id or slot out of range, ctx_b > max_ctx, a bounded wait that
 *   ran out) are written to a device status word (see pa_read_status); the
 *   offending work item is skipped, never faulted.
 */
#ifndef PAGED_ATTN_H
#define PAGED_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { PA_F16 = 0, PA_BF16 = 1 } pa_dtype;

typedef enum {
    PA_OK = 0,
    PA_ERR_ARG = -1,         /* a size, pointer or count is invalid */
    PA_ERR_UNSUPPORTED = -2, /* d not in {64,128}, H_q % H_kv != 0, q_len > 8 in decode, ... */
    PA_ERR_ALIGN = -3,       /* a pointer is not 16-byte aligned */
    PA_ERR_WORKSPACE = -4,   /* workspace NULL or smaller than the *_workspace_bytes query */
    PA_ERR_CUDA = -5,        /* a CUDA runtime call failed (launch, attribute, driver entry point) */
    PA_ERR_TIMEOUT = -6,     /* device: a bounded wait on an asynchronous copy ran out */
    PA_ERR_BOUNDS = -7,      /* device: a block id, slot or length was out of range; item skipped */
    PA_ERR_SEQ = -8,         /* device: cu_seqlens_q / context_lens inconsistent (q_b < 1, ctx_b < q_b, ...) */
    PA_ERR_TOO_LARGE = -9    /* pa_paged_attn_decode_noalloc: the sizes need more than its fixed scratch */
} pa_status;

/* Size of the device status word area at the start of every workspace, bytes. */
#define PA_STATUS_BYTES 256

/*
 * pa_kv_cache_write -- scatter the step's new K/V rows into the paged cache.
 * For every token t with s = slot_mapping[t] >= 0:
 *     key_cache[s / 16][h][s % 16][:] = k_new[t][h][:]   (h < H_kv), same for V.
 * A negative slot marks a padding token and is skipped.  Slots >= 16*num_blocks
 * are skipped and reported through `status` (PA_ERR_BOUNDS) when status != NULL.
 * Bit-exact copy.  Slots must be distinct (two tokens on one slot: either wins).
 * Follows: "Continuous Batching" answer of the interview Q&A page (a new
 * token goes into the current block, a new block when it is full) and the
 * page-table figure of iopencloud section 3.2.
 *   k_new, v_new  [T][H_kv][d]         slot_mapping int32 [T]
 *   status        optional device int32 (may be NULL); written only on error
 */
int pa_kv_cache_write(const void *k_new, const void *v_new, const int32_t *slot_mapping, int64_t T,
                      void *key_cache, void *value_cache, int64_t num_blocks, int H_kv, int d, pa_dtype dtype,
                      int32_t *status, void *stream);

/*
 * pa_kv_block_copy -- copy-on-write of shared blocks.  For each pair
 * (src, dst) = (pairs[2i], pairs[2i+1]) copy K and V of every head and all 16
 * rows of block src to block dst.  Pairs with an id outside [0, num_blocks)
 * are skipped and reported through `status`.  A dst must not be the src of
 * another pair in the same call (the copies run concurrently).  Bit-exact.
 * Follows: zhihu roofline page, "显存管理" (refcounted blocks shared by
 * several sequences are copied when one of them writes).
 *   pairs  int32 [n][2], device memory
 */
int pa_kv_block_copy(void *key_cache, void *value_cache, int64_t num_blocks, int H_kv, int d, pa_dtype dtype,
                     const int32_t *pairs, int64_t n, int32_t *status, void *stream);

/* Directions of pa_kv_block_swap. */
#define PA_SWAP_OUT 0 /* device cache -> host pool */
#define PA_SWAP_IN 1  /* host pool -> device cache */

/*
 * pa_kv_block_swap -- move whole blocks between the device caches and a pool
 * of blocks in page-locked host memory: the swap-out of a preempted request's
 * KV blocks to CPU memory, and their swap-in when it resumes (the interview
 * Q&A page, its answer on combining continuous batching with PagedAttention:
 * preemption under memory pressure).  For each pair (dev, host) =
 * (pairs[2i], pairs[2i+1]) copy K and V of every head and all 16 rows of
 * device block `dev` to host block `host` (PA_SWAP_OUT) or back (PA_SWAP_IN).
 * Pairs with an id outside [0, num_blocks) / [0, host_blocks) are skipped and
 * reported through `status`.  No destination may appear twice in one call.
 * Bit-exact.  One kernel reads and writes the host pool over the host link
 * through its device-mapped address; nothing is staged.
 *   host_key, host_value  [host_blocks][H_kv][16][d], page-locked host memory
 *                         that the device can address (cudaHostAlloc or a
 *                         pinned torch tensor); anything else -> PA_ERR_ARG,
 *                         before any launch.  Owned by the caller.
 *   pairs                 int32 [n][2], device memory
 *   direction             PA_SWAP_OUT or PA_SWAP_IN
 */
int pa_kv_block_swap(void *key_cache, void *value_cache, int64_t num_blocks, void *host_key, void *host_value,
                     int64_t host_blocks, int H_kv, int d, pa_dtype dtype, const int32_t *pairs, int64_t n,
                     int direction, int32_t *status, void *stream);

/*
 * pa_decode_workspace_bytes -- device workspace that pa_paged_attn_decode needs
 * for these sizes: the status word area, the order in which the sequences are
 * scheduled (B int32, most pages first, written by the call itself), and with
 * more than one KV split the split-KV partial outputs and log-sum-exps.
 * Pure host function.  Returns 0 for invalid sizes.
 */
size_t pa_decode_workspace_bytes(int64_t T, int B, int H_q, int H_kv, int d, int max_ctx);

/*
 * pa_paged_attn_decode -- attention for 1..8 new query tokens per sequence
 * (decode, and speculative verification of up to 7 drafted tokens), all
 * query heads of one KV head processed together (GQA rows share each K/V tile).
 * The KV range of each sequence is split across CTAs (split-KV decoding); each
 * split keeps its own running max / sum and the splits are merged by
 * log-sum-exp in a second kernel on the same stream ("FlashDecoding" answer
 * of the interview Q&A page: split the long KV sequence over blocks, local
 * softmax per block, then a cross-block reduction).  A one-CTA kernel first orders the
 * sequences by page count, longest first, so that the CTAs of the longest
 * sequences start first and short ones fill the last wave; the order changes
 * no result.
 *   out          [T][H_q][d] written (same dtype as q)
 *   q            [T][H_q][d], T = cu_seqlens_q[B]
 *   cu_seqlens_q [B+1], each q_b in 1..8      context_lens [B], q_b <= ctx_b <= max_ctx
 *   max_ctx      host upper bound of context_lens (sizes the split grid and workspace)
 *   scale        multiplies Q K^T (normally 1/sqrt(d))
 *   workspace    >= pa_decode_workspace_bytes(T, B, H_q, H_kv, d, max_ctx) bytes; its
 *                first PA_STATUS_BYTES hold the status word, which this call resets
 *                to PA_OK on `stream`: its first kernel clears it before any other
 *                kernel of the call runs (a call with B = 0 or T = 0 launches nothing and
 *                clears it with a memset).  After a call that returns an error code
 *                it holds no result of that call.
 */
int pa_paged_attn_decode(void *out, const void *q, const void *key_cache, const void *value_cache,
                         int64_t num_blocks, const int32_t *block_tables, int max_blocks_per_seq,
                         const int32_t *cu_seqlens_q, const int32_t *context_lens, int B, int max_ctx, int64_t T,
                         int H_q, int H_kv, int d, float scale, pa_dtype dtype, void *workspace,
                         size_t workspace_bytes, void *stream);

/*
 * pa_paged_attn_decode_tree -- pa_paged_attn_decode for tree-attention
 * verification of speculative drafts (the interview Q&A page, speculative
 * decoding with a tree of drafts): the q_b new tokens of a sequence are the
 * nodes of a draft tree, and token t sees every cached key before the new
 * tokens plus new token j exactly when bit j of tree_mask[t] is set (its own
 * bit and its ancestors' in the usual case).  The chain mask, bits 0..i for
 * the i-th new token, is the causal verify of pa_paged_attn_decode.  Same
 * sizes, layouts, workspace and errors as pa_paged_attn_decode, plus:
 *   tree_mask  int32 [T], device memory; only bits 0 .. q_b - 1 are read.
 *              NULL -> PA_ERR_ARG.  A token that sees no key at all gets O = 0.
 */
int pa_paged_attn_decode_tree(void *out, const void *q, const void *key_cache, const void *value_cache,
                              int64_t num_blocks, const int32_t *block_tables, int max_blocks_per_seq,
                              const int32_t *cu_seqlens_q, const int32_t *context_lens, const int32_t *tree_mask,
                              int B, int max_ctx, int64_t T, int H_q, int H_kv, int d, float scale, pa_dtype dtype,
                              void *workspace, size_t workspace_bytes, void *stream);

/*
 * Shared-prefix decode -- pa_paged_attn_decode for batches in which groups of
 * sequences share the blocks of a common prompt prefix (page-level sharing of
 * one prompt prefix by several requests: iopencloud "大模型推理加速技术全景"
 * section 3.2; refcounted shared blocks on the PagedAttention section of the
 * fourth page).  The shared blocks are read once per (group, KV head) for all
 * the group's query rows, instead of once per sequence; each sequence's own
 * keys (after the prefix) are read as in pa_paged_attn_decode, and the two
 * partial softmaxes are merged by log-sum-exp.  The result is the attention of
 * pa_paged_attn_decode over the same tables (the pages only say that blocks
 * are shared; reading them once and merging is this library's reading of it).
 *
 * pa_shared_prefix_workspace_bytes -- workspace for these sizes (status word,
 * sequence order, per-sequence prefix lengths, the prefix partials and the
 * sequences' own split partials).  Pure host function; 0 for invalid sizes.
 */
size_t pa_shared_prefix_workspace_bytes(int64_t T, int B, int H_q, int H_kv, int d, int max_ctx, int n_groups,
                                        int max_prefix_blocks, int max_group_tokens);

/*
 * pa_paged_attn_decode_shared_prefix -- sizes, layouts and errors of
 * pa_paged_attn_decode, plus:
 *   n_groups           1 .. B + 1 (else PA_ERR_ARG)
 *   group_start        int32 [n_groups + 1], device: group v is the sequences
 *                      group_start[v] .. group_start[v+1]-1 (consecutive runs,
 *                      group_start[0] = 0, group_start[n_groups] = B; a
 *                      sequence sharing nothing is a group of its own with 0
 *                      prefix blocks)
 *   prefix_blocks      int32 [n_groups], device: the first prefix_blocks[v]
 *                      entries of the block tables of group v are the shared
 *                      blocks (whole blocks, before every new token)
 *   max_prefix_blocks  host bound on prefix_blocks (<= max_blocks_per_seq)
 *   max_group_tokens   host bound on the new tokens of one group (sizes the
 *                      prefix pass: rows = tokens x H_q/H_kv per KV head)
 * A sequence whose table does not start with its group leader's prefix
 * blocks, or whose new tokens start inside the prefix, is computed over its
 * own table alone (same result, no sharing).  Groups that are not a partition
 * of the sequences into consecutive runs, prefix_blocks outside
 * 0..max_blocks_per_seq, or a group with more new tokens than
 * max_group_tokens set PA_ERR_ARG in the status word (every sequence is then
 * computed alone).  Launches: a one-CTA plan kernel, the sequence order, the
 * attention kernel (prefix CTAs first, then the sequences'), the merge.
 * When the sharing saves little -- estimated from the host bounds as
 * (n - 1) / n x 16 max_prefix_blocks / max_ctx < 1/4 with n = B / n_groups --
 * the call runs the plain decode over the same tables instead (same result,
 * faster there; the groups are still checked).
 */
int pa_paged_attn_decode_shared_prefix(void *out, const void *q, const void *key_cache, const void *value_cache,
                                       int64_t num_blocks, const int32_t *block_tables, int max_blocks_per_seq,
                                       const int32_t *cu_seqlens_q, const int32_t *context_lens, int B, int max_ctx,
                                       int64_t T, int H_q, int H_kv, int d, float scale, pa_dtype dtype,
                                       const int32_t *group_start, const int32_t *prefix_blocks, int n_groups,
                                       int max_prefix_blocks, int max_group_tokens, void *workspace,
                                       size_t workspace_bytes, void *stream);

/*
 * FP8 (E4M3) KV cache -- an 8-bit cache with one float scale per stored row
 * (the FP8 KV-cache option of the serving page; FP8 with scaling on the
 * interview Q&A page): half the HBM bytes of a 16-bit cache per key.
 *   key_cache               uint8 [num_blocks][H_kv][16][d]: E4M3 codes
 *                           (OCP FP8: bias 7, 3 mantissa bits, no infinities,
 *                           largest finite 448)
 *   value_cache             uint8 [num_blocks][H_kv][d][16]: E4M3 codes,
 *                           transposed within each block (vLLM's value-cache
 *                           layout), so a slot's row is a column of its block
 *   key_scale, value_scale  float [num_blocks][H_kv][16]: the row's scale;
 *                           the stored value is code x scale (16-byte
 *                           aligned for the decode call, else PA_ERR_ALIGN)
 * A row's scale is fixed when the row is written (amax / 448), so nothing
 * stored is ever requantised.
 *
 * pa_kv_cache_write_fp8 -- pa_kv_cache_write into the FP8 cache: each new row
 * (16-bit, `dtype`) gets scale = amax / 448 (1 for an all-zero row) and codes
 * = the E4M3 value nearest to x / scale (ties to even, saturated at +-448),
 * both divisions IEEE round-to-nearest: bit-exact given the inputs.
 */
int pa_kv_cache_write_fp8(const void *k_new, const void *v_new, const int32_t *slot_mapping, int64_t T,
                          uint8_t *key_cache, uint8_t *value_cache, float *key_scale, float *value_scale,
                          int64_t num_blocks, int H_kv, int d, pa_dtype dtype, int32_t *status, void *stream);

/*
 * pa_paged_attn_decode_fp8 -- pa_paged_attn_decode over the FP8 cache: the
 * same sizes, workspace, scheduling and errors.  The codes are widened exactly
 * to `dtype` (the type of q and out; every E4M3 value is an f16 and a bf16
 * value) in registers, and the row scales multiply the fp32 scores (K) and
 * the probabilities before P V (V).  NULL scales -> PA_ERR_ARG.
 */
int pa_paged_attn_decode_fp8(void *out, const void *q, const uint8_t *key_cache, const uint8_t *value_cache,
                             const float *key_scale, const float *value_scale, int64_t num_blocks,
                             const int32_t *block_tables, int max_blocks_per_seq, const int32_t *cu_seqlens_q,
                             const int32_t *context_lens, int B, int max_ctx, int64_t T, int H_q, int H_kv, int d,
                             float scale, pa_dtype dtype, void *workspace, size_t workspace_bytes, void *stream);

/*
 * pa_paged_attn_decode_noalloc -- pa_paged_attn_decode without a caller workspace.
 * The pages have no counterpart: this is an interface for callers that may not
 * allocate device memory when they call, such as plugins inside an engine that
 * owns all device memory and forbids allocation while work is enqueued, or
 * latency-critical code that cannot take cudaMalloc's implicit synchronisation
 * or a possible allocation failure mid-step.  Same arguments, argument checks,
 * error codes and results as pa_paged_attn_decode, except:
 *   - the scratch (status word + split partials) is a fixed array of
 *     PA_DECODE_NOALLOC_SCRATCH_BYTES inside the library; every GPU that loads
 *     it holds that memory until the process exits;
 *   - sizes whose pa_decode_workspace_bytes(...) exceeds that maximum are
 *     rejected with PA_ERR_TOO_LARGE before anything is launched;
 *   - the first call on each device (with that device current) looks up the
 *     array's device address (cudaGetSymbolAddress) and keeps it: make that
 *     first call before any stream capture;
 *   - all calls on a device share the array and it keeps the last call's
 *     contents; the status word is cleared on `stream` by each call, as in
 *     pa_paged_attn_decode.
 *     Calls that overlap on the GPU (different streams without ordering) race;
 *   - status: optional device int32 (may be NULL) that receives the call's
 *     device status word (copied on `stream` after the kernels).
 * Nothing is allocated: no cudaMalloc, cudaFree or allocating library routine.
 */
#define PA_DECODE_NOALLOC_SCRATCH_BYTES (32u << 20)
int pa_paged_attn_decode_noalloc(void *out, const void *q, const void *key_cache, const void *value_cache,
                                 int64_t num_blocks, const int32_t *block_tables, int max_blocks_per_seq,
                                 const int32_t *cu_seqlens_q, const int32_t *context_lens, int B, int max_ctx,
                                 int64_t T, int H_q, int H_kv, int d, float scale, pa_dtype dtype, int32_t *status,
                                 void *stream);

/*
 * pa_prefill_workspace_bytes -- device workspace of pa_paged_attn_prefill:
 * the status word area (with the work counter of the tile scheduler), the
 * order in which the (query-tile pair, sequence) work is handed out (most K/V
 * tiles first), and, for calls whose work items would keep at most 3/4 of the
 * SMs busy (n_pairs * B * H_kv <= 3/4 of min(SMs, 160), n_pairs =
 * ceil(ceil(max_q_len / (128 / G)) / 2); a long-context chunk among few
 * items), the split schedule's per-SM starts and arrival counters and the
 * partial outputs (fp32) and log-sum-exps of two pieces per SM:
 * 2 * 160 * 2 * 128 * (d + 1) * 4 bytes more (42 MB at d = 128).  All of it
 * is written by the call itself.  Host function (reads the SM count of the
 * current device once).
 */
size_t pa_prefill_workspace_bytes(int B, int H_q, int H_kv, int d, int max_q_len);

/*
 * pa_paged_attn_prefill -- causal variable-length attention for prompts or
 * prompt chunks whose K/V were already written into the paged cache (by
 * pa_kv_cache_write).  Sequences are packed through cu_seqlens_q (no padding,
 * block-diagonal mask: the ragged-batching answer of the interview Q&A page);
 * a chunk with earlier context attends to that context too (chunked prefill).
 * Tiles of 128 queries x 128 keys run on the tcgen05 tensor cores with fp32
 * accumulators in tensor memory, fed by TMA from the cache blocks; the online
 * softmax of iopencloud section 2.2 runs between the two products.  Work
 * items too long for a balanced share of an SM are cut along the keys into
 * pieces on neighbouring SMs and their partial results merged by log-sum-exp
 * (the split-KV and merge of the FlashDecoding answer, interview Q&A page).
 *   out, q        [T][H_q][d]        cu_seqlens_q [B+1] (q_b >= 1)   context_lens [B]
 *   max_q_len     host upper bound of q_b;  max_ctx host upper bound of ctx_b
 *   workspace     >= pa_prefill_workspace_bytes(...) bytes; status word reset on stream
 *                 (by the call's first kernel, as in pa_paged_attn_decode).
 */
int pa_paged_attn_prefill(void *out, const void *q, const void *key_cache, const void *value_cache,
                          int64_t num_blocks, const int32_t *block_tables, int max_blocks_per_seq,
                          const int32_t *cu_seqlens_q, const int32_t *context_lens, int B, int max_q_len,
                          int max_ctx, int64_t T, int H_q, int H_kv, int d, float scale, pa_dtype dtype,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * pa_selftest_wait_timeout -- exercise the failure path that every kernel of
 * this library shares (no counterpart on the pages): one warp waits on an
 * mbarrier phase that nothing completes, bounded by `timeout_ns` of
 * %globaltimer, then records PA_ERR_TIMEOUT in *status (if it still holds
 * PA_OK) and returns; the context stays usable.  No fault, trap or endless
 * loop is involved.
 *   status      int32, device memory, owned by the caller (set it to PA_OK first)
 *   timeout_ns  1 .. 100,000,000 (0.1 s); else PA_ERR_ARG, nothing launched
 */
int pa_selftest_wait_timeout(int32_t *status, uint64_t timeout_ns, void *stream);

/*
 * pa_read_status -- copy the device status word at the start of `workspace`
 * (or any device int32 given to the write/copy calls) into *host_status.
 * This call synchronises `stream`.  Returns PA_OK or PA_ERR_CUDA.
 */
int pa_read_status(const void *workspace, int32_t *host_status, void *stream);

/*
 * pa_get_status -- the device status word at the start of `workspace` (or any
 * device int32 given to the write/copy calls), returned directly.  It first
 * waits for all work on the current device (every stream), so it suits a
 * check after a step, not the middle of a pipeline (pa_read_status waits for
 * one stream only).  Returns the word (PA_OK or a device-detected pa_status),
 * or PA_ERR_ARG for NULL, PA_ERR_CUDA if the runtime fails.
 */
int pa_get_status(const void *workspace);

/* pa_strerror -- static text for a pa_status value. */
const char *pa_strerror(int code);

/* pa_launch_count -- number of kernels this library has launched in this process. */
uint64_t pa_launch_count(void);

/* pa_version -- library ABI version (major * 100 + minor). */
int pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_ATTN_H */
