// Declarations shared by the decode kernels of libpagedattn (the mma.sync rows kernel and the
// tcgen05 rows kernel): their parameters, the attention modes and the work unit of a CTA.
#pragma once

#include <stdint.h>

#include "pa_device.cuh"

namespace pa {

constexpr int kRowsPerCta = 64;
constexpr int kPagesPerStage = 4;
constexpr int kMaxTablePages = 256;  // page ids of one split (split_pages <= this)
constexpr int kThreads = 128;

// What the rows of a decode CTA see: causal (the new tokens in order), a tree-verification mask
// over the new tokens, or the shared-prefix pass (causal sequence CTAs plus prefix CTAs whose
// rows see every prefix key).
constexpr int kModeCausal = 0;
constexpr int kModeTree = 1;
constexpr int kModeShared = 2;

struct RowsParams {
    const void *q;
    void *out;
    const int32_t *block_tables;
    const int32_t *cu_seqlens;
    const int32_t *context_lens;
    float *ws_o;    // [max_splits][T][H_q][D] normalised partial outputs
    float *ws_lse;  // [max_splits][T][H_q] log2-sum-exp of the scaled scores
    const int32_t *order;  // [B] sequences by decreasing page count: grid z -> sequence
    const int32_t *tree;   // [T] tree verification: bit j = the token sees new token j; nullptr = causal
    const float *k_scale;  // FP8 cache: [num_blocks][H_kv][16] scale of every stored K row
    const float *v_scale;  // ... and V row
    // shared-prefix decode
    const int32_t *group_start;    // [n_groups + 1] the sequences of group v: [group_start[v], group_start[v+1])
    const int32_t *prefix_blocks;  // [n_groups] blocks shared by group v at the head of its tables
    int32_t *seq_prefix;           // [B] prefix blocks of each sequence's group (set by the plan kernel)
    int n_groups;
    int prefix_split_pages;  // pages per split of a prefix
    int prefix_slots;        // workspace slots of the prefix splits (the sequences' own splits follow)
    int32_t *status;
    int64_t num_blocks;
    int64_t T;
    int max_blocks;
    int B, H_q, H_kv, G;
    int max_ctx;
    int max_q_len;
    int n_rg;         // row groups per (sequence, KV head): of kRowsPerCta rows, or the tcgen05 kernel's rows
    int split_pages;  // pages per split
    float scale_log2;  // scale * log2(e)
};

__device__ __forceinline__ int seq_of_token(const int32_t *cu, int B, int64_t t)
{
    int lo = 0, hi = B;  // cu[lo] <= t < cu[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(cu + mid) <= t)
            lo = mid;
        else
            hi = mid;
    }
    return lo;
}

// Sequence checks shared by the attention and merge kernels.
__device__ __forceinline__ bool seq_ok(int qb, int ctx, const RowsParams &p, int64_t q1)
{
    return qb >= 1 && ctx >= qb && qb <= p.max_q_len && ctx <= p.max_ctx && ctx <= p.max_blocks * 16 && q1 <= p.T;
}

// The keys one decode CTA covers, before its row group and split are applied.
struct DecodeUnit {
    int q0, q1;        // the CTA's new tokens [q0, q1)
    int ctx;           // keys of its sequence (of the shared prefix, for a prefix CTA)
    int page_base;     // first page of the keys its splits cover
    int sp;            // pages per split
    int slot0;         // workspace slot of its first split
    bool prefix_cta;   // shared-prefix pass: the rows of a group against the group's shared blocks
    const int32_t *table;
};

// Which keys the CTA at blockIdx.z covers.  Shared-prefix mode: grid z < n_groups is the prefix of
// group z -- every token of the group's sequences against the group's shared blocks, read once for
// all of them (no mask: the prefix precedes every new token); z >= n_groups is one sequence's own
// keys, from the first block after its group's prefix.  Other modes: z is one sequence (through
// the longest-first order).  False when the CTA has no work; an inconsistent sequence is reported
// (PA_ERR_SEQ) by one of its CTAs.
template <int MODE>
__device__ __forceinline__ bool decode_unit(const RowsParams &p, int tid, DecodeUnit &u)
{
    u.page_base = 0;
    u.sp = p.split_pages;
    u.slot0 = 0;
    u.prefix_cta = false;
    if constexpr (MODE == kModeShared) {
        const int sp_pre = p.prefix_split_pages;
        if (static_cast<int>(blockIdx.z) < p.n_groups) {
            // the group's arrays were checked by the plan kernel (status); clamp them here so a
            // bad call stays inside its buffers
            const int v = blockIdx.z;
            const int s0 = min(max(__ldg(p.group_start + v), 0), p.B);
            const int s1 = min(max(__ldg(p.group_start + v + 1), s0), p.B);
            if (s0 >= s1)
                return false;
            u.q0 = __ldg(p.cu_seqlens + s0);
            u.q1 = max(__ldg(p.cu_seqlens + s1), u.q0);
            u.ctx = min(max(__ldg(p.prefix_blocks + v), 0), min(p.max_blocks, p.prefix_slots * sp_pre)) * 16;
            u.table = p.block_tables + (int64_t)s0 * p.max_blocks;
            u.sp = p.prefix_split_pages;
            u.prefix_cta = true;
            if (u.q0 < 0 || u.q1 > p.T || u.ctx == 0)
                return false;
            return true;
        }
        const int b = __ldg(p.order + (blockIdx.z - p.n_groups));
        u.q0 = __ldg(p.cu_seqlens + b);
        u.q1 = __ldg(p.cu_seqlens + b + 1);
        u.ctx = __ldg(p.context_lens + b);
        if (!seq_ok(u.q1 - u.q0, u.ctx, p, u.q1)) {
            if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0)
                set_status(p.status, PA_ERR_SEQ);
            return false;
        }
        u.table = p.block_tables + (int64_t)b * p.max_blocks;
        u.page_base = min(max(__ldg(p.seq_prefix + b), 0), (u.ctx - (u.q1 - u.q0)) / 16);
        u.slot0 = p.prefix_slots;
        return true;
    } else {
        const int b = __ldg(p.order + blockIdx.z);
        u.q0 = __ldg(p.cu_seqlens + b);
        u.q1 = __ldg(p.cu_seqlens + b + 1);
        u.ctx = __ldg(p.context_lens + b);
        if (!seq_ok(u.q1 - u.q0, u.ctx, p, u.q1)) {
            if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0)
                set_status(p.status, PA_ERR_SEQ);
            return false;
        }
        u.table = p.block_tables + (int64_t)b * p.max_blocks;
        return true;
    }
}

// The tcgen05 rows kernel (rows_tc.cu) for wide row groups: the rows one CTA holds for G query
// heads per KV head and at most max_tokens new tokens per sequence (a multiple of G, at most 128;
// 0 when G is too large), and its launch for the grid (splits, H_kv x row groups, sequences
// [+ prefix groups]) of `rp` (rp.n_rg row groups of rows_per_cta rows).
int rows_tc_rows_per_cta(int G, int max_tokens);
int launch_rows_tc(const RowsParams &rp, const CUtensorMap &tk, const CUtensorMap &tv, int d, pa_dtype dtype,
                   int mode, int rows_per_cta, dim3 grid, cudaStream_t stream);

}  // namespace pa
