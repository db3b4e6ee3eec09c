// Host-side internals of libpagedattn shared between translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/paged_attn.h"

#include <nvtx3/nvToolsExt.h>

namespace pa {

// An NVTX range around one library call, named after its entry point, for timelines in the
// profilers; free when no profiler is attached (NVTX v3 is header-only and looks for a tool on
// first use).
struct CallRange {
    explicit CallRange(const char *name) { nvtxRangePushA(name); }
    ~CallRange() { nvtxRangePop(); }
    CallRange(const CallRange &) = delete;
    CallRange &operator=(const CallRange &) = delete;
};

// Counts every kernel launch of the library (pa_launch_count).
void count_launch(uint64_t n = 1);

// Launches `kern` as a programmatic dependent of the kernel before it on `stream`: its CTAs may be
// scheduled while that kernel still runs, and every kernel of the library calls griddep_wait()
// before it touches memory (a kernel launched the ordinary way before it, or any other stream
// operation, still completes first).  Hides the launch latency between kernels.
#ifndef PA_DEPENDENT_LAUNCH
#define PA_DEPENDENT_LAUNCH 1
#endif
template <typename... Params, typename... Args>
cudaError_t launch_dependent(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             Args &&...args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = PA_DEPENDENT_LAUNCH;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

// True when p is non-null and 16-byte aligned.
inline bool aligned16(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// 2-D tensor map over a paged cache [num_blocks][H_kv][16][d] viewed as
// rows of d elements; box = 64 elements x 16 rows, 128-byte swizzle.
// Returns PA_OK or PA_ERR_CUDA / PA_ERR_ARG.
int make_cache_tmap_fp8(CUtensorMap *map, const void *cache, int64_t num_blocks, int H_kv, int d);
int make_cache_tmap(CUtensorMap *map, const void *cache, int64_t num_blocks, int H_kv, int d, pa_dtype dtype);

// 2-D tensor map over FP8 row scales [num_blocks][H_kv][16] floats viewed as num_blocks * H_kv rows
// of 16; box = one row (the 16 scales of one (block, head) page), no swizzle.
int make_scale_tmap(CUtensorMap *map, const float *scale, int64_t num_blocks, int H_kv);

// 3-D tensor map over Q [T][H_q][d] for query tiles of `tok` tokens x G heads of one
// KV head: dims (d, H_q, T), box (64, G, tok), 128-byte swizzle.
int make_q_tmap(CUtensorMap *map, const void *q, int64_t T, int H_q, int d, int G, int tok, pa_dtype dtype);

// The size and shape checks of decode and prefill, before any pointer or workspace check:
// PA_OK, PA_ERR_ARG or PA_ERR_UNSUPPORTED.
struct AttnArgs;
int check_attn_shape(const AttnArgs &a, bool decode);

// Reset the status word at the start of a workspace on `stream`.
int reset_status(void *workspace, cudaStream_t stream);

int sm_count();

// ---- launchers (one per translation unit) --------------------------------------------

struct AttnArgs {
    void *out;
    const void *q;
    const void *key_cache;
    const void *value_cache;
    int64_t num_blocks;
    const int32_t *block_tables;
    int max_blocks;
    const int32_t *cu_seqlens_q;
    const int32_t *context_lens;
    int B;
    int max_q_len;
    int max_ctx;
    int64_t T;
    int H_q;
    int H_kv;
    int d;
    float scale;
    pa_dtype dtype;
    void *workspace;
    size_t workspace_bytes;
    cudaStream_t stream;
    const int32_t *tree_mask = nullptr;  // decode only: per-token visibility bits of the new tokens
    const float *key_scale = nullptr;    // FP8 cache (decode only): per-row scales, else nullptr
    const float *value_scale = nullptr;
    // shared-prefix decode (decode only): groups of consecutive sequences whose tables start
    // with the same prefix_blocks[v] blocks; nullptr = none
    const int32_t *group_start = nullptr;    // [n_groups + 1] device
    const int32_t *prefix_blocks = nullptr;  // [n_groups] device
    int n_groups = 0;
    int max_prefix_blocks = 0;  // host bound on prefix_blocks[v]
    int max_group_tokens = 0;   // host bound on the new tokens of one group
};

// Split-KV decode plan: pages per split and the number of splits.
struct DecodePlan {
    int split_pages;
    int max_splits;
    int row_groups;
};
DecodePlan decode_plan(int B, int H_q, int H_kv, int d, int max_ctx);
size_t decode_workspace_bytes(int64_t T, int B, int H_q, int H_kv, int d, int max_ctx);

// Shared-prefix decode plan: the decode plan of the sequences' own keys plus the prefix pass.
struct SharedPlan {
    DecodePlan own;
    int row_groups;          // per KV head: covers a sequence's rows and a group's rows
    int prefix_split_pages;  // pages per split of a prefix
    int prefix_slots;        // workspace slots of the prefix splits
};
SharedPlan shared_plan(int B, int H_q, int H_kv, int d, int max_ctx, int n_groups, int max_prefix_blocks,
                       int max_group_tokens);
size_t shared_workspace_bytes(int64_t T, int B, int H_q, int H_kv, int d, int max_ctx, int n_groups,
                              int max_prefix_blocks, int max_group_tokens);

// Sequence order by decreasing page count (one CTA, on `stream`): order[r] = the sequence of rank r.
// The workspace holds it right after the status area, seq_order_bytes(B) bytes.  The kernel is the
// first of its call and also clears the call's status word.
size_t seq_order_bytes(int B);
int launch_seq_order(const int32_t *context_lens, int B, int32_t *order, int32_t *status, cudaStream_t stream);
int launch_decode(const AttnArgs &a);
size_t prefill_workspace_bytes(int B, int H_q, int H_kv, int d, int max_q_len);
int launch_prefill(const AttnArgs &a);

}  // namespace pa
