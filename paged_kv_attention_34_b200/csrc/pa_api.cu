// Host side of the C ABI: argument validation, TMA tensor maps, the status
// word and small utilities.  No device memory is allocated here or anywhere
// else in the library.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <mutex>

#include "pa_internal.h"

namespace pa {

static std::atomic<uint64_t> g_launches{0};

void count_launch(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

int sm_count()
{
    static int cached = -1;
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    if (cached < 0) {
        int dev = 0, n = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;  // B200
        cached = n;
    }
    return cached;
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

int make_cache_tmap(CUtensorMap *map, const void *cache, int64_t num_blocks, int H_kv, int d, pa_dtype dtype)
{
    auto fn = encode_fn();
    if (!fn)
        return PA_ERR_CUDA;
    const int64_t rows = num_blocks * H_kv * 16;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
    cuuint32_t box[2] = {64, 16};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                    const_cast<void *>(cache), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? PA_OK : PA_ERR_CUDA;
}

// FP8 cache: the same rows of d one-byte codes; one box = a page (16 rows x d bytes), no swizzle.
int make_cache_tmap_fp8(CUtensorMap *map, const void *cache, int64_t num_blocks, int H_kv, int d)
{
    auto fn = encode_fn();
    if (!fn)
        return PA_ERR_CUDA;
    const int64_t rows = num_blocks * H_kv * 16;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(d)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(d), 16};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(cache), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? PA_OK : PA_ERR_CUDA;
}

int make_scale_tmap(CUtensorMap *map, const float *scale, int64_t num_blocks, int H_kv)
{
    auto fn = encode_fn();
    if (!fn)
        return PA_ERR_CUDA;
    cuuint64_t dims[2] = {16, static_cast<cuuint64_t>(num_blocks * H_kv)};
    cuuint64_t strides[1] = {16 * sizeof(float)};
    cuuint32_t box[2] = {16, 1};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(scale), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? PA_OK : PA_ERR_CUDA;
}

int make_q_tmap(CUtensorMap *map, const void *q, int64_t T, int H_q, int d, int G, int tok, pa_dtype dtype)
{
    auto fn = encode_fn();
    if (!fn)
        return PA_ERR_CUDA;
    if (G < 1 || G > 256 || tok < 1 || tok > 256)
        return PA_ERR_UNSUPPORTED;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H_q), static_cast<cuuint64_t>(T)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H_q) * d * 2};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(tok)};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                    const_cast<void *>(q), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? PA_OK : PA_ERR_CUDA;
}

int reset_status(void *workspace, cudaStream_t stream)
{
    return cudaMemsetAsync(workspace, 0, sizeof(int32_t), stream) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// Size and shape checks shared by decode and prefill (no pointer is looked at).  Largest TMA
// row coordinate used is (num_blocks + 1) * H_kv * 16 (one past the pool marks a bad block id),
// which must stay below 2^31.
int check_attn_shape(const AttnArgs &a, bool decode)
{
    if (a.B < 0 || a.T < 0 || a.H_q < 1 || a.H_kv < 1 || a.num_blocks < 1 || a.max_blocks < 1 || a.max_ctx < 0)
        return PA_ERR_ARG;
    if (a.dtype != PA_F16 && a.dtype != PA_BF16)
        return PA_ERR_ARG;
    if (a.d != 64 && a.d != 128)
        return PA_ERR_UNSUPPORTED;
    if (a.H_q % a.H_kv != 0)
        return PA_ERR_UNSUPPORTED;
    if ((a.num_blocks + 1) * (int64_t)a.H_kv * 16 >= (int64_t(1) << 31))
        return PA_ERR_UNSUPPORTED;
    if (!decode && a.max_q_len < 1)
        return PA_ERR_ARG;
    return PA_OK;
}

// Every host-side check of decode and prefill: sizes and shapes, then workspace and pointers.
static int check_attn(const AttnArgs &a, bool decode)
{
    const int rc = check_attn_shape(a, decode);
    if (rc != PA_OK)
        return rc;
    if (!a.workspace)
        return PA_ERR_WORKSPACE;
    if (!aligned16(a.workspace))
        return PA_ERR_ALIGN;
    if (a.B == 0 || a.T == 0)
        return PA_OK;
    if (!aligned16(a.out) || !aligned16(a.q) || !aligned16(a.key_cache) || !aligned16(a.value_cache))
        return PA_ERR_ALIGN;
    if (!aligned4(a.block_tables) || !aligned4(a.cu_seqlens_q) || !aligned4(a.context_lens))
        return PA_ERR_ALIGN;
    if (!std::isfinite(a.scale))
        return PA_ERR_ARG;
    return PA_OK;
}

}  // namespace pa

using namespace pa;

extern "C" size_t pa_decode_workspace_bytes(int64_t T, int B, int H_q, int H_kv, int d, int max_ctx)
{
    if (T < 0 || B < 0 || H_q < 1 || H_kv < 1 || (d != 64 && d != 128) || max_ctx < 0 || H_q % H_kv)
        return 0;
    return decode_workspace_bytes(T, B, H_q, H_kv, d, max_ctx);
}

extern "C" int pa_paged_attn_decode(void *out, const void *q, const void *key_cache, const void *value_cache,
                                    int64_t num_blocks, const int32_t *block_tables, int max_blocks_per_seq,
                                    const int32_t *cu_seqlens_q, const int32_t *context_lens, int B, int max_ctx,
                                    int64_t T, int H_q, int H_kv, int d, float scale, pa_dtype dtype,
                                    void *workspace, size_t workspace_bytes, void *stream)
{
    CallRange range(__func__);
    AttnArgs a{out, q, key_cache, value_cache, num_blocks, block_tables, max_blocks_per_seq, cu_seqlens_q,
               context_lens, B, 8, max_ctx, T, H_q, H_kv, d, scale, dtype, workspace, workspace_bytes,
               static_cast<cudaStream_t>(stream)};
    int rc = check_attn(a, true);
    if (rc != PA_OK)
        return rc;
    if (workspace_bytes < decode_workspace_bytes(T, B, H_q, H_kv, d, max_ctx))
        return PA_ERR_WORKSPACE;
    if (B == 0 || T == 0)
        return reset_status(workspace, a.stream);  // nothing to launch
    return launch_decode(a);  // its first kernel clears the status word
}

extern "C" int pa_paged_attn_decode_tree(void *out, const void *q, const void *key_cache, const void *value_cache,
                                         int64_t num_blocks, const int32_t *block_tables, int max_blocks_per_seq,
                                         const int32_t *cu_seqlens_q, const int32_t *context_lens,
                                         const int32_t *tree_mask, int B, int max_ctx, int64_t T, int H_q, int H_kv,
                                         int d, float scale, pa_dtype dtype, void *workspace, size_t workspace_bytes,
                                         void *stream)
{
    CallRange range(__func__);
    AttnArgs a{out, q, key_cache, value_cache, num_blocks, block_tables, max_blocks_per_seq, cu_seqlens_q,
               context_lens, B, 8, max_ctx, T, H_q, H_kv, d, scale, dtype, workspace, workspace_bytes,
               static_cast<cudaStream_t>(stream), tree_mask};
    int rc = check_attn(a, true);
    if (rc != PA_OK)
        return rc;
    if (B > 0 && T > 0) {
        if (!tree_mask)
            return PA_ERR_ARG;
        if (!aligned4(tree_mask))
            return PA_ERR_ALIGN;
    }
    if (workspace_bytes < decode_workspace_bytes(T, B, H_q, H_kv, d, max_ctx))
        return PA_ERR_WORKSPACE;
    if (B == 0 || T == 0)
        return reset_status(workspace, a.stream);  // nothing to launch
    return launch_decode(a);  // its first kernel clears the status word
}

extern "C" size_t pa_shared_prefix_workspace_bytes(int64_t T, int B, int H_q, int H_kv, int d, int max_ctx,
                                                    int n_groups, int max_prefix_blocks, int max_group_tokens)
{
    if (T < 0 || B < 0 || H_q < 1 || H_kv < 1 || (d != 64 && d != 128) || max_ctx < 0 || H_q % H_kv ||
        n_groups < 1 || max_prefix_blocks < 0 || max_group_tokens < 0)
        return 0;
    return shared_workspace_bytes(T, B, H_q, H_kv, d, max_ctx, n_groups, max_prefix_blocks, max_group_tokens);
}

extern "C" int pa_paged_attn_decode_shared_prefix(void *out, const void *q, const void *key_cache,
                                                  const void *value_cache, int64_t num_blocks,
                                                  const int32_t *block_tables, int max_blocks_per_seq,
                                                  const int32_t *cu_seqlens_q, const int32_t *context_lens, int B,
                                                  int max_ctx, int64_t T, int H_q, int H_kv, int d, float scale,
                                                  pa_dtype dtype, const int32_t *group_start,
                                                  const int32_t *prefix_blocks, int n_groups, int max_prefix_blocks,
                                                  int max_group_tokens, void *workspace, size_t workspace_bytes,
                                                  void *stream)
{
    CallRange range(__func__);
    AttnArgs a{out, q, key_cache, value_cache, num_blocks, block_tables, max_blocks_per_seq, cu_seqlens_q,
               context_lens, B, 8, max_ctx, T, H_q, H_kv, d, scale, dtype, workspace, workspace_bytes,
               static_cast<cudaStream_t>(stream)};
    a.group_start = group_start;
    a.prefix_blocks = prefix_blocks;
    a.n_groups = n_groups;
    a.max_prefix_blocks = max_prefix_blocks;
    a.max_group_tokens = max_group_tokens;
    int rc = check_attn(a, true);
    if (rc != PA_OK)
        return rc;
    if (n_groups < 1 || n_groups > B + 1 || max_prefix_blocks < 0 || max_prefix_blocks > max_blocks_per_seq ||
        max_group_tokens < 0 || (int64_t)max_group_tokens > T)
        return PA_ERR_ARG;
    if (B > 0 && T > 0) {
        if (!group_start || !prefix_blocks)
            return PA_ERR_ARG;
        if (!aligned4(group_start) || !aligned4(prefix_blocks))
            return PA_ERR_ALIGN;
    }
    if (workspace_bytes <
        shared_workspace_bytes(T, B, H_q, H_kv, d, max_ctx, n_groups, max_prefix_blocks, max_group_tokens))
        return PA_ERR_WORKSPACE;
    if (B == 0 || T == 0)
        return reset_status(workspace, a.stream);  // nothing to launch
    return launch_decode(a);  // its first kernel clears the status word
}

extern "C" int pa_paged_attn_decode_fp8(void *out, const void *q, const uint8_t *key_cache,
                                        const uint8_t *value_cache, const float *key_scale, const float *value_scale,
                                        int64_t num_blocks, const int32_t *block_tables, int max_blocks_per_seq,
                                        const int32_t *cu_seqlens_q, const int32_t *context_lens, int B, int max_ctx,
                                        int64_t T, int H_q, int H_kv, int d, float scale, pa_dtype dtype,
                                        void *workspace, size_t workspace_bytes, void *stream)
{
    CallRange range(__func__);
    AttnArgs a{out, q, key_cache, value_cache, num_blocks, block_tables, max_blocks_per_seq, cu_seqlens_q,
               context_lens, B, 8, max_ctx, T, H_q, H_kv, d, scale, dtype, workspace, workspace_bytes,
               static_cast<cudaStream_t>(stream), nullptr, key_scale, value_scale};
    int rc = check_attn(a, true);
    if (rc != PA_OK)
        return rc;
    if (B > 0 && T > 0) {
        if (!key_scale || !value_scale)
            return PA_ERR_ARG;
        if (!aligned16(key_scale) || !aligned16(value_scale))
            return PA_ERR_ALIGN;
    }
    if (workspace_bytes < decode_workspace_bytes(T, B, H_q, H_kv, d, max_ctx))
        return PA_ERR_WORKSPACE;
    if (B == 0 || T == 0)
        return reset_status(workspace, a.stream);  // nothing to launch
    return launch_decode(a);  // its first kernel clears the status word
}

extern "C" size_t pa_prefill_workspace_bytes(int B, int H_q, int H_kv, int d, int max_q_len)
{
    if (B < 0 || H_q < 1 || H_kv < 1 || (d != 64 && d != 128) || max_q_len < 0 || H_q % H_kv)
        return 0;
    return prefill_workspace_bytes(B, H_q, H_kv, d, max_q_len);
}

extern "C" int pa_paged_attn_prefill(void *out, const void *q, const void *key_cache, const void *value_cache,
                                     int64_t num_blocks, const int32_t *block_tables, int max_blocks_per_seq,
                                     const int32_t *cu_seqlens_q, const int32_t *context_lens, int B,
                                     int max_q_len, int max_ctx, int64_t T, int H_q, int H_kv, int d, float scale,
                                     pa_dtype dtype, void *workspace, size_t workspace_bytes, void *stream)
{
    CallRange range(__func__);
    AttnArgs a{out, q, key_cache, value_cache, num_blocks, block_tables, max_blocks_per_seq, cu_seqlens_q,
               context_lens, B, max_q_len, max_ctx, T, H_q, H_kv, d, scale, dtype, workspace, workspace_bytes,
               static_cast<cudaStream_t>(stream)};
    int rc = check_attn(a, false);
    if (rc != PA_OK)
        return rc;
    if (workspace_bytes < pa_prefill_workspace_bytes(B, H_q, H_kv, d, max_q_len))
        return PA_ERR_WORKSPACE;
    if (B == 0 || T == 0)
        return reset_status(workspace, a.stream);  // nothing to launch
    return launch_prefill(a);  // its first kernel clears the status word
}

extern "C" int pa_read_status(const void *workspace, int32_t *host_status, void *stream)
{
    CallRange range(__func__);
    if (!workspace || !host_status)
        return PA_ERR_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(host_status, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return PA_ERR_CUDA;
    return cudaStreamSynchronize(s) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" int pa_get_status(const void *workspace)
{
    CallRange range(__func__);
    if (!workspace)
        return PA_ERR_ARG;
    int32_t word = 0;
    if (cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpy(&word, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
        return PA_ERR_CUDA;
    return word;
}

extern "C" const char *pa_strerror(int code)
{
    switch (code) {
    case PA_OK: return "success";
    case PA_ERR_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported shape (head size, GQA ratio, q_len or pool size)";
    case PA_ERR_ALIGN: return "pointer not 16-byte aligned";
    case PA_ERR_WORKSPACE: return "workspace missing or too small";
    case PA_ERR_CUDA: return "CUDA runtime error";
    case PA_ERR_TIMEOUT: return "device wait on an asynchronous copy timed out";
    case PA_ERR_BOUNDS: return "block id, slot or length out of range (item skipped)";
    case PA_ERR_SEQ: return "inconsistent cu_seqlens_q / context_lens (sequence skipped)";
    case PA_ERR_TOO_LARGE: return "sizes need more scratch than the allocation-free decode entry point holds";
    default: return "unknown status";
    }
}

extern "C" uint64_t pa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

extern "C" int pa_version(void) { return 100; }
