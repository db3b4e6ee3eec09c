// pa_paged_attn_decode_noalloc: split-KV decode whose scratch (the status word
// and the per-split partial outputs / log-sum-exps) lives in a fixed array
// inside the library instead of a caller-provided workspace.
//
// It exists for callers that must not allocate device memory at call time:
// plugins inside a host engine that owns every byte of device memory through
// its own pool and forbids raw allocations while work is being enqueued, and
// latency-critical code that cannot accept cudaMalloc's implicit device
// synchronisation or its possible failure in the middle of a step.
//
// The array is a file-scope __device__ object: every GPU that loads this part
// of the library holds PA_DECODE_NOALLOC_SCRATCH_BYTES of it until the process
// exits.  Host code cannot use the array's name as a device address (on the
// host it names a stand-in object), so the first call on each device, with that
// device current, looks the address up with cudaGetSymbolAddress and keeps it.
// Do that first call before any stream capture.  All calls on a device share
// the one array and it keeps the last call's contents: the status word is
// cleared on the stream before every launch (the partials need no clearing;
// every split that the merge reads is written first by its own CTA), and calls
// whose work overlaps on the GPU (different streams, no ordering) race on it.
#include <mutex>

#include "pa_internal.h"

namespace pa {
namespace {

static __device__ __align__(256) uint8_t g_decode_scratch[PA_DECODE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up once per device).
int scratch_address(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return PA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices)
        return PA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p)
            return PA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return PA_OK;
}

}  // namespace
}  // namespace pa

extern "C" int pa_paged_attn_decode_noalloc(void *out, const void *q, const void *key_cache,
                                            const void *value_cache, int64_t num_blocks,
                                            const int32_t *block_tables, int max_blocks_per_seq,
                                            const int32_t *cu_seqlens_q, const int32_t *context_lens, int B,
                                            int max_ctx, int64_t T, int H_q, int H_kv, int d, float scale,
                                            pa_dtype dtype, int32_t *status, void *stream)
{
    pa::CallRange range(__func__);
    // the same size and shape checks as pa_paged_attn_decode, so both return the same code
    pa::AttnArgs a{out, q, key_cache, value_cache, num_blocks, block_tables, max_blocks_per_seq, cu_seqlens_q,
                   context_lens, B, 8, max_ctx, T, H_q, H_kv, d, scale, dtype, nullptr, 0,
                   static_cast<cudaStream_t>(stream)};
    const int shape_rc = pa::check_attn_shape(a, true);
    if (shape_rc != PA_OK)
        return shape_rc;
    const size_t need = pa_decode_workspace_bytes(T, B, H_q, H_kv, d, max_ctx);
    if (need == 0)
        return PA_ERR_ARG;
    if (need > PA_DECODE_NOALLOC_SCRATCH_BYTES)
        return PA_ERR_TOO_LARGE;
    if (status && (reinterpret_cast<uintptr_t>(status) & 3u))
        return PA_ERR_ALIGN;
    void *scratch = nullptr;
    int rc = pa::scratch_address(&scratch);
    if (rc != PA_OK)
        return rc;
    rc = pa_paged_attn_decode(out, q, key_cache, value_cache, num_blocks, block_tables, max_blocks_per_seq,
                              cu_seqlens_q, context_lens, B, max_ctx, T, H_q, H_kv, d, scale, dtype, scratch,
                              PA_DECODE_NOALLOC_SCRATCH_BYTES, stream);
    if (rc == PA_OK && status &&
        cudaMemcpyAsync(status, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice,
                        static_cast<cudaStream_t>(stream)) != cudaSuccess)
        rc = PA_ERR_CUDA;
    return rc;
}
