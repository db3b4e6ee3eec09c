// kv_cache_write and kv_block_copy: the two byte-moving steps of the paged
// KV cache.  Both are pure HBM streams; each thread moves 16-byte vectors,
// consecutive threads touch consecutive 16-byte chunks of one (block, head,
// row) so every warp reads and writes whole 128-byte lines.
//
// Cache layout [num_blocks][H_kv][16][d]: the PagedAttention block pool of
// iopencloud "大模型推理加速技术全景" section 3.2 (16-token pages, per-request
// page table); copy-on-write of refcounted blocks follows the zhihu roofline
// page, "显存管理".
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

// One item = one 16-byte chunk of one (token, head) row, for K and for V.
// CH = chunks per row = d * 2 / 16.
template <int CH>
__global__ void __launch_bounds__(256) kv_cache_write_kernel(const uint4 *__restrict__ k_new,
                                                             const uint4 *__restrict__ v_new,
                                                             const int32_t *__restrict__ slot_mapping, int64_t T,
                                                             uint4 *__restrict__ key_cache,
                                                             uint4 *__restrict__ value_cache, int64_t num_blocks,
                                                             int H_kv, int32_t *status)
{
    const int64_t items = T * H_kv * CH;
    const int64_t n_slots = num_blocks * 16;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < items; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = i / CH;  // t * H_kv + h
        const int c = static_cast<int>(i - row * CH);
        const int64_t t = row / H_kv;
        const int h = static_cast<int>(row - t * H_kv);
        const int64_t slot = __ldg(slot_mapping + t);
        if (slot < 0)
            continue;  // padding token
        if (slot >= n_slots) {
            set_status(status, PA_ERR_BOUNDS);
            continue;
        }
        const int64_t blk = slot >> 4, off = slot & 15;
        const int64_t dst = ((blk * H_kv + h) * 16 + off) * CH + c;
        const uint4 kv = ldg_nc_v4(k_new + i);
        const uint4 vv = ldg_nc_v4(v_new + i);
        key_cache[dst] = kv;
        value_cache[dst] = vv;
    }
}

// One item = one 16-byte chunk of one block (all heads, 16 rows), K and V.
__global__ void __launch_bounds__(256) kv_block_copy_kernel(uint4 *__restrict__ key_cache,
                                                            uint4 *__restrict__ value_cache, int64_t num_blocks,
                                                            int64_t chunks_per_block,
                                                            const int32_t *__restrict__ pairs, int64_t n,
                                                            int32_t *status)
{
    const int64_t items = n * chunks_per_block;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < items; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t p = i / chunks_per_block;
        const int64_t c = i - p * chunks_per_block;
        const int64_t src = __ldg(pairs + 2 * p), dst = __ldg(pairs + 2 * p + 1);
        if (src < 0 || dst < 0 || src >= num_blocks || dst >= num_blocks) {
            set_status(status, PA_ERR_BOUNDS);
            continue;
        }
        const uint4 kv = ldg_nc_v4(key_cache + src * chunks_per_block + c);
        const uint4 vv = ldg_nc_v4(value_cache + src * chunks_per_block + c);
        key_cache[dst * chunks_per_block + c] = kv;
        value_cache[dst * chunks_per_block + c] = vv;
    }
}

// One item = one 16-byte chunk of one block (all heads, 16 rows), K and V, between the device cache
// and a pool of blocks in page-locked host memory (read and written over the host link through its
// device-mapped address).
__global__ void __launch_bounds__(256) kv_block_swap_kernel(uint4 *__restrict__ key_cache,
                                                            uint4 *__restrict__ value_cache, int64_t num_blocks,
                                                            uint4 *__restrict__ host_key, uint4 *__restrict__ host_value,
                                                            int64_t host_blocks, int64_t chunks_per_block,
                                                            const int32_t *__restrict__ pairs, int64_t n, int to_host,
                                                            int32_t *status)
{
    const int64_t items = n * chunks_per_block;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < items; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t p = i / chunks_per_block;
        const int64_t c = i - p * chunks_per_block;
        const int64_t dev = __ldg(pairs + 2 * p), hst = __ldg(pairs + 2 * p + 1);
        if (dev < 0 || hst < 0 || dev >= num_blocks || hst >= host_blocks) {
            set_status(status, PA_ERR_BOUNDS);
            continue;
        }
        const int64_t di = dev * chunks_per_block + c, hi = hst * chunks_per_block + c;
        if (to_host) {
            const uint4 kv = ldg_nc_v4(key_cache + di);
            const uint4 vv = ldg_nc_v4(value_cache + di);
            host_key[hi] = kv;
            host_value[hi] = vv;
        } else {
            const uint4 kv = host_key[hi];
            const uint4 vv = host_value[hi];
            key_cache[di] = kv;
            value_cache[di] = vv;
        }
    }
}

static int grid_for(int64_t items, int threads)
{
    const int64_t need = (items + threads - 1) / threads;
    const int64_t cap = (int64_t)sm_count() * 8;  // enough resident warps to saturate HBM
    return static_cast<int>(need < cap ? need : cap);
}

}  // namespace pa

using namespace pa;

extern "C" int pa_kv_cache_write(const void *k_new, const void *v_new, const int32_t *slot_mapping, int64_t T,
                                 void *key_cache, void *value_cache, int64_t num_blocks, int H_kv, int d,
                                 pa_dtype dtype, int32_t *status, void *stream)
{
    if (T < 0 || num_blocks < 1 || H_kv < 1)
        return PA_ERR_ARG;
    if (dtype != PA_F16 && dtype != PA_BF16)
        return PA_ERR_ARG;
    if (d != 64 && d != 128)
        return PA_ERR_UNSUPPORTED;
    if (T == 0)
        return PA_OK;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(key_cache) || !aligned16(value_cache))
        return PA_ERR_ALIGN;
    if (!aligned4(slot_mapping) || (status && !aligned4(status)))
        return PA_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int threads = 256;
    if (d == 128) {
        const int64_t items = T * H_kv * 16;
        kv_cache_write_kernel<16><<<grid_for(items, threads), threads, 0, s>>>(
            static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new), slot_mapping, T,
            static_cast<uint4 *>(key_cache), static_cast<uint4 *>(value_cache), num_blocks, H_kv, status);
    } else {
        const int64_t items = T * H_kv * 8;
        kv_cache_write_kernel<8><<<grid_for(items, threads), threads, 0, s>>>(
            static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new), slot_mapping, T,
            static_cast<uint4 *>(key_cache), static_cast<uint4 *>(value_cache), num_blocks, H_kv, status);
    }
    count_launch();
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" int pa_kv_block_copy(void *key_cache, void *value_cache, int64_t num_blocks, int H_kv, int d,
                                pa_dtype dtype, const int32_t *pairs, int64_t n, int32_t *status, void *stream)
{
    if (n < 0 || num_blocks < 1 || H_kv < 1)
        return PA_ERR_ARG;
    if (dtype != PA_F16 && dtype != PA_BF16)
        return PA_ERR_ARG;
    if (d != 64 && d != 128)
        return PA_ERR_UNSUPPORTED;
    if (n == 0)
        return PA_OK;
    if (!aligned16(key_cache) || !aligned16(value_cache) || !aligned4(pairs) || (status && !aligned4(status)))
        return PA_ERR_ALIGN;
    const int64_t chunks = (int64_t)H_kv * 16 * d * 2 / 16;
    const int threads = 256;
    kv_block_copy_kernel<<<grid_for(n * chunks, threads), threads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint4 *>(key_cache), static_cast<uint4 *>(value_cache), num_blocks, chunks, pairs, n, status);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// The device-mapped address of page-locked host memory at `p`, or nullptr when `p` is not
// page-locked host memory that the device can address (pageable memory, device memory, NULL).
static void *mapped_host(void *p)
{
    if (!p)
        return nullptr;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (at.type != cudaMemoryTypeHost || !at.devicePointer)
        return nullptr;
    return at.devicePointer;
}

extern "C" int pa_kv_block_swap(void *key_cache, void *value_cache, int64_t num_blocks, void *host_key,
                                void *host_value, int64_t host_blocks, int H_kv, int d, pa_dtype dtype,
                                const int32_t *pairs, int64_t n, int direction, int32_t *status, void *stream)
{
    if (n < 0 || num_blocks < 1 || host_blocks < 1 || H_kv < 1)
        return PA_ERR_ARG;
    if (dtype != PA_F16 && dtype != PA_BF16)
        return PA_ERR_ARG;
    if (direction != PA_SWAP_OUT && direction != PA_SWAP_IN)
        return PA_ERR_ARG;
    if (d != 64 && d != 128)
        return PA_ERR_UNSUPPORTED;
    if (n == 0)
        return PA_OK;
    // the host pools must be page-locked memory the device can address: anything else is refused
    // here, before any launch
    void *hk = mapped_host(host_key), *hv = mapped_host(host_value);
    if (!hk || !hv)
        return PA_ERR_ARG;
    if (!aligned16(key_cache) || !aligned16(value_cache) || !aligned16(hk) || !aligned16(hv) || !aligned4(pairs) ||
        (status && !aligned4(status)))
        return PA_ERR_ALIGN;
    const int64_t chunks = (int64_t)H_kv * 16 * d * 2 / 16;
    const int threads = 256;
    kv_block_swap_kernel<<<grid_for(n * chunks, threads), threads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint4 *>(key_cache), static_cast<uint4 *>(value_cache), num_blocks, static_cast<uint4 *>(hk),
        static_cast<uint4 *>(hv), host_blocks, chunks, pairs, n, direction == PA_SWAP_OUT ? 1 : 0, status);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
