// kv_cache_write and kv_block_copy: the two byte-moving steps of the paged
// KV cache.  Both are pure HBM streams; each thread moves 16-byte vectors,
// consecutive threads touch consecutive 16-byte chunks of one (block, head,
// row) so every warp reads and writes whole 128-byte lines.
//
// Cache layout [num_blocks][H_kv][16][d]: the PagedAttention block pool of
// iopencloud "大模型推理加速技术全景" section 3.2 (16-token pages, per-request
// page table); copy-on-write of refcounted blocks follows the zhihu roofline
// page, "显存管理".
#include <cuda_fp8.h>

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
    // a programmatic dependent of the kernel before it on the stream: wait for it before any access
    griddep_wait();
    griddep_release();
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
    // a programmatic dependent of the kernel before it on the stream: wait for it before any access
    griddep_wait();
    griddep_release();
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
    // a programmatic dependent of the kernel before it on the stream: wait for it before any access
    griddep_wait();
    griddep_release();
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

// FP8 cache write: one warp per (token, KV head) row of K and of V.  The row's scale is
// amax / 448 (1 for an all-zero row) and every value becomes the E4M3 code nearest to value /
// scale (saturated at +-448); both divisions are IEEE round-to-nearest, so the codes follow from
// the 16-bit inputs alone.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) kv_cache_write_fp8_kernel(const void *__restrict__ k_new,
                                                                 const void *__restrict__ v_new,
                                                                 const int32_t *__restrict__ slot_mapping, int64_t T,
                                                                 int H_kv, uint8_t *__restrict__ key_cache,
                                                                 uint8_t *__restrict__ value_cache, float *key_scale,
                                                                 float *value_scale, int64_t num_blocks, int32_t *status)
{
    // a programmatic dependent of the kernel before it on the stream: wait for it before any access
    griddep_wait();
    griddep_release();
    constexpr int VPL = D / 32;  // values per lane (2 or 4)
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); r < T * H_kv; r += warps) {
        const int64_t t = r / H_kv;
        const int h = static_cast<int>(r % H_kv);
        const int64_t slot = __ldg(slot_mapping + t);
        if (slot < 0)
            continue;  // padding token
        if (slot >= num_blocks * 16) {
            if (lane == 0)
                set_status(status, PA_ERR_BOUNDS);
            continue;
        }
        const int64_t row = ((slot / 16) * H_kv + h) * 16 + slot % 16;
#pragma unroll
        for (int kv = 0; kv < 2; ++kv) {
            const uint16_t *src = static_cast<const uint16_t *>(kv ? v_new : k_new) + (t * H_kv + h) * D + lane * VPL;
            float x[VPL], amax = 0.f;
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const uint16_t u = src[i];
                if constexpr (BF16)
                    x[i] = __bfloat162float(__ushort_as_bfloat16(u));
                else
                    x[i] = __half2float(__ushort_as_half(u));
                amax = fmaxf(amax, fabsf(x[i]));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            const float sc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
            uint8_t code[VPL];
#pragma unroll
            for (int i = 0; i < VPL; i += 2) {
                const float2 qv = make_float2(__fdiv_rn(x[i], sc), __fdiv_rn(x[i + 1], sc));
                const __nv_fp8x2_storage_t pr = __nv_cvt_float2_to_fp8x2(qv, __NV_SATFINITE, __NV_E4M3);
                code[i] = static_cast<uint8_t>(pr & 0xffu);
                code[i + 1] = static_cast<uint8_t>(pr >> 8);
            }
            if (kv) {
                // V codes are transposed within the block ([d][16 slots]): this row is a column
                uint8_t *dst = value_cache + ((slot / 16) * H_kv + h) * 16 * D + (lane * VPL) * 16 + slot % 16;
#pragma unroll
                for (int i = 0; i < VPL; ++i)
                    dst[i * 16] = code[i];
            } else {
                uint8_t *dst = key_cache + row * D + lane * VPL;
                if constexpr (VPL == 4)
                    *reinterpret_cast<uint32_t *>(dst) =
                        code[0] | (code[1] << 8) | (code[2] << 16) | (uint32_t(code[3]) << 24);
                else
                    *reinterpret_cast<uint16_t *>(dst) = static_cast<uint16_t>(code[0] | (code[1] << 8));
            }
            if (lane == 0)
                (kv ? value_scale : key_scale)[row] = sc;
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
    CallRange range(__func__);
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
    cudaError_t e;
    if (d == 128) {
        const int64_t items = T * H_kv * 16;
        e = launch_dependent(kv_cache_write_kernel<16>, dim3(grid_for(items, threads)), dim3(threads), 0, s,
                             static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new), slot_mapping, T,
                             static_cast<uint4 *>(key_cache), static_cast<uint4 *>(value_cache), num_blocks, H_kv,
                             status);
    } else {
        const int64_t items = T * H_kv * 8;
        e = launch_dependent(kv_cache_write_kernel<8>, dim3(grid_for(items, threads)), dim3(threads), 0, s,
                             static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new), slot_mapping, T,
                             static_cast<uint4 *>(key_cache), static_cast<uint4 *>(value_cache), num_blocks, H_kv,
                             status);
    }
    count_launch();
    const cudaError_t e2 = cudaGetLastError();
    return e == cudaSuccess && e2 == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" int pa_kv_block_copy(void *key_cache, void *value_cache, int64_t num_blocks, int H_kv, int d,
                                pa_dtype dtype, const int32_t *pairs, int64_t n, int32_t *status, void *stream)
{
    CallRange range(__func__);
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
    const cudaError_t e = launch_dependent(kv_block_copy_kernel, dim3(grid_for(n * chunks, threads)), dim3(threads), 0,
                                           static_cast<cudaStream_t>(stream), static_cast<uint4 *>(key_cache),
                                           static_cast<uint4 *>(value_cache), num_blocks, chunks, pairs, n, status);
    count_launch();
    const cudaError_t e2 = cudaGetLastError();
    return e == cudaSuccess && e2 == cudaSuccess ? PA_OK : PA_ERR_CUDA;
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
    CallRange range(__func__);
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
    const cudaError_t e = launch_dependent(
        kv_block_swap_kernel, dim3(grid_for(n * chunks, threads)), dim3(threads), 0, static_cast<cudaStream_t>(stream),
        static_cast<uint4 *>(key_cache), static_cast<uint4 *>(value_cache), num_blocks, static_cast<uint4 *>(hk),
        static_cast<uint4 *>(hv), host_blocks, chunks, pairs, n, direction == PA_SWAP_OUT ? 1 : 0, status);
    count_launch();
    const cudaError_t e2 = cudaGetLastError();
    return e == cudaSuccess && e2 == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" int pa_kv_cache_write_fp8(const void *k_new, const void *v_new, const int32_t *slot_mapping, int64_t T,
                                     uint8_t *key_cache, uint8_t *value_cache, float *key_scale, float *value_scale,
                                     int64_t num_blocks, int H_kv, int d, pa_dtype dtype, int32_t *status, void *stream)
{
    CallRange range(__func__);
    if (T < 0 || num_blocks < 1 || H_kv < 1)
        return PA_ERR_ARG;
    if (dtype != PA_F16 && dtype != PA_BF16)
        return PA_ERR_ARG;
    if (d != 64 && d != 128)
        return PA_ERR_UNSUPPORTED;
    if (T == 0)
        return PA_OK;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(key_cache) || !aligned16(value_cache) ||
        !aligned4(key_scale) || !aligned4(value_scale) || !aligned4(slot_mapping) || (status && !aligned4(status)))
        return PA_ERR_ALIGN;
    const int threads = 256;
    const int64_t warps_needed = T * H_kv;
    const int grid = grid_for(warps_needed * 32, threads);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
#define PA_LAUNCH_WRITE8(DD, BB)                                                                                   \
    launch_dependent(kv_cache_write_fp8_kernel<DD, BB>, dim3(grid), dim3(threads), 0, s, k_new, v_new, slot_mapping, T, \
                     H_kv, key_cache, value_cache, key_scale, value_scale, num_blocks, status)
    cudaError_t e;
    if (d == 128)
        e = dtype == PA_BF16 ? PA_LAUNCH_WRITE8(128, true) : PA_LAUNCH_WRITE8(128, false);
    else
        e = dtype == PA_BF16 ? PA_LAUNCH_WRITE8(64, true) : PA_LAUNCH_WRITE8(64, false);
#undef PA_LAUNCH_WRITE8
    count_launch();
    const cudaError_t e2 = cudaGetLastError();
    return e == cudaSuccess && e2 == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
