// Device-side building blocks shared by the kernels of libpagedattn:
// mbarriers with bounded waits, TMA tile loads, ldmatrix, warp-level MMA,
// 16-bit packing and the status word.  sm_100a only.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/paged_attn.h"

namespace pa {

// A bounded wait gives up after this long and reports PA_ERR_TIMEOUT.
constexpr uint64_t kWaitTimeoutNs = 1000000000ull;  // 1 s

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Record the first error of a launch; later errors do not overwrite it.
__device__ __forceinline__ void set_status(int32_t *status, int code)
{
    if (status)
        atomicCAS(reinterpret_cast<int *>(status), PA_OK, code);
}

// ---- mbarrier -----------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking: has phase `parity` of `bar` completed?
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of `bar` to complete; false if it has not after `timeout_ns`.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t timeout_ns = kWaitTimeoutNs)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = globaltimer();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity))
                return true;
        if (globaltimer() - t0 > timeout_ns)
            return false;
    }
}

// ---- programmatic dependent launch ---------------------------------------------------
// griddep_wait: in a kernel started by launch_dependent, returns once the kernel before it on the
// stream has completed and its writes are visible (at once for a kernel launched the ordinary
// way).  griddep_release: lets the kernel after this one on the stream be scheduled early.

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---- TMA ------------------------------------------------------------------------

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *m)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 2-D tiled load of one box into shared memory; completion is counted on `bar`.
// x (innermost, elements) must keep x * 2 bytes a multiple of 16.
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *m, int x, int y, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// ---- ldmatrix / mma.sync -----------------------------------------------------------

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D(16x8, f32) += A(16x16) * B(16x8), A row-major, B column-major, 16-bit inputs.
template <bool BF16>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    if constexpr (BF16) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    } else {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
}

// ---- numerics -------------------------------------------------------------------------

// 2^x on the SFU (ex2.approx; 2^-inf = +0).
__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---- packed fp32 pairs (f32x2 instructions of sm_100) ----------------------------------

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void f2_unpack(uint64_t v, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// max of three floats in one instruction
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Two floats -> packed 16-bit pair (round to nearest even); `lo` in the low half.
template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    if constexpr (BF16) {
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&v);
    } else {
        __half2 v = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&v);
    }
}

// Four floats -> four 16-bit values stored with one 8-byte store.
template <bool BF16>
__device__ __forceinline__ void store4(void *dst, float a, float b, float c, float d)
{
    uint2 v;
    v.x = pack2<BF16>(a, b);
    v.y = pack2<BF16>(c, d);
    *reinterpret_cast<uint2 *>(dst) = v;
}

// One 32-byte store of 8 words; `dst` must be 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void *dst, const uint32_t *w)
{
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(w[0]), "r"(w[1]),
                 "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// ---- longest-first ordering -------------------------------------------------------------------

constexpr int kOrderKeys = 4096;
constexpr int kOrderThreads = 1024;
constexpr int kOrderSmall = 256;  // up to this many elements: ranks by comparison

// One CTA of kOrderThreads threads, all of which call this: order[r] = the element of rank r when
// the n elements are sorted by decreasing key_of(e) in [0, kOrderKeys) (a counting sort; elements
// with equal keys in arbitrary order; up to kOrderSmall elements, ranks by comparison, equal keys
// by index).
template <class KeyOf>
__device__ void order_by_key_desc(int n, KeyOf key_of, int32_t *order)
{
    const int tid = threadIdx.x;
    if (n <= kOrderSmall) {
        // few elements: each one's rank by comparison with all of them (ties by index), one barrier
        __shared__ int key[kOrderSmall];
        if (tid < n)
            key[tid] = key_of(tid);
        __syncthreads();
        if (tid < n) {
            const int k = key[tid];
            int r = 0;
            for (int u = 0; u < n; ++u) {
                const int ku = key[u];
                r += (ku > k || (ku == k && u < tid)) ? 1 : 0;
            }
            order[r] = tid;
        }
        return;
    }
    __shared__ int cnt[kOrderKeys];
    __shared__ int warp_tot[kOrderThreads / 32];
    const int lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < kOrderKeys; i += kOrderThreads)
        cnt[i] = 0;
    __syncthreads();
    for (int e = tid; e < n; e += kOrderThreads)
        atomicAdd(&cnt[key_of(e)], 1);
    __syncthreads();
    // exclusive prefix sum in descending key order: thread t owns keys kOrderKeys-1-PER*t downwards
    constexpr int PER = kOrderKeys / kOrderThreads;
    int v[PER], run = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        v[i] = cnt[kOrderKeys - 1 - (tid * PER + i)];
        run += v[i];
    }
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o)
            incl += y;
    }
    if (lane == 31)
        warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int t = warp_tot[lane];
        int ti = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, ti, o);
            if (lane >= o)
                ti += y;
        }
        warp_tot[lane] = ti - t;  // exclusive over warps
    }
    __syncthreads();
    int base = warp_tot[warp] + incl - run;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        cnt[kOrderKeys - 1 - (tid * PER + i)] = base;
        base += v[i];
    }
    __syncthreads();
    for (int e = tid; e < n; e += kOrderThreads)
        order[atomicAdd(&cnt[key_of(e)], 1)] = e;
}

}  // namespace pa
