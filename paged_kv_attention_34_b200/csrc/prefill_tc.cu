// Causal variable-length prefill over the paged KV cache on the tcgen05 tensor
// cores (sm_100a).
//
// What it computes: for every query row (token i of sequence b, query head h)
// O = softmax(scale * q K^T) V over keys 0 .. ctx_b - q_b + i, with K/V read
// through the block table (iopencloud "大模型推理加速技术全景" section 3.2).
// Sequences are packed by cu_seqlens (ragged batching answer of the interview
// Q&A page); a chunk with earlier context sees it (chunked prefill).
//
// Tiling (the online softmax of iopencloud section 2.2, on Blackwell units):
//   * a work item = (sequence, KV head, query tile).  A query tile holds
//     128 rows = 128/G tokens x the G query heads of the KV head, so every K/V
//     tile is shared by the whole GQA group;
//   * K/V tiles of 128 keys = 8 pages of 16 keys, each page fetched by TMA
//     (64-element x 16-row boxes, 128-byte swizzle) straight from its block;
//   * S = Q K^T: tcgen05.mma M=128 N=128, both operands in shared memory
//     (K-major), fp32 accumulator in TMEM (two S buffers);
//   * softmax: 4 warps, one thread per row (= TMEM lane) read S with
//     tcgen05.ld, keep the running max m and sum l in registers, write
//     P (16-bit) back over S in TMEM;
//   * O += P V: tcgen05.mma with A = P from TMEM, B = V in shared memory
//     (MN-major), fp32 accumulator in TMEM (two O buffers, one per item in
//     flight).  O is rescaled only when a row's max grows by more than 2^8
//     (exact: the same stale max is used for P and for l, and O / l is taken
//     once at the end);
//   * warp roles: warp 0 issues TMA (Q, K, V), warp 1 allocates TMEM and issues
//     the MMAs, warps 2-5 run the softmax and the epilogue.  Persistent CTAs,
//     one per SM, walk the items heaviest first (later query tiles see more keys).
// All waits are bounded; a wait that runs out records PA_ERR_TIMEOUT and the
// CTA winds down (its copies and MMAs in flight are waited for, TMEM freed).
#include <cmath>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "tc_device.cuh"

namespace pa {
namespace tcp {

constexpr int kRows = 128;     // query rows per tile (TMEM lanes)
constexpr int kKeys = 128;     // keys per K/V tile
constexpr int kStages = 2;     // K/V ring depth
constexpr int kThreads = 192;  // 6 warps
constexpr int kMaxTable = 1024;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct Params {
    const int32_t *block_tables;
    const int32_t *cu_seqlens;
    const int32_t *context_lens;
    void *out;
    int32_t *status;
    int64_t num_blocks;
    int64_t T;
    int max_blocks;
    int B, H_q, H_kv, G;
    int max_q_len, max_ctx;
    int tok_per_tile;   // 128 / G (floor)
    int rows_per_tile;  // tok_per_tile * G
    int n_qt_max;       // ceil(max_q_len / tok_per_tile)
    int n_items;        // n_qt_max * B * H_kv
    int oob_row;        // first row past the pool in the cache tensor map
    float scale_log2;
};

template <int D>
struct Smem {
    static constexpr int kKB = D / 64;                 // 128-byte column blocks
    static constexpr int kTile = kKB * kRows * 128;    // one 128-row x D tile (Q, K or V)
    static constexpr int kQ = 0;                       // 2 Q buffers
    static constexpr int kKV = 2 * kTile;              // kStages x (K tile, V tile)
    static constexpr int kTable = kKV + kStages * 2 * kTile;
    static constexpr int kBars = kTable + 4 * kMaxTable;
    // q_full[2] q_empty[2] kv_full[S] kv_empty[S] s_full[2] s_free[2] p_full[2] o_full[2] o_free[2] drain
    static constexpr int kNumBars = 2 + 2 + 2 * kStages + 2 + 2 + 2 + 2 + 2 + 1;
    static constexpr int kTmemSlot = kBars + 8 * kNumBars;
    static constexpr int kAbort = kTmemSlot + 8;
    static constexpr int kBytes = kAbort + 8;
    static constexpr int kAlloc = kBytes + 1024;
};

struct Item {
    int b, g, t_begin, n_tok, q0, qb, ctx, lim_hi, n_pages, n_kv;
};

__device__ __forceinline__ bool get_item(const Params &p, int it, Item &I, bool report)
{
    const int per = p.B * p.H_kv;
    const int qt = p.n_qt_max - 1 - it / per;
    const int rem = it % per;
    I.b = rem / p.H_kv;
    I.g = rem % p.H_kv;
    I.q0 = __ldg(p.cu_seqlens + I.b);
    const int q1 = __ldg(p.cu_seqlens + I.b + 1);
    I.qb = q1 - I.q0;
    I.ctx = __ldg(p.context_lens + I.b);
    const bool ok = I.qb >= 1 && I.ctx >= I.qb && I.qb <= p.max_q_len && I.ctx <= p.max_ctx &&
                    I.ctx <= p.max_blocks * 16 && q1 <= p.T && I.q0 >= 0;
    if (!ok) {
        if (report && qt == 0 && I.g == 0)
            set_status(p.status, PA_ERR_SEQ);
        return false;
    }
    I.t_begin = qt * p.tok_per_tile;
    if (I.t_begin >= I.qb)
        return false;
    I.n_tok = min(p.tok_per_tile, I.qb - I.t_begin);
    I.lim_hi = I.ctx - I.qb + I.t_begin + I.n_tok - 1;
    I.n_pages = I.lim_hi / 16 + 1;
    I.n_kv = I.lim_hi / kKeys + 1;
    return true;
}

// Bounded wait that also gives up once another role has aborted.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int32_t *status)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = globaltimer();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity))
                return true;
        if (*abort_flag)
            return false;
        if (globaltimer() - t0 > kWaitTimeoutNs) {
            *abort_flag = 1;
            set_status(status, PA_ERR_TIMEOUT);
            return false;
        }
    }
}

template <int D, bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
    pa_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v, const Params p)
{
    using L = Smem<D>;
    constexpr int KB = L::kKB;
    constexpr uint32_t kTmemCols = 512;
    constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + 128;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBars);
    uint64_t *q_full = bars, *q_empty = bars + 2;
    uint64_t *kv_full = bars + 4, *kv_empty = bars + 4 + kStages;
    uint64_t *s_full = bars + 4 + 2 * kStages, *s_free = s_full + 2, *p_full = s_full + 4;
    uint64_t *o_full = s_full + 6, *o_free = s_full + 8, *drain = s_full + 10;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kTmemSlot);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kAbort);
    int32_t *s_table = reinterpret_cast<int32_t *>(smem + L::kTable);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], 1);
            mbar_init(&s_full[i], 1);
            mbar_init(&s_free[i], 1);
            mbar_init(&p_full[i], 128);
            mbar_init(&o_full[i], 1);
            mbar_init(&o_free[i], 128);
        }
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&kv_full[i], 1);
            mbar_init(&kv_empty[i], 1);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&tmap_q);
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, kTmemCols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ===================== TMA producer =====================
        int kv_n = 0, n_it = 0, kv_issued = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < p.n_items && ok; it += gridDim.x) {
            Item I;
            if (!get_item(p, it, I, lane == 0))
                continue;
            const int32_t *table = p.block_tables + (int64_t)I.b * p.max_blocks;
            for (int i = lane; i < min(I.n_pages, kMaxTable); i += 32) {
                int pg = __ldg(table + i);
                if (pg < 0 || pg >= p.num_blocks) {
                    set_status(p.status, PA_ERR_BOUNDS);
                    pg = -1;
                }
                s_table[i] = pg;
            }
            __syncwarp();
            if (lane == 0) {
                const int qbuf = n_it & 1;
                ok = wait_bar(&q_empty[qbuf], ((n_it >> 1) & 1) ^ 1, abort_flag, p.status);
                if (ok) {
                    uint8_t *qs = smem + L::kQ + qbuf * L::kTile;
                    mbar_arrive_expect_tx(&q_full[qbuf], KB * p.rows_per_tile * 128);
                    for (int kb = 0; kb < KB; ++kb)
                        tc::tma_load_3d(qs + kb * kRows * 128, &tmap_q, kb * 64, I.g * p.G, I.q0 + I.t_begin,
                                        &q_full[qbuf]);
                }
                for (int j = 0; j < I.n_kv && ok; ++j) {
                    const int n = kv_n + j, s = n % kStages;
                    ok = wait_bar(&kv_empty[s], ((n / kStages) & 1) ^ 1, abort_flag, p.status);
                    if (!ok)
                        break;
                    uint8_t *ks = smem + L::kKV + s * 2 * L::kTile;
                    uint8_t *vs = ks + L::kTile;
                    mbar_arrive_expect_tx(&kv_full[s], 2 * L::kTile);
                    ++kv_issued;
                    for (int pg = 0; pg < 8; ++pg) {
                        const int pidx = j * 8 + pg;
                        int y = p.oob_row;  // pages past this item's range: zero-filled by TMA
                        if (pidx < I.n_pages) {
                            int id = pidx < kMaxTable ? s_table[pidx] : __ldg(table + pidx);
                            if (id < 0 || id >= p.num_blocks) {
                                set_status(p.status, PA_ERR_BOUNDS);
                                id = -1;
                            }
                            if (id >= 0)
                                y = (id * p.H_kv + I.g) * 16;
                        }
#pragma unroll
                        for (int kb = 0; kb < KB; ++kb) {
                            tma_load_2d(ks + kb * kRows * 128 + pg * 2048, &tmap_k, kb * 64, y, &kv_full[s]);
                            tma_load_2d(vs + kb * kRows * 128 + pg * 2048, &tmap_v, kb * 64, y, &kv_full[s]);
                        }
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            kv_issued = __shfl_sync(0xffffffffu, kv_issued, 0);
            __syncwarp();
            kv_n += I.n_kv;
            ++n_it;
        }
        if (lane == 0 && *abort_flag) {
            // let the copies already issued land before shared memory is released: the
            // last arming of stage s was its ((issued_s - 1))-th use
            for (int s = 0; s < kStages; ++s) {
                const int issued_s = kv_issued / kStages + (s < kv_issued % kStages ? 1 : 0);
                if (issued_s > 0)
                    mbar_wait(&kv_full[s], (issued_s - 1) & 1, kWaitTimeoutNs / 10);
            }
        }
    } else if (warp == 1) {
        // ===================== MMA issuer =====================
        if (lane == 0) {
            constexpr uint32_t idesc_qk = tc::idesc_f16(BF16, kRows, kKeys, false);
            constexpr uint32_t idesc_pv = tc::idesc_f16(BF16, kRows, D, true);
            int kv_n = 0, n_it = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < p.n_items && ok; it += gridDim.x) {
                Item I;
                if (!get_item(p, it, I, false))
                    continue;
                const int qbuf = n_it & 1, ob = n_it & 1;
                const uint32_t o_tmem = tmem + (ob ? kColO1 : kColO0);
                ok = wait_bar(&q_full[qbuf], (n_it >> 1) & 1, abort_flag, p.status);
                const uint32_t q_addr = smem_u32(smem + L::kQ + qbuf * L::kTile);
                for (int j = 0; j <= I.n_kv && ok; ++j) {
                    if (j < I.n_kv) {
                        const int n = kv_n + j, s = n % kStages, sb = n & 1;
                        ok = wait_bar(&kv_full[s], (n / kStages) & 1, abort_flag, p.status) &&
                             wait_bar(&s_free[sb], ((n >> 1) & 1) ^ 1, abort_flag, p.status);
                        if (!ok)
                            break;
                        tc::fence_after_sync();
                        const uint32_t k_addr = smem_u32(smem + L::kKV + s * 2 * L::kTile);
                        const uint32_t s_tmem = tmem + (sb ? kColS1 : kColS0);
#pragma unroll
                        for (int ks = 0; ks < D / 16; ++ks) {
                            const uint32_t off = (ks >> 2) * (kRows * 128) + (ks & 3) * 32;
                            tc::mma_ss(s_tmem, tc::desc_k_sw128(q_addr + off), tc::desc_k_sw128(k_addr + off),
                                       idesc_qk, ks > 0 ? 1u : 0u);
                        }
                        tc::commit(&s_full[sb]);
                        if (j == I.n_kv - 1)
                            tc::commit(&q_empty[qbuf]);
                    }
                    if (j >= 1) {
                        const int n = kv_n + j - 1, s = n % kStages, sb = n & 1;
                        ok = wait_bar(&p_full[sb], (n >> 1) & 1, abort_flag, p.status);
                        if (ok && j == 1)
                            ok = wait_bar(&o_free[ob], ((n_it >> 1) & 1) ^ 1, abort_flag, p.status);
                        if (!ok)
                            break;
                        tc::fence_after_sync();
                        const uint32_t v_addr = smem_u32(smem + L::kKV + s * 2 * L::kTile + L::kTile);
                        const uint32_t p_tmem = tmem + (sb ? kColS1 : kColS0);
#pragma unroll
                        for (int ks = 0; ks < kKeys / 16; ++ks)
                            tc::mma_ts(o_tmem, p_tmem + ks * 8, tc::desc_mn_sw128(v_addr + ks * 2048, kRows * 128),
                                       idesc_pv, (j > 1 || ks > 0) ? 1u : 0u);
                        tc::commit(&kv_empty[s]);
                        tc::commit(&s_free[sb]);
                        if (j == I.n_kv)
                            tc::commit(&o_full[ob]);
                    }
                }
                kv_n += I.n_kv;
                ++n_it;
            }
            // every MMA issued so far must be complete before TMEM is released
            tc::commit(drain);
            mbar_wait(drain, 0, kWaitTimeoutNs / 10);
        }
        __syncwarp();
    } else {
        // ===================== softmax + epilogue (warps 2-5) =====================
        const int sub = warp & 3;        // TMEM sub-partition of this warp
        const int r = sub * 32 + lane;   // query row of this thread in the tile
        const uint32_t lane_addr = static_cast<uint32_t>(sub * 32) << 16;
        const float sl2 = p.scale_log2;
        int kv_n = 0, n_it = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < p.n_items && ok; it += gridDim.x) {
            Item I;
            if (!get_item(p, it, I, false))
                continue;
            const int ob = n_it & 1;
            const uint32_t o_tmem = tmem + lane_addr + (ob ? kColO1 : kColO0);
            const int tl = r / p.G, gi = r % p.G;
            const bool row_valid = r < p.rows_per_tile && tl < I.n_tok;
            const int lim = row_valid ? I.ctx - I.qb + I.t_begin + tl : -1;
            float m = -INFINITY, l = 0.f;
            for (int j = 0; j < I.n_kv; ++j) {
                const int n = kv_n + j, sb = n & 1;
                ok = wait_bar(&s_full[sb], (n >> 1) & 1, abort_flag, p.status);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok)
                    break;
                tc::fence_after_sync();
                const uint32_t s_tmem = tmem + lane_addr + (sb ? kColS1 : kColS0);
                float s[kKeys];
                {
                    uint32_t raw[kKeys];
                    tc::ld128(s_tmem, raw);
#pragma unroll
                    for (int i = 0; i < kKeys; ++i)
                        s[i] = __uint_as_float(raw[i]);
                }
                const int key0 = j * kKeys;
                float mx = -INFINITY;
                if (key0 + kKeys - 1 <= lim) {
#pragma unroll
                    for (int c = 0; c < kKeys; ++c)
                        mx = fmaxf(mx, s[c]);
                } else {
#pragma unroll
                    for (int c = 0; c < kKeys; ++c) {
                        s[c] = (key0 + c <= lim) ? s[c] : -INFINITY;
                        mx = fmaxf(mx, s[c]);
                    }
                }
                const float mx_s = mx * sl2;  // scaled max (-inf stays -inf)
                float factor = 1.f;
                bool grow = false;
                if (j == 0) {
                    m = mx_s;
                } else if (mx_s > m + kRescaleThreshold) {
                    factor = fast_exp2(m - mx_s);
                    l *= factor;
                    m = mx_s;
                    grow = true;
                }
                if (__any_sync(0xffffffffu, grow)) {
                    // O must hold P_(n-1) V_(n-1) before it is rescaled
                    ok = wait_bar(&s_free[(n - 1) & 1], ((n - 1) >> 1) & 1, abort_flag, p.status);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok)
                        break;
                    tc::fence_after_sync();
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tc::ld32(o_tmem + c * 32, o);
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
                        tc::st32(o_tmem + c * 32, o);
                    }
                    tc::wait_st();
                }
                const float base = m == -INFINITY ? 0.f : m;
                uint32_t pk[kKeys / 2];
                float rs = 0.f;
#pragma unroll
                for (int c = 0; c < kKeys; c += 2) {
                    const float p0 = fast_exp2(fmaf(s[c], sl2, -base));
                    const float p1 = fast_exp2(fmaf(s[c + 1], sl2, -base));
                    rs += p0 + p1;
                    pk[c / 2] = pack2<BF16>(p0, p1);
                }
                l += rs;
                tc::st32(s_tmem, pk);
                tc::st32(s_tmem + 32, pk + 32);
                tc::wait_st();
                // keys past the context end in the sequence's last page may hold anything:
                // zero their V rows before P V reads them (P is 0 there, but 0 * NaN is NaN)
                if (j == I.n_kv - 1 && warp == 2) {
                    const int last_page = (I.ctx + 15) / 16 - 1;
                    const int pg = last_page - 8 * j;
                    if ((I.ctx & 15) && I.n_pages == last_page + 1 && pg >= 0 && pg < 8) {
                        const int s = n % kStages;
                        ok = wait_bar(&kv_full[s], (n / kStages) & 1, abort_flag, p.status);
                        if (ok) {
                            uint8_t *vs = smem + L::kKV + s * 2 * L::kTile + L::kTile;
                            const int r0 = I.ctx & 15;
                            const int nz = (16 - r0) * 8 * KB;  // 16-byte chunks to clear
                            for (int i = lane; i < nz; i += 32) {
                                const int kb = i / ((16 - r0) * 8);
                                const int rem = i % ((16 - r0) * 8);
                                const int row = pg * 16 + r0 + rem / 8;
                                *reinterpret_cast<uint4 *>(vs + kb * kRows * 128 + row * 128 + (rem & 7) * 16) =
                                    make_uint4(0, 0, 0, 0);
                            }
                            fence_proxy_async_smem();
                        }
                        ok = __all_sync(0xffffffffu, ok);
                        __syncwarp();
                    }
                }
                tc::fence_before_sync();
                mbar_arrive(&p_full[sb]);
                if (!ok)
                    break;
            }
            if (!ok)
                break;
            // epilogue: O / l -> out
            ok = wait_bar(&o_full[ob], (n_it >> 1) & 1, abort_flag, p.status);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok)
                break;
            tc::fence_after_sync();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            uint8_t *orow = static_cast<uint8_t *>(p.out) +
                            ((int64_t)(I.q0 + I.t_begin + tl) * p.H_q + I.g * p.G + gi) * (D * 2);
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tc::ld32(o_tmem + c * 32, o);
                if (row_valid) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint4 v;
                        v.x = pack2<BF16>(__uint_as_float(o[i + 0]) * inv, __uint_as_float(o[i + 1]) * inv);
                        v.y = pack2<BF16>(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
                        v.z = pack2<BF16>(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv);
                        v.w = pack2<BF16>(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv);
                        *reinterpret_cast<uint4 *>(orow + (c * 32 + i) * 2) = v;
                    }
                }
            }
            tc::fence_before_sync();
            mbar_arrive(&o_free[ob]);
            kv_n += I.n_kv;
            ++n_it;
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1)
        tc::tmem_dealloc(tmem, kTmemCols);
}

// ---- host ---------------------------------------------------------------------------------------

template <int D, bool BF16>
static int run(const AttnArgs &a)
{
    using L = Smem<D>;
    const int G = a.H_q / a.H_kv;
    if (G > kRows)
        return PA_ERR_UNSUPPORTED;
    Params p{};
    p.block_tables = a.block_tables;
    p.cu_seqlens = a.cu_seqlens_q;
    p.context_lens = a.context_lens;
    p.out = a.out;
    p.status = static_cast<int32_t *>(a.workspace);
    p.num_blocks = a.num_blocks;
    p.T = a.T;
    p.max_blocks = a.max_blocks;
    p.B = a.B;
    p.H_q = a.H_q;
    p.H_kv = a.H_kv;
    p.G = G;
    p.max_q_len = a.max_q_len;
    p.max_ctx = a.max_ctx;
    p.tok_per_tile = kRows / G;
    p.rows_per_tile = p.tok_per_tile * G;
    p.n_qt_max = (a.max_q_len + p.tok_per_tile - 1) / p.tok_per_tile;
    const int64_t items = (int64_t)p.n_qt_max * a.B * a.H_kv;
    if (items > (int64_t(1) << 30) || a.T > (int64_t(1) << 31) - 256)
        return PA_ERR_UNSUPPORTED;
    p.n_items = static_cast<int>(items);
    p.oob_row = static_cast<int>(a.num_blocks * a.H_kv * 16);
    p.scale_log2 = a.scale * 1.4426950408889634f;

    CUtensorMap tq, tk, tv;
    int rc = make_q_tmap(&tq, a.q, a.T, a.H_q, D, G, p.tok_per_tile, a.dtype);
    if (rc == PA_OK)
        rc = make_cache_tmap(&tk, a.key_cache, a.num_blocks, a.H_kv, D, a.dtype);
    if (rc == PA_OK)
        rc = make_cache_tmap(&tv, a.value_cache, a.num_blocks, a.H_kv, D, a.dtype);
    if (rc != PA_OK)
        return rc;

    auto kern = pa_prefill_tc_kernel<D, BF16>;
    static uint64_t configured = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return PA_ERR_CUDA;
    const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
    if (!bit || !(configured & bit)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) != cudaSuccess)
            return PA_ERR_CUDA;
        configured |= bit;
    }
    const int grid = static_cast<int>(std::min<int64_t>(items, sm_count()));
    kern<<<grid, kThreads, L::kAlloc, a.stream>>>(tq, tk, tv, p);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace tcp

int launch_prefill(const AttnArgs &a)
{
    if (a.d == 128)
        return a.dtype == PA_BF16 ? tcp::run<128, true>(a) : tcp::run<128, false>(a);
    return a.dtype == PA_BF16 ? tcp::run<64, true>(a) : tcp::run<64, false>(a);
}

}  // namespace pa
