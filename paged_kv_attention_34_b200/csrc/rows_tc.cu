// Paged decode attention for wide row groups on the tcgen05 tensor cores (sm_100a).
//
// What it computes is what pa_attn_rows_kernel computes for the same grid: for one (sequence,
// KV head, row group, split) the rows are the G query heads x the new tokens of the sequence
// (of a shared-prefix group, for a prefix CTA), the keys those of the split's pages, read through
// the block table (iopencloud "大模型推理加速技术全景" section 3.2); each split keeps its own
// running max and sum (online softmax, section 2.2 there) and writes either the final rows or a
// normalised partial with its log2-sum-exp for the split merge ("FlashDecoding" answer of the
// interview Q&A page).  Rows see keys causally, through a tree-verification mask, or -- prefix
// CTAs -- every prefix key.
//
// Why a second kernel: with 16 or more rows per KV head (verify rows of speculative decoding, the
// rows of a whole group on a shared prefix) the mma.sync kernel spends most of its time on the
// matrix products of every page.  Here they go to the tensor core:
//   * rows on the MMA's M side (M = 128 = the TMEM lanes; G x tokens rows, the rest padding) and
//     Q staged once by TMA (one 3-D box per 64 columns: tokens x G heads);
//   * keys in tiles of 64 = 4 pages, each page one TMA box per 64 columns (128-byte swizzle)
//     straight from its block, K and V of a tile in one stage of a ring of 2-4 stages (as deep as
//     two CTAs per SM allow once Q has its rows);
//   * S = Q K^T (M = 128, N = 64, fp32 in TMEM) double-buffered: S(j+1) is computed while the
//     softmax of tile j runs, so the softmax never waits for a product;
//   * one thread per row (warps 4-7, TMEM lane = row; a warp without a row sits out) loads its S
//     row, masks, keeps m and l, and writes P (16-bit) back over S; O += P V with P from TMEM and
//     V (MN-major) from shared memory, fp32 in TMEM; O is rescaled only when a row's max grows by
//     more than 2^8 (after the products already issued for that row have completed);
//   * warp 0 loads Q and feeds the K tiles, warp 2 the V tiles (lanes 0-3 one page each; K of a
//     tile is released once its S is complete, V once its P V is), warp 1 issues the MMAs (one
//     thread).
// TMEM: S0, S1 (64 columns each) and O (d columns) in 256 columns; up to 113 KB of shared memory:
// two CTAs per SM.  Every wait is bounded; a wait that runs out records PA_ERR_TIMEOUT and the CTA
// winds down (copies and products in flight are waited for, TMEM freed).
#include <algorithm>
#include <cmath>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "rows_common.cuh"
#include "tc_device.cuh"

namespace pa {
namespace rtc {

constexpr int kRows = 128;                 // TMEM lanes = rows of a CTA
constexpr int kTileKeys = 64;              // keys per K/V tile
constexpr int kTilePages = kTileKeys / 16;
constexpr int kThreads = 256;              // warps 0, 2 TMA, warp 1 MMA, warps 4-7 softmax and epilogue
constexpr uint32_t kTmemCols = 256;        // S0, S1, O
constexpr uint32_t kColO = 128;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

constexpr int kMaxStages = 4;
// Shared memory of one CTA: two must fit on an SM.
constexpr int kSmemPerCta = 113 * 1024;

// Layout (1024-byte aligned base): Q as kKB column blocks of q_rows rows x 128 B (q_rows = the
// CTA's rows rounded up to a whole 8-row swizzle atom; the MMA's padding rows beyond them read
// whatever follows, which only ever reaches rows no thread stores), then the ring of `stages`
// stages (K tile then V tile), then barriers and flags.
template <int D>
struct Smem {
    static constexpr int kKB = D / 64;                   // 128-byte column blocks
    static constexpr int kBlk = kTileKeys * 128;         // one column block of a K or V tile
    static constexpr int kTile = kKB * kBlk;             // a K (or V) tile
    // q_full, k_full, v_full, k_empty, v_empty [kMaxStages each], s_full[2], p_full[2], pv_done,
    // o_done, land, drain
    static constexpr int kNumBars = 1 + 4 * kMaxStages + 2 + 2 + 4;
    static constexpr int kTail = 8 * kNumBars + 16;      // barriers, TMEM slot, abort flag
    __host__ __device__ static constexpr int q_rows(int rows) { return (rows + 7) / 8 * 8; }
    __host__ __device__ static constexpr int ring(int rows) { return kKB * q_rows(rows) * 128; }
    __host__ __device__ static constexpr int bars(int rows, int stages) { return ring(rows) + stages * 2 * kTile; }
    __host__ __device__ static constexpr int alloc(int rows, int stages) { return bars(rows, stages) + kTail + 1024; }
    // the deepest ring (at most kMaxStages) that keeps two CTAs on an SM
    static int stages_for(int rows)
    {
        int st = kMaxStages;
        while (st > 2 && alloc(rows, st) > kSmemPerCta)
            --st;
        return st;
    }
};

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

__device__ __forceinline__ uint32_t full_par(int k) { return static_cast<uint32_t>(k & 1); }
__device__ __forceinline__ uint32_t free_par(int k) { return static_cast<uint32_t>((k & 1) ^ 1); }

template <int D, bool BF16, int MODE>
__global__ void __launch_bounds__(kThreads, 2)
    pa_attn_rows_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                           const __grid_constant__ CUtensorMap tmap_v, const RowsParams p, int rows_per_cta,
                           int n_st, int oob_row)
{
    using L = Smem<D>;
    constexpr int KB = L::kKB;
    const int q_blk = L::q_rows(rows_per_cta) * 128;  // bytes of one Q column block
    const int ring_off = L::ring(rows_per_cta);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *tail = smem + L::bars(rows_per_cta, n_st);
    uint64_t *bars = reinterpret_cast<uint64_t *>(tail);
    uint64_t *q_full = bars;
    uint64_t *k_full = bars + 1;               // [n_st] K of a tile landed
    uint64_t *v_full = k_full + kMaxStages;    // [n_st] V of a tile landed (tail rows cleared)
    uint64_t *k_empty = v_full + kMaxStages;   // [n_st] S of the tile complete
    uint64_t *v_empty = k_empty + kMaxStages;  // [n_st] P V of the tile complete
    uint64_t *s_full = v_empty + kMaxStages;   // [2] S buffer b computed
    uint64_t *p_full = s_full + 2;             // [2] P written into S buffer b (128 arrivals)
    uint64_t *pv_done = p_full + 2;            // one completion per O += P V
    uint64_t *o_done = pv_done + 1;            // every product of the CTA complete
    uint64_t *land = o_done + 1;               // the tile with the context end landed (V rows not yet cleared)
    uint64_t *drain = land + 1;                // wind-down after an abort
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tail + 8 * L::kNumBars);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tail + 8 * L::kNumBars + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    griddep_wait();     // the sequence order comes from the kernel before this one
    griddep_release();  // the split merge after this kernel may be scheduled (it waits for this grid)

    // ---- the CTA's rows and keys (uniform over the CTA: early returns precede every barrier) ----
    const int split = blockIdx.x;
    // the heaviest row groups (the last tokens, which see the most keys) are dispatched first
    const int g = blockIdx.y / p.n_rg, rg = p.n_rg - 1 - static_cast<int>(blockIdx.y % p.n_rg);
    DecodeUnit u;
    if (!decode_unit<MODE>(p, tid, u))
        return;
    const int qb = u.q1 - u.q0;
    const int G = p.G;
    const int R = G * qb;
    const int row0 = rg * rows_per_cta;
    if (row0 >= R)
        return;
    const int rows_here = min(rows_per_cta, R - row0);
    const bool see_all = MODE == kModeTree || u.prefix_cta;
    const int ctx = u.ctx;
    const int base = ctx - qb;  // first new token of the sequence
    const int lim_cta = see_all ? ctx - 1 : ctx - qb + (row0 + rows_here - 1) / G;
    const int pages_need = lim_cta / 16 + 1;
    const int pages_ctx = (ctx + 15) / 16;
    const int n_splits = (pages_ctx - u.page_base + u.sp - 1) / u.sp;
    if (split >= n_splits)
        return;
    const int page_lo = u.page_base + split * u.sp;
    const int page_hi = min(page_lo + u.sp, pages_need);
    const int n_pages = max(0, page_hi - page_lo);
    const int n_tiles = (n_pages + kTilePages - 1) / kTilePages;
    const bool final_out = MODE != kModeShared && n_splits == 1;
    // softmax warps that hold at least one of the rows (warp 4 + i holds rows 32 i .. 32 i + 31);
    // the others have nothing to compute or store and stay out of the P barrier: their TMEM lanes
    // keep S where the products read P, which reaches only their own (never stored) rows of O
    const int act_warps = (rows_here + 31) / 32;

    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < n_st; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&v_full[i], 1);
            mbar_init(&k_empty[i], 1);
            mbar_init(&v_empty[i], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&p_full[b], 32 * act_warps);
        }
        mbar_init(pv_done, 1);
        mbar_init(o_done, 1);
        mbar_init(land, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&tmap_q);
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, kTmemCols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 || warp == 2) {
        // ===================== producers: warp 0 = Q once and the K tiles, warp 2 = the V tiles =====================
        // K of a tile is released once its S is complete, V once its P V is: each ring runs as far
        // ahead as its own consumer allows.
        const bool is_v = warp == 2;
        const CUtensorMap *tmap = is_v ? &tmap_v : &tmap_k;
        uint64_t *full = is_v ? v_full : k_full;
        uint64_t *empty = is_v ? v_empty : k_empty;
        int n_issued = 0, z_n = 0;
        bool ok = true;
        if (!is_v && lane == 0 && n_tiles > 0) {
            mbar_arrive_expect_tx(q_full, KB * rows_per_cta * 128);
#pragma unroll
            for (int kb = 0; kb < KB; ++kb)
                tc::tma_load_3d(smem + kb * q_blk, &tmap_q, kb * 64, g * G, u.q0 + row0 / G, q_full);
        }
        // The last page of the context may be partly filled: its V rows past the end can hold
        // anything (NaN included) and P is 0 there, but 0 * NaN is NaN, so the V warp clears them in
        // shared memory before the tile is handed on.
        const int last_page = pages_ctx - 1;
        const int zr0 = ctx & 15;  // first row of the last page to clear (0: the page is full)
        for (int j = 0; j < n_tiles && ok; ++j) {
            const int st = j % n_st;
            const int pidx = j * kTilePages + lane;
            int y = oob_row;  // pages past the split read rows past the pool: zero fill
            if (lane < kTilePages && pidx < n_pages) {
                const int id = __ldg(u.table + page_lo + pidx);
                if (id >= 0 && id < p.num_blocks)
                    y = (id * p.H_kv + g) * 16;
                else if (!is_v)
                    set_status(p.status, PA_ERR_BOUNDS);
            }
            const int zk = last_page - page_lo - j * kTilePages;  // tile page holding the context end
            const bool z = is_v && zr0 != 0 && zk >= 0 && zk < kTilePages && zk < n_pages - j * kTilePages;
            uint64_t *done = z ? land : &full[st];
            if (lane == 0) {
                ok = wait_bar(&empty[st], free_par(j / n_st), abort_flag, p.status);
                if (ok)
                    mbar_arrive_expect_tx(done, L::kTile);
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok)
                break;
            ++n_issued;
            uint8_t *dst = smem + ring_off + st * 2 * L::kTile + (is_v ? L::kTile : 0);
            if (lane < kTilePages) {
#pragma unroll
                for (int kb = 0; kb < KB; ++kb)
                    tma_load_2d(dst + kb * L::kBlk + lane * 2048, tmap, kb * 64, y, done);
            }
            if (z) {
                ++z_n;
                ok = wait_bar(land, full_par(z_n - 1), abort_flag, p.status);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok)
                    break;
                const int per_kb = (16 - zr0) * 8;  // 16-byte chunks to clear per column block
                for (int i = lane; i < per_kb * KB; i += 32) {
                    const int kb = i / per_kb, rem = i % per_kb;
                    const int row = zk * 16 + zr0 + rem / 8;
                    *reinterpret_cast<uint4 *>(dst + kb * L::kBlk + row * 128 + (rem & 7) * 16) =
                        make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();  // generic writes before the tensor core reads the tile
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&full[st]);
            }
        }
        if (lane == 0 && *abort_flag) {
            // let the copies already issued land before shared memory is released
            if (!is_v && n_tiles > 0)
                mbar_wait(q_full, 0, kWaitTimeoutNs / 10);
            for (int st = 0; st < n_st; ++st) {
                const int uses = n_issued / n_st + (st < n_issued % n_st ? 1 : 0);
                if (uses > 0)
                    mbar_wait(&full[st], full_par(uses - 1), kWaitTimeoutNs / 10);
            }
            if (z_n > 0)
                mbar_wait(land, full_par(z_n - 1), kWaitTimeoutNs / 10);
        }
    } else if (warp == 1) {
        // ===================== MMA issuer (one thread) =====================
        // Iteration j issues S(j) into buffer j & 1, then -- once the softmax has written P(j-1) --
        // O += P(j-1) V(j-1).  S(j) overwrites buffer j & 1 after the product that read P(j-2) there
        // (issued earlier by this thread; tcgen05.mma operations of one thread execute in order).
        if (lane == 0) {
            constexpr uint32_t idesc_s = tc::idesc_f16(BF16, kRows, kTileKeys, false);
            constexpr uint32_t idesc_pv = tc::idesc_f16(BF16, kRows, D, true);
            const uint32_t q_addr = smem_u32(smem);
            bool ok = n_tiles == 0 || wait_bar(q_full, 0, abort_flag, p.status);
            for (int j = 0; j <= n_tiles && ok; ++j) {
                if (j < n_tiles) {
                    ok = wait_bar(&k_full[j % n_st], full_par(j / n_st), abort_flag, p.status);
                    if (!ok)
                        break;
                    tc::fence_after_sync();
                    const uint32_t k_addr = smem_u32(smem + ring_off + (j % n_st) * 2 * L::kTile);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t qo = (ks >> 2) * q_blk + (ks & 3) * 32;
                        const uint32_t ko = (ks >> 2) * L::kBlk + (ks & 3) * 32;
                        tc::mma_ss(tmem + (j & 1) * kTileKeys, tc::desc_k_sw128(q_addr + qo),
                                   tc::desc_k_sw128(k_addr + ko), idesc_s, ks > 0 ? 1u : 0u);
                    }
                    tc::commit(&s_full[j & 1]);
                    tc::commit(&k_empty[j % n_st]);
                }
                if (j >= 1) {
                    const int jp = j - 1;
                    ok = wait_bar(&p_full[jp & 1], full_par(jp >> 1), abort_flag, p.status);
                    if (ok)
                        ok = wait_bar(&v_full[jp % n_st], full_par(jp / n_st), abort_flag, p.status);
                    if (!ok)
                        break;
                    tc::fence_after_sync();
                    const uint32_t v_addr = smem_u32(smem + ring_off + (jp % n_st) * 2 * L::kTile + L::kTile);
#pragma unroll
                    for (int ks = 0; ks < kTileKeys / 16; ++ks)
                        tc::mma_ts(tmem + kColO, tmem + (jp & 1) * kTileKeys + ks * 8,
                                   tc::desc_mn_sw128(v_addr + ks * 2048, L::kBlk), idesc_pv,
                                   (jp > 0 || ks > 0) ? 1u : 0u);
                    tc::commit(&v_empty[jp % n_st]);
                    tc::commit(pv_done);
                }
            }
            // o_done completes when every product issued above has (also with no product at all)
            tc::commit(ok ? o_done : drain);
            if (!ok)
                mbar_wait(drain, 0, kWaitTimeoutNs / 10);
        }
        __syncwarp();
    } else if (warp >= 4 && warp - 4 < act_warps) {
        // ===================== softmax and epilogue: thread r = row r = TMEM lane r =====================
        const int sub = warp & 3;
        const int r = sub * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(sub * 32) << 16;
        const bool row_valid = r < rows_here;
        const int ridx = row0 + r;
        const int lim = row_valid ? (see_all ? ctx - 1 : ctx - qb + ridx / G) : -1;
        uint32_t bits = ~0u;
        if (MODE == kModeTree && row_valid)
            bits = static_cast<uint32_t>(__ldg(p.tree + u.q0 + ridx / G));
        const float sl2 = p.scale_log2;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j) {
            ok = wait_bar(&s_full[j & 1], full_par(j >> 1), abort_flag, p.status);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok)
                break;
            tc::fence_after_sync();
            const uint32_t s_tm = tmem + lane_addr + (j & 1) * kTileKeys;
            uint32_t raw[kTileKeys];
            tc::ld64(s_tm, raw);
            // keys past the row's limit (causal / context end) and, among the new tokens, those the
            // row's tree mask hides become -inf
            const int key0 = (page_lo + j * kTilePages) * 16;
            const bool tree_here = MODE == kModeTree && key0 + kTileKeys > base;
            if (key0 + kTileKeys - 1 > lim || tree_here) {
#pragma unroll
                for (int c = 0; c < kTileKeys; ++c) {
                    const int key = key0 + c;
                    bool vis = key <= lim;
                    if (MODE == kModeTree)
                        vis = vis && (key < base || ((bits >> min(max(key - base, 0), 31)) & 1u));
                    if (!vis)
                        raw[c] = 0xff800000u;  // -inf
                }
            }
            float mx4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                mx4[i] = fmaxf(__uint_as_float(raw[2 * i]), __uint_as_float(raw[2 * i + 1]));
#pragma unroll
            for (int c = 8; c < kTileKeys; c += 2)
                mx4[(c >> 1) & 3] = fmax3(mx4[(c >> 1) & 3], __uint_as_float(raw[c]), __uint_as_float(raw[c + 1]));
            const float mx_s = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * sl2;  // -inf stays -inf
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
                // O holds the products of P(0 .. j-1); P(j-1) V(j-1) may still be in flight: wait for
                // it (S(j), complete here, was issued after P(j-2) V(j-2), so at most that one is open)
                ok = __all_sync(0xffffffffu, wait_bar(pv_done, full_par(j - 1), abort_flag, p.status));
                if (!ok)
                    break;
                tc::fence_after_sync();
#pragma unroll 1
                for (int c = 0; c < D / 16; ++c) {
                    uint32_t o[16];
                    tc::ld16(tmem + lane_addr + kColO + c * 16, o);
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
                    tc::st16(tmem + lane_addr + kColO + c * 16, o);
                }
            }
            // P = 2^(s * scale * log2 e - m) (masked keys: 2^-inf = 0), packed to 16 bits in place
            const float nb = m == -INFINITY ? 0.f : -m;
            const uint64_t sl2_2 = f2_pack(sl2, sl2), nb_2 = f2_pack(nb, nb);
            uint64_t acc[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
            for (int q = 0; q < kTileKeys / 2; ++q) {
                float x0, x1;
                f2_unpack(f2_fma(f2_pack(__uint_as_float(raw[2 * q]), __uint_as_float(raw[2 * q + 1])), sl2_2, nb_2),
                          x0, x1);
                const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
                acc[q & 1] = f2_add(acc[q & 1], f2_pack(p0, p1));
                raw[q] = pack2<BF16>(p0, p1);
            }
            {
                float a0, a1, b0, b1;
                f2_unpack(acc[0], a0, a1);
                f2_unpack(acc[1], b0, b1);
                l += (a0 + a1) + (b0 + b1);
            }
            tc::st32(s_tm, raw);
            tc::wait_st();
            tc::fence_before_sync();
            mbar_arrive(&p_full[j & 1]);
        }
        // ---- epilogue: O / l -> out (one split) or the normalised partial and its log2-sum-exp ----
        if (ok)
            ok = __all_sync(0xffffffffu, wait_bar(o_done, 0, abort_flag, p.status));
        if (ok) {
            tc::fence_after_sync();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const int64_t t = u.q0 + ridx / G;
            const int h = g * G + ridx % G;
            const int64_t orow = t * p.H_q + h;
            const int64_t prow = (int64_t)(u.slot0 + split) * p.T * p.H_q + orow;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                if (n_tiles > 0) {
                    tc::ld32(tmem + lane_addr + kColO + c * 32, o);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        o[i] = 0u;
                }
                if (!row_valid)
                    continue;
                if (final_out) {
                    uint8_t *dst = static_cast<uint8_t *>(p.out) + (orow * D + c * 32) * 2;
#pragma unroll
                    for (int i = 0; i < 32; i += 8)
                        *reinterpret_cast<uint4 *>(dst + i * 2) =
                            make_uint4(pack2<BF16>(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv),
                                       pack2<BF16>(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv),
                                       pack2<BF16>(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv),
                                       pack2<BF16>(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv));
                } else {
                    float *dst = p.ws_o + prow * D + c * 32;
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4 *>(dst + i) =
                            make_float4(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv,
                                        __uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
                }
            }
            if (row_valid && !final_out)
                p.ws_lse[prow] = l > 0.f ? m + log2f(l) : -INFINITY;
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0)
        tc::tmem_dealloc(tmem, kTmemCols);
}

template <int D, bool BF16, int MODE>
static int launch(const RowsParams &rp, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                  int rows_per_cta, dim3 grid, cudaStream_t stream)
{
    using L = Smem<D>;
    auto kern = pa_attn_rows_tc_kernel<D, BF16, MODE>;
    static uint64_t configured = 0;  // one bit per device, per template instance
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return PA_ERR_CUDA;
    const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
    if (!bit || !(configured & bit)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemPerCta) != cudaSuccess)
            return PA_ERR_CUDA;
        configured |= bit;
    }
    const int n_st = L::stages_for(rows_per_cta);
    const int bytes = L::alloc(rows_per_cta, n_st);
    if (bytes > kSmemPerCta)
        return PA_ERR_UNSUPPORTED;
    const int oob_row = static_cast<int>(rp.num_blocks * rp.H_kv * 16);
    const cudaError_t e =
        launch_dependent(kern, grid, dim3(kThreads), bytes, stream, tq, tk, tv, rp, rows_per_cta, n_st, oob_row);
    count_launch();
    const cudaError_t e2 = cudaGetLastError();
    return e == cudaSuccess && e2 == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace rtc

int rows_tc_rows_per_cta(int G, int max_tokens)
{
    if (G < 1 || G > rtc::kRows || max_tokens < 1)
        return 0;
    return std::min(rtc::kRows / G, max_tokens) * G;
}

int launch_rows_tc(const RowsParams &rp, const CUtensorMap &tk, const CUtensorMap &tv, int d, pa_dtype dtype,
                   int mode, int rows_per_cta, dim3 grid, cudaStream_t stream)
{
    if (rows_per_cta < 1 || rows_per_cta > rtc::kRows || rows_per_cta % rp.G)
        return PA_ERR_UNSUPPORTED;
    CUtensorMap tq;
    const int rc = make_q_tmap(&tq, rp.q, rp.T, rp.H_q, d, rp.G, rows_per_cta / rp.G, dtype);
    if (rc != PA_OK)
        return rc;
    const bool bf16 = dtype == PA_BF16;
#define PA_RTC_CASE(DD, BB, MM)                                                                    \
    if (d == DD && bf16 == BB && mode == MM)                                                       \
        return rtc::launch<DD, BB, MM>(rp, tq, tk, tv, rows_per_cta, grid, stream);
    PA_RTC_CASE(128, true, kModeCausal)
    PA_RTC_CASE(128, false, kModeCausal)
    PA_RTC_CASE(128, true, kModeTree)
    PA_RTC_CASE(128, false, kModeTree)
    PA_RTC_CASE(128, true, kModeShared)
    PA_RTC_CASE(128, false, kModeShared)
    PA_RTC_CASE(64, true, kModeCausal)
    PA_RTC_CASE(64, false, kModeCausal)
    PA_RTC_CASE(64, true, kModeTree)
    PA_RTC_CASE(64, false, kModeTree)
    PA_RTC_CASE(64, true, kModeShared)
    PA_RTC_CASE(64, false, kModeShared)
#undef PA_RTC_CASE
    return PA_ERR_UNSUPPORTED;
}

}  // namespace pa
