// Paged attention for groups of up to 64 query rows that share one KV head.
//
// Decode ("FlashDecoding" answer of the interview Q&A page): the rows of a
// CTA are the G query heads x q_b new tokens of one (sequence, KV head); the
// sequence's pages are split into ranges of `split_pages` pages handled by
// different CTAs; each split keeps its own running max m and sum l (online
// softmax, iopencloud "大模型推理加速技术全景" section 2.2) and writes a
// normalised partial O_s with its log-sum-exp; pa_split_merge_kernel then
// combines the splits ("cross-block reduction").  A sequence short enough
// for one split is written straight to `out`.
//
// Data movement: TMA box loads (64 elements x 16 rows, 128-byte swizzle) of
// whole (block, head) pages straight from the block pool into a ring of three
// shared-memory stages; completion is tracked by mbarriers with bounded waits.
// The page ids come from the block table (iopencloud section 3.2): the first
// stages are issued at once from the table in global memory, the rest from a
// copy in shared memory.  A stage is refilled by the last warp to finish with
// it, so no warp waits for the others between stages.  Q is staged through the
// last stage's buffer before that buffer's first load.  K/V bytes are read
// once per CTA.
//
// Compute: four warps; each owns a 16-row m-tile and a subset of the pages of
// every stage (several warps on different pages when there are <= 32 rows,
// merged at the end like splits).  S = Q K^T and O += P V run on mma.sync
// m16n8k16 with fp32 accumulators; P is rounded to the input type for P V.
#include <algorithm>
#include <cmath>

#include <cuda_fp8.h>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "rows_common.cuh"

namespace pa {

// Epilogue buffer of a rows CTA: partial O, max and sum of every warp's 16 rows.
template <int D>
struct RowsEpi {
    static constexpr int kStride = D + 8;  // floats per row of the epilogue buffer
    static constexpr int kBytes = (4 * 16 * kStride + 2 * 64) * 4;
};

template <int D, int STAGES>
struct RowsSmem {
    static constexpr int kPageBytes = 16 * D * 2;
    static constexpr int kStageBytes = 2 * kPagesPerStage * kPageBytes;  // K pages then V pages
    static constexpr int kQBytes = kRowsPerCta * D * 2;
    static_assert(RowsEpi<D>::kBytes <= STAGES * kStageBytes, "epilogue must fit in the stage ring");
    static_assert(kQBytes <= kStageBytes, "Q is staged through one stage buffer");
    static constexpr int kStageOff = 0;
    static constexpr int kQOff = (STAGES - 1) * kStageBytes;  // aliases the last stage during set-up
    static constexpr int kBarOff = STAGES * kStageBytes;
    static constexpr int kCountOff = kBarOff + 8 * STAGES;    // warps done with each stage
    static constexpr int kIssuedOff = kCountOff + 4 * STAGES; // loads issued into each stage
    static constexpr int kTableOff = kIssuedOff + 4 * STAGES;
    static constexpr int kFlagOff = kTableOff + 4 * kMaxTablePages;
    static constexpr int kBytes = kFlagOff + 16;
    static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 B (swizzle atoms)
};

// One 16-key page for one warp: S = Q K^T for its m-tile (mma.sync m16n8k16 from ldmatrix of the
// swizzled K page), mask, online softmax of its two rows, O += P V.  `kbase` and `vbase` are shared
// addresses of the page's K and V in the 128-byte-swizzled 16-bit layout; keys j0 .. j0 + 15.
// Key k is visible to a row when k <= lim and, among the new tokens (k >= base), its bit is set.
// SCALED (the FP8 cache): K and V hold the codes' values unscaled and ksc / vsc the 16 row scales
// of the page in shared memory; a key's K scale multiplies its score, its V scale its P (the row
// sum l takes the unscaled P), which is K x scale and V x scale exactly up to rounding.
template <int D, bool BF16, bool SCALED = false, bool TREE = false>
__device__ __forceinline__ void rows_page(uint32_t kbase, uint32_t vbase, int j0, int lane,
                                          const uint32_t (&qa)[D / 16][4], float (&o)[D / 8][4], float &m_a,
                                          float &m_b, float &l_a, float &l_b, int lim_a, int lim_b, uint32_t bits_a,
                                          uint32_t bits_b, int base, int ctx, float sl2, const float *ksc = nullptr,
                                          const float *vsc = nullptr)
{
    constexpr int KSTEPS = D / 16;  // k-steps of S = Q K^T
    constexpr int NT = D / 8;       // n-tiles of O
    const int kq = lane & 3;
    auto visible = [&](int key, int lim, uint32_t bits) {
        if constexpr (TREE)
            return key <= lim && (key < base || ((bits >> (key - base)) & 1u));
        else
            return key <= lim;
    };

    // S (16 rows x 16 keys) = Q K^T
    float s[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
        s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
        const int mi = lane >> 3, rr = lane & 7;
        const int key = (mi >> 1) * 8 + rr;
        const int c = 2 * ks + (mi & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kbase + (c >> 3) * 2048 + key * 128 + (((c & 7) ^ (key & 7)) << 4), b0, b1, b2, b3);
        mma16816<BF16>(s[0], qa[ks], b0, b1);
        mma16816<BF16>(s[1], qa[ks], b2, b3);
    }
    // mask (causal / context end), scale to log2 units, online softmax
    float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int key = j0 + nt * 8 + 2 * kq + c;
            float f = sl2;
            if constexpr (SCALED)
                f *= ksc[nt * 8 + 2 * kq + c];
            s[nt][c] = visible(key, lim_a, bits_a) ? s[nt][c] * f : -INFINITY;
            s[nt][2 + c] = visible(key, lim_b, bits_b) ? s[nt][2 + c] * f : -INFINITY;
            mx_a = fmaxf(mx_a, s[nt][c]);
            mx_b = fmaxf(mx_b, s[nt][2 + c]);
        }
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
    const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
    const float base_a = mn_a == -INFINITY ? 0.f : mn_a;
    const float base_b = mn_b == -INFINITY ? 0.f : mn_b;
    const float al_a = fast_exp2(m_a - base_a), al_b = fast_exp2(m_b - base_b);
    m_a = mn_a;
    m_b = mn_b;
    float ps_a = 0.f, ps_b = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        s[nt][0] = fast_exp2(s[nt][0] - base_a);
        s[nt][1] = fast_exp2(s[nt][1] - base_a);
        s[nt][2] = fast_exp2(s[nt][2] - base_b);
        s[nt][3] = fast_exp2(s[nt][3] - base_b);
        ps_a += s[nt][0] + s[nt][1];
        ps_b += s[nt][2] + s[nt][3];
    }
    l_a = l_a * al_a + ps_a;
    l_b = l_b * al_b + ps_b;
    if (__any_sync(0xffffffffu, al_a != 1.f || al_b != 1.f)) {
#pragma unroll
        for (int nd = 0; nd < NT; ++nd) {
            o[nd][0] *= al_a;
            o[nd][1] *= al_a;
            o[nd][2] *= al_b;
            o[nd][3] *= al_b;
        }
    }
    if constexpr (SCALED) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const float vs = vsc[nt * 8 + 2 * kq + c];
                s[nt][c] *= vs;
                s[nt][2 + c] *= vs;
            }
    }
    uint32_t pa_[4];
    pa_[0] = pack2<BF16>(s[0][0], s[0][1]);
    pa_[1] = pack2<BF16>(s[0][2], s[0][3]);
    pa_[2] = pack2<BF16>(s[1][0], s[1][1]);
    pa_[3] = pack2<BF16>(s[1][2], s[1][3]);

    // keys past the context end may hold anything (NaN): zero their V
    uint32_t vm_lo = 0xffffffffu, vm_hi = 0xffffffffu;
    if (j0 + 16 > ctx) {
        const int valid = ctx - j0;
        const int k0 = 2 * kq;
        vm_lo = (k0 < valid ? 0x0000ffffu : 0u) | (k0 + 1 < valid ? 0xffff0000u : 0u);
        vm_hi = (k0 + 8 < valid ? 0x0000ffffu : 0u) | (k0 + 9 < valid ? 0xffff0000u : 0u);
    }
    // O (16 x D) += P (16 x 16 keys) V (16 keys x D)
#pragma unroll
    for (int ndp = 0; ndp < NT / 2; ++ndp) {
        const int mi = lane >> 3, rr = lane & 7;
        const int key = (mi & 1) * 8 + rr;
        const int c = 2 * ndp + (mi >> 1);
        uint32_t r0, r1, r2, r3;
        ldsm_x4_t(vbase + (c >> 3) * 2048 + key * 128 + (((c & 7) ^ (key & 7)) << 4), r0, r1, r2, r3);
        r0 &= vm_lo;
        r1 &= vm_hi;
        r2 &= vm_lo;
        r3 &= vm_hi;
        mma16816<BF16>(o[2 * ndp], pa_, r0, r1);
        mma16816<BF16>(o[2 * ndp + 1], pa_, r2, r3);
    }
}

// Epilogue of a rows CTA: merge the warps of each m-tile (several warps on different pages of the
// same rows, like splits) through shared memory `e_o` (at least RowsEpi<D>::kBytes), normalise,
// and store the rows: straight to `out` when `final_out`, else the normalised partial and its
// log2-sum-exp to workspace slot `slot`.
template <int D, bool BF16>
__device__ __forceinline__ void rows_epilogue(float *e_o, const RowsParams &p, const float (&o)[D / 8][4], float m_a,
                                              float m_b, float l_a, float l_b, bool has_rows, int rows_here,
                                              int row0, int q0, int g, int slot, bool final_out, int KG)
{
    constexpr int NT = D / 8;
    constexpr int kEpiStride = RowsEpi<D>::kStride;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, kq = lane & 3;
    const int G = p.G;
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    float *e_m = e_o + 4 * 16 * kEpiStride;        // [4][16]
    float *e_l = e_m + 64;                            // [4][16]
    if (has_rows) {
        const int la = lane >> 2, lb = la + 8;
#pragma unroll
        for (int nd = 0; nd < NT; ++nd) {
            const int col = nd * 8 + 2 * kq;
            *reinterpret_cast<float2 *>(e_o + (warp * 16 + la) * kEpiStride + col) = make_float2(o[nd][0], o[nd][1]);
            *reinterpret_cast<float2 *>(e_o + (warp * 16 + lb) * kEpiStride + col) = make_float2(o[nd][2], o[nd][3]);
        }
        if (kq == 0) {
            e_m[warp * 16 + la] = m_a;
            e_m[warp * 16 + lb] = m_b;
            e_l[warp * 16 + la] = l_a;
            e_l[warp * 16 + lb] = l_b;
        }
    }
    __syncthreads();
    for (int i = tid; i < rows_here * (D / 4); i += kThreads) {
        const int r = i / (D / 4), c4 = i % (D / 4);
        const int mtr = r >> 4, lr = r & 15;
        float M = -INFINITY;
        for (int k = 0; k < KG; ++k)
            M = fmaxf(M, e_m[(mtr * KG + k) * 16 + lr]);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float Lsum = 0.f;
        for (int k = 0; k < KG; ++k) {
            const int w = mtr * KG + k;
            const float mk = e_m[w * 16 + lr];
            const float wt = mk == -INFINITY ? 0.f : fast_exp2(mk - M);
            Lsum += wt * e_l[w * 16 + lr];
            const float4 v = *reinterpret_cast<const float4 *>(e_o + (w * 16 + lr) * kEpiStride + c4 * 4);
            acc.x += wt * v.x;
            acc.y += wt * v.y;
            acc.z += wt * v.z;
            acc.w += wt * v.w;
        }
        const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
        const int ridx = row0 + r;
        const int64_t t = q0 + ridx / G;
        const int h = g * G + ridx % G;
        const int64_t orow = t * p.H_q + h;
        if (final_out) {
            store4<BF16>(static_cast<uint8_t *>(p.out) + (orow * D + c4 * 4) * 2, acc.x * inv, acc.y * inv,
                         acc.z * inv, acc.w * inv);
        } else {
            const int64_t prow = (int64_t)slot * p.T * p.H_q + orow;
            *reinterpret_cast<float4 *>(p.ws_o + prow * D + c4 * 4) =
                make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
            if (c4 == 0)
                p.ws_lse[prow] = Lsum > 0.f ? M + log2f(Lsum) : -INFINITY;
        }
    }
}

// CTAs of the 16-bit rows kernel resident on an SM (sets the register budget), and its ring depth.
#ifndef PA_ROWS_MIN_BLOCKS
#define PA_ROWS_MIN_BLOCKS 3
#endif
#ifndef PA_ROWS_STAGES
#define PA_ROWS_STAGES 2
#endif

template <int D, bool BF16, int STAGES, int MODE>
__global__ void __launch_bounds__(kThreads, PA_ROWS_MIN_BLOCKS)
    pa_attn_rows_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                        const RowsParams p)
{
    using L = RowsSmem<D, STAGES>;
    constexpr int CH = D / 8;       // 16-byte chunks per row
    constexpr int BOXES = D / 64;   // TMA boxes per page
    constexpr int KSTEPS = D / 16;  // k-steps of S = Q K^T
    constexpr int NT = D / 8;       // n-tiles of O

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *s_stage = smem + L::kStageOff;
    uint8_t *s_q = smem + L::kQOff;
    uint64_t *s_bar = reinterpret_cast<uint64_t *>(smem + L::kBarOff);
    int *s_count = reinterpret_cast<int *>(smem + L::kCountOff);
    int *s_issued = reinterpret_cast<int *>(smem + L::kIssuedOff);
    int32_t *s_pages = reinterpret_cast<int32_t *>(smem + L::kTableOff);
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + L::kFlagOff);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    griddep_wait();     // the sequence order comes from the kernel before this one
    griddep_release();  // the split merge after this kernel may be scheduled (it waits for this grid)

    // ---- which (sequence, KV head, row group, split) --------------------------------
    const int split = blockIdx.x;
    const int g = blockIdx.y / p.n_rg, rg = blockIdx.y % p.n_rg;
    DecodeUnit u;
    if (!decode_unit<MODE>(p, tid, u))
        return;
    const int q0 = u.q0, q1 = u.q1, ctx = u.ctx, page_base = u.page_base, sp = u.sp, slot0 = u.slot0;
    const bool prefix_cta = u.prefix_cta;
    const int32_t *table = u.table;
    const int qb = q1 - q0;
    const int G = p.G;
    const int R = G * qb;
    const int row0 = rg * kRowsPerCta;
    if (row0 >= R)
        return;
    const int rows_here = min(kRowsPerCta, R - row0);
    constexpr bool tree = MODE == kModeTree;  // p.tree is set exactly in this mode
    const int base = ctx - qb;  // first new token of the sequence
    // rows that see every key: tree rows (their mask decides among the new tokens) and the rows
    // of a shared prefix
    const bool see_all = tree || prefix_cta;
    // last key any row here sees
    const int lim_cta = see_all ? ctx - 1 : ctx - qb + (row0 + rows_here - 1) / G;
    const int pages_need = lim_cta / 16 + 1;
    const int pages_ctx = (ctx + 15) / 16;
    const int n_splits = (pages_ctx - page_base + sp - 1) / sp;
    if (split >= n_splits)
        return;
    const int page_lo = page_base + split * sp;
    const int page_hi = min(page_lo + sp, pages_need);
    const int n_pages = max(0, page_hi - page_lo);
    const int n_stages = (n_pages + kPagesPerStage - 1) / kPagesPerStage;

    // warp roles: MT m-tiles of 16 rows, KG warps per m-tile on different pages
    const int MT = rows_here <= 16 ? 1 : (rows_here <= 32 ? 2 : 4);
    const int KG = 4 / MT;
    const int mt = warp / KG, kg = warp % KG;
    const bool has_rows = mt * 16 < rows_here;

    // ---- set-up: barriers and the first loads, page ids, Q tile ---------------------------
    auto checked = [&](int pg) -> int {
        if (pg < 0 || pg >= p.num_blocks) {
            set_status(p.status, PA_ERR_BOUNDS);
            pg = static_cast<int>(p.num_blocks);  // past the pool: TMA fills zeros
        }
        return pg;
    };
    auto issue = [&](int st) {  // one thread; the page ids from the shared-memory copy
        const int slot = st % STAGES;
        uint8_t *kb = s_stage + slot * L::kStageBytes;
        uint8_t *vb = kb + kPagesPerStage * L::kPageBytes;
        const int np = min(kPagesPerStage, n_pages - st * kPagesPerStage);
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&s_bar[slot], np * 2 * L::kPageBytes);
        s_issued[slot] += 1;
        for (int k = 0; k < np; ++k) {
            const int i = st * kPagesPerStage + k;
            const int pg = s_pages[i];
            const int y = (pg * p.H_kv + g) * 16;
#pragma unroll
            for (int bx = 0; bx < BOXES; ++bx) {
                tma_load_2d(kb + k * L::kPageBytes + bx * 2048, &tmap_k, bx * 64, y, &s_bar[slot]);
                tma_load_2d(vb + k * L::kPageBytes + bx * 2048, &tmap_v, bx * 64, y, &s_bar[slot]);
            }
        }
    };
    if (warp == 0) {
        // the first stages go out before anything else: lane i < (STAGES - 1) * 4 reads the id of
        // page i straight from the table in global memory and issues that page's boxes, so the
        // id loads overlap instead of following one another
        if (lane == 0) {
            for (int s = 0; s < STAGES; ++s) {
                mbar_init(&s_bar[s], 1);
                s_count[s] = 0;
                s_issued[s] = 0;
            }
            *s_abort = 0;
            fence_barrier_init();
            prefetch_tmap(&tmap_k);
            prefetch_tmap(&tmap_v);
        }
        const int first = min(STAGES - 1, n_stages);
        const int i = lane;
        const bool mine = i < first * kPagesPerStage && i < n_pages;
        const int pg = mine ? checked(__ldg(table + page_lo + i)) : 0;
        __syncwarp();
        if (lane == 0) {
            for (int st = 0; st < first; ++st) {
                const int np = min(kPagesPerStage, n_pages - st * kPagesPerStage);
                mbar_arrive_expect_tx(&s_bar[st], np * 2 * L::kPageBytes);
                s_issued[st] += 1;
            }
        }
        __syncwarp();
        if (mine) {
            const int st = i / kPagesPerStage, k = i % kPagesPerStage;
            uint8_t *kb = s_stage + st * L::kStageBytes;
            uint8_t *vb = kb + kPagesPerStage * L::kPageBytes;
            const int y = (pg * p.H_kv + g) * 16;
#pragma unroll
            for (int bx = 0; bx < BOXES; ++bx) {
                tma_load_2d(kb + k * L::kPageBytes + bx * 2048, &tmap_k, bx * 64, y, &s_bar[st]);
                tma_load_2d(vb + k * L::kPageBytes + bx * 2048, &tmap_v, bx * 64, y, &s_bar[st]);
            }
        }
    }
    for (int i = tid; i < n_pages; i += kThreads)
        s_pages[i] = checked(__ldg(table + page_lo + i));
    for (int i = tid; i < kRowsPerCta * CH; i += kThreads) {
        const int r = i / CH, c = i % CH;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < rows_here) {
            const int ridx = row0 + r;
            const int64_t t = q0 + ridx / G;
            const int h = g * G + ridx % G;
            v = __ldg(reinterpret_cast<const uint4 *>(p.q) + (t * p.H_q + h) * CH + c);
        }
        *reinterpret_cast<uint4 *>(s_q + r * (D * 2) + ((c ^ (r & 7)) << 4)) = v;
    }
    __syncthreads();

    // ---- per-thread row state --------------------------------------------------------------
    // This thread holds rows ra = lane/4 and rb = ra + 8 of its warp's m-tile.
    // Key k is visible to a row when k <= lim and, among the new tokens (k >= base), its bit is set:
    // causal rows see keys up to their own position with every bit set; tree rows see up to the
    // last key with their own mask.
    const int ra = mt * 16 + (lane >> 2), rb = ra + 8;
    const int lim_a = ra < rows_here ? (see_all ? ctx - 1 : ctx - qb + (row0 + ra) / G) : -1;
    const int lim_b = rb < rows_here ? (see_all ? ctx - 1 : ctx - qb + (row0 + rb) / G) : -1;
    const uint32_t bits_a = tree && ra < rows_here ? static_cast<uint32_t>(__ldg(p.tree + q0 + (row0 + ra) / G)) : ~0u;
    const uint32_t bits_b = tree && rb < rows_here ? static_cast<uint32_t>(__ldg(p.tree + q0 + (row0 + rb) / G)) : ~0u;
    const int lim_warp =
        has_rows ? (see_all ? ctx - 1 : ctx - qb + (row0 + min(mt * 16 + 15, rows_here - 1)) / G) : -1;

    uint32_t qa[KSTEPS][4];
    if (has_rows) {
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
            const int mi = lane >> 3, rr = lane & 7;
            const int r = mt * 16 + (mi & 1) * 8 + rr;
            const int c = 2 * ks + (mi >> 1);
            ldsm_x4(smem_u32(s_q + r * (D * 2) + ((c ^ (r & 7)) << 4)), qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3]);
        }
    }
    __syncthreads();  // Q is in registers: the last stage buffer can be loaded
    if (tid == 0 && STAGES - 1 < n_stages)
        issue(STAGES - 1);
    float o[NT][4];
#pragma unroll
    for (int i = 0; i < NT; ++i)
        o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
    const float sl2 = p.scale_log2;

    // ---- main loop over stages ---------------------------------------------------------------
    int it = 0;
    for (; it < n_stages; ++it) {
        const int slot = it % STAGES;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&s_bar[slot], (it / STAGES) & 1));
        if (!ok) {
            *s_abort = 1;
            set_status(p.status, PA_ERR_TIMEOUT);
        }
        if (ok && has_rows) {
            const uint8_t *kst = s_stage + slot * L::kStageBytes;
            const uint8_t *vst = kst + kPagesPerStage * L::kPageBytes;
            for (int k = kg; k < kPagesPerStage; k += KG) {
                const int pidx = it * kPagesPerStage + k;
                if (pidx >= n_pages)
                    break;
                const int j0 = (page_lo + pidx) * 16;
                if (j0 > lim_warp)
                    continue;  // every row of this warp is causally masked on this page
                const uint32_t kbase = smem_u32(kst + k * L::kPageBytes);
                const uint32_t vbase = smem_u32(vst + k * L::kPageBytes);
                rows_page<D, BF16, false, MODE == kModeTree>(kbase, vbase, j0, lane, qa, o, m_a, m_b, l_a, l_b, lim_a, lim_b, bits_a, bits_b,
                                   base, ctx, sl2);
            }
        }
        // the last warp done with this slot refills it
        __syncwarp();
        if (lane == 0 && atomicAdd(&s_count[slot], 1) == 3) {
            s_count[slot] = 0;
            if (it + STAGES < n_stages && !*s_abort)
                issue(it + STAGES);
        }
        if (*s_abort)
            break;
    }
    __syncthreads();
    if (*s_abort) {
        // let the copies still in flight land (bounded) before the CTA releases its shared memory
        if (tid == 0)
            for (int s = 0; s < STAGES; ++s)
                if (s_issued[s] > 0)
                    mbar_wait(&s_bar[s], (s_issued[s] - 1) & 1, kWaitTimeoutNs / 10);
        return;
    }

    // ---- epilogue ---------------------------------------------------------------------------
    // a shared-prefix pass always leaves partials for the merge: prefix splits in slots
    // [0, prefix_slots), a sequence's own splits after them
    rows_epilogue<D, BF16>(reinterpret_cast<float *>(s_stage), p, o, m_a, m_b, l_a, l_b, has_rows, rows_here, row0, q0, g,
                           slot0 + split, MODE != kModeShared && n_splits == 1, KG);
}

// ---- FP8 (E4M3) cache -----------------------------------------------------------------------
// The split-KV decode over an 8-bit cache with one float scale per stored row.  Per (block, KV
// head) the K codes are [16 keys][d] and the V codes [d][16 keys] (transposed, like vLLM's value
// cache), so both reach the mma.sync operand fragments through plain shared-memory loads and are
// widened to 16 bits in registers, with no dequantised copy of the page:
//  - S = Q K^T sums over d in any order: k-step ks of lane quad kq takes the columns
//    d = kq*(D/4) + 4ks + {0..3} (Q's fragments are built in the same order), so a lane reads
//    D/4 contiguous code bytes of a key row;
//  - the keys of a page sit in S's columns so that the four keys a lane quad holds in P (the A
//    operand of P V) are 4kq .. 4kq+3: one 32-bit word of a transposed V row per n-tile.
// The row scales of every page of the split are loaded into shared memory once; they multiply the
// fp32 scores (K) and the probabilities before P V (V).  Pipeline and epilogue as the 16-bit
// kernel: a four-stage TMA ring (one 16 x d-byte box per page for K and one for V), refilled by
// the last warp done with a stage.
#ifndef PA_FP8_NARROW_STAGES
#define PA_FP8_NARROW_STAGES 2
#endif
#ifndef PA_FP8_NARROW_CTAS
#define PA_FP8_NARROW_CTAS 5
#endif
constexpr int kFp8Stages = 4;
constexpr int kNarrowStages = PA_FP8_NARROW_STAGES;  // narrow variant: a shallower ring ...
constexpr int kNarrowCtasPerSm = PA_FP8_NARROW_CTAS;  // ... and more CTAs on an SM

// Epilogue buffer of a narrow FP8 CTA: O^T, max and sum of every warp's 8 rows.
template <int D>
struct NarrowEpi {
    static constexpr int kStride = D + 4;  // floats per (warp, row) of O
    static constexpr int kBytes = (4 * 8 * kStride + 2 * 4 * 8) * 4;
};

// NARROW: no scale table for the whole split; each stage carries its pages' scales (K then V, 16
// floats per page), loaded by TMA with the codes, so five CTAs fit on an SM.
template <int D, bool NARROW>
struct Fp8Smem {
    static constexpr int kStages = NARROW ? kNarrowStages : kFp8Stages;
    static constexpr int kPage = 16 * D;                       // codes of one page of K or of V
    static constexpr int kStage = 2 * kPagesPerStage * kPage;  // K pages then V pages
    static_assert(NARROW || RowsEpi<D>::kBytes <= kStages * kStage, "the epilogue reuses the ring");
    static_assert(NarrowEpi<D>::kBytes <= kStages * kStage, "the epilogue reuses the ring");
    static constexpr int kRingOff = 0;
    // NARROW: floats of a stage's scales, [K, V][page of the stage][32]: 16 keys and 16 floats of
    // padding, as a TMA destination in shared memory must be 128-byte aligned
    static constexpr int kScaleSlot = 32;
    static constexpr int kStageScales = 2 * kPagesPerStage * kScaleSlot;
    // wide: [page of the split][K, V][16 keys]; NARROW: [stage][K, V][page of the stage][32]
    static constexpr int kScaleOff = kStages * kStage;
    static constexpr int kBarOff = kScaleOff + (NARROW ? kStages * kStageScales * 4 : kMaxTablePages * 2 * 16 * 4);
    static constexpr int kCountOff = kBarOff + 8 * kStages;     // warps done with each stage
    static constexpr int kIssuedOff = kCountOff + 4 * kStages;  // loads issued into each stage
    static constexpr int kTableOff = kIssuedOff + 4 * kStages;
    static constexpr int kFlagOff = kTableOff + 4 * kMaxTablePages;
    static constexpr int kBytes = kFlagOff + 16;
    static constexpr int kAlloc = kBytes + 128;  // slack to align the base to 128 B
};

// Four E4M3 codes (the bytes of `w`, lowest first) -> two words of two 16-bit values: lo = codes 0,
// 1 and hi = codes 2, 3; exact, as every E4M3 value is an f16 and a bf16 value.  The f16 form is
// two conversions on the halves of the word, with no repacking around them.
template <bool BF16>
__device__ __forceinline__ void widen_e4m3x4(uint32_t w, uint32_t &lo, uint32_t &hi)
{
    asm volatile("{\n\t.reg .b16 c0, c1;\n\t"
        "mov.b32 {c0, c1}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, c0;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, c1;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
    if constexpr (BF16) {
        const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&lo));
        const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&hi));
        lo = pack2<true>(a.x, a.y);
        hi = pack2<true>(b.x, b.y);
    }
}

// One page of 16 keys for the 16 rows of a warp's m-tile, straight from the codes in shared memory
// (kp: K [16][D], vp: V [D][16]) and the page's scales (sc: 16 for K, then 16 for V).  Rows and
// state as rows_page; keys past `ctx` may hold anything (NaN codes, any scale) and are masked.
template <int D, bool BF16>
__device__ __forceinline__ void rows_page_fp8(const uint8_t *kp, const uint8_t *vp, const float *sc, int j0, int lane,
                                              const uint32_t (&qa)[D / 16][4], float (&o)[D / 8][4], float &m_a,
                                              float &m_b, float &l_a, float &l_b, int lim_a, int lim_b, int ctx,
                                              float sl2)
{
    constexpr int KSTEPS = D / 16;  // k-steps of S = Q K^T
    constexpr int NT = D / 8;       // n-tiles of O
    constexpr int SPAN = D / 4;     // code bytes of a key row per lane quad
    const int r = lane >> 2, kq = lane & 3;

    // S (16 rows x 16 keys) = Q K^T.  Column r of n-tile t is key 4(r/2) + 2t + r%2; the k-steps
    // alternate between two accumulators, which halves the chain of dependent MMAs.
    float s[2][4], s2[2][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            s[t][i] = s2[t][i] = 0.f;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const uint8_t *row = kp + (4 * (r >> 1) + 2 * t + (r & 1)) * D + kq * SPAN;
        uint32_t w[SPAN / 4];
#pragma unroll
        for (int i = 0; i < SPAN / 16; ++i) {
            const uint4 v = *reinterpret_cast<const uint4 *>(row + i * 16);
            w[4 * i] = v.x;
            w[4 * i + 1] = v.y;
            w[4 * i + 2] = v.z;
            w[4 * i + 3] = v.w;
        }
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
            uint32_t b0, b1;
            widen_e4m3x4<BF16>(w[ks], b0, b1);
            if (ks & 1)
                mma16816<BF16>(s2[t], qa[ks], b0, b1);
            else
                mma16816<BF16>(s[t], qa[ks], b0, b1);
        }
    }
    // key scales, mask (causal / context end), log2 units, online softmax.  This lane's keys are
    // 4kq + {0, 1} (n-tile 0) and 4kq + {2, 3} (n-tile 1).
    const float4 kf4 = *reinterpret_cast<const float4 *>(sc + 4 * kq);
    const float kf[4] = {kf4.x, kf4.y, kf4.z, kf4.w};
    float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int key = j0 + 4 * kq + 2 * t + c;
            const float f = sl2 * kf[2 * t + c];
            s[t][c] = key <= lim_a ? (s[t][c] + s2[t][c]) * f : -INFINITY;
            s[t][2 + c] = key <= lim_b ? (s[t][2 + c] + s2[t][2 + c]) * f : -INFINITY;
            mx_a = fmaxf(mx_a, s[t][c]);
            mx_b = fmaxf(mx_b, s[t][2 + c]);
        }
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
    const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
    const float base_a = mn_a == -INFINITY ? 0.f : mn_a;
    const float base_b = mn_b == -INFINITY ? 0.f : mn_b;
    const float al_a = fast_exp2(m_a - base_a), al_b = fast_exp2(m_b - base_b);
    m_a = mn_a;
    m_b = mn_b;
    float ps_a = 0.f, ps_b = 0.f;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        s[t][0] = fast_exp2(s[t][0] - base_a);
        s[t][1] = fast_exp2(s[t][1] - base_a);
        s[t][2] = fast_exp2(s[t][2] - base_b);
        s[t][3] = fast_exp2(s[t][3] - base_b);
        ps_a += s[t][0] + s[t][1];
        ps_b += s[t][2] + s[t][3];
    }
    l_a = l_a * al_a + ps_a;
    l_b = l_b * al_b + ps_b;
    if (__any_sync(0xffffffffu, al_a != 1.f || al_b != 1.f)) {
#pragma unroll
        for (int nd = 0; nd < NT; ++nd) {
            o[nd][0] *= al_a;
            o[nd][1] *= al_a;
            o[nd][2] *= al_b;
            o[nd][3] *= al_b;
        }
    }
    // value scales into P, then P in the A layout of P V: logical keys 2kq + {0, 1} are n-tile 0's
    // columns, 2kq + 8 + {0, 1} n-tile 1's, i.e. the lane's keys 4kq + {0, 1} and 4kq + {2, 3}
    const float4 vf4 = *reinterpret_cast<const float4 *>(sc + 16 + 4 * kq);
    const float vf[4] = {vf4.x, vf4.y, vf4.z, vf4.w};
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            s[t][c] *= vf[2 * t + c];
            s[t][2 + c] *= vf[2 * t + c];
        }
    uint32_t pa_[4];
    pa_[0] = pack2<BF16>(s[0][0], s[0][1]);
    pa_[1] = pack2<BF16>(s[0][2], s[0][3]);
    pa_[2] = pack2<BF16>(s[1][0], s[1][1]);
    pa_[3] = pack2<BF16>(s[1][2], s[1][3]);

    // codes of keys past the context end may be NaN: zero them (code 0 is +0)
    uint32_t vmask = 0xffffffffu;
    if (j0 + 16 > ctx) {
        const int valid = ctx - j0;
        vmask = 0u;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            vmask |= (4 * kq + i < valid ? 0xffu : 0u) << (8 * i);
    }
    // O (16 x D) += P (16 x 16 keys) V (16 keys x D): lane (r, kq) of n-tile nd reads the codes of
    // keys 4kq .. 4kq+3 in V's row d = 8nd + r
#pragma unroll
    for (int nd = 0; nd < NT; ++nd) {
        const uint32_t w = *reinterpret_cast<const uint32_t *>(vp + (8 * nd + r) * 16 + 4 * kq) & vmask;
        uint32_t b0, b1;
        widen_e4m3x4<BF16>(w, b0, b1);
        mma16816<BF16>(o[nd], pa_, b0, b1);
    }
}

// FP8 page step with the keys on the MMA's M side, for CTAs of at most 8 query rows (single-token
// decode with G <= 8), where the 16-row m-tile of rows_page_fp8 would be mostly padding:
// S^T = K Q^T (m = 16 keys, n = 8 rows, k = 16 columns of d) and O^T += V^T P^T (m = 16 columns
// of d, n = 8 rows, k = 16 keys) -- half the MMAs per page, and V^T's operand is one 32-bit word
// of a transposed V row.  A-row g of S^T is key 2g and A-row g + 8 key 2g + 1; the d order of the
// k-steps is rows_page_fp8's.  kf, vf: the K and V scales of keys 2g, 2g + 1 (0 past the context
// end).  State per lane (g = lane/4, t = lane%4): rows 2t and 2t + 1, their
// running max m (uniform over the 8 lanes of a t) and partial sum l (summed over g at the end),
// and O^T rows d = 16 mt + g, 16 mt + g + 8.
template <int D, bool BF16>
__device__ __forceinline__ void narrow_page_fp8(const uint8_t *kp, const uint8_t *vp, float2 kf, float2 vf, int j0, int lane,
                                                const uint32_t (&qb)[D / 16][2], float (&o)[D / 16][4], float (&m)[2],
                                                float (&l)[2], const int (&lim)[2], int ctx, float sl2)
{
    constexpr int MT = D / 16;      // m-tiles of O^T
    constexpr int SPAN = D / 4;     // code bytes of a key row per lane quad
    const int g = lane >> 2, t = lane & 3;

    // S^T (16 keys x 8 rows); the k-steps alternate between two accumulators
    float s[4] = {0.f, 0.f, 0.f, 0.f}, s2[4] = {0.f, 0.f, 0.f, 0.f};
    {
        const uint8_t *r0 = kp + (2 * g) * D + t * SPAN;
        const uint8_t *r1 = r0 + D;
        // 16 bytes of each key row at a time (four k-steps), converted next to their products
#pragma unroll
        for (int i = 0; i < SPAN / 16; ++i) {
            const uint4 a4 = *reinterpret_cast<const uint4 *>(r0 + i * 16);
            const uint4 b4 = *reinterpret_cast<const uint4 *>(r1 + i * 16);
            const uint32_t w0[4] = {a4.x, a4.y, a4.z, a4.w}, w1[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int ks = 4 * i + q;
                uint32_t a[4];
                widen_e4m3x4<BF16>(w0[q], a[0], a[2]);
                widen_e4m3x4<BF16>(w1[q], a[1], a[3]);
                if (ks & 1)
                    mma16816<BF16>(s2, a, qb[ks][0], qb[ks][1]);
                else
                    mma16816<BF16>(s, a, qb[ks][0], qb[ks][1]);
            }
        }
    }
    // x0 = (key 2g, row 2t), x1 = (2g, 2t+1), x2 = (2g+1, 2t), x3 = (2g+1, 2t+1): key scales,
    // mask, log2 units; max over the page's keys (this lane's two, then the 8 lanes of its t)
    const int key0 = j0 + 2 * g, key1 = key0 + 1;
    const float x0 = key0 <= lim[0] ? (s[0] + s2[0]) * (sl2 * kf.x) : -INFINITY;
    const float x1 = key0 <= lim[1] ? (s[1] + s2[1]) * (sl2 * kf.x) : -INFINITY;
    const float x2 = key1 <= lim[0] ? (s[2] + s2[2]) * (sl2 * kf.y) : -INFINITY;
    const float x3 = key1 <= lim[1] ? (s[3] + s2[3]) * (sl2 * kf.y) : -INFINITY;
    float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float mn0 = fmaxf(m[0], mx0), mn1 = fmaxf(m[1], mx1);
    const float b0 = mn0 == -INFINITY ? 0.f : mn0;
    const float b1 = mn1 == -INFINITY ? 0.f : mn1;
    const float al0 = fast_exp2(m[0] - b0), al1 = fast_exp2(m[1] - b1);
    m[0] = mn0;
    m[1] = mn1;
    const float p0 = fast_exp2(x0 - b0), p1 = fast_exp2(x1 - b1);
    const float p2 = fast_exp2(x2 - b0), p3 = fast_exp2(x3 - b1);
    l[0] = l[0] * al0 + p0 + p2;
    l[1] = l[1] * al1 + p1 + p3;
    if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            o[mt][0] *= al0;
            o[mt][1] *= al1;
            o[mt][2] *= al0;
            o[mt][3] *= al1;
        }
    }
    // value scales into P, packed per row as (key 2g, key 2g + 1); P^T's operand for lane (g, t)
    // is row g's keys 4t, 4t + 1 (held by lane (2t, g/2)) and 4t + 2, 4t + 3 (lane (2t + 1, g/2))
    const uint32_t pk0 = pack2<BF16>(p0 * vf.x, p2 * vf.y);  // row 2t
    const uint32_t pk1 = pack2<BF16>(p1 * vf.x, p3 * vf.y);  // row 2t + 1
    const int src = (2 * t) * 4 + (g >> 1);
    const uint32_t u0 = __shfl_sync(0xffffffffu, pk0, src), u1 = __shfl_sync(0xffffffffu, pk1, src);
    const uint32_t v0 = __shfl_sync(0xffffffffu, pk0, src + 4), v1 = __shfl_sync(0xffffffffu, pk1, src + 4);
    const uint32_t pb0 = (g & 1) ? u1 : u0, pb1 = (g & 1) ? v1 : v0;

    // codes of keys past the context end may be NaN: zero them (code 0 is +0)
    uint32_t vmask = 0xffffffffu;
    if (j0 + 16 > ctx) {
        const int valid = ctx - j0;
        vmask = 0u;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            vmask |= (4 * t + i < valid ? 0xffu : 0u) << (8 * i);
    }
    // O^T += V^T P^T: m-tile mt holds d = 16 mt + g (A rows g) and 16 mt + g + 8; the word of V
    // row d at bytes 4t .. 4t + 3 is keys 4t .. 4t + 3 = MMA k indices 2t, 2t+1, 2t+8, 2t+9
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const uint32_t wa = *reinterpret_cast<const uint32_t *>(vp + (16 * mt + g) * 16 + 4 * t) & vmask;
        const uint32_t wb = *reinterpret_cast<const uint32_t *>(vp + (16 * mt + g + 8) * 16 + 4 * t) & vmask;
        uint32_t a[4];
        widen_e4m3x4<BF16>(wa, a[0], a[2]);
        widen_e4m3x4<BF16>(wb, a[1], a[3]);
        mma16816<BF16>(o[mt], a, pb0, pb1);
    }
}

// Epilogue of a narrow FP8 CTA: the four warps (different pages of the same <= 8 rows) merge
// through shared memory `e` (at least NarrowEpi<D>::kBytes) like splits; then as rows_epilogue.

template <int D, bool BF16>
__device__ __forceinline__ void narrow_epilogue(float *e, const RowsParams &p, const float (&o)[D / 16][4],
                                                const float (&m)[2], float (&l)[2], int rows_here, int row0, int q0,
                                                int g, int slot, bool final_out)
{
    constexpr int S = NarrowEpi<D>::kStride;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gr = lane >> 2, t = lane & 3;
    const int G = p.G;
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        l[0] += __shfl_xor_sync(0xffffffffu, l[0], off);
        l[1] += __shfl_xor_sync(0xffffffffu, l[1], off);
    }
    float *e_o = e;                   // [4 warps][8 rows][S]
    float *e_m = e + 4 * 8 * S;       // [4][8]
    float *e_l = e_m + 32;            // [4][8]
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
        const int d0 = 16 * mt + gr;
        e_o[(warp * 8 + 2 * t) * S + d0] = o[mt][0];
        e_o[(warp * 8 + 2 * t + 1) * S + d0] = o[mt][1];
        e_o[(warp * 8 + 2 * t) * S + d0 + 8] = o[mt][2];
        e_o[(warp * 8 + 2 * t + 1) * S + d0 + 8] = o[mt][3];
    }
    if (gr == 0) {
        e_m[warp * 8 + 2 * t] = m[0];
        e_m[warp * 8 + 2 * t + 1] = m[1];
        e_l[warp * 8 + 2 * t] = l[0];
        e_l[warp * 8 + 2 * t + 1] = l[1];
    }
    __syncthreads();
    for (int i = tid; i < rows_here * (D / 4); i += kThreads) {
        const int r = i / (D / 4), c4 = i % (D / 4);
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w)
            M = fmaxf(M, e_m[w * 8 + r]);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float Lsum = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const float mw = e_m[w * 8 + r];
            const float wt = mw == -INFINITY ? 0.f : fast_exp2(mw - M);
            Lsum += wt * e_l[w * 8 + r];
            const float4 v = *reinterpret_cast<const float4 *>(e_o + (w * 8 + r) * S + c4 * 4);
            acc.x += wt * v.x;
            acc.y += wt * v.y;
            acc.z += wt * v.z;
            acc.w += wt * v.w;
        }
        const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
        const int ridx = row0 + r;
        const int64_t tok = q0 + ridx / G;
        const int h = g * G + ridx % G;
        const int64_t orow = tok * p.H_q + h;
        if (final_out) {
            store4<BF16>(static_cast<uint8_t *>(p.out) + (orow * D + c4 * 4) * 2, acc.x * inv, acc.y * inv,
                         acc.z * inv, acc.w * inv);
        } else {
            const int64_t prow = (int64_t)slot * p.T * p.H_q + orow;
            *reinterpret_cast<float4 *>(p.ws_o + prow * D + c4 * 4) =
                make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
            if (c4 == 0)
                p.ws_lse[prow] = Lsum > 0.f ? M + log2f(Lsum) : -INFINITY;
        }
    }
}

template <int D, bool BF16, bool NARROW>
__global__ void __launch_bounds__(kThreads, NARROW ? kNarrowCtasPerSm : 1)
    pa_attn_rows_fp8_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                            const __grid_constant__ CUtensorMap tmap_ks, const __grid_constant__ CUtensorMap tmap_vs,
                            const RowsParams p)
{
    using L = Fp8Smem<D, NARROW>;
    constexpr int STAGES = L::kStages;
    constexpr int KSTEPS = D / 16;  // k-steps of S = Q K^T
    constexpr int NT = D / 8;       // n-tiles of O

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint8_t *s_ring = smem + L::kRingOff;
    float *s_scale = reinterpret_cast<float *>(smem + L::kScaleOff);
    uint64_t *s_bar = reinterpret_cast<uint64_t *>(smem + L::kBarOff);
    int *s_count = reinterpret_cast<int *>(smem + L::kCountOff);
    int *s_issued = reinterpret_cast<int *>(smem + L::kIssuedOff);
    int32_t *s_pages = reinterpret_cast<int32_t *>(smem + L::kTableOff);
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + L::kFlagOff);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    griddep_wait();     // the sequence order comes from the kernel before this one
    griddep_release();  // the split merge after this kernel may be scheduled (it waits for this grid)

    // ---- which (sequence, KV head, row group, split): as the 16-bit kernel ----------------
    const int b = __ldg(p.order + blockIdx.z);
    const int split = blockIdx.x;
    const int g = blockIdx.y / p.n_rg, rg = blockIdx.y % p.n_rg;
    const int q0 = __ldg(p.cu_seqlens + b), q1 = __ldg(p.cu_seqlens + b + 1);
    const int qb = q1 - q0, ctx = __ldg(p.context_lens + b);
    if (!seq_ok(qb, ctx, p, q1)) {
        if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0)
            set_status(p.status, PA_ERR_SEQ);
        return;
    }
    const int G = p.G;
    const int R = G * qb;
    const int row0 = rg * kRowsPerCta;
    if (row0 >= R)
        return;
    const int rows_here = min(kRowsPerCta, R - row0);
    const int lim_cta = ctx - qb + (row0 + rows_here - 1) / G;
    const int pages_need = lim_cta / 16 + 1;
    const int pages_ctx = (ctx + 15) / 16;
    const int n_splits = (pages_ctx + p.split_pages - 1) / p.split_pages;
    if (split >= n_splits)
        return;
    const int page_lo = split * p.split_pages;
    const int page_hi = min(page_lo + p.split_pages, pages_need);
    const int n_pages = max(0, page_hi - page_lo);
    const int n_stages = (n_pages + kPagesPerStage - 1) / kPagesPerStage;
    const int MT = rows_here <= 16 ? 1 : (rows_here <= 32 ? 2 : 4);
    const int KG = 4 / MT;
    const int mt = warp / KG, kg = warp % KG;
    const bool has_rows = mt * 16 < rows_here;
    if (NARROW && rows_here > 8) {  // the host picks this variant for single-token decode with G <= 8 only
        if (tid == 0)
            set_status(p.status, PA_ERR_UNSUPPORTED);
        return;
    }

    // ---- set-up: barriers and the first loads, page ids and scales, Q fragments -------------
    const int32_t *table = p.block_tables + (int64_t)b * p.max_blocks;
    auto checked = [&](int pg) -> int {
        if (pg < 0 || pg >= p.num_blocks) {
            set_status(p.status, PA_ERR_BOUNDS);
            pg = static_cast<int>(p.num_blocks);  // past the pool: TMA fills zeros, scales 0
        }
        return pg;
    };
    // bytes a page brings into a stage: its K and V codes and, NARROW, its 16 K and 16 V scales
    constexpr int kPageTx = 2 * L::kPage + (NARROW ? 2 * 16 * 4 : 0);
    auto load_page = [&](int slot, int k, int pg) {
        uint8_t *kb = s_ring + slot * L::kStage;
        const int y = (pg * p.H_kv + g) * 16;
        tma_load_2d(kb + k * L::kPage, &tmap_k, 0, y, &s_bar[slot]);
        tma_load_2d(kb + (kPagesPerStage + k) * L::kPage, &tmap_v, 0, y, &s_bar[slot]);
        if constexpr (NARROW) {
            // a bad page id was replaced by num_blocks: its scale row is past the map, zero filled
            float *sc = s_scale + slot * L::kStageScales;
            tma_load_2d(sc + k * L::kScaleSlot, &tmap_ks, 0, pg * p.H_kv + g, &s_bar[slot]);
            tma_load_2d(sc + (kPagesPerStage + k) * L::kScaleSlot, &tmap_vs, 0, pg * p.H_kv + g, &s_bar[slot]);
        }
    };
    auto issue = [&](int st) {  // one thread; the page ids from the shared-memory copy
        const int slot = st % STAGES;
        const int np = min(kPagesPerStage, n_pages - st * kPagesPerStage);
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&s_bar[slot], np * kPageTx);
        s_issued[slot] += 1;
        for (int k = 0; k < np; ++k)
            load_page(slot, k, s_pages[st * kPagesPerStage + k]);
    };
    if (warp == 0) {
        // every stage of the ring goes out at once: lane i reads the id of page i from the table
        // in global memory and issues that page's two boxes
        static_assert(STAGES * kPagesPerStage <= 32, "one lane per page of the first stages");
        if (lane == 0) {
            for (int s = 0; s < STAGES; ++s) {
                mbar_init(&s_bar[s], 1);
                s_count[s] = 0;
                s_issued[s] = 0;
            }
            *s_abort = 0;
            fence_barrier_init();
            prefetch_tmap(&tmap_k);
            prefetch_tmap(&tmap_v);
            if constexpr (NARROW) {
                prefetch_tmap(&tmap_ks);
                prefetch_tmap(&tmap_vs);
            }
        }
        const int first = min(STAGES, n_stages);
        const bool mine = lane < first * kPagesPerStage && lane < n_pages;
        const int pg = mine ? checked(__ldg(table + page_lo + lane)) : 0;
        __syncwarp();
        if (lane == 0) {
            for (int st = 0; st < first; ++st) {
                mbar_arrive_expect_tx(&s_bar[st], min(kPagesPerStage, n_pages - st * kPagesPerStage) * kPageTx);
                s_issued[st] += 1;
            }
        }
        __syncwarp();
        if (mine)
            load_page(lane / kPagesPerStage, lane % kPagesPerStage, pg);
    }
    // page ids and the scales of the split's keys; keys past the context end (or of a bad page)
    // get scale 0
    for (int i = tid; i < n_pages; i += kThreads) {
        const int pg = checked(__ldg(table + page_lo + i));
        s_pages[i] = pg;
        if constexpr (NARROW)
            continue;
        const int keys_left = ctx - (page_lo + i) * 16;
#pragma unroll
        for (int kv = 0; kv < 2; ++kv) {
            const float4 *src =
                reinterpret_cast<const float4 *>((kv ? p.v_scale : p.k_scale) + ((int64_t)pg * p.H_kv + g) * 16);
            float4 *dst = reinterpret_cast<float4 *>(s_scale + (i * 2 + kv) * 16);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (pg < p.num_blocks)
                    v = __ldg(src + j);
                v.x = 4 * j < keys_left ? v.x : 0.f;
                v.y = 4 * j + 1 < keys_left ? v.y : 0.f;
                v.z = 4 * j + 2 < keys_left ? v.z : 0.f;
                v.w = 4 * j + 3 < keys_left ? v.w : 0.f;
                dst[j] = v;
            }
        }
    }

    // This thread holds rows ra = lane/4 and rb = ra + 8 of its warp's m-tile.
    const int ra = mt * 16 + (lane >> 2), rb = ra + 8;
    const int lim_a = ra < rows_here ? ctx - qb + (row0 + ra) / G : -1;
    const int lim_b = rb < rows_here ? ctx - qb + (row0 + rb) / G : -1;
    const int lim_warp = has_rows ? ctx - qb + (row0 + min(mt * 16 + 15, rows_here - 1)) / G : -1;
    // Q fragments in the column order of rows_page_fp8: qa[ks][0] = Q[ra][c0 + 4ks + {0, 1}] and
    // qa[ks][2] = Q[ra][c0 + 4ks + {2, 3}] with c0 = (lane % 4) * D/4; [1] and [3] likewise for rb.
    // The narrow variant's B operand (Q^T) is the same two words of row lane/4: qn[ks][0], [1].
    uint32_t qa[KSTEPS][4], qn[KSTEPS][2];
    int lim_n[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int r = 2 * (lane & 3) + i;
        lim_n[i] = r < rows_here ? ctx - qb + (row0 + r) / G : -1;
    }
#pragma unroll
    for (int half = 0; half < (NARROW ? 1 : 2); ++half) {
        const int rr = NARROW ? (lane >> 2) : (half ? rb : ra);
        uint32_t w[D / 8];
#pragma unroll
        for (int i = 0; i < D / 8; ++i)
            w[i] = 0u;
        if (has_rows && rr < rows_here) {
            const int ridx = row0 + rr;
            const int64_t t = q0 + ridx / G;
            const int h = g * G + ridx % G;
            const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(p.q) +
                                                               ((t * p.H_q + h) * D + (lane & 3) * (D / 4)) * 2);
#pragma unroll
            for (int i = 0; i < D / 32; ++i) {
                const uint4 v = __ldg(src + i);
                w[4 * i] = v.x;
                w[4 * i + 1] = v.y;
                w[4 * i + 2] = v.z;
                w[4 * i + 3] = v.w;
            }
        }
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
            if constexpr (NARROW) {
                qn[ks][0] = w[2 * ks];
                qn[ks][1] = w[2 * ks + 1];
            } else {
                qa[ks][half] = w[2 * ks];
                qa[ks][2 + half] = w[2 * ks + 1];
            }
        }
    }
    __syncthreads();  // page ids, scales and barriers are set
    float o[NT][4];
#pragma unroll
    for (int i = 0; i < NT; ++i)
        o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
    float on[D / 16][4], m_n[2] = {-INFINITY, -INFINITY}, l_n[2] = {0.f, 0.f};
#pragma unroll
    for (int i = 0; i < D / 16; ++i)
        on[i][0] = on[i][1] = on[i][2] = on[i][3] = 0.f;
    const float sl2 = p.scale_log2;


    // ---- main loop over stages (as the 16-bit kernel) ------------------------------------------
    for (int it = 0; it < n_stages; ++it) {
        const int slot = it % STAGES;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&s_bar[slot], (it / STAGES) & 1));
        if (!ok) {
            *s_abort = 1;
            set_status(p.status, PA_ERR_TIMEOUT);
        }
        if constexpr (NARROW) {
            // one page per warp per stage (KG = 4); the scales of its keys 2g, 2g + 1.  A key past
            // the context end is masked from the scores whatever its K scale; its V scale (which
            // may be anything, NaN included) becomes 0 so that P = 0 stays 0.
            const int pidx = it * kPagesPerStage + kg;
            const int j0 = (page_lo + pidx) * 16;
            if (ok && has_rows && pidx < n_pages && j0 <= lim_warp) {
                const float *sc = s_scale + slot * L::kStageScales + 2 * (lane >> 2);
                const float2 kf = *reinterpret_cast<const float2 *>(sc + kg * L::kScaleSlot);
                float2 vf = *reinterpret_cast<const float2 *>(sc + (kPagesPerStage + kg) * L::kScaleSlot);
                const int key0 = j0 + 2 * (lane >> 2);
                vf.x = key0 < ctx ? vf.x : 0.f;
                vf.y = key0 + 1 < ctx ? vf.y : 0.f;
                const uint8_t *st = s_ring + slot * L::kStage;
                narrow_page_fp8<D, BF16>(st + kg * L::kPage, st + (kPagesPerStage + kg) * L::kPage, kf, vf, j0, lane,
                                         qn, on, m_n, l_n, lim_n, ctx, sl2);
            }
        } else if (ok && has_rows) {
            const uint8_t *st = s_ring + slot * L::kStage;
            for (int k = kg; k < kPagesPerStage; k += KG) {
                const int pidx = it * kPagesPerStage + k;
                if (pidx >= n_pages)
                    break;
                const int j0 = (page_lo + pidx) * 16;
                if (j0 > lim_warp)
                    continue;  // every row of this warp is causally masked on this page
                rows_page_fp8<D, BF16>(st + k * L::kPage, st + (kPagesPerStage + k) * L::kPage, s_scale + pidx * 32,
                                       j0, lane, qa, o, m_a, m_b, l_a, l_b, lim_a, lim_b, ctx, sl2);
            }
        }
        // the last warp done with this slot refills it
        __syncwarp();
        if (lane == 0 && atomicAdd(&s_count[slot], 1) == 3) {
            s_count[slot] = 0;
            if (it + STAGES < n_stages && !*s_abort)
                issue(it + STAGES);
        }
        if (*s_abort)
            break;
    }
    __syncthreads();
    if (*s_abort) {
        // let the copies still in flight land (bounded) before the CTA releases its shared memory
        if (tid == 0)
            for (int s = 0; s < STAGES; ++s)
                if (s_issued[s] > 0)
                    mbar_wait(&s_bar[s], (s_issued[s] - 1) & 1, kWaitTimeoutNs / 10);
        return;
    }
    if constexpr (NARROW)
        narrow_epilogue<D, BF16>(reinterpret_cast<float *>(s_ring), p, on, m_n, l_n, rows_here, row0, q0, g, split,
                                 n_splits == 1);
    else
        rows_epilogue<D, BF16>(reinterpret_cast<float *>(s_ring), p, o, m_a, m_b, l_a, l_b, has_rows, rows_here, row0,
                               q0, g, split, n_splits == 1, KG);
}

// One warp per (token, query head) row of a sequence with more than one split:
// O = sum_s 2^(lse_s - lse) O_s,  lse = log2 sum_s 2^lse_s.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) pa_split_merge_kernel(const RowsParams p)
{
    griddep_wait();  // the partials of the attention kernel
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 8 + warp;
    if (row >= p.T * p.H_q)
        return;
    const int64_t t = row / p.H_q;
    const int b = seq_of_token(p.cu_seqlens, p.B, t);
    const int q0 = __ldg(p.cu_seqlens + b), q1 = __ldg(p.cu_seqlens + b + 1);
    const int ctx = __ldg(p.context_lens + b);
    if (!seq_ok(q1 - q0, ctx, p, q1))
        return;
    const int pages_ctx = (ctx + 15) / 16;
    // shared-prefix decode: the prefix's splits sit in slots [0, nps), the sequence's own splits
    // from prefix_slots on, and every row goes through the merge
    const bool shared = p.seq_prefix != nullptr;
    int nps = 0, own_lo = 0, own_slot = 0;
    if (shared) {
        own_lo = min(max(__ldg(p.seq_prefix + b), 0), (ctx - (q1 - q0)) / 16);
        nps = (own_lo + p.prefix_split_pages - 1) / p.prefix_split_pages;
        own_slot = p.prefix_slots;
    }
    const int ns = nps + (pages_ctx - own_lo + p.split_pages - 1) / p.split_pages;
    if (!shared && ns <= 1)
        return;
    auto slot = [&](int s) -> int64_t { return s < nps ? s : own_slot + (s - nps); };
    const int64_t stride = p.T * p.H_q;
    constexpr int LANES = D / 4;
    if (ns <= 32) {
        // one split per lane: its log2-sum-exp read once, the weights 2^(lse_s - max) / sum in
        // registers, then the partials read four splits at a time (independent loads in flight)
        const float l = lane < ns ? p.ws_lse[slot(lane) * stride + row] : -INFINITY;
        float M = l;
#pragma unroll
        for (int o = 16; o; o >>= 1)
            M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float w = l == -INFINITY ? 0.f : fast_exp2(l - M);
        float Z = w;
#pragma unroll
        for (int o = 16; o; o >>= 1)
            Z += __shfl_xor_sync(0xffffffffu, Z, o);
        w *= Z > 0.f ? 1.f / Z : 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s0 = 0; s0 < ns; s0 += 4) {
            float ws[4];
            float4 v[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                ws[k] = __shfl_sync(0xffffffffu, w, (s0 + k) & 31);
                if (s0 + k >= ns)
                    ws[k] = 0.f;
                v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (ws[k] != 0.f && lane < LANES)
                    v[k] = *reinterpret_cast<const float4 *>(p.ws_o + (slot(s0 + k) * stride + row) * D + lane * 4);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (ws[k] == 0.f)
                    continue;
                acc.x += ws[k] * v[k].x;
                acc.y += ws[k] * v[k].y;
                acc.z += ws[k] * v[k].z;
                acc.w += ws[k] * v[k].w;
            }
        }
        if (lane < LANES)
            store4<BF16>(static_cast<uint8_t *>(p.out) + (row * D + lane * 4) * 2, acc.x, acc.y, acc.z, acc.w);
        return;
    }
    float M = -INFINITY;
    for (int s = lane; s < ns; s += 32)
        M = fmaxf(M, p.ws_lse[slot(s) * stride + row]);
#pragma unroll
    for (int o = 16; o; o >>= 1)
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float Z = 0.f;
    for (int s = lane; s < ns; s += 32) {
        const float l = p.ws_lse[slot(s) * stride + row];
        Z += l == -INFINITY ? 0.f : fast_exp2(l - M);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
        Z += __shfl_xor_sync(0xffffffffu, Z, o);
    const float invZ = Z > 0.f ? 1.f / Z : 0.f;
    if (lane < LANES) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s = 0; s < ns; ++s) {
            const float l = p.ws_lse[slot(s) * stride + row];
            if (l == -INFINITY)
                continue;
            const float w = fast_exp2(l - M) * invZ;
            const float4 v = *reinterpret_cast<const float4 *>(p.ws_o + (slot(s) * stride + row) * D + lane * 4);
            acc.x += w * v.x;
            acc.y += w * v.y;
            acc.z += w * v.z;
            acc.w += w * v.w;
        }
        store4<BF16>(static_cast<uint8_t *>(p.out) + (row * D + lane * 4) * 2, acc.x, acc.y, acc.z, acc.w);
    }
}

// Shared-prefix decode, before the rows kernel (one CTA): the longest-first order of the
// sequences, the checks of the groups and, with fill_prefix, seq_prefix[b] = the prefix blocks of
// sequence b's group, or 0 where the shared pass must not be used for b -- its table does not
// start with the group leader's prefix blocks, or the prefix reaches its new tokens; such a
// sequence is computed over its own table alone (the result is the same).  Malformed groups (not a
// partition of the sequences into consecutive runs, a prefix outside the table, more new tokens
// than the rows planned for a group, a prefix longer than the planned bound) set PA_ERR_ARG and
// turn every sequence into the unshared case.
__global__ void __launch_bounds__(kOrderThreads) pa_shared_plan_kernel(const RowsParams p, int32_t *order,
                                                                         int fill_prefix)
{
    griddep_wait();  // the kernel before this call's on the stream (its writes are visible after this)
    if (threadIdx.x == 0)
        *p.status = PA_OK;  // the call's status word: this is its first kernel
    __syncthreads();        // before any thread records a malformed group
    griddep_release();      // the attention kernel waits for the order and the group checks
    // first the longest-first order of the sequences (as pa_seq_order_kernel), in this same launch
    order_by_key_desc(
        p.B,
        [&](int b) {
            const int ctx = __ldg(p.context_lens + b);
            const int pages = ctx > 0 ? (ctx + 15) / 16 : 0;
            return min(pages, kOrderKeys - 1);
        },
        order);
    __shared__ int bad;
    const int tid = threadIdx.x;
    if (tid == 0)
        bad = __ldg(p.group_start) != 0 || __ldg(p.group_start + p.n_groups) != p.B;
    __syncthreads();
    for (int v = tid; v < p.n_groups; v += blockDim.x) {
        const int s0 = __ldg(p.group_start + v), s1 = __ldg(p.group_start + v + 1);
        const int P = __ldg(p.prefix_blocks + v);
        if (s0 < 0 || s1 < s0 || s1 > p.B || P < 0 || P > p.max_blocks || P > p.prefix_slots * p.prefix_split_pages)
            bad = 1;
        else if (s1 > s0 && (int64_t)(__ldg(p.cu_seqlens + s1) - __ldg(p.cu_seqlens + s0)) * p.G >
                                (int64_t)p.n_rg * kRowsPerCta)
            bad = 1;
    }
    __syncthreads();
    if (bad) {
        if (tid == 0)
            set_status(p.status, PA_ERR_ARG);
        for (int b = tid; b < p.B && fill_prefix; b += blockDim.x)
            p.seq_prefix[b] = 0;
        return;
    }
    if (!fill_prefix)  // the plain decode computes the result: only the checks above are wanted
        return;
    // one warp per sequence: its lanes compare the prefix entries with the leader's side by side
    const int lane = tid & 31;
    for (int b = tid >> 5; b < p.B; b += blockDim.x >> 5) {
        // b's group: the last v with group_start[v] <= b (groups may be empty)
        int lo = 0, hi = p.n_groups - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) / 2;
            if (__ldg(p.group_start + mid) <= b)
                lo = mid;
            else
                hi = mid - 1;
        }
        const int s0 = __ldg(p.group_start + lo);
        const int P = __ldg(p.prefix_blocks + lo);
        const int q_b = __ldg(p.cu_seqlens + b + 1) - __ldg(p.cu_seqlens + b);
        const int use = (int64_t)P * 16 <= (int64_t)__ldg(p.context_lens + b) - q_b ? P : 0;
        const int32_t *mine = p.block_tables + (int64_t)b * p.max_blocks;
        const int32_t *lead = p.block_tables + (int64_t)s0 * p.max_blocks;
        bool same = true;
        for (int i = lane; i < use; i += 32)
            same &= __ldg(mine + i) == __ldg(lead + i);
        same = __all_sync(0xffffffffu, same);
        if (lane == 0)
            p.seq_prefix[b] = same ? use : 0;
    }
}

// ---- host side ------------------------------------------------------------------------------

constexpr int kStages = PA_ROWS_STAGES;
// Rows per (sequence, KV head) from which a 16-bit decode goes to the tcgen05 rows kernel.
#ifndef PA_WIDE_ROWS
#define PA_WIDE_ROWS 16
#endif
constexpr int kWideRows = PA_WIDE_ROWS;

template <int D, bool BF16, int MODE>
static int launch_rows(const RowsParams &rp, const CUtensorMap &tk, const CUtensorMap &tv, dim3 grid,
                       cudaStream_t stream)
{
    using L = RowsSmem<D, kStages>;
    auto kern = pa_attn_rows_kernel<D, BF16, kStages, MODE>;
    static uint64_t configured = 0;  // one bit per device, per template instance
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return PA_ERR_CUDA;
    const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
    if (!bit || !(configured & bit)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) != cudaSuccess)
            return PA_ERR_CUDA;
        configured |= bit;
    }
    const cudaError_t e = launch_dependent(kern, grid, dim3(kThreads), L::kAlloc, stream, tk, tv, rp);
    count_launch();
    const cudaError_t e2 = cudaGetLastError();
    return e == cudaSuccess && e2 == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <int D, bool BF16, bool NARROW>
static int launch_rows_fp8(const RowsParams &rp, const CUtensorMap &tk, const CUtensorMap &tv,
                           const CUtensorMap &tks, const CUtensorMap &tvs, dim3 grid, cudaStream_t stream)
{
    using L = Fp8Smem<D, NARROW>;
    auto kern = pa_attn_rows_fp8_kernel<D, BF16, NARROW>;
    static uint64_t configured = 0;  // one bit per device, per template instance
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return PA_ERR_CUDA;
    const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
    if (!bit || !(configured & bit)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) != cudaSuccess)
            return PA_ERR_CUDA;
        configured |= bit;
    }
    const cudaError_t e = launch_dependent(kern, grid, dim3(kThreads), L::kAlloc, stream, tk, tv, tks, tvs, rp);
    count_launch();
    const cudaError_t e2 = cudaGetLastError();
    return e == cudaSuccess && e2 == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// Longest sequences first: decode CTAs are dispatched in grid order, so putting the sequences with
// the most pages at the front leaves short CTAs for the last wave (longest-processing-time-first
// list scheduling; the order among equal page counts is arbitrary and changes no result).
__global__ void __launch_bounds__(kOrderThreads)
    pa_seq_order_kernel(const int32_t *context_lens, int B, int32_t *order, int32_t *status)
{
    griddep_wait();  // the kernel before this call's on the stream (its writes are visible after this)
    if (threadIdx.x == 0)
        *status = PA_OK;  // the call's status word: this is its first kernel
    griddep_release();    // the attention kernel's CTAs may be scheduled now; they wait for the order
    order_by_key_desc(
        B,
        [&](int b) {
            const int ctx = __ldg(context_lens + b);
            const int pages = ctx > 0 ? (ctx + 15) / 16 : 0;
            return min(pages, kOrderKeys - 1);
        },
        order);
}

int launch_seq_order(const int32_t *context_lens, int B, int32_t *order, int32_t *status, cudaStream_t stream)
{
    const cudaError_t e = launch_dependent(pa_seq_order_kernel, dim3(1), dim3(kOrderThreads), 0, stream, context_lens, B,
                                           order, status);
    count_launch();
    const cudaError_t e2 = cudaGetLastError();
    return e == cudaSuccess && e2 == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <int D, bool BF16>
static int launch_merge(const RowsParams &rp, cudaStream_t stream)
{
    const int64_t rows = rp.T * rp.H_q;
    const int64_t blocks = (rows + 7) / 8;
    const cudaError_t e =
        launch_dependent(pa_split_merge_kernel<D, BF16>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream, rp);
    count_launch();
    const cudaError_t e2 = cudaGetLastError();
    return e == cudaSuccess && e2 == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

static int split_pages_override()
{
    static int v = -2;
    if (v == -2) {
        const char *e = getenv("PA_DECODE_SPLIT_PAGES");
        v = e ? atoi(e) : -1;
    }
    return v;
}

// Decode CTAs the split planner counts on per SM.
#ifndef PA_PLAN_CTAS_PER_SM
#define PA_PLAN_CTAS_PER_SM 3
#endif

// Pages per split for `units` independent (sequence, KV head, row group) units of up to `pages`
// pages on `slots` resident CTAs: the multiple of the stage size in [16, kMaxTablePages] that
// minimises the time of a batch whose every unit has `pages` pages, modelled as (full waves of
// CTAs) x (split length + a fixed per-CTA cost of `cta_cost` pages).  Longer splits mean fewer CTAs
// and less fixed cost; the wave count rounds up, so a split that fills the last wave beats a
// slightly shorter one that leaves it nearly empty.
static int plan_split_pages(int64_t units, int64_t pages, int64_t slots, int64_t cta_cost)
{
    int64_t sp = kMaxTablePages, best = -1;
    for (int64_t c = kMaxTablePages; c >= 16 && units > 0 && pages > 0; c -= kPagesPerStage) {
        const int64_t ctas = units * ((pages + c - 1) / c);
        const int64_t waves = (ctas + slots - 1) / slots;
        const int64_t len = c < pages ? c : pages;
        const int64_t cost = waves * (len + cta_cost);
        if (best < 0 || cost < best) {
            best = cost;
            sp = c;
        }
    }
    return static_cast<int>(sp);
}

DecodePlan decode_plan(int B, int H_q, int H_kv, int d, int max_ctx)
{
    DecodePlan pl;
    const int G = H_q / H_kv;
    pl.row_groups = (8 * G + kRowsPerCta - 1) / kRowsPerCta;
    const int64_t pages = (int64_t)(max_ctx + 15) / 16;
    // the mma.sync kernels: PA_PLAN_CTAS_PER_SM CTAs per SM, a per-CTA cost of ~80 KB of streaming
    const int64_t page_bytes = 2 * 16 * (int64_t)d * 2;
    const int64_t cta_cost = (80 * 1024 + page_bytes - 1) / page_bytes;
    int64_t sp = plan_split_pages((int64_t)B * H_kv * pl.row_groups, pages, (int64_t)sm_count() * PA_PLAN_CTAS_PER_SM,
                                  cta_cost);
    const int ov = split_pages_override();
    if (ov > 0)
        sp = ov < kMaxTablePages ? ov : kMaxTablePages;
    pl.split_pages = static_cast<int>(sp);
    pl.max_splits = pages > 0 ? static_cast<int>((pages + sp - 1) / sp) : 1;
    return pl;
}

// Split plan of the tcgen05 rows kernel for `units` (sequence, KV head, row group) units: two CTAs
// per SM, and a per-CTA cost of 32 pages (its TMEM allocation, Q load and the first K/V tiles'
// latency before the ring streams, the partials and the merge of every extra split) -- fitted to
// tree verification of 64 sequences x 8 drafts over contexts U[512, 4096] with 32/8 heads, where
// splits of 64 / 128 / 256 pages measured 0.141 / 0.126 / 0.113 ms.  Never finer than `ws`, the
// plan the workspace was sized for.
static DecodePlan decode_plan_tc(int64_t units, int max_ctx, const DecodePlan &ws)
{
    DecodePlan pl = ws;
    const int64_t pages = (int64_t)(max_ctx + 15) / 16;
    int sp = plan_split_pages(units, pages, (int64_t)sm_count() * 2, 32);
    if (split_pages_override() > 0 || sp < ws.split_pages)
        sp = ws.split_pages;
    pl.split_pages = sp;
    pl.max_splits = pages > 0 ? static_cast<int>((pages + sp - 1) / sp) : 1;
    return pl;
}

// Workspace: status word area, the sequence order, then (with more than one split) the partial
// outputs and their log-sum-exps.
size_t seq_order_bytes(int B) { return (static_cast<size_t>(B) * sizeof(int32_t) + 255) / 256 * 256; }

size_t decode_workspace_bytes(int64_t T, int B, int H_q, int H_kv, int d, int max_ctx)
{
    const DecodePlan pl = decode_plan(B, H_q, H_kv, d, max_ctx);
    size_t bytes = PA_STATUS_BYTES + seq_order_bytes(B);
    if (pl.max_splits > 1) {
        const size_t rows = static_cast<size_t>(pl.max_splits) * static_cast<size_t>(T) * H_q;
        bytes += rows * d * sizeof(float);
        bytes += rows * sizeof(float);
        bytes += 256;
    }
    return bytes;
}

SharedPlan shared_plan(int B, int H_q, int H_kv, int d, int max_ctx, int n_groups, int max_prefix_blocks,
                       int max_group_tokens)
{
    SharedPlan sp;
    sp.own = decode_plan(B, H_q, H_kv, d, max_ctx);
    const int G = H_q / H_kv;
    const int rg_prefix = max(1, (max_group_tokens * G + kRowsPerCta - 1) / kRowsPerCta);
    sp.row_groups = max(sp.own.row_groups, rg_prefix);
    // prefix splits: about one wave of prefix CTAs (two per SM), at least 16 pages each
    const int64_t units = (int64_t)max(n_groups, 1) * H_kv * rg_prefix;
    const int64_t slots = (int64_t)sm_count() * 2;
    const int64_t want = (slots + units - 1) / units;  // >= 1
    int64_t len = max_prefix_blocks > 0 ? (max_prefix_blocks + want - 1) / want : 16;
    len = (len + kPagesPerStage - 1) / kPagesPerStage * kPagesPerStage;
    len = len < 16 ? 16 : (len > kMaxTablePages ? kMaxTablePages : len);
    sp.prefix_split_pages = static_cast<int>(len);
    sp.prefix_slots = max_prefix_blocks > 0 ? static_cast<int>((max_prefix_blocks + len - 1) / len) : 0;
    return sp;
}

// Workspace of the shared-prefix decode: status, sequence order, seq_prefix, then the partials of
// the prefix splits and of the sequences' own splits (every row is merged).
size_t shared_workspace_bytes(int64_t T, int B, int H_q, int H_kv, int d, int max_ctx, int n_groups,
                              int max_prefix_blocks, int max_group_tokens)
{
    const SharedPlan sp = shared_plan(B, H_q, H_kv, d, max_ctx, n_groups, max_prefix_blocks, max_group_tokens);
    const size_t rows = static_cast<size_t>(sp.prefix_slots + sp.own.max_splits) * static_cast<size_t>(T) * H_q;
    return PA_STATUS_BYTES + 2 * seq_order_bytes(B) + rows * d * sizeof(float) + rows * sizeof(float) + 256;
}

// Does the shared-prefix pass pay for itself?  Reading a group's prefix once saves (n - 1) / n of
// the prefix keys of a group of n sequences, about (n - 1) / n x prefix / context of the keys the
// batch reads; the pass costs the prefix CTAs (a whole group's rows on every prefix page), a
// partial output for every row and the merge.  Below a quarter of the keys saved it loses to the
// plain decode, which also finds repeated prefix blocks in L2 (measured: 16 sequences sharing 2048
// of 32768 tokens, 6 % of the keys: 0.89x the plain decode; 64 requests in groups of 16 sharing
// 4096 of <= 4608 tokens, 83 %: 4.7x).  Host bounds only: mean group size B / n_groups, prefix
// max_prefix_blocks, context max_ctx (an overestimate, so the plain path is taken when unsure).
static bool shared_pass_pays(const AttnArgs &a)
{
    if (a.n_groups < 1 || a.max_ctx < 1 || a.max_prefix_blocks < 1)
        return false;
    const double n = static_cast<double>(a.B) / a.n_groups;
    const double prefix = 16.0 * a.max_prefix_blocks;
    const double saved = (n - 1.0) / n * (prefix < a.max_ctx ? prefix : a.max_ctx) / a.max_ctx;
    return saved >= 0.25;
}

template <int D, bool BF16>
static int run(const AttnArgs &a)
{
    const bool fp8 = a.key_scale != nullptr;
    CUtensorMap tk, tv;
    int rc = fp8 ? make_cache_tmap_fp8(&tk, a.key_cache, a.num_blocks, a.H_kv, D)
                 : make_cache_tmap(&tk, a.key_cache, a.num_blocks, a.H_kv, D, a.dtype);
    if (rc == PA_OK)
        rc = fp8 ? make_cache_tmap_fp8(&tv, a.value_cache, a.num_blocks, a.H_kv, D)
                 : make_cache_tmap(&tv, a.value_cache, a.num_blocks, a.H_kv, D, a.dtype);
    CUtensorMap tks{}, tvs{};  // FP8: the row scales, which the narrow kernel loads with each stage
    if (rc == PA_OK && fp8)
        rc = make_scale_tmap(&tks, a.key_scale, a.num_blocks, a.H_kv);
    if (rc == PA_OK && fp8)
        rc = make_scale_tmap(&tvs, a.value_scale, a.num_blocks, a.H_kv);
    if (rc != PA_OK)
        return rc;
    RowsParams rp{};
    rp.q = a.q;
    rp.out = a.out;
    rp.block_tables = a.block_tables;
    rp.cu_seqlens = a.cu_seqlens_q;
    rp.context_lens = a.context_lens;
    rp.status = static_cast<int32_t *>(a.workspace);
    rp.num_blocks = a.num_blocks;
    rp.T = a.T;
    rp.max_blocks = a.max_blocks;
    rp.B = a.B;
    rp.H_q = a.H_q;
    rp.H_kv = a.H_kv;
    rp.G = a.H_q / a.H_kv;
    rp.max_ctx = a.max_ctx;
    rp.max_q_len = a.max_q_len;
    rp.scale_log2 = a.scale * 1.4426950408889634f;
    rp.tree = a.tree_mask;
    rp.k_scale = a.key_scale;
    rp.v_scale = a.value_scale;
    if (a.group_start) {
        const SharedPlan sp = shared_plan(a.B, a.H_q, a.H_kv, a.d, a.max_ctx, a.n_groups, a.max_prefix_blocks,
                                          a.max_group_tokens);
        rp.n_rg = sp.row_groups;
        rp.split_pages = sp.own.split_pages;
        rp.prefix_split_pages = sp.prefix_split_pages;
        rp.prefix_slots = sp.prefix_slots;
        rp.n_groups = a.n_groups;
        rp.group_start = a.group_start;
        rp.prefix_blocks = a.prefix_blocks;
        uint8_t *ws = static_cast<uint8_t *>(a.workspace) + PA_STATUS_BYTES;
        int32_t *order = reinterpret_cast<int32_t *>(ws);
        int32_t *seq_prefix = reinterpret_cast<int32_t *>(ws + seq_order_bytes(a.B));
        rp.order = order;
        rp.seq_prefix = seq_prefix;
        const size_t rows = static_cast<size_t>(sp.prefix_slots + sp.own.max_splits) * static_cast<size_t>(a.T) * a.H_q;
        uint8_t *part = ws + 2 * seq_order_bytes(a.B);
        rp.ws_o = reinterpret_cast<float *>(part);
        rp.ws_lse = reinterpret_cast<float *>(part + rows * D * sizeof(float));
        const int64_t z = (int64_t)a.n_groups + a.B;
        if (z > 65535 || (int64_t)a.H_kv * sp.row_groups > 65535)
            return PA_ERR_UNSUPPORTED;
        dim3 grid(max(sp.own.max_splits, sp.prefix_slots), a.H_kv * sp.row_groups, static_cast<unsigned>(z));
        // one launch writes the sequence order and checks the groups (status), whichever path
        // computes the result
        const bool pays = shared_pass_pays(a);
        const cudaError_t e =
            launch_dependent(pa_shared_plan_kernel, dim3(1), dim3(kOrderThreads), 0, a.stream, rp, order, pays ? 1 : 0);
        count_launch();
        const cudaError_t e2 = cudaGetLastError();
        rc = e == cudaSuccess && e2 == cudaSuccess ? PA_OK : PA_ERR_CUDA;
        if (rc != PA_OK)
            return rc;
        if (pays) {
            // (the prefix rows of a group stay on the mma.sync kernel: with three CTAs per SM it
            // beat the tcgen05 rows kernel on the prefix pass, which it shares one launch with)
            if (rc == PA_OK)
                rc = launch_rows<D, BF16, kModeShared>(rp, tk, tv, grid, a.stream);
            if (rc == PA_OK)
                rc = launch_merge<D, BF16>(rp, a.stream);
            return rc;
        }
        // the plain decode over the same tables: its workspace (status, order, partials) is no
        // larger than this one and starts at the same place (the plan kernel wrote no per-sequence
        // prefix lengths)
        rp.group_start = nullptr;
        rp.prefix_blocks = nullptr;
        rp.seq_prefix = nullptr;
        rp.n_groups = 0;
        rp.prefix_slots = 0;
        rp.ws_o = nullptr;
        rp.ws_lse = nullptr;
    }
    {
        const DecodePlan pl = decode_plan(a.B, a.H_q, a.H_kv, a.d, a.max_ctx);
        rp.n_rg = pl.row_groups;
        rp.split_pages = pl.split_pages;
        int32_t *order = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(a.workspace) + PA_STATUS_BYTES);
        rp.order = order;
        if (pl.max_splits > 1) {
            const size_t rows = static_cast<size_t>(pl.max_splits) * static_cast<size_t>(a.T) * a.H_q;
            uint8_t *ws = static_cast<uint8_t *>(a.workspace) + PA_STATUS_BYTES + seq_order_bytes(a.B);
            rp.ws_o = reinterpret_cast<float *>(ws);
            rp.ws_lse = reinterpret_cast<float *>(ws + rows * D * sizeof(float));
        }
        if (a.B > 65535 || (int64_t)a.H_kv * pl.row_groups > 65535)
            return PA_ERR_UNSUPPORTED;
        dim3 grid(pl.max_splits, a.H_kv * pl.row_groups, a.B);
        // 16-bit cache where every sequence has 16 or more rows per KV head (G query heads x its
        // new tokens, at least T - 8 (B - 1) of them): the tcgen05 rows kernel.  A batch that
        // mixes narrow and wide sequences stays on the mma.sync kernel: one launch over all of
        // them beats two launches in a row (measured on the mixed continuous-batching step).
        const int64_t max_q = std::min<int64_t>(8, a.T - a.B + 1);
        const int64_t min_q = std::max<int64_t>(1, a.T - 8 * (int64_t)(a.B - 1));
        const int tc_rows = rows_tc_rows_per_cta(rp.G, static_cast<int>(max_q));
        const bool all_wide = !fp8 && tc_rows > 0 && (int64_t)rp.G * min_q >= kWideRows;
        if (!a.group_start)  // the shared-prefix call's plan kernel has written the order already
            rc = launch_seq_order(a.context_lens, a.B, order, rp.status, a.stream);
        int merge_splits = pl.max_splits;  // splits of the kernel launched below
        if (rc == PA_OK && all_wide) {
            rp.n_rg = static_cast<int>(((int64_t)rp.G * max_q + tc_rows - 1) / tc_rows);
            const DecodePlan tp = decode_plan_tc((int64_t)a.B * a.H_kv * rp.n_rg, a.max_ctx, pl);
            rp.split_pages = tp.split_pages;
            merge_splits = tp.max_splits;
            const dim3 grid_tc(tp.max_splits, a.H_kv * rp.n_rg, a.B);
            rc = launch_rows_tc(rp, tk, tv, D, a.dtype, rp.tree ? kModeTree : kModeCausal, tc_rows, grid_tc,
                                a.stream);
        }
        if (rc == PA_OK && !all_wide) {
            // single-token decode with at most 8 query heads per KV head: keys on the MMA's M side
            rc = fp8 && a.T == a.B && rp.G <= 8 ? launch_rows_fp8<D, BF16, true>(rp, tk, tv, tks, tvs, grid, a.stream)
                 : fp8     ? launch_rows_fp8<D, BF16, false>(rp, tk, tv, tks, tvs, grid, a.stream)
                 : rp.tree ? launch_rows<D, BF16, kModeTree>(rp, tk, tv, grid, a.stream)
                           : launch_rows<D, BF16, kModeCausal>(rp, tk, tv, grid, a.stream);
        }
        if (rc == PA_OK && merge_splits > 1)
            rc = launch_merge<D, BF16>(rp, a.stream);
        return rc;
    }
}

int launch_decode(const AttnArgs &a)
{
    if (a.d == 128)
        return a.dtype == PA_BF16 ? run<128, true>(a) : run<128, false>(a);
    return a.dtype == PA_BF16 ? run<64, true>(a) : run<64, false>(a);
}

}  // namespace pa
