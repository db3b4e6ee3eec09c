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
//   * a query tile holds 128 rows = 128/G tokens x the G query heads of one KV
//     head, so every K/V tile is shared by the whole GQA group.  A work item is
//     a PAIR of consecutive query tiles (A, B) of one (sequence, KV head): both
//     tiles read the same K/V tiles, and while one softmax warpgroup works on
//     its scores the tensor core runs the other tile's products;
//   * K/V tiles of 128 keys = 8 pages of 16 keys, each page fetched by TMA
//     (64-element x 16-row boxes, 128-byte swizzle) straight from its block,
//     on separate K and V rings;
//   * S_X = Q_X K^T (X = A, B): tcgen05.mma M=128 N=128, K-major operands in
//     shared memory, fp32 accumulator in TMEM;
//   * softmax warpgroup X (one thread per row = TMEM lane) reads S_X with
//     tcgen05.ld, keeps the running max m and sum l in registers and writes
//     P_X (16-bit) back over S_X in TMEM;
//   * O_X += P_X V: tcgen05.mma with A = P_X from TMEM and B = V (MN-major) in
//     shared memory, fp32 accumulator in TMEM.  O_X is rescaled only when a
//     row's max grows by more than 2^8 (exact: the same stale max is used for
//     P and for l, and O / l is taken once at the end);
//   * the MMAs of tile X are issued by one thread of their own (warp 0 for A, warp 1 for B), in
//     the order S_X(j), O_X += P_X(j) V_j, S_X(j+1), ...; S_X(j+1) goes after the product that
//     reads the TMEM columns it overwrites (tcgen05.mma operations of one thread execute in issue
//     order), and the two threads feed the tensor core independently, so one tile's products run
//     while the other tile's softmax runs;
//   * warp 2 hands out work items from a global counter, heaviest first (sequences with the most
//     pages first, and within one the later query tiles, which see more keys), loads the Q tiles
//     and feeds the K ring.  A call with too few items to give most SMs one (a long-context chunk:
//     a few query tiles over many keys) runs the split instance of the kernel instead: the items
//     are laid end to end by cost and cut into equal consecutive ranges, one per CTA
//     (McNaughton's wrap-around rule), so an item crossing a cut runs as pieces on neighbouring
//     CTAs, each over its own K/V tiles; a piece writes its normalised partial O and log2-sum-exp
//     to the workspace, and the last piece of each row to finish (a per-warp arrival counter)
//     combines them and writes the output (the split-KV and merge of the FlashDecoding answer,
//     interview Q&A page).  Warp 3 feeds the V ring and clears the
//     V rows past the context end in the tile that holds it (P is 0 there, but 0 * NaN is NaN);
//     lanes 0-7 each fetch one page of a tile (one thread issuing all boxes of a tile is limited
//     by the per-instruction issue cost of TMA).  The first warpgroup shrinks its register budget
//     so the softmax warpgroups can grow theirs; warps 4-7 and 8-11 are the two softmax
//     warpgroups (rescale and epilogue included).  One persistent CTA per SM.
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
constexpr int kStages = 2;     // depth of the K ring and of the V ring
constexpr int kThreads = 384;  // 3 warpgroups: MMA/TMA/scheduling, softmax A, softmax B
// Register budgets: launched at 168 per thread (65536 / 384, rounded to 8); the first warpgroup
// gives registers back, the softmax warpgroups take them: 128 * 104 + 256 * 200 <= 384 * 168.
constexpr int kLaunchRegs = 168;
constexpr uint32_t kRegsControl = 104;
constexpr uint32_t kRegsSoftmax = 200;
static_assert(128 * kRegsControl + 256 * kRegsSoftmax <= kThreads * kLaunchRegs, "register split over budget");
constexpr int kItemSlots = 2;
constexpr int kItemReaders = 11;  // warps 0, 1, 3 and 4-11 each acknowledge a work item
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr size_t kCounterOffset = 64;      // work counter inside the status area of the workspace
constexpr size_t kPlanOffset = 128;        // split schedule: T, the cost range of a CTA
// The split schedule: costs in K/V tiles, plus kItemCost per item for its start and end (the first
// tiles' latency, the epilogue); at most kMaxCtas CTAs (the workspace holds two partial slots per
// CTA) and kMaxPieces pieces per item.  A call takes it when its items would keep at most 3/4 of
// the CTAs busy (4 items <= 3 CTAs).
constexpr int kMaxCtas = 160;
constexpr int kItemCost = 2;
constexpr int kMaxPieces = 8;

struct Params {
    const int32_t *block_tables;
    const int32_t *cu_seqlens;
    const int32_t *context_lens;
    const int32_t *order;  // [n_pairs_max * B] (pair, sequence) entries by decreasing K/V tiles
    void *out;
    int32_t *status;
    int *counter;
    int64_t num_blocks;
    int64_t T;
    int max_blocks;
    int B, H_q, H_kv, G;
    int max_q_len, max_ctx;
    int tok_per_tile;   // 128 / G (floor)
    int rows_per_tile;  // tok_per_tile * G
    int n_pairs_max;    // ceil(ceil(max_q_len / tok_per_tile) / 2)
    int n_items;        // n_pairs_max * B * H_kv
    int oob_row;        // first row past the pool in the cache tensor map
    int out_align32;    // out is 32-byte aligned: 32-byte stores in the epilogue
    float scale_log2;
};

// The split schedule's buffers (in the workspace), a kernel argument of their own.
struct SplitParams {
    int *plan;       // [0] = T, the cost range of a CTA (written by the plan kernel)
    int4 *starts;    // [kMaxCtas] CTA c's first item {b, g, pair, its start relative to c T}
    int *merge_cnt;  // [kMaxCtas][2 tiles][4 warps] arrivals of the pieces of the item that starts in c
    float *part_o;   // [2 kMaxCtas slots][2 tiles][D][kRows] normalised partial O (column-major)
    float *part_lse; // [2 kMaxCtas slots][2 tiles][kRows] log2-sum-exp of the scaled scores
    int n_ctas;      // grid size
};

// One query tile of a work item.
struct Tile {
    bool on;      // the tile has at least one query token
    int t_begin;  // first token (within the sequence) of the tile
    int n_tok;    // tokens in the tile
    int n_kv;     // K/V tiles it needs (causal)
};

struct Item {
    int b, g, q0, qb, ctx;
    Tile A, Bt;
    int n_kv;     // K/V tiles of the item (= the larger of the two)
    int n_pages;  // pages of the item
};

// What the scheduler hands to the other roles: the item index (-1 = no more work) and the
// decoded item, so that no role re-reads the sequence metadata from global memory.
// The split schedule's piece of an item, handed to the roles with it (the tile counts in the
// item are the piece's).
struct Split {
    int k0;        // first K/V tile of the piece
    int n_kv_all;  // K/V tiles of the whole item (its last one may hold the context end)
    int c0;        // the CTA whose range the item starts in
    int j;         // this piece (running on CTA c0 + j)
    int ns[2];     // per query tile: pieces holding its keys (1: its output is written directly)
    int jf[2];     // ... and the first of them
};

template <bool SPLIT>
struct ItemSlot {
    int it;
    Item I;
};
template <>
struct ItemSlot<true> {
    int it;
    Item I;
    Split sp;
};

template <int D, bool SPLIT>
struct Smem {
    static constexpr int kKB = D / 64;               // 128-byte column blocks
    static constexpr int kTile = kKB * kRows * 128;  // one 128-row x D tile
    static constexpr int kQ = 0;                     // Q_A, Q_B
    static constexpr int kK = 2 * kTile;             // K ring
    static constexpr int kV = kK + kStages * kTile;  // V ring
    static constexpr int kBars = kV + kStages * kTile;
    static constexpr int kNumBars = 2 * 2 + 4 * kStages + 4 * 2 + 2 * kItemSlots + 4;
    static constexpr int kItems = kBars + 8 * kNumBars;
    static constexpr int kTmemSlot = kItems + ((int(sizeof(ItemSlot<SPLIT>)) * kItemSlots + 15) / 16) * 16;
    static constexpr int kAbort = kTmemSlot + 8;
    static constexpr int kBytes = kAbort + 8;
    static constexpr int kAlloc = kBytes + 1024;
};

__device__ __forceinline__ void make_tile(const Params &p, const Item &I, int qt, Tile &t)
{
    t.t_begin = qt * p.tok_per_tile;
    t.on = t.t_begin < I.qb;
    t.n_tok = t.on ? min(p.tok_per_tile, I.qb - t.t_begin) : 0;
    t.n_kv = t.on ? (I.ctx - I.qb + t.t_begin + t.n_tok - 1) / kKeys + 1 : 0;
}

// K/V tiles read by query-tile pair `pair` of a sequence (0 when it has no query token or the
// sequence's lengths are invalid): the work of its items.
__device__ __forceinline__ int pair_kv_tiles(int pair, int qb, int ctx, int tok_per_tile)
{
    const int64_t t0 = 2ll * pair * tok_per_tile;
    if (qb < 1 || ctx < qb || t0 >= qb)
        return 0;
    const int64_t end = t0 + 2 * tok_per_tile;
    const int last = static_cast<int>(end < qb ? end : qb) - 1;
    return (ctx - qb + last) / kKeys + 1;
}

// Longest-processing-time-first order of the work: the (pair, sequence) entries by decreasing
// K/V tiles, so the heaviest items are drawn first and short ones fill the end.
__global__ void __launch_bounds__(kOrderThreads) pa_prefill_order_kernel(const int32_t *cu_seqlens,
                                                                           const int32_t *context_lens, int B,
                                                                           int n_pairs, int tok_per_tile, int32_t *order,
                                                                           int *counter, int32_t *status)
{
    griddep_wait();  // the kernel before this call's on the stream (its writes are visible after this)
    if (threadIdx.x == 0) {
        *status = PA_OK;  // the call's status word: this is its first kernel
        *counter = 0;     // the work counter the attention kernel's CTAs draw items from
    }
    griddep_release();  // the attention kernel's CTAs may be scheduled now; they wait for this grid
    order_by_key_desc(
        n_pairs * B,
        [&](int e) {
            const int b = e % B;
            const int qb = __ldg(cu_seqlens + b + 1) - __ldg(cu_seqlens + b);
            return min(pair_kv_tiles(e / B, qb, __ldg(context_lens + b), tok_per_tile), kOrderKeys - 1);
        },
        order);
}

// Decode work item `it` (the KV heads of one entry of the order are consecutive items); false when
// it has no query token (or its sequence is invalid).
__device__ __forceinline__ bool get_item(const Params &p, int it, Item &I, bool report)
{
    const int e = __ldg(p.order + it / p.H_kv);
    const int pair = e / p.B;
    I.b = e % p.B;
    I.g = it % p.H_kv;
    I.q0 = __ldg(p.cu_seqlens + I.b);
    const int q1 = __ldg(p.cu_seqlens + I.b + 1);
    I.qb = q1 - I.q0;
    I.ctx = __ldg(p.context_lens + I.b);
    const bool ok = I.qb >= 1 && I.ctx >= I.qb && I.qb <= p.max_q_len && I.ctx <= p.max_ctx &&
                    I.ctx <= p.max_blocks * 16 && q1 <= p.T && I.q0 >= 0;
    if (!ok) {
        if (report && pair == 0 && I.g == 0)
            set_status(p.status, PA_ERR_SEQ);
        return false;
    }
    make_tile(p, I, 2 * pair, I.A);
    make_tile(p, I, 2 * pair + 1, I.Bt);
    if (!I.A.on)
        return false;
    I.n_kv = max(I.A.n_kv, I.Bt.n_kv);
    const int lim_hi = I.ctx - I.qb + (I.Bt.on ? I.Bt.t_begin + I.Bt.n_tok : I.A.t_begin + I.A.n_tok) - 1;
    I.n_pages = lim_hi / 16 + 1;
    return true;
}

// ---- the split schedule ------------------------------------------------------------------------

// The checks every sequence of a call must pass (PA_ERR_SEQ otherwise; its items are skipped).
__device__ __forceinline__ bool seq_valid(const Params &p, int q0, int q1, int ctx)
{
    const int qb = q1 - q0;
    return qb >= 1 && ctx >= qb && qb <= p.max_q_len && ctx <= p.max_ctx && ctx <= p.max_blocks * 16 && q1 <= p.T &&
           q0 >= 0;
}

// Query-tile pairs of a sequence with qb new tokens.
__device__ __forceinline__ int seq_pairs(int qb, int tok_per_tile) { return (qb + 2 * tok_per_tile - 1) / (2 * tok_per_tile); }

__device__ __forceinline__ long long floor_div(long long a, long long b) { return a >= 0 ? a / b : -((-a + b - 1) / b); }

// The split schedule's plan (one CTA, the call's first kernel): clears the status word and the
// merge counters, reports inconsistent sequences, and lays the items end to end in (sequence b,
// KV head g, query-tile pair) order, an item costing its K/V tiles + kItemCost.  With W the cost
// of all items and M the largest, a CTA's range is T = ceil(W / n_ctas), at least kItemCost + 1
// (so that only the first piece of an item can be empty) and at least M / (kMaxPieces - 1) (so
// that no item has more than kMaxPieces pieces); CTA c takes [c T, (c + 1) T), and starts[c] is
// the item holding position c T.  The call takes this schedule only with B <= kOrderThreads.
__global__ void __launch_bounds__(kOrderThreads) pa_prefill_split_plan_kernel(const Params p, const SplitParams sq)
{
    griddep_wait();  // the kernel before this call's on the stream (its writes are visible after this)
    const int tid = threadIdx.x;
    if (tid == 0)
        *p.status = PA_OK;  // the call's status word: this is its first kernel
    for (int i = tid; i < kMaxCtas * 8; i += kOrderThreads)
        sq.merge_cnt[i] = 0;
    __syncthreads();    // the status word is clear before any thread reports
    griddep_release();  // the attention kernel's CTAs may be scheduled now; they wait for this grid
    const int tpt = p.tok_per_tile;
    __shared__ long long pre[kOrderThreads + 1];  // exclusive prefix of the sequences' costs
    __shared__ long long red_s[kOrderThreads / 32];
    __shared__ int red_m[kOrderThreads / 32];
    const int lane = tid & 31, warp = tid >> 5;
    // sequence tid: the cost of its items (all KV heads) and its largest item
    long long c = 0;
    int m = 0;
    if (tid < p.B) {
        const int q0 = __ldg(p.cu_seqlens + tid), q1 = __ldg(p.cu_seqlens + tid + 1);
        const int ctx = __ldg(p.context_lens + tid);
        if (!seq_valid(p, q0, q1, ctx)) {
            set_status(p.status, PA_ERR_SEQ);
        } else {
            const int np = seq_pairs(q1 - q0, tpt);
            for (int pr = 0; pr < np; ++pr) {
                const int k = pair_kv_tiles(pr, q1 - q0, ctx, tpt) + kItemCost;
                c += k;
                m = max(m, k);
            }
            c *= p.H_kv;
        }
    }
    // block-wide inclusive scan of c (warp shuffles, then the warp totals) and max of m
    long long incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o)
            incl += y;
        m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    }
    if (lane == 31)
        red_s[warp] = incl;
    if (lane == 0)
        red_m[warp] = m;
    __syncthreads();
    long long base = 0, W = 0;
    int M = 0;
    for (int i = 0; i < kOrderThreads / 32; ++i) {
        if (i < warp)
            base += red_s[i];
        W += red_s[i];
        M = max(M, red_m[i]);
    }
    pre[tid] = base + incl - c;
    if (tid == 0)
        pre[kOrderThreads] = W;
    __syncthreads();
    long long T = (W + sq.n_ctas - 1) / sq.n_ctas;
    T = max(T, (long long)kItemCost + 1);
    T = max(T, (long long)((M + kMaxPieces - 2) / (kMaxPieces - 1)));
    if (T >= (1ll << 30)) {
        if (tid == 0)
            set_status(p.status, PA_ERR_TOO_LARGE);
        T = 1ll << 30;
    }
    for (int cta = tid; cta < sq.n_ctas; cta += kOrderThreads) {
        const long long pos = (long long)cta * T;
        int4 st = make_int4(-1, 0, 0, 0);
        if (pos < W) {
            int lo = 0, hi = p.B;  // pre[lo] <= pos < pre[hi] (pre[B] = W)
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (pre[mid] <= pos)
                    lo = mid;
                else
                    hi = mid;
            }
            const int b = lo;
            const int q0 = __ldg(p.cu_seqlens + b), qb = __ldg(p.cu_seqlens + b + 1) - q0;
            const int ctx = __ldg(p.context_lens + b);
            const long long cb = (pre[b + 1] - pre[b]) / p.H_kv;  // one KV head's items of b
            const long long off = pos - pre[b];
            const int g = static_cast<int>(off / cb);
            const long long r = off - g * cb;
            int pr = 0;
            long long acc = 0;
            for (;; ++pr) {
                const long long k = pair_kv_tiles(pr, qb, ctx, tpt) + kItemCost;
                if (acc + k > r)
                    break;
                acc += k;
            }
            st = make_int4(b, g, pr, static_cast<int>(acc - r));
        }
        sq.starts[cta] = st;
    }
    if (tid == 0)
        sq.plan[0] = static_cast<int>(T);
}

// Item (b, g, pair) of the split schedule, with the whole item's tile counts; false when the pair
// has no query token or the sequence is invalid (the plan kernel reports it).
__device__ __forceinline__ bool item_of(const Params &p, int b, int g, int pair, Item &I)
{
    I.b = b;
    I.g = g;
    I.q0 = __ldg(p.cu_seqlens + b);
    const int q1 = __ldg(p.cu_seqlens + b + 1);
    I.qb = q1 - I.q0;
    I.ctx = __ldg(p.context_lens + b);
    if (!seq_valid(p, I.q0, q1, I.ctx))
        return false;
    make_tile(p, I, 2 * pair, I.A);
    make_tile(p, I, 2 * pair + 1, I.Bt);
    if (!I.A.on)
        return false;
    I.n_kv = max(I.A.n_kv, I.Bt.n_kv);
    const int lim_hi = I.ctx - I.qb + (I.Bt.on ? I.Bt.t_begin + I.Bt.n_tok : I.A.t_begin + I.A.n_tok) - 1;
    I.n_pages = lim_hi / 16 + 1;
    return true;
}

// Where a CTA of the split schedule is in its range: the next item (b, g, pair) and its start
// relative to the range's start.
struct Walk {
    int b, g, pair;
    long long rel;
};

// The next piece of this CTA's range [0, T) (relative positions), advancing `w`; false when the
// range is exhausted.  An item is cut where the CTA ranges cut its cost: with prel its start
// within the range of the CTA c0 where it begins, piece i covers the K/V tiles [kc(i), kc(i + 1)),
// kc(i) = clamp(i T - prel - kItemCost, 0, tiles) for 0 < i < n, kc(0) = 0, kc(n) = tiles, and
// runs on CTA c0 + i.  I gets the piece's tile counts, sp the rest.
__device__ bool walk_next(const Params &p, int T, Walk &w, Item &I, Split &sp)
{
    const int tpt = p.tok_per_tile;
    while (w.b < p.B && w.rel < T) {
        const int b = w.b, g = w.g, pair = w.pair;
        const int q0 = __ldg(p.cu_seqlens + b), q1 = __ldg(p.cu_seqlens + b + 1), ctx = __ldg(p.context_lens + b);
        const int np = seq_valid(p, q0, q1, ctx) ? seq_pairs(q1 - q0, tpt) : 0;
        if (np == 0) {  // no cost in the plan
            w.b = b + 1;
            w.g = 0;
            w.pair = 0;
            continue;
        }
        const int t = pair_kv_tiles(pair, q1 - q0, ctx, tpt);
        const long long start = w.rel, cost = t + kItemCost;
        w.rel += cost;
        if (++w.pair >= np) {
            w.pair = 0;
            if (++w.g >= p.H_kv) {
                w.g = 0;
                ++w.b;
            }
        }
        const long long lo = start < 0 ? -start - kItemCost : 0;
        const long long hi = start + cost > T ? T - start - kItemCost : t;
        const int k0 = static_cast<int>(min(max(lo, 0ll), (long long)t));
        const int k1 = static_cast<int>(min(max(hi, 0ll), (long long)t));
        // nothing here but the item's start or end cost; or no query token (not for pair < np)
        if (k0 >= k1 || !item_of(p, b, g, pair, I))
            continue;
        const long long sh = floor_div(start, T);
        const long long prel = start - sh * T;  // in [0, T)
        sp.c0 = static_cast<int>(blockIdx.x + sh);
        sp.j = static_cast<int>(-sh);
        sp.k0 = k0;
        sp.n_kv_all = I.n_kv;
        const int n = static_cast<int>((prel + cost + T - 1) / T);
        auto kc = [&](int i) -> int {
            if (i <= 0)
                return 0;
            if (i >= n)
                return t;
            return static_cast<int>(min(max((long long)i * T - prel - kItemCost, 0ll), (long long)t));
        };
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            Tile &tl = x == 0 ? I.A : I.Bt;
            int ns = 0, jf = 0;
            if (tl.on) {
                for (int i = 0; i < n && i < kMaxPieces; ++i) {
                    const int a = kc(i);
                    if (a < kc(i + 1) && a < tl.n_kv) {
                        if (ns == 0)
                            jf = i;
                        ++ns;
                    }
                }
                tl.n_kv = max(0, min(k1, tl.n_kv) - k0);
                tl.on = tl.n_kv > 0;
            }
            sp.ns[x] = ns;
            sp.jf[x] = jf;
        }
        if (!I.A.on && !I.Bt.on)
            continue;
        I.n_kv = k1 - k0;
        return true;
    }
    return false;
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

// Parity to wait for the k-th completion (0-based) of a barrier; and for the k-th
// "slot is free again" wait on a barrier whose slot starts out free.
__device__ __forceinline__ uint32_t full_par(int k) { return static_cast<uint32_t>(k & 1); }
__device__ __forceinline__ uint32_t free_par(int k) { return static_cast<uint32_t>((k & 1) ^ 1); }

// Epilogue of one query tile (x) of a piece of a split item, for the row of this thread: the
// piece's normalised partial O and its log2-sum-exp go to the piece's slot -- 2 (c0 + j) + 1 for
// the piece that begins an item in CTA c0's range (the last item of that range), 2 (c0 + j) for a
// piece that goes on from an earlier range (the first item of its range) -- then each warp counts
// itself in on the item's counter, and the warp whose arrival completes the count combines the
// pieces of its 32 rows, O = sum_i 2^(lse_i - M) O_i / sum_i 2^(lse_i - M), M = max_i lse_i,
// and writes them out.  `o_free` is arrived on once O has been read from TMEM.
template <int D, bool BF16>
__device__ __forceinline__ void split_epilogue(const Params &p, const SplitParams &sq, const Split &sp, int x, int sub,
                                               int r, int lane,
                                               uint32_t o_tmem, float inv, float m, float l, bool row_valid,
                                               uint8_t *orow, uint64_t *o_free)
{
    auto slot_of = [&](int jj) { return 2 * (sp.c0 + jj) + (jj == 0 ? 1 : 0); };
    const int own = slot_of(sp.j);
    {
        float *po = sq.part_o + ((int64_t)own * 2 + x) * (D * kRows) + r;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tc::ld32(o_tmem + c * 32, o);
#pragma unroll
            for (int i = 0; i < 32; ++i)
                __stcg(po + (c * 32 + i) * kRows, __uint_as_float(o[i]) * inv);
        }
    }
    tc::fence_before_sync();
    mbar_arrive(o_free);  // O_X has been read
    __stcg(sq.part_lse + (own * 2 + x) * kRows + r, l > 0.f ? m + __log2f(l) : -INFINITY);
    __threadfence();  // the partial is visible device-wide before the warp counts itself in
    __syncwarp();
    int prev = 0;
    if (lane == 0)
        prev = atomicAdd(sq.merge_cnt + (sp.c0 * 2 + x) * 4 + sub, 1);
    prev = __shfl_sync(0xffffffffu, prev, 0);
    const int ns = sp.ns[x];
    if (prev != ns - 1)
        return;
    __threadfence();  // every other piece's partial of these rows is visible
    float lse[kMaxPieces], M = -INFINITY;
#pragma unroll
    for (int i = 0; i < kMaxPieces; ++i) {
        lse[i] = i < ns ? __ldcg(sq.part_lse + (slot_of(sp.jf[x] + i) * 2 + x) * kRows + r) : -INFINITY;
        M = fmaxf(M, lse[i]);
    }
    if (!row_valid || M == -INFINITY)
        return;
    float wgt[kMaxPieces], Z = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxPieces; ++i) {
        wgt[i] = lse[i] == -INFINITY ? 0.f : fast_exp2(lse[i] - M);
        Z += wgt[i];
    }
    const float iz = 1.f / Z;  // Z >= 1: the largest term is 2^0
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
        float acc[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
            acc[i] = 0.f;
#pragma unroll
        for (int k = 0; k < kMaxPieces; ++k) {
            if (wgt[k] == 0.f)
                continue;
            const float *src =
                sq.part_o + ((int64_t)slot_of(sp.jf[x] + k) * 2 + x) * (D * kRows) + (c * 32) * kRows + r;
            const float wk = wgt[k] * iz;
#pragma unroll
            for (int i = 0; i < 32; ++i)
                acc[i] += wk * __ldcg(src + i * kRows);
        }
        uint32_t o[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2)
            o[i >> 1] = pack2<BF16>(acc[i], acc[i + 1]);
        uint8_t *dst = orow + c * 64;
        if (p.out_align32) {
            st_global_v8(dst, o);
            st_global_v8(dst + 32, o + 8);
        } else {
#pragma unroll
            for (int i = 0; i < 16; i += 4)
                *reinterpret_cast<uint4 *>(dst + i * 4) = make_uint4(o[i], o[i + 1], o[i + 2], o[i + 3]);
        }
    }
}

// SPLIT: the split schedule (pieces of items, walked per CTA); otherwise the queue.
template <int D, bool BF16, bool SPLIT>
__global__ void __launch_bounds__(kThreads, 1)
    pa_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v, const Params p, const SplitParams sq)
{
    using L = Smem<D, SPLIT>;
    constexpr int KB = L::kKB;
    constexpr uint32_t kTmemCols = 512;
    // TMEM columns: S_A, S_B (P written over their first 64 columns), O_A, O_B

    griddep_wait();  // the item order and the zeroed work counter come from the order kernel
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBars);
    uint64_t *q_full = bars;                    // [2] Q_X landed
    uint64_t *q_empty = bars + 2;               // [2] Q_X no longer read
    uint64_t *k_full = bars + 4;                // [kStages]
    uint64_t *k_empty = k_full + kStages;       // [kStages] released by both MMA threads
    uint64_t *v_full = k_empty + kStages;       // [kStages]
    uint64_t *v_empty = v_full + kStages;       // [kStages] released by both MMA threads
    uint64_t *s_full = v_empty + kStages;       // [2] S_X computed
    uint64_t *p_full = s_full + 2;              // [2] P_X written (128 arrivals)
    uint64_t *o_full = p_full + 2;              // [2] O_X final for the item
    uint64_t *o_free = o_full + 2;              // [2] epilogue of X has read O_X (128 arrivals)
    uint64_t *item_full = o_free + 2;           // [kItemSlots]
    uint64_t *item_empty = item_full + kItemSlots;
    uint64_t *drain = item_empty + kItemSlots;  // [1] both MMA threads' products complete
    uint64_t *v_land = drain + 1;               // [1] V tile with a context end landed (before zeroing)
    uint64_t *tok = v_land + 1;                 // [2] tok[X]: MMA thread X may issue its next batch
    ItemSlot<SPLIT> *item_slot = reinterpret_cast<ItemSlot<SPLIT> *>(smem + L::kItems);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kTmemSlot);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kAbort);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int x = 0; x < 2; ++x) {
            mbar_init(&q_full[x], 1);
            mbar_init(&q_empty[x], 1);
            mbar_init(&s_full[x], 1);
            mbar_init(&p_full[x], 128);
            mbar_init(&o_full[x], 1);
            mbar_init(&o_free[x], 128);
        }
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 2);
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 2);
        }
        for (int i = 0; i < kItemSlots; ++i) {
            mbar_init(&item_full[i], 1);
            mbar_init(&item_empty[i], kItemReaders);
        }
        mbar_init(drain, 2);
        mbar_init(v_land, 1);
        mbar_init(&tok[0], 1);
        mbar_init(&tok[1], 1);
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
    // TMEM columns of tile X: S_X at 128 X, O_X at 256 + 128 X

    if (warp < 4) {
    // first warpgroup: give registers back (all four warps), then split into roles
    tc::regs_shrink<kRegsControl>();
    if (warp < 2) {
        // ===================== MMA issuers: warp 0 for tile A, warp 1 for tile B (one thread each) =====================
        // Per K/V tile j: S_X(j) = Q_X K_j^T, then O_X += P_X(j) V_j once the softmax has written P_X(j);
        // S_X(j+1) is issued after that product, which reads the TMEM columns S_X(j+1) overwrites
        // (tcgen05.mma operations of one thread execute in issue order).  The two threads feed the
        // tensor core independently, so one tile's waits overlap the other tile's products.  Each
        // thread releases every K and V tile of the item (the empty barriers count two arrivals),
        // always after waiting for the tile to land, so that neither can arrive twice on a stage
        // before the other has arrived once.
        const int x = warp;
        constexpr uint32_t idesc_qk = tc::idesc_f16(BF16, kRows, kKeys, false);
        constexpr uint32_t idesc_pv = tc::idesc_f16(BF16, kRows, D, true);
        const uint32_t q_addr = smem_u32(smem + L::kQ + x * L::kTile);
        const uint32_t s_tm = tmem + 128u * x;
        const uint32_t o_tm = tmem + 256u + 128u * x;
        int n_item = 0, k_base = 0, q_n = 0, pv_n = 0, o_n = 0, n_batch = 0;
        bool ok = true;
        for (;;) {
            const int slot = n_item % kItemSlots;
            ok = wait_bar(&item_full[slot], full_par(n_item / kItemSlots), abort_flag, p.status);
            ok = __all_sync(0xffffffffu, ok);
            const int it = ok ? item_slot[slot].it : -1;
            Item I;
            if (it >= 0)
                I = item_slot[slot].I;
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&item_empty[slot]);
            ++n_item;
            if (it < 0)
                break;
            if (lane == 0) {
                const int nt = x == 0 ? I.A.n_kv : I.Bt.n_kv;  // 0 for a tile without tokens
                const int n = I.n_kv;
                auto wait_k = [&](int j) {
                    const int kg = k_base + j;
                    return wait_bar(&k_full[kg % kStages], full_par(kg / kStages), abort_flag, p.status);
                };
                auto wait_v = [&](int j) {
                    const int vg = k_base + j;
                    return wait_bar(&v_full[vg % kStages], full_par(vg / kStages), abort_flag, p.status);
                };
                // S_X(j) = Q_X K_j^T
                auto issue_s = [&](int j) {
                    const uint32_t k_addr = smem_u32(smem + L::kK + ((k_base + j) % kStages) * L::kTile);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t off = (ks >> 2) * (kRows * 128) + (ks & 3) * 32;
                        tc::mma_ss(s_tm, tc::desc_k_sw128(q_addr + off), tc::desc_k_sw128(k_addr + off), idesc_qk,
                                   ks > 0 ? 1u : 0u);
                    }
                    tc::commit(&s_full[x]);
                    if (j == nt - 1)
                        tc::commit(&q_empty[x]);  // Q_X no longer needed
                };
                // O_X += P_X(j) V_j
                auto issue_pv = [&](int j) {
                    const uint32_t v_addr = smem_u32(smem + L::kV + ((k_base + j) % kStages) * L::kTile);
#pragma unroll
                    for (int ks = 0; ks < kKeys / 16; ++ks)
                        tc::mma_ts(o_tm, s_tm + ks * 8, tc::desc_mn_sw128(v_addr + ks * 2048, kRows * 128), idesc_pv,
                                   (j > 0 || ks > 0) ? 1u : 0u);
                    ++pv_n;
                    if (j == nt - 1) {
                        tc::commit(&o_full[x]);
                        ++o_n;
                    }
                };
                // Batch 0 of the item is S_X(0); batch j + 1 is P_X(j) V_j followed by S_X(j + 1).  The
                // two threads issue their batches in turn (a token passed through tok[]), every
                // thread n + 1 batches per item (empty ones where its tile has fewer K/V tiles), so the
                // tensor core runs one tile's batch while the other tile's softmax runs.  All waits
                // for data come before the token is taken.
                auto take_turn = [&]() {
                    const uint32_t par = x == 0 ? free_par(n_batch) : full_par(n_batch);
                    return wait_bar(&tok[x], par, abort_flag, p.status);
                };
                auto pass_turn = [&]() {
                    mbar_arrive(&tok[x ^ 1]);
                    ++n_batch;
                };
                ok = wait_k(0);
                if (ok && nt > 0) {
                    ok = wait_bar(&q_full[x], full_par(q_n), abort_flag, p.status);
                    ++q_n;
                }
                if (ok)
                    ok = take_turn();
                if (ok) {
                    if (nt > 0) {
                        tc::fence_after_sync();
                        issue_s(0);
                    }
                    pass_turn();
                    tc::commit(&k_empty[k_base % kStages]);
                }
                for (int j = 0; j < n && ok; ++j) {
                    // V_j and K_(j+1) are normally in place long before P_X(j)
                    ok = wait_v(j);
                    if (ok && j + 1 < n)
                        ok = wait_k(j + 1);
                    if (ok && j < nt) {
                        ok = wait_bar(&p_full[x], full_par(pv_n), abort_flag, p.status);
                        if (ok && j == 0)
                            ok = wait_bar(&o_free[x], free_par(o_n), abort_flag, p.status);
                    }
                    if (ok)
                        ok = take_turn();
                    if (!ok)
                        break;
                    if (j < nt) {
                        tc::fence_after_sync();
                        issue_pv(j);
                        if (j + 1 < nt)
                            issue_s(j + 1);
                    }
                    pass_turn();
                    tc::commit(&v_empty[(k_base + j) % kStages]);
                    if (j + 1 < n)
                        tc::commit(&k_empty[(k_base + j + 1) % kStages]);
                }
                k_base += n;
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            k_base = __shfl_sync(0xffffffffu, k_base, 0);
            q_n = __shfl_sync(0xffffffffu, q_n, 0);
            pv_n = __shfl_sync(0xffffffffu, pv_n, 0);
            o_n = __shfl_sync(0xffffffffu, o_n, 0);
            n_batch = __shfl_sync(0xffffffffu, n_batch, 0);
            if (!ok)
                break;
        }
        if (lane == 0) {
            // every MMA issued so far must be complete before TMEM is released
            tc::commit(drain);
            mbar_wait(drain, 0, kWaitTimeoutNs / 10);
        }
        __syncwarp();
    } else {
        // ===================== producers: warp 2 = scheduler + Q + K ring, warp 3 = V ring =====================
        // One TMA box is 16 keys x 64 columns of one page; lanes 0-7 each fetch one page of a tile
        // (one thread issuing every box of a tile is limited by the per-instruction issue cost).
        const bool is_v = warp == 3;
        const CUtensorMap *tmap = is_v ? &tmap_v : &tmap_k;
        uint64_t *full = is_v ? v_full : k_full;
        uint64_t *empty = is_v ? v_empty : k_empty;
        uint8_t *ring = smem + (is_v ? L::kV : L::kK);
        int n_item = 0, n_tiles = 0, q_n[2] = {0, 0}, z_n = 0;
        bool ok = true;
        // split schedule: the scheduler walks this CTA's range from its first item
        Walk walk{p.B, 0, 0, 0};
        int split_T = 0;
        if constexpr (SPLIT) {
            if (!is_v) {
                split_T = sq.plan[0];
                const int4 s0 = sq.starts[blockIdx.x];
                if (s0.x >= 0)
                    walk = Walk{s0.x, s0.y, s0.z, s0.w};
            }
        }
        for (;;) {
            int it = -1;
            Item I;
            Split sp;
            if (!is_v) {
                if constexpr (SPLIT) {
                    // the next piece of this CTA's range (every lane walks the same state; lane 0
                    // decides whether to go on, the abort flag may change between lanes' reads)
                    int go = 0;
                    if (lane == 0)
                        go = ok && !*abort_flag;
                    go = __shfl_sync(0xffffffffu, go, 0);
                    if (go && walk_next(p, split_T, walk, I, sp))
                        it = 0;
                } else {
                    // next work item that has query tokens (lane 0 draws, the warp follows)
                    for (;;) {
                        // lane 0 decides for the whole warp (the abort flag may change between lanes' reads)
                        int cand = -1;
                        if (lane == 0 && ok && !*abort_flag)
                            cand = atomicAdd(p.counter, 1);
                        cand = __shfl_sync(0xffffffffu, cand, 0);
                        if (cand < 0 || cand >= p.n_items)
                            break;
                        if (get_item(p, cand, I, lane == 0)) {
                            it = cand;
                            break;
                        }
                    }
                }
                // publish it (or the end marker -1) to the other roles
                if (lane == 0) {
                    const int slot = n_item % kItemSlots;
                    const bool got = wait_bar(&item_empty[slot], free_par(n_item / kItemSlots), abort_flag, p.status);
                    ok = ok && got;
                    item_slot[slot].it = ok ? it : -1;
                    item_slot[slot].I = I;
                    if constexpr (SPLIT)
                        item_slot[slot].sp = sp;
                    mbar_arrive(&item_full[slot]);
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok)
                    it = -1;
            } else {
                const int slot = n_item % kItemSlots;
                ok = wait_bar(&item_full[slot], full_par(n_item / kItemSlots), abort_flag, p.status);
                ok = __all_sync(0xffffffffu, ok);
                it = ok ? item_slot[slot].it : -1;
                if (it >= 0) {
                    I = item_slot[slot].I;
                    if constexpr (SPLIT)
                        sp = item_slot[slot].sp;
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&item_empty[slot]);
            }
            ++n_item;
            if (it < 0)
                break;
            // K/V tile j of the item is tile k_first + j of its whole causal range (a piece of a split
            // item starts later), and n_kv_all the whole range's tiles
            int k_first = 0, n_kv_all = I.n_kv;
            if constexpr (SPLIT) {
                k_first = sp.k0;
                n_kv_all = sp.n_kv_all;
            }
            const int32_t *table = p.block_tables + (int64_t)I.b * p.max_blocks;
            // TMA row of page `pidx` of the item (lanes 0-7); pages past the item's range, and bad
            // block ids, read rows past the pool, which TMA fills with zeros
            auto page_row = [&](int pidx) -> int {
                int y = p.oob_row;
                if (lane < 8 && pidx < I.n_pages) {
                    const int id = __ldg(table + pidx);
                    if (id >= 0 && id < p.num_blocks)
                        y = (id * p.H_kv + I.g) * 16;
                    else
                        set_status(p.status, PA_ERR_BOUNDS);
                }
                return y;
            };
            // The last page of the context may be partly filled: its V rows past the context end can
            // hold anything (NaN included) and P is 0 there, but 0 * NaN is NaN, so the V warp clears
            // them before the tile is handed on.  That happens only when this item reads up to the
            // context end, in the last tile of its whole range.
            const int last_page = (I.ctx + 15) / 16 - 1;
            const int zpg = last_page - 8 * (n_kv_all - 1);  // page of the last tile holding the context end
            const int zr0 = I.ctx & 15;                     // first row to clear
            const bool zero_tail = is_v && zr0 != 0 && I.n_pages == last_page + 1 && zpg >= 0 && zpg < 8;
            int y = page_row(k_first * 8 + lane);
            for (int j = 0; j < I.n_kv; ++j) {
                const int y_next = j + 1 < I.n_kv ? page_row((k_first + j + 1) * 8 + lane) : p.oob_row;  // in flight meanwhile
                const int st = n_tiles % kStages;
                const bool z = zero_tail && k_first + j == n_kv_all - 1;
                uint64_t *done = z ? v_land : &full[st];
                if (lane == 0) {
                    ok = wait_bar(&empty[st], free_par(n_tiles / kStages), abort_flag, p.status);
                    if (ok)
                        mbar_arrive_expect_tx(done, L::kTile);
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok)
                    break;
                ++n_tiles;
                uint8_t *dst = ring + st * L::kTile;
                if (lane < 8) {
#pragma unroll
                    for (int kb = 0; kb < KB; ++kb)
                        tma_load_2d(dst + lane * 2048 + kb * kRows * 128, tmap, kb * 64, y, done);
                }
                y = y_next;
                if (z) {
                    ++z_n;
                    ok = wait_bar(v_land, full_par(z_n - 1), abort_flag, p.status);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok)
                        break;
                    const int per_kb = (16 - zr0) * 8;  // 16-byte chunks to clear per column block
                    for (int i = lane; i < per_kb * KB; i += 32) {
                        const int kb = i / per_kb, rem = i % per_kb;
                        const int row = zpg * 16 + zr0 + rem / 8;
                        *reinterpret_cast<uint4 *>(dst + kb * kRows * 128 + row * 128 + (rem & 7) * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();  // generic writes before the tensor core reads the tile
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&full[st]);
                }
                if (!is_v && j == 0) {
                    // Q_A and Q_B of the item, after its first K tile
                    if (lane == 0) {
#pragma unroll
                        for (int xq = 0; xq < 2 && ok; ++xq) {
                            const Tile &tq = xq == 0 ? I.A : I.Bt;
                            if (!tq.on)
                                continue;
                            ok = wait_bar(&q_empty[xq], free_par(q_n[xq]), abort_flag, p.status);
                            if (!ok)
                                break;
                            uint8_t *qs = smem + L::kQ + xq * L::kTile;
                            mbar_arrive_expect_tx(&q_full[xq], KB * p.rows_per_tile * 128);
                            for (int kb = 0; kb < KB; ++kb)
                                tc::tma_load_3d(qs + kb * kRows * 128, &tmap_q, kb * 64, I.g * p.G,
                                                I.q0 + tq.t_begin, &q_full[xq]);
                            ++q_n[xq];
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                    q_n[0] = __shfl_sync(0xffffffffu, q_n[0], 0);
                    q_n[1] = __shfl_sync(0xffffffffu, q_n[1], 0);
                    if (!ok)
                        break;
                }
            }
            if (!ok)
                break;
        }
        if (lane == 0 && *abort_flag) {
            // let the copies already issued land before shared memory is released
            for (int st = 0; st < kStages; ++st) {
                const int uses = n_tiles / kStages + (st < n_tiles % kStages ? 1 : 0);
                if (uses > 0)
                    mbar_wait(&full[st], full_par(uses - 1), kWaitTimeoutNs / 10);
            }
            if (z_n > 0)
                mbar_wait(v_land, full_par(z_n - 1), kWaitTimeoutNs / 10);
            for (int xq = 0; xq < 2; ++xq)
                if (q_n[xq] > 0)
                    mbar_wait(&q_full[xq], full_par(q_n[xq] - 1), kWaitTimeoutNs / 10);
        }
    }
    } else {
        tc::regs_grow<kRegsSoftmax>();
        // ===================== softmax warpgroups: warps 4-7 -> tile A, 8-11 -> tile B =====================
        const int x = (warp - 4) >> 2;  // 0 = A, 1 = B
        const int sub = warp & 3;       // TMEM sub-partition of this warp
        const int r = sub * 32 + lane;  // query row of this thread in its tile
        const uint32_t lane_addr = static_cast<uint32_t>(sub * 32) << 16;
        const uint32_t s_tmem = tmem + lane_addr + 128u * x;
        const uint32_t o_tmem = tmem + lane_addr + 256u + 128u * x;
        const float sl2 = p.scale_log2;
        int n_item = 0, s_n = 0, o_n = 0;
        bool ok = true;
        for (;;) {
            const int slot = n_item % kItemSlots;
            ok = wait_bar(&item_full[slot], full_par(n_item / kItemSlots), abort_flag, p.status);
            ok = __all_sync(0xffffffffu, ok);
            const int it = ok ? item_slot[slot].it : -1;
            Item I;
            Split sp;
            if (it >= 0) {
                I = item_slot[slot].I;
                if constexpr (SPLIT)
                    sp = item_slot[slot].sp;
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&item_empty[slot]);
            ++n_item;
            if (it < 0)
                break;
            int k_first = 0;  // first K/V tile of a piece of a split item
            if constexpr (SPLIT)
                k_first = sp.k0;
            const Tile &t = x == 0 ? I.A : I.Bt;
            if (!t.on)
                continue;
            const int tl = r / p.G, gi = r % p.G;
            const bool row_valid = r < p.rows_per_tile && tl < t.n_tok;
            const int lim = row_valid ? I.ctx - I.qb + t.t_begin + tl : -1;
            const int n_kv_t = t.n_kv;
            uint8_t *orow = static_cast<uint8_t *>(p.out) +
                            ((int64_t)(I.q0 + t.t_begin + tl) * p.H_q + I.g * p.G + gi) * (D * 2);
            float m = -INFINITY, l = 0.f;
            for (int j = 0; j < n_kv_t; ++j) {
                ok = wait_bar(&s_full[x], full_par(s_n), abort_flag, p.status);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok)
                    break;
                ++s_n;
                tc::fence_after_sync();
                // the whole S row in one TMEM load; masked keys (causal / context end) become -inf
                const int key0 = (k_first + j) * kKeys;
                uint32_t raw[kKeys];
                tc::ld128(s_tmem, raw);
                if (key0 + kKeys - 1 > lim) {
#pragma unroll
                    for (int c = 0; c < kKeys; ++c)
                        if (key0 + c > lim)
                            raw[c] = 0xff800000u;  // -inf
                }
                float mx4[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    mx4[i] = fmaxf(__uint_as_float(raw[2 * i]), __uint_as_float(raw[2 * i + 1]));
#pragma unroll
                for (int c = 8; c < kKeys; c += 2)
                    mx4[(c >> 1) & 3] = fmax3(mx4[(c >> 1) & 3], __uint_as_float(raw[c]), __uint_as_float(raw[c + 1]));
                const float mx = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
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
                    // every earlier P V product of this tile is complete: S_X(j) was issued after them
                    // by the same thread, and its completion (s_full) covers them
                    tc::fence_after_sync();
#pragma unroll 1
                    for (int c = 0; c < D / 16; ++c) {
                        uint32_t o[16];
                        tc::ld16(o_tmem + c * 16, o);
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
                        tc::st16(o_tmem + c * 16, o);
                    }
                }
                // P = 2^(s * scale * log2 e - m), packed to 16 bits in place and stored over the
                // first 64 columns of S
                // P = 2^(s * scale * log2 e - m) (masked keys: 2^-inf = 0), packed to 16 bits in place
                const float nb = m == -INFINITY ? 0.f : -m;
                const uint64_t sl2_2 = f2_pack(sl2, sl2), nb_2 = f2_pack(nb, nb);
                uint64_t acc[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
                for (int q = 0; q < kKeys / 2; ++q) {
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
                tc::st32(s_tmem, raw);
                tc::st32(s_tmem + 32, raw + 32);
                tc::wait_st();
                tc::fence_before_sync();
                mbar_arrive(&p_full[x]);
            }
            if (!ok)
                break;
            // epilogue: O_X / l -> out
            ok = wait_bar(&o_full[x], full_par(o_n), abort_flag, p.status);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok)
                break;
            ++o_n;
            tc::fence_after_sync();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            if constexpr (SPLIT) {
                if (sp.ns[x] > 1) {
                    split_epilogue<D, BF16>(p, sq, sp, x, sub, r, lane, o_tmem, inv, m, l, row_valid, orow,
                                            &o_free[x]);
                    continue;
                }
            }
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tc::ld32(o_tmem + c * 32, o);
#pragma unroll
                for (int i = 0; i < 32; i += 2)
                    o[i >> 1] = pack2<BF16>(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv);
                if (row_valid) {
                    uint8_t *dst = orow + c * 64;
                    if (p.out_align32) {
                        st_global_v8(dst, o);
                        st_global_v8(dst + 32, o + 8);
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; i += 4)
                            *reinterpret_cast<uint4 *>(dst + i * 4) = make_uint4(o[i], o[i + 1], o[i + 2], o[i + 3]);
                    }
                }
            }
            tc::fence_before_sync();
            mbar_arrive(&o_free[x]);
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0)
        tc::tmem_dealloc(tmem, kTmemCols);
}

// ---- host ---------------------------------------------------------------------------------------

// The split schedule is taken when the call's items would keep at most 3/4 of the CTAs busy.
static bool use_split(int64_t items, int n_ctas, int B) { return B <= kOrderThreads && 4 * items <= 3 * (int64_t)n_ctas; }

// Workspace of a call: the status area (status word, work counter, split plan word), the queue
// order, and for the split schedule the CTAs' starts, the merge counters and two partial slots
// (O and log2-sum-exp of both query tiles) per CTA.
struct WsLayout {
    size_t order, starts, merge_cnt, part_lse, part_o, bytes;
};

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

static WsLayout ws_layout(int B, int64_t n_pairs, int D, bool split)
{
    WsLayout w;
    w.order = PA_STATUS_BYTES;
    w.starts = w.order + align256(static_cast<size_t>(n_pairs) * B * sizeof(int32_t));
    w.merge_cnt = w.starts + (split ? align256(kMaxCtas * sizeof(int4)) : 0);
    w.part_lse = w.merge_cnt + (split ? align256(kMaxCtas * 8 * sizeof(int)) : 0);
    w.part_o = w.part_lse + (split ? align256(static_cast<size_t>(2 * kMaxCtas) * 2 * kRows * sizeof(float)) : 0);
    w.bytes = w.part_o + (split ? static_cast<size_t>(2 * kMaxCtas) * 2 * D * kRows * sizeof(float) : 0);
    return w;
}

// Launch one instance of the attention kernel (per device, once: the check of the register count
// the warpgroups' register split relies on, and the shared-memory attribute).
template <int D, bool BF16, bool SPLIT>
static int launch_attention(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv, const Params &p,
                            const SplitParams &sq, int grid, cudaStream_t stream)
{
    using L = Smem<D, SPLIT>;
    auto kern = pa_prefill_tc_kernel<D, BF16, SPLIT>;
    static uint64_t configured = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return PA_ERR_CUDA;
    const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
    if (!bit || !(configured & bit)) {
        // the per-warpgroup register split assumes exactly kLaunchRegs registers per thread at
        // launch; with any other count the growing warpgroups could wait forever, so refuse
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess)
            return PA_ERR_CUDA;
        if (fa.numRegs != kLaunchRegs)
            return PA_ERR_UNSUPPORTED;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) != cudaSuccess)
            return PA_ERR_CUDA;
        configured |= bit;
    }
    const cudaError_t e = launch_dependent(kern, dim3(grid), dim3(kThreads), L::kAlloc, stream, tq, tk, tv, p, sq);
    count_launch();
    const cudaError_t e2 = cudaGetLastError();
    return e == cudaSuccess && e2 == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <int D, bool BF16>
static int run(const AttnArgs &a)
{
    const int G = a.H_q / a.H_kv;
    if (G > kRows)
        return PA_ERR_UNSUPPORTED;
    Params p{};
    SplitParams sq{};
    uint8_t *ws = static_cast<uint8_t *>(a.workspace);
    p.block_tables = a.block_tables;
    p.cu_seqlens = a.cu_seqlens_q;
    p.context_lens = a.context_lens;
    p.out = a.out;
    p.status = reinterpret_cast<int32_t *>(ws);
    p.counter = reinterpret_cast<int *>(ws + kCounterOffset);
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
    const int n_qt = (a.max_q_len + p.tok_per_tile - 1) / p.tok_per_tile;
    p.n_pairs_max = (n_qt + 1) / 2;
    const int64_t items = (int64_t)p.n_pairs_max * a.B * a.H_kv;
    if (items > (int64_t(1) << 30) || a.T > (int64_t(1) << 31) - 256)
        return PA_ERR_UNSUPPORTED;
    p.n_items = static_cast<int>(items);
    p.oob_row = static_cast<int>(a.num_blocks * a.H_kv * 16);
    p.out_align32 = (reinterpret_cast<uintptr_t>(a.out) & 31u) == 0;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    const int n_ctas = std::min(sm_count(), kMaxCtas);
    const bool split = use_split(items, n_ctas, a.B);
    const WsLayout wl = ws_layout(a.B, p.n_pairs_max, D, split);
    int32_t *order = reinterpret_cast<int32_t *>(ws + wl.order);
    p.order = order;

    CUtensorMap tq, tk, tv;
    int rc = make_q_tmap(&tq, a.q, a.T, a.H_q, D, G, p.tok_per_tile, a.dtype);
    if (rc == PA_OK)
        rc = make_cache_tmap(&tk, a.key_cache, a.num_blocks, a.H_kv, D, a.dtype);
    if (rc == PA_OK)
        rc = make_cache_tmap(&tv, a.value_cache, a.num_blocks, a.H_kv, D, a.dtype);
    if (rc != PA_OK)
        return rc;
    if (split) {
        // every CTA walks its share of the items laid end to end (one CTA per SM, also when that
        // is more CTAs than items: the items are cut to give every CTA a share)
        sq.plan = reinterpret_cast<int *>(ws + kPlanOffset);
        sq.starts = reinterpret_cast<int4 *>(ws + wl.starts);
        sq.merge_cnt = reinterpret_cast<int *>(ws + wl.merge_cnt);
        sq.part_lse = reinterpret_cast<float *>(ws + wl.part_lse);
        sq.part_o = reinterpret_cast<float *>(ws + wl.part_o);
        sq.n_ctas = n_ctas;
        const cudaError_t eo =
            launch_dependent(pa_prefill_split_plan_kernel, dim3(1), dim3(kOrderThreads), 0, a.stream, p, sq);
        count_launch();
        if (eo != cudaSuccess || cudaGetLastError() != cudaSuccess)
            return PA_ERR_CUDA;
        return launch_attention<D, BF16, true>(tq, tk, tv, p, sq, n_ctas, a.stream);
    }
    const cudaError_t eo = launch_dependent(pa_prefill_order_kernel, dim3(1), dim3(kOrderThreads), 0, a.stream,
                                            a.cu_seqlens_q, a.context_lens, a.B, p.n_pairs_max, p.tok_per_tile, order,
                                            p.counter, p.status);
    count_launch();
    if (eo != cudaSuccess || cudaGetLastError() != cudaSuccess)
        return PA_ERR_CUDA;
    const int grid = static_cast<int>(std::min<int64_t>(items, sm_count()));
    return launch_attention<D, BF16, false>(tq, tk, tv, p, sq, grid, a.stream);
}

}  // namespace tcp

// Workspace: see ws_layout (the split schedule's areas only for calls that take it).
size_t prefill_workspace_bytes(int B, int H_q, int H_kv, int d, int max_q_len)
{
    const int G = H_q / H_kv;
    const int tok = G >= 1 && G <= tcp::kRows ? tcp::kRows / G : 1;
    const int64_t n_pairs = ((int64_t)(max_q_len + tok - 1) / tok + 1) / 2;
    const int n_ctas = std::min(sm_count(), tcp::kMaxCtas);
    return tcp::ws_layout(B, n_pairs, d, tcp::use_split(n_pairs * B * H_kv, n_ctas, B)).bytes;
}

int launch_prefill(const AttnArgs &a)
{
    if (a.d == 128)
        return a.dtype == PA_BF16 ? tcp::run<128, true>(a) : tcp::run<128, false>(a);
    return a.dtype == PA_BF16 ? tcp::run<64, true>(a) : tcp::run<64, false>(a);
}

}  // namespace pa
