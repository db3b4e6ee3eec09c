"""A host model of the prefill call's work schedule, for the tests.

The prefill call runs its work items (sequence b, KV head g, query-tile pair) on one of two
schedules, chosen on the host from the call's sizes:
  * the queue: items are drawn from a global counter, the (pair, sequence) entries in decreasing
    K/V tiles (longest-processing-time-first);
  * the split schedule, when the items would keep at most 3/4 of the CTAs busy (a long-context
    chunk among few items): McNaughton's wrap-around rule for splittable work -- the plan kernel
    lays the items end to end by cost (K/V tiles + ITEM_COST) in (b, g, pair) order, and CTA c
    takes the cost range [c T, (c + 1) T).  An item crossing a cut runs as pieces on
    neighbouring CTAs, each over its own K/V tiles, and the pieces' partial outputs are merged
    (the split-and-merge of the FlashDecoding answer on the interview Q&A page).

This module restates that schedule in plain Python so that the tests can (a) check its invariants
on the CPU for many shapes -- every item's K/V tiles covered exactly once, merge slots and
counters used by one item each -- and (b) compare the plan the kernel writes into its workspace
with this one on the GPU.  It holds no attention arithmetic.
"""
from dataclasses import dataclass
from typing import List, Optional, Tuple

KEYS = 128  # keys per K/V tile
ROWS = 128  # query rows per tile
ITEM_COST = 2
MAX_PIECES = 8
MAX_CTAS = 160
ORDER_THREADS = 1024
MODE_QUEUE, MODE_WRAP = 0, 1


def n_pairs_max(max_q_len: int, G: int) -> int:
    tpt = ROWS // G
    return ((max_q_len + tpt - 1) // tpt + 1) // 2


def takes_split(B: int, max_q_len: int, H_kv: int, G: int, n_ctas: int) -> bool:
    """The host's choice: the split schedule when 4 x items <= 3 x CTAs (and B <= ORDER_THREADS)."""
    items = n_pairs_max(max_q_len, G) * B * H_kv
    return B <= ORDER_THREADS and 4 * items <= 3 * n_ctas


def pair_kv_tiles(pair: int, qb: int, ctx: int, tpt: int) -> int:
    """K/V tiles the query-tile pair `pair` of a sequence reads (causal, bottom-right aligned)."""
    t0 = 2 * pair * tpt
    if qb < 1 or ctx < qb or t0 >= qb:
        return 0
    last = min(t0 + 2 * tpt, qb) - 1
    return (ctx - qb + last) // KEYS + 1


def seq_pairs(qb: int, tpt: int) -> int:
    return (qb + 2 * tpt - 1) // (2 * tpt)


@dataclass
class Plan:
    mode: int
    T: int
    starts: List[Tuple[int, int, int, int]]  # per CTA: (b, g, pair, start relative to c T); b = -1: none
    W: int
    M: int


def plan(q_lens, ctx_lens, H_kv: int, G: int, n_ctas: int) -> Plan:
    """The split schedule's plan for valid sequences (q_b >= 1, ctx_b >= q_b); mode says whether
    the call takes it (the host's choice, with max_q_len = max(q_lens))."""
    tpt = ROWS // G
    B = len(q_lens)
    costs = []  # per sequence: the cost of one KV head's items
    m = 0
    for qb, ctx in zip(q_lens, ctx_lens):
        c = 0
        for pr in range(seq_pairs(qb, tpt)):
            k = pair_kv_tiles(pr, qb, ctx, tpt) + ITEM_COST
            c += k
            m = max(m, k)
        costs.append(c)
    W = sum(costs) * H_kv
    T = -(-W // n_ctas)
    T = max(T, ITEM_COST + 1, -(-m // (MAX_PIECES - 1)))
    mode = MODE_WRAP if takes_split(B, max(q_lens), H_kv, G, n_ctas) else MODE_QUEUE
    pre = [0]
    for c in costs:
        pre.append(pre[-1] + c * H_kv)
    starts = []
    for cta in range(n_ctas):
        pos = cta * T
        if pos >= W:
            starts.append((-1, 0, 0, 0))
            continue
        b = max(i for i in range(B) if pre[i] <= pos)
        cb = costs[b]
        off = pos - pre[b]
        g, r = divmod(off, cb)
        acc, pr = 0, 0
        while True:
            k = pair_kv_tiles(pr, q_lens[b], ctx_lens[b], tpt) + ITEM_COST
            if acc + k > r:
                break
            acc += k
            pr += 1
        starts.append((b, g, pr, acc - r))
    return Plan(mode, T, starts, W, m)


@dataclass
class Piece:
    cta: int
    b: int
    g: int
    pair: int
    k0: int
    k1: int
    c0: int      # the CTA whose range the item starts in
    j: int       # piece index (runs on CTA c0 + j)
    tiles: List[Optional[Tuple[int, int, int]]]  # per query tile X: (K/V tiles in the piece, n_split, j_first) or None


def tile_kv(qt: int, qb: int, ctx: int, tpt: int) -> int:
    t_begin = qt * tpt
    if t_begin >= qb:
        return 0
    n_tok = min(tpt, qb - t_begin)
    return (ctx - qb + t_begin + n_tok - 1) // KEYS + 1


def walk(p: Plan, q_lens, ctx_lens, H_kv: int, G: int, cta: int) -> List[Piece]:
    """The pieces CTA `cta` runs under the wrap-around plan, as its scheduler walks its range."""
    tpt = ROWS // G
    B = len(q_lens)
    T = p.T
    b, g, pair, rel = p.starts[cta]
    if b < 0:
        return []
    out = []
    while b < B and rel < T:
        qb, ctx = q_lens[b], ctx_lens[b]
        np_ = seq_pairs(qb, tpt)
        t = pair_kv_tiles(pair, qb, ctx, tpt)
        start, cost = rel, t + ITEM_COST
        cb, cg, cpair = b, g, pair
        rel += cost
        pair += 1
        if pair >= np_:
            pair = 0
            g += 1
            if g >= H_kv:
                g = 0
                b += 1
        lo = -start - ITEM_COST if start < 0 else 0
        hi = T - start - ITEM_COST if start + cost > T else t
        k0, k1 = min(max(lo, 0), t), min(max(hi, 0), t)
        if k0 >= k1:
            continue
        sh = start // T  # floor division
        prel = start - sh * T
        c0, j = cta + sh, -sh
        n = -(-(prel + cost) // T)

        def kc(i):
            if i <= 0:
                return 0
            if i >= n:
                return t
            return min(max(i * T - prel - ITEM_COST, 0), t)

        tiles = []
        for x in range(2):
            full = tile_kv(2 * cpair + x, qb, ctx, tpt)
            if full == 0:
                tiles.append(None)
                continue
            ns, jf = 0, 0
            for i in range(min(n, MAX_PIECES)):
                a = kc(i)
                if a < kc(i + 1) and a < full:
                    if ns == 0:
                        jf = i
                    ns += 1
            nkv = max(0, min(k1, full) - k0)
            tiles.append((nkv, ns, jf) if nkv > 0 else None)
        if tiles[0] is None and tiles[1] is None:
            continue
        out.append(Piece(cta, cb, cg, cpair, k0, k1, c0, j, tiles))
    return out


def slot_of(c0: int, j: int) -> int:
    """Merge slot of piece j of an item that starts in CTA c0's range."""
    return 2 * (c0 + j) + (1 if j == 0 else 0)
