"""CPU checks of the prefill call's work schedule (the host model in prefill_schedule_model.py):
every item's K/V tiles are covered exactly once by its pieces, the merge bookkeeping of a split
item (piece counts, slots, arrival counters) is consistent across its pieces, and no two items
share a slot or a counter.  The GPU tests compare the plan the kernel writes with this model."""
import random
from collections import defaultdict

import pytest

import prefill_schedule_model as S


def _check_wrap(q_lens, ctx_lens, H_kv, G, n_ctas):
    # the split plan of any shape, whether or not the host would choose it for these sizes
    p = S.plan(q_lens, ctx_lens, H_kv, G, n_ctas)
    tpt = S.ROWS // G
    assert p.T >= S.ITEM_COST + 1 and p.T * (S.MAX_PIECES - 1) >= p.M
    pieces = [pc for c in range(n_ctas) for pc in S.walk(p, q_lens, ctx_lens, H_kv, G, c)]
    by_item = defaultdict(list)
    for pc in pieces:
        assert pc.cta == pc.c0 + pc.j and 0 <= pc.c0 <= pc.cta < n_ctas
        assert 0 <= pc.j < S.MAX_PIECES and 0 <= pc.k0 < pc.k1
        by_item[(pc.b, pc.g, pc.pair)].append(pc)
    # every item with work: its tiles partitioned by its pieces, in CTA order
    for b, (qb, ctx) in enumerate(zip(q_lens, ctx_lens)):
        for g in range(H_kv):
            for pr in range(S.seq_pairs(qb, tpt)):
                t = S.pair_kv_tiles(pr, qb, ctx, tpt)
                ps = sorted(by_item.pop((b, g, pr), []), key=lambda x: x.cta)
                assert ps, (b, g, pr)
                assert ps[0].k0 == 0 and ps[-1].k1 == t
                for a, c in zip(ps, ps[1:]):
                    assert a.k1 == c.k0 and c.cta == a.cta + 1 and c.j == a.j + 1 and c.c0 == a.c0
                # per query tile: the pieces that hold its keys agree on (n_split, j_first), are
                # pieces j_first .. j_first + n_split - 1, and cover its K/V tiles exactly
                for x in range(2):
                    full = S.tile_kv(2 * pr + x, qb, ctx, tpt)
                    on = [pc for pc in ps if pc.tiles[x] is not None]
                    if full == 0:
                        assert not on
                        continue
                    assert {(pc.tiles[x][1], pc.tiles[x][2]) for pc in on} == {(len(on), on[0].j)}
                    assert [pc.j for pc in on] == list(range(on[0].j, on[0].j + len(on)))
                    assert sum(pc.tiles[x][0] for pc in on) == full
                    assert on[0].k0 == 0
    assert not by_item, "pieces of items that have no work"
    # split items: slots (2 per CTA) and arrival counters (per item) are each used by one item
    slot_owner, cnt_owner = {}, {}
    items = defaultdict(list)
    for pc in pieces:
        items[(pc.b, pc.g, pc.pair)].append(pc)
    for key, ps in items.items():
        if all(pc.tiles[x] is None or pc.tiles[x][1] == 1 for pc in ps for x in range(2)):
            continue
        assert cnt_owner.setdefault(ps[0].c0, key) == key
        for pc in ps:
            s = S.slot_of(pc.c0, pc.j)
            assert 0 <= s < 2 * n_ctas
            assert slot_owner.setdefault(s, key) == key
    return p


def _rand_case(rng):
    G = rng.choice([1, 2, 4, 5, 8, 16])
    H_kv = rng.choice([1, 2, 8])
    B = rng.choice([1, 2, 3, 4, 7, 16])
    q_lens, ctx_lens = [], []
    for _ in range(B):
        qb = rng.randint(1, rng.choice([40, 300, 1024]))
        ctx = qb + rng.choice([0, rng.randint(0, 600), rng.randint(0, 20000)])
        q_lens.append(qb)
        ctx_lens.append(ctx)
    return q_lens, ctx_lens, H_kv, G, rng.choice([148, 37, 5, 1])


@pytest.mark.parametrize("seed", range(40))
def test_wrap_schedule_covers_every_tile_once(seed):
    rng = random.Random(seed)
    for _ in range(10):
        _check_wrap(*_rand_case(rng))


def test_long_context_chunk_takes_the_split_schedule():
    # one 512-token chunk over a 32 K context (8 KV heads, G 4): 64 items on 148 SMs; cut into
    # pieces of at most T tiles, so every CTA gets a share
    p = _check_wrap([512], [32768], 8, 4, 148)
    assert p.mode == S.MODE_WRAP and p.T < p.M / 2
    n = sum(len(S.walk(p, [512], [32768], 8, 4, c)) for c in range(148))
    assert n >= 148


def test_many_items_keep_the_queue():
    # eight causal prompts of 273-1422 tokens, 40 heads: 1280 short items
    q = [612, 273, 871, 1223, 1150, 1216, 325, 1422]
    assert S.plan(q, q, 40, 1, 148).mode == S.MODE_QUEUE
    # the mixed step's four 512-token chunks, 8 KV heads: 256 items on 148 SMs
    assert S.plan([512] * 4, [2311, 6183, 8512, 911], 8, 4, 148).mode == S.MODE_QUEUE
    # the host's rule: at most 3/4 of the CTAs busy
    assert S.takes_split(1, 512, 8, 4, 148) and not S.takes_split(2, 512, 8, 4, 148)
    assert S.takes_split(111, 64, 1, 1, 148) and not S.takes_split(112, 64, 1, 1, 148)


def test_few_items_split_across_ctas():
    # 16 items of ~30 K/V tiles on 148 CTAs: every item is cut into pieces of about T tiles
    p = _check_wrap([512], [4000], 2, 4, 148)
    assert p.mode == S.MODE_WRAP
    n = sum(len(S.walk(p, [512], [4000], 2, 4, c)) for c in range(148))
    assert n > 16 * 4  # more pieces than items


def test_piece_cap_sets_the_range_for_very_long_items():
    # two items of ~1560 K/V tiles on 148 CTAs: the balanced share (~22) would cut each into ~70
    # pieces; T is raised to M / 7 so that no item has more than 8, and CTAs past the work get none
    q, c = [512], [200000]
    p = _check_wrap(q, c, 1, 4, 148)
    assert p.T == -(-p.M // (S.MAX_PIECES - 1)) > -(-p.W // 148)
    per_item = {}
    for cta in range(148):
        for pc in S.walk(p, q, c, 1, 4, cta):
            per_item.setdefault((pc.b, pc.g, pc.pair), []).append(pc)
    assert all(len(v) <= S.MAX_PIECES for v in per_item.values())
    assert p.starts[147][0] == -1  # positions past W: no work
