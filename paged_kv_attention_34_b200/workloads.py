"""Seeded synthetic workloads for paged KV attention.

This module only draws inputs: sequence lengths, block tables, slot mappings
and N(0,1) tensors.  It holds none of the attention arithmetic, so both the
CUDA library and the CPU oracle can be fed from it without sharing any code
of the method itself.

Layouts (the pages fix none of them):

* ``q``, ``k_new``, ``v_new``: token-major ``[T, H, d]``; tokens of sequence
  ``b`` occupy rows ``cu_seqlens_q[b] .. cu_seqlens_q[b+1]``.
* ``key_cache`` / ``value_cache``: ``[num_blocks, H_kv, 16, d]``, i.e. one
  (block, kv-head) pair is a contiguous ``16 x d`` tile.  This is the
  fixed-size 16-token page of "PagedAttention" (iopencloud, "大模型推理加速技术
  全景", section 3.2; ybb.press, section 2; the zhihu roofline page,
  "显存管理：从碎片化到分页", which names 16 tokens as the default).
* ``block_tables``: ``int32 [B, max_blocks]``; page ``p`` of sequence ``b`` is
  physical block ``block_tables[b, p]``.  Entries past a sequence's last page
  are 0 and are never read.
* ``context_lens``: ``int32 [B]``, keys of sequence ``b`` in the cache
  *including* the step's new tokens.  Query ``i`` of sequence ``b`` sits at
  absolute position ``ctx_b - q_b + i``.
* ``slot_mapping``: ``int32 [T]``, ``slot = block * 16 + offset`` for each new
  token; negative means "padding, skip".

Every workload is seeded (``seed = 34_000 + config index`` by default) and
drawn with a torch CPU generator, so the same call always returns the same
bytes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import torch

BLOCK_SIZE = 16

F16 = torch.float16
BF16 = torch.bfloat16


@dataclass
class AttnCall:
    """One attention launch inside a step: a contiguous range of sequences."""

    kind: str  # "decode" or "prefill"
    seq_lo: int
    seq_hi: int  # exclusive


@dataclass
class Workload:
    name: str
    dtype: torch.dtype
    H_q: int
    H_kv: int
    d: int
    q_lens: List[int]
    ctx_lens: List[int]
    num_blocks: int
    block_tables: torch.Tensor  # int32 [B, max_blocks]
    slot_mapping: torch.Tensor  # int32 [T]
    q: torch.Tensor  # [T, H_q, d]
    k_new: torch.Tensor  # [T, H_kv, d]
    v_new: torch.Tensor  # [T, H_kv, d]
    key_cache: torch.Tensor  # [NB, H_kv, 16, d] state before the step
    value_cache: torch.Tensor
    scale: float
    calls: List[AttnCall]
    copy_pairs: Optional[torch.Tensor] = None  # int32 [n, 2] (src, dst), run before the write
    shared_blocks: int = 0  # physical blocks referenced by more than one sequence (counted once)
    notes: dict = field(default_factory=dict)

    # ---- derived views ------------------------------------------------------
    @property
    def B(self) -> int:
        return len(self.q_lens)

    @property
    def T(self) -> int:
        return int(sum(self.q_lens))

    @property
    def max_blocks(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def cu_seqlens_q(self) -> torch.Tensor:
        cu = [0]
        for n in self.q_lens:
            cu.append(cu[-1] + n)
        return torch.tensor(cu, dtype=torch.int32)

    @property
    def context_lens(self) -> torch.Tensor:
        return torch.tensor(self.ctx_lens, dtype=torch.int32)

    def call_args(self, call: AttnCall) -> dict:
        """Host tensors for one attention call (sequence subset, rebased cu_seqlens)."""
        lo, hi = call.seq_lo, call.seq_hi
        cu_all = self.cu_seqlens_q
        t0, t1 = int(cu_all[lo]), int(cu_all[hi])
        cu = (cu_all[lo : hi + 1] - t0).to(torch.int32).contiguous()
        return dict(
            t0=t0,
            t1=t1,
            cu_seqlens_q=cu,
            context_lens=self.context_lens[lo:hi].contiguous(),
            block_tables=self.block_tables[lo:hi].contiguous(),
            B=hi - lo,
            max_q_len=max(self.q_lens[lo:hi]),
            max_ctx=max(self.ctx_lens[lo:hi]),
        )


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _randn(shape, dtype, g) -> torch.Tensor:
    return torch.randn(shape, generator=g, dtype=torch.float32).to(dtype)


def _fill_cache_randn(cache: torch.Tensor, g: torch.Generator, chunk_blocks: int = 2048) -> None:
    """Fill a [NB, H, 16, d] cache with N(0,1) values in chunks (bounded host memory)."""
    nb = cache.shape[0]
    for s in range(0, nb, chunk_blocks):
        e = min(nb, s + chunk_blocks)
        cache[s:e] = torch.randn(cache[s:e].shape, generator=g, dtype=torch.float32).to(cache.dtype)


def build_workload(
    name: str,
    *,
    q_lens: List[int],
    ctx_lens: List[int],
    H_q: int,
    H_kv: int,
    d: int,
    dtype: torch.dtype,
    seed: int,
    calls: List[AttnCall],
    pool_extra: int = 0,
    pool_blocks: Optional[int] = None,
    fill: str = "nan",
    scale: Optional[float] = None,
) -> Workload:
    """Generic builder: every sequence owns its pages; the pool is a seeded shuffle.

    The cache holds N(0,1) K/V for the existing tokens (positions ``< ctx_b - q_b``);
    the step's new tokens come as ``k_new``/``v_new`` + ``slot_mapping``.  Every
    other slot (unused blocks, the tail of a last partial block, and the new
    tokens' slots before they are written) holds ``fill``: NaN by default, so a
    kernel that reads past a sequence's context shows up as a NaN.
    """
    assert len(q_lens) == len(ctx_lens)
    for qb, cb in zip(q_lens, ctx_lens):
        assert 1 <= qb <= cb, (qb, cb)
    g = _gen(seed)
    B = len(q_lens)
    pages = [math.ceil(c / BLOCK_SIZE) for c in ctx_lens]
    used = sum(pages)
    nb = pool_blocks if pool_blocks is not None else used + pool_extra
    assert nb >= used
    perm = torch.randperm(nb, generator=g).to(torch.int32)
    max_blocks = max(pages)
    bt = torch.zeros((B, max_blocks), dtype=torch.int32)
    pos = 0
    for b in range(B):
        bt[b, : pages[b]] = perm[pos : pos + pages[b]]
        pos += pages[b]

    T = sum(q_lens)
    q = _randn((T, H_q, d), dtype, g)
    k_new = _randn((T, H_kv, d), dtype, g)
    v_new = _randn((T, H_kv, d), dtype, g)
    slot = torch.empty(T, dtype=torch.int32)
    t = 0
    for b in range(B):
        for i in range(q_lens[b]):
            p = ctx_lens[b] - q_lens[b] + i
            slot[t] = int(bt[b, p // BLOCK_SIZE]) * BLOCK_SIZE + p % BLOCK_SIZE
            t += 1

    kc, vc = _make_caches(nb, H_kv, d, dtype, fill)
    # existing context: random K/V written slot by slot range (whole blocks where possible)
    for b in range(B):
        n_old = ctx_lens[b] - q_lens[b]
        _fill_existing(kc, vc, bt[b], n_old, g)
    return Workload(
        name=name,
        dtype=dtype,
        H_q=H_q,
        H_kv=H_kv,
        d=d,
        q_lens=list(q_lens),
        ctx_lens=list(ctx_lens),
        num_blocks=nb,
        block_tables=bt,
        slot_mapping=slot,
        q=q,
        k_new=k_new,
        v_new=v_new,
        key_cache=kc,
        value_cache=vc,
        scale=scale if scale is not None else 1.0 / math.sqrt(d),
        calls=calls,
    )


def _make_caches(nb, H_kv, d, dtype, fill):
    shape = (nb, H_kv, BLOCK_SIZE, d)
    if fill == "nan":
        kc = torch.full(shape, float("nan"), dtype=dtype)
        vc = torch.full(shape, float("nan"), dtype=dtype)
    elif fill == "zero":
        kc = torch.zeros(shape, dtype=dtype)
        vc = torch.zeros(shape, dtype=dtype)
    else:
        raise ValueError(fill)
    return kc, vc


def _fill_existing(kc, vc, table_row, n_old, g):
    """Write N(0,1) K/V for logical positions [0, n_old) of one sequence."""
    full, rem = divmod(n_old, BLOCK_SIZE)
    if full:
        blocks = table_row[:full].long()
        shp = (full,) + tuple(kc.shape[1:])
        kc[blocks] = _randn(shp, kc.dtype, g)
        vc[blocks] = _randn(shp, vc.dtype, g)
    if rem:
        blk = int(table_row[full])
        shp = (kc.shape[1], rem, kc.shape[3])
        kc[blk, :, :rem] = _randn(shp, kc.dtype, g)
        vc[blk, :, :rem] = _randn(shp, vc.dtype, g)


# ---------------------------------------------------------------------------
# The five configurations
# ---------------------------------------------------------------------------

CONFIG_NAMES = {
    1: "tiny decode: 3 seqs ctx {1,17,50}, q_len 1, 4/4 heads, d 64, fp16",
    2: "LLaMA-2-13B-shaped decode layer: B 64, q_len 1, 40/40 heads, d 128, fp16, ctx U[128,4096]",
    3: "causal varlen prefill: 8 prompts U[256,2048], 40/40 heads, d 128, bf16",
    4: "long-context GQA decode: B 16, 64/8 heads, d 128, bf16, ctx 32768, 2048-token shared prefix, one kv_block_copy",
    5: "mixed continuous-batching step: 4x512-token chunks + 16 verify (q 6) + 128 decode, 32/8 heads, d 128, bf16",
}


def _uniform_int(g, lo, hi, n) -> List[int]:
    """n integers uniform on [lo, hi] (inclusive)."""
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g)]


def config1(seed: int = 34_001, fill: str = "nan") -> Workload:
    """Tiny decode: ctx {1,17,50}, pool of 16 blocks assigned by a seeded permutation."""
    ctx = [1, 17, 50]
    return build_workload(
        "cfg1",
        q_lens=[1, 1, 1],
        ctx_lens=ctx,
        H_q=4,
        H_kv=4,
        d=64,
        dtype=F16,
        seed=seed,
        calls=[AttnCall("decode", 0, 3)],
        pool_blocks=16,
        fill=fill,
        scale=1.0 / math.sqrt(64),
    )


def config2(seed: int = 34_002, fill: str = "nan", B: int = 64) -> Workload:
    g = _gen(seed + 1_000_000)
    ctx = _uniform_int(g, 128, 4096, B)
    return build_workload(
        "cfg2",
        q_lens=[1] * B,
        ctx_lens=ctx,
        H_q=40,
        H_kv=40,
        d=128,
        dtype=F16,
        seed=seed,
        calls=[AttnCall("decode", 0, B)],
        fill=fill,
    )


def config3(seed: int = 34_003, fill: str = "nan", B: int = 8) -> Workload:
    g = _gen(seed + 1_000_000)
    L = _uniform_int(g, 256, 2048, B)
    return build_workload(
        "cfg3",
        q_lens=L,
        ctx_lens=L,
        H_q=40,
        H_kv=40,
        d=128,
        dtype=BF16,
        seed=seed,
        calls=[AttnCall("prefill", 0, B)],
        fill=fill,
    )


def config4(
    seed: int = 34_004,
    fill: str = "nan",
    B: int = 16,
    ctx: int = 32768,
    shared_tokens: int = 2048,
    fork_tokens: int = 8,
) -> Workload:
    """GQA decode over a long context whose first blocks are shared by every sequence.

    The state before the step: blocks ``0 .. shared_tokens/16 - 1`` of every
    sequence map to the same physical blocks (refcount B).  Logical block
    ``shared_tokens/16`` was filled with ``fork_tokens`` shared tokens before
    the fork and is still shared.  The step then (1) copies that block for
    B-1 sequences (copy-on-write; the last sequence keeps the original),
    (2) writes each sequence's own tokens for the rest of that block and its
    newest token (position ctx-1), (3) decodes one query per sequence.
    Positions after the divergent block up to ctx-2 are already cached and
    unique per sequence.
    """
    g = _gen(seed)
    H_q, H_kv, d, dt = 64, 8, 128, BF16
    assert shared_tokens % BLOCK_SIZE == 0 and 0 < fork_tokens < BLOCK_SIZE
    n_pages = math.ceil(ctx / BLOCK_SIZE)
    n_shared = shared_tokens // BLOCK_SIZE
    fork_page = n_shared
    # pool: shared blocks + the shared fork block + (B-1) copies + unique blocks
    n_unique = n_pages - n_shared - 1
    nb = n_shared + 1 + (B - 1) + B * n_unique
    perm = torch.randperm(nb, generator=g).to(torch.int32)
    shared_ids = perm[:n_shared]
    fork_id = int(perm[n_shared])
    copy_ids = perm[n_shared + 1 : n_shared + B]
    uniq = perm[n_shared + B :].view(B, n_unique)
    bt = torch.zeros((B, n_pages), dtype=torch.int32)
    for b in range(B):
        bt[b, :n_shared] = shared_ids
        bt[b, fork_page] = int(copy_ids[b]) if b < B - 1 else fork_id
        bt[b, fork_page + 1 :] = uniq[b]
    pairs = torch.stack([torch.full((B - 1,), fork_id, dtype=torch.int32), copy_ids], dim=1).contiguous()

    kc, vc = _make_caches(nb, H_kv, d, dt, fill)
    _fill_cache_blocks(kc, vc, shared_ids, g)
    shp = (H_kv, fork_tokens, d)
    kc[fork_id, :, :fork_tokens] = _randn(shp, dt, g)
    vc[fork_id, :, :fork_tokens] = _randn(shp, dt, g)
    # unique blocks: every position except the newest one (ctx-1) is already cached
    for b in range(B):
        ids = uniq[b]
        _fill_cache_blocks(kc, vc, ids, g)
        last_pos = ctx - 1
        lp, lo = divmod(last_pos, BLOCK_SIZE)
        blk = int(bt[b, lp])
        kc[blk, :, lo:] = float("nan") if fill == "nan" else 0.0
        vc[blk, :, lo:] = float("nan") if fill == "nan" else 0.0

    # new tokens: rest of the fork block (fork_tokens..15) + newest token, per sequence
    n_fork_new = BLOCK_SIZE - fork_tokens
    q_lens = [1] * B
    T_write = B * (n_fork_new + 1)
    slot = torch.empty(T_write, dtype=torch.int32)
    t = 0
    for b in range(B):
        for o in range(fork_tokens, BLOCK_SIZE):
            slot[t] = int(bt[b, fork_page]) * BLOCK_SIZE + o
            t += 1
    for b in range(B):
        p = ctx - 1
        slot[t] = int(bt[b, p // BLOCK_SIZE]) * BLOCK_SIZE + p % BLOCK_SIZE
        t += 1
    k_new_all = _randn((T_write, H_kv, d), dt, g)
    v_new_all = _randn((T_write, H_kv, d), dt, g)
    q = _randn((B, H_q, d), dt, g)
    w = Workload(
        name="cfg4",
        dtype=dt,
        H_q=H_q,
        H_kv=H_kv,
        d=d,
        q_lens=q_lens,
        ctx_lens=[ctx] * B,
        num_blocks=nb,
        block_tables=bt,
        slot_mapping=slot,
        q=q,
        k_new=k_new_all,
        v_new=v_new_all,
        key_cache=kc,
        value_cache=vc,
        scale=1.0 / math.sqrt(d),
        calls=[AttnCall("decode", 0, B)],
        copy_pairs=pairs,
        shared_blocks=n_shared,
        notes=dict(shared_tokens=shared_tokens, fork_tokens=fork_tokens, write_tokens=T_write),
    )
    return w


def _fill_cache_blocks(kc, vc, ids, g, chunk=1024):
    ids = ids.long()
    for s in range(0, ids.numel(), chunk):
        sub = ids[s : s + chunk]
        shp = (sub.numel(),) + tuple(kc.shape[1:])
        kc[sub] = _randn(shp, kc.dtype, g)
        vc[sub] = _randn(shp, vc.dtype, g)


def lognormal_ctx(g, n, mean=1500.0, sigma=1.0, cap=8192) -> List[int]:
    """Integer context lengths with a lognormal law of the given mean, clamped to [1, cap]."""
    mu = math.log(mean) - sigma * sigma / 2.0
    z = torch.randn(n, generator=g, dtype=torch.float64)
    vals = torch.exp(mu + sigma * z).round().clamp(1, cap)
    return [int(v) for v in vals]


def config5(
    seed: int = 34_005,
    fill: str = "nan",
    n_chunks: int = 4,
    chunk: int = 512,
    n_verify: int = 16,
    verify_q: int = 6,
    n_decode: int = 128,
) -> Workload:
    """Mixed continuous-batching step.

    Sequence order: chunked-prefill requests, then speculative-verify requests,
    then plain decode requests.  One ``kv_cache_write`` covers every new token;
    one prefill call covers the chunks and one decode call covers verify + decode.
    """
    g = _gen(seed + 1_000_000)
    existing = _uniform_int(g, 0, 8192, n_chunks)
    ver_ctx = _uniform_int(g, 512, 4096, n_verify)
    dec_ctx = lognormal_ctx(g, n_decode)
    q_lens = [chunk] * n_chunks + [verify_q] * n_verify + [1] * n_decode
    ctx = [e + chunk for e in existing] + ver_ctx + dec_ctx
    calls = [AttnCall("prefill", 0, n_chunks), AttnCall("decode", n_chunks, n_chunks + n_verify + n_decode)]
    return build_workload(
        "cfg5",
        q_lens=q_lens,
        ctx_lens=ctx,
        H_q=32,
        H_kv=8,
        d=128,
        dtype=BF16,
        seed=seed,
        calls=calls,
        fill=fill,
    )


def random_tree_masks(seed: int, q_lens) -> torch.Tensor:
    """Draft-tree visibility masks for tree-attention verification, int32 [sum(q_lens)].

    The q_b new tokens of a sequence are the nodes of a random forest drafted in order: node i has
    a parent drawn uniformly from the earlier nodes or none (a new root).  Bit j of node i's mask
    is set when node j is node i itself or one of its ancestors.
    """
    g = _gen(seed)
    masks = []
    for qb in q_lens:
        m = []
        for i in range(int(qb)):
            parent = int(torch.randint(-1, i, (1,), generator=g)) if i > 0 else -1
            m.append((m[parent] if parent >= 0 else 0) | (1 << i))
        masks.extend(m)
    return torch.tensor(masks, dtype=torch.int32)


def chain_masks(q_lens) -> torch.Tensor:
    """The causal verify as a tree: node i sees nodes 0 .. i."""
    return torch.tensor([(1 << (i + 1)) - 1 for qb in q_lens for i in range(int(qb))], dtype=torch.int32)


def tree_verify(seed: int = 34_105, fill: str = "nan", B: int = 64, q: int = 8) -> Workload:
    """Tree-attention verification of speculative drafts: B sequences with q drafted tokens each
    (a random draft forest, ``random_tree_masks``) on contexts U[512, 4096] (the verify rows of the
    mixed step, with a tree instead of a chain); 32/8 heads, d 128, bf16."""
    g = _gen(seed + 1_000_000)
    ctx = _uniform_int(g, 512, 4096, B)
    return build_workload(
        "tree_verify",
        q_lens=[q] * B,
        ctx_lens=ctx,
        H_q=32,
        H_kv=8,
        d=128,
        dtype=BF16,
        seed=seed,
        calls=[AttnCall("decode", 0, B)],
        fill=fill,
    )


def share_prefixes(w: Workload, group_sizes: List[int], prefix_blocks: List[int]) -> Workload:
    """Make consecutive runs of sequences share prompt-prefix blocks, in place: group v is the next
    group_sizes[v] sequences, and the first prefix_blocks[v] entries of each member's table are
    pointed at its first sequence's blocks (whose contents then stand for the shared prompt; the
    members' own former prefix blocks stay in the pool unused).  A prefix must end before every
    member's new tokens.  Returns w with notes group_start / prefix_blocks."""
    assert sum(group_sizes) == w.B and len(group_sizes) == len(prefix_blocks)
    starts = [0]
    for n in group_sizes:
        starts.append(starts[-1] + n)
    for v, P in enumerate(prefix_blocks):
        lead = starts[v]
        for b in range(lead, starts[v + 1]):
            assert P * BLOCK_SIZE <= w.ctx_lens[b] - w.q_lens[b], (b, P)
            if b != lead:
                w.block_tables[b, :P] = w.block_tables[lead, :P]
    w.shared_blocks = sum(P for v, P in enumerate(prefix_blocks) if group_sizes[v] > 1)
    w.notes = {**w.notes, "group_start": starts, "prefix_blocks": list(prefix_blocks)}
    return w


def shared_prefix_batch(seed: int = 34_106, fill: str = "nan", B: int = 64, n_groups: int = 4,
                        prefix_tokens: int = 4096, suffix=(16, 512), q_max: int = 1, H_q: int = 40, H_kv: int = 40,
                        d: int = 128, dtype: torch.dtype = F16) -> Workload:
    """Decode batch of requests that share prompts: B sequences in n_groups consecutive groups of
    (nearly) equal size; each group shares a prefix_tokens-token prompt (whole blocks), and each
    sequence has its own suffix of U[suffix] tokens after it, the last q_b of them new this step.
    Defaults: the 13B-shaped decode layer (40/40 heads, d 128, fp16) with 4 prompts of 4096 tokens
    and 16 requests each."""
    assert prefix_tokens % BLOCK_SIZE == 0
    g = _gen(seed + 1_000_000)
    q_lens = [int(x) for x in torch.randint(1, q_max + 1, (B,), generator=g)]
    suf = _uniform_int(g, suffix[0], suffix[1], B)
    ctx = [prefix_tokens + max(sb, qb) for sb, qb in zip(suf, q_lens)]
    w = build_workload("shared_prefix", q_lens=q_lens, ctx_lens=ctx, H_q=H_q, H_kv=H_kv, d=d, dtype=dtype,
                       seed=seed, calls=[AttnCall("decode", 0, B)], fill=fill)
    sizes = [B // n_groups + (1 if v < B % n_groups else 0) for v in range(n_groups)]
    return share_prefixes(w, sizes, [prefix_tokens // BLOCK_SIZE] * n_groups)


def make_config(idx: int, **kw) -> Workload:
    return {1: config1, 2: config2, 3: config3, 4: config4, 5: config5}[idx](**kw)


def random_workload(
    seed: int,
    *,
    B: int,
    q_max: int,
    ctx_max: int,
    H_kv: int,
    G: int,
    d: int,
    dtype: torch.dtype,
    kind: str,
    pool_extra: int = 3,
) -> Workload:
    """Small seeded random case for sweeps (ragged contexts, partial last blocks)."""
    g = _gen(seed)
    q_lens, ctx_lens = [], []
    for _ in range(B):
        qb = int(torch.randint(1, q_max + 1, (1,), generator=g))
        cb = int(torch.randint(qb, max(qb, ctx_max) + 1, (1,), generator=g))
        q_lens.append(qb)
        ctx_lens.append(cb)
    return build_workload(
        f"rand{seed}",
        q_lens=q_lens,
        ctx_lens=ctx_lens,
        H_q=H_kv * G,
        H_kv=H_kv,
        d=d,
        dtype=dtype,
        seed=seed + 7,
        calls=[AttnCall(kind, 0, B)],
        pool_extra=pool_extra,
    )
