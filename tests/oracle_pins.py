"""Pins that tie the fp64 oracle to facts outside itself.

Each ``pin_*`` takes a loaded oracle library ``L`` and raises AssertionError
when the oracle disagrees with:

* a library routine (numpy's binary16 decoding, torch's bfloat16 widening,
  numpy/torch fancy indexing, torch's fp64 ``scaled_dot_product_attention``);
* a closed form (one key returns its value row; equal scores return the mean;
  two keys give a logistic weight);
* an invariant the pages fix (paged equals contiguous and is blind to which
  physical blocks hold the pages; a tiled online softmax equals the full
  softmax; split partials merged by log-sum-exp equal the unsplit result);
* the worked page-table figure of the iopencloud page (section 3.2).

The same pins run against copies of the oracle with a planted mistake
(``test_oracle_mutants.py``); each plant must trip at least one pin.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch
import torch.nn.functional as F

import oracle
from paged_kv_attention_34_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---- helpers independent of the oracle ------------------------------------------

def gather_contiguous(cache: torch.Tensor, table_row: torch.Tensor, n: int) -> torch.Tensor:
    """[NB, H, 16, d] paged cache -> [H, n, d] contiguous keys of one sequence (torch indexing)."""
    pages = table_row[: (n + 15) // 16].long()
    x = cache[pages].double()  # [P, H, 16, d]
    x = x.permute(1, 0, 2, 3).reshape(cache.shape[1], -1, cache.shape[3])
    return x[:, :n]


def sdpa_reference(w: W.Workload, tree_mask=None) -> np.ndarray:
    """torch fp64 scaled_dot_product_attention per sequence on gathered K/V -> [T, H_q, d]; with
    ``tree_mask`` each new token sees the cached keys and the new tokens whose bits are set."""
    G = w.H_q // w.H_kv
    kc, vc = w.key_cache.clone(), w.value_cache.clone()
    # the step's new tokens are part of the context
    for t in range(w.k_new.shape[0]):
        s = int(w.slot_mapping[t])
        if s < 0:
            continue
        kc[s // 16, :, s % 16] = w.k_new[t]
        vc[s // 16, :, s % 16] = w.v_new[t]
    out = torch.empty((w.T, w.H_q, w.d), dtype=torch.float64)
    cu = w.cu_seqlens_q
    for b in range(w.B):
        ctx, qb = w.ctx_lens[b], w.q_lens[b]
        K = gather_contiguous(kc, w.block_tables[b], ctx).repeat_interleave(G, dim=0)  # [H_q, ctx, d]
        V = gather_contiguous(vc, w.block_tables[b], ctx).repeat_interleave(G, dim=0)
        Q = w.q[int(cu[b]) : int(cu[b + 1])].double().permute(1, 0, 2)  # [H_q, qb, d]
        i = torch.arange(qb).unsqueeze(1)
        j = torch.arange(ctx).unsqueeze(0)
        if tree_mask is None:
            mask = j <= (ctx - qb + i)
        else:
            bits = tree_mask[int(cu[b]) : int(cu[b + 1])].long().unsqueeze(1)  # [qb, 1]
            new = j - (ctx - qb)                                               # index among the new tokens
            mask = (new < 0) | ((bits >> new.clamp(min=0)) & 1).bool()
        o = F.scaled_dot_product_attention(Q, K, V, attn_mask=mask, scale=w.scale)
        out[int(cu[b]) : int(cu[b + 1])] = o.permute(1, 0, 2)
    return out.numpy()


def oracle_step(w: W.Workload, L, rows=None, n_threads: int = 0, tree_mask=None):
    """Run the step on the oracle: block copies, cache write, then attention over all sequences
    (tree-attention verification when ``tree_mask`` is given)."""
    kc = oracle._u16(w.key_cache).copy()
    vc = oracle._u16(w.value_cache).copy()
    if w.copy_pairs is not None:
        assert oracle.kv_block_copy(kc, vc, w.copy_pairs, L=L) == 0
    assert oracle.kv_cache_write(w.k_new, w.v_new, w.slot_mapping, kc, vc, L=L) == 0
    out = oracle.paged_attention(
        w.q, kc, vc, oracle.dtype_code(w.dtype), w.block_tables, w.cu_seqlens_q, w.context_lens, w.H_kv,
        w.scale, rows=rows, n_threads=n_threads, L=L, tree_mask=tree_mask,
    )
    return out, kc, vc


def _small_cases():
    cases = []
    for seed, (B, q_max, ctx_max, H_kv, G, d, dt) in enumerate(
        [
            (3, 1, 50, 2, 1, 64, W.F16),
            (4, 4, 70, 2, 4, 64, W.BF16),
            (2, 8, 40, 1, 8, 32, W.F16),
            (3, 20, 33, 2, 2, 16, W.BF16),
        ]
    ):
        cases.append(
            W.random_workload(100 + seed, B=B, q_max=q_max, ctx_max=ctx_max, H_kv=H_kv, G=G, d=d, dtype=dt,
                              kind="decode")
        )
    return cases


# ---- pins ---------------------------------------------------------------------------

def pin_f16_decoding(L):
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([L.oracle_f16_to_f64(int(b)) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all(), f"binary16 decode differs at {np.flatnonzero(~same)[:5]}"


def pin_bf16_decoding(L):
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).double().numpy()
    got = np.array([L.oracle_bf16_to_f64(int(b) & 0xFFFF) for b in bits.tolist()])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all(), f"bfloat16 decode differs at {np.flatnonzero(~same)[:5]}"


def pin_cache_write(L):
    g = torch.Generator().manual_seed(5)
    NB, H, d, T = 9, 3, 16, 40
    kc = torch.randn((NB, H, 16, d), generator=g).half()
    vc = torch.randn((NB, H, 16, d), generator=g).half()
    kn = torch.randn((T, H, d), generator=g).half()
    vn = torch.randn((T, H, d), generator=g).half()
    slots = torch.randperm(NB * 16, generator=g)[:T].to(torch.int32)
    slots[3] = -1
    slots[17] = -5
    ref_k, ref_v = kc.clone(), vc.clone()
    keep = slots >= 0
    s = slots[keep].long()
    rk = ref_k.permute(0, 2, 1, 3).reshape(NB * 16, H, d).clone()
    rv = ref_v.permute(0, 2, 1, 3).reshape(NB * 16, H, d).clone()
    rk[s] = kn[keep]
    rv[s] = vn[keep]
    rk = rk.view(NB, 16, H, d).permute(0, 2, 1, 3).contiguous()
    rv = rv.view(NB, 16, H, d).permute(0, 2, 1, 3).contiguous()
    k16, v16 = oracle._u16(kc).copy(), oracle._u16(vc).copy()
    bad = oracle.kv_cache_write(kn, vn, slots, k16, v16, L=L)
    assert bad == 0
    assert np.array_equal(k16, oracle._u16(rk)) and np.array_equal(v16, oracle._u16(rv))
    # an out-of-range slot is reported and not written
    slots2 = torch.tensor([NB * 16], dtype=torch.int32)
    before = k16.copy()
    assert oracle.kv_cache_write(kn[:1], vn[:1], slots2, k16, v16, L=L) == 1
    assert np.array_equal(before, k16)


def pin_block_copy(L):
    g = torch.Generator().manual_seed(6)
    NB, H, d = 8, 2, 16
    kc = torch.randn((NB, H, 16, d), generator=g).bfloat16()
    vc = torch.randn((NB, H, 16, d), generator=g).bfloat16()
    pairs = torch.tensor([[1, 4], [1, 5], [7, 0]], dtype=torch.int32)
    rk, rv = kc.clone(), vc.clone()
    for s, t in pairs.tolist():
        rk[t] = kc[s]
        rv[t] = vc[s]
    k16, v16 = oracle._u16(kc).copy(), oracle._u16(vc).copy()
    assert oracle.kv_block_copy(k16, v16, pairs, L=L) == 0
    assert np.array_equal(k16, oracle._u16(rk)) and np.array_equal(v16, oracle._u16(rv))
    assert oracle.kv_block_copy(k16, v16, torch.tensor([[0, NB]], dtype=torch.int32), L=L) == 1


def pin_block_swap(L):
    """Swap-out then swap-in into other device blocks restores their contents bit for bit; blocks
    outside the pairs are untouched; out-of-range pairs are skipped and counted."""
    g = torch.Generator().manual_seed(16)
    NB, HB, H, d = 8, 5, 2, 16
    kc = torch.randn((NB, H, 16, d), generator=g).half()
    vc = torch.randn((NB, H, 16, d), generator=g).half()
    k16, v16 = oracle._u16(kc).copy(), oracle._u16(vc).copy()
    hk, hv = np.zeros((HB, H, 16, d), np.uint16), np.zeros((HB, H, 16, d), np.uint16)
    out_pairs = torch.tensor([[6, 0], [2, 3], [5, 1]], dtype=torch.int32)
    assert oracle.kv_block_swap(k16, v16, hk, hv, out_pairs, to_host=True, L=L) == 0
    assert np.array_equal(k16, oracle._u16(kc)) and np.array_equal(v16, oracle._u16(vc))  # source untouched
    assert not hk[2].any() and not hk[4].any()                                              # unused host blocks
    # the device blocks are reused for something else, then the request resumes in other blocks
    k16[[6, 2, 5]] = 0
    v16[[6, 2, 5]] = 0
    in_pairs = torch.tensor([[7, 0], [0, 3], [4, 1]], dtype=torch.int32)
    assert oracle.kv_block_swap(k16, v16, hk, hv, in_pairs, to_host=False, L=L) == 0
    for (src, _), (dst, _) in zip(out_pairs.tolist(), in_pairs.tolist()):
        assert np.array_equal(k16[dst], oracle._u16(kc)[src]) and np.array_equal(v16[dst], oracle._u16(vc)[src])
    for b in (1, 3):  # neither swapped out nor in
        assert np.array_equal(k16[b], oracle._u16(kc)[b]) and np.array_equal(v16[b], oracle._u16(vc)[b])
    before = (k16.copy(), hk.copy())
    bad = torch.tensor([[NB, 0], [0, HB], [-1, 2]], dtype=torch.int32)
    assert oracle.kv_block_swap(k16, v16, hk, hv, bad, to_host=True, L=L) == 3
    assert oracle.kv_block_swap(k16, v16, hk, hv, bad, to_host=False, L=L) == 3
    assert np.array_equal(before[0], k16) and np.array_equal(before[1], hk)


def _e4m3_values(codes) -> torch.Tensor:
    """E4M3 codes -> float64 through torch's float8_e4m3fn (a decoder independent of the oracle)."""
    return torch.as_tensor(codes, dtype=torch.uint8).view(torch.float8_e4m3fn).double()


def pin_e4m3_codec(L):
    """The oracle's E4M3 decode and nearest-even encode against the format's definition (worked
    codes), torch's float8_e4m3fn decoder and encoder (finite range), and saturation at +-448."""
    worked = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x3F: 1.875, 0x40: 2.0,
              0x70: 128.0, 0x77: 240.0, 0x7E: 448.0, 0xFE: -448.0, 0xB8: -1.0}
    for c, v in worked.items():
        assert oracle.e4m3_to_f64(c, L=L) == v, hex(c)
    assert math.isnan(oracle.e4m3_to_f64(0x7F, L=L)) and math.isnan(oracle.e4m3_to_f64(0xFF, L=L))
    finite = [c for c in range(256) if c not in (0x7F, 0xFF)]
    ref = _e4m3_values(finite).tolist()
    for c, v in zip(finite, ref):
        assert oracle.e4m3_to_f64(c, L=L) == v, hex(c)
        assert oracle.f64_to_e4m3(v, L=L) == c, hex(c)  # every code round-trips (including -0)
    g = torch.Generator().manual_seed(8)
    xs = torch.cat([torch.randn(3000, generator=g) * 40, torch.randn(1000, generator=g) * 0.01,
                    (torch.rand(1000, generator=g) * 2 - 1) * 447.9])
    want = xs.to(torch.float8_e4m3fn).view(torch.uint8).tolist()
    for x, c in zip(xs.tolist(), want):
        assert oracle.f64_to_e4m3(x, L=L) == c, (x, c)
    # ties go to the even code; beyond 448 the codes saturate
    assert oracle.f64_to_e4m3(1.0625, L=L) == 0x38 and oracle.f64_to_e4m3(1.1875, L=L) == 0x3A
    assert oracle.f64_to_e4m3(1.5 * 2.0 ** -9, L=L) == 0x02 and oracle.f64_to_e4m3(0.5 * 2.0 ** -9, L=L) == 0x00
    for x in (448.5, 464.0, 500.0, 1e30):
        assert oracle.f64_to_e4m3(x, L=L) == 0x7E and oracle.f64_to_e4m3(-x, L=L) == 0xFE


def _fp8_case(seed, B=3, q_max=1, ctx_max=60, H_kv=2, G=2, d=32, dt=W.BF16):
    """A small decode workload with its cache written to FP8 by the oracle (every context row);
    V codes are [NB, H_kv, d, 16], transposed within each block."""
    w = W.random_workload(seed, B=B, q_max=q_max, ctx_max=ctx_max, H_kv=H_kv, G=G, d=d, dtype=dt, kind="decode")
    NB = w.key_cache.shape[0]
    kc8 = np.zeros((NB, H_kv, 16, d), np.uint8)
    vc8 = np.zeros((NB, H_kv, d, 16), np.uint8)
    ks = np.ones((NB, H_kv, 16), np.float32)
    vs = np.ones((NB, H_kv, 16), np.float32)
    # every stored row (the cached context and the step's new tokens) goes through the FP8 write
    rows_k = w.key_cache.reshape(NB, H_kv, 16, d).permute(0, 2, 1, 3).reshape(NB * 16, H_kv, d)
    rows_v = w.value_cache.reshape(NB, H_kv, 16, d).permute(0, 2, 1, 3).reshape(NB * 16, H_kv, d)
    slots = torch.arange(NB * 16, dtype=torch.int32)
    dtc = oracle.dtype_code(w.dtype)
    assert oracle.kv_cache_write_fp8(rows_k.contiguous(), rows_v.contiguous(), dtc, slots, kc8, vc8, ks, vs) == 0
    assert oracle.kv_cache_write_fp8(w.k_new, w.v_new, dtc, w.slot_mapping, kc8, vc8, ks, vs) == 0
    return w, kc8, vc8, ks, vs


def pin_fp8_write(L):
    """FP8 write: the row maximum lands on 448 exactly, the scale is amax / 448 in float, every
    value is within half an E4M3 step of the original, a zero row gets scale 1; bad slots count."""
    g = torch.Generator().manual_seed(12)
    T, H, d = 6, 3, 64
    kn = torch.randn((T, H, d), generator=g).bfloat16()
    vn = (torch.randn((T, H, d), generator=g) * 30).bfloat16()
    vn[2, 1] = 0
    NB = 2
    kc8, vc8 = np.zeros((NB, H, 16, d), np.uint8), np.zeros((NB, H, d, 16), np.uint8)
    ks, vs = np.zeros((NB, H, 16), np.float32), np.zeros((NB, H, 16), np.float32)
    slots = torch.tensor([0, 5, 17, 31, -1, 16], dtype=torch.int32)
    assert oracle.kv_cache_write_fp8(kn, vn, oracle.dtype_code(W.BF16), slots, kc8, vc8, ks, vs, L=L) == 0
    for t, sl in enumerate(slots.tolist()):
        if sl < 0:
            continue
        for h in range(H):
            # a V row is a column of its block: V codes are [NB, H, d, 16]
            for new, c8, sc in ((kn, kc8, ks), (vn, vc8.transpose(0, 1, 3, 2), vs)):
                x = new[t, h].double()
                amax = float(x.abs().max())
                s_ref = np.float32(amax) / np.float32(448.0) if amax > 0 else np.float32(1.0)
                assert sc[sl // 16, h, sl % 16] == s_ref
                deq = _e4m3_values(c8[sl // 16, h, sl % 16]) * float(s_ref)
                if amax > 0:
                    assert float(deq.abs().max()) == 448.0 * float(s_ref)
                # E4M3 keeps 3 mantissa bits: relative error <= 2^-4 for normals, absolute 2^-10 * scale below
                bound = torch.maximum(x.abs() * 2.0 ** -4, torch.full_like(x, 2.0 ** -10 * float(s_ref)))
                assert bool(((deq - x).abs() <= bound + 1e-12).all())
    assert not vc8[1, 1, :, 1].any() and vs[1, 1, 1] == 1.0  # the zero row (token 2 -> slot 17)
    # writing one slot touches only that slot's column of the V block
    assert not vc8[0, :, :, [c for c in range(16) if c not in (0, 5)]].any()
    assert oracle.kv_cache_write_fp8(kn[:1], vn[:1], oracle.dtype_code(W.BF16), torch.tensor([NB * 16], dtype=torch.int32), kc8, vc8,
                                     ks, vs, L=L) == 1


def pin_fp8_attention(L):
    """Attention over the FP8 cache == torch fp64 SDPA on the cache dequantised through torch's
    float8 decoder (ragged, GQA, causal verify rows)."""
    for seed, kw in ((21, {}), (22, dict(q_max=6, G=4, d=64, dt=W.F16)), (23, dict(B=2, q_max=3, ctx_max=90))):
        w, kc8, vc8, ks, vs = _fp8_case(seed, **kw)
        got = oracle.paged_attention_fp8(w.q, oracle.dtype_code(w.dtype), kc8, vc8, ks, vs, w.block_tables,
                                         w.cu_seqlens_q, w.context_lens, w.H_kv, w.scale, L=L)
        deq = lambda c8, sc: (_e4m3_values(c8.reshape(-1)).reshape(c8.shape) * torch.from_numpy(sc).double()[..., None])
        vrows = np.ascontiguousarray(vc8.transpose(0, 1, 3, 2))  # back to [NB, H_kv, 16, d]
        w2 = W.Workload(**{**vars(w), "key_cache": deq(kc8, ks), "value_cache": deq(vrows, vs),
                           "slot_mapping": torch.full_like(w.slot_mapping, -1)})
        ref = sdpa_reference(w2)
        err = np.abs(got - ref).max()
        assert err < 1e-12, f"fp8 oracle vs SDPA max err {err}"


def pin_sdpa_library(L):
    """Paged fp64 oracle == torch fp64 SDPA on the gathered contiguous K/V (ragged, GQA, causal)."""
    for w in _small_cases():
        got, _, _ = oracle_step(w, L)
        ref = sdpa_reference(w)
        err = np.abs(got - ref).max()
        assert err < 1e-12, f"{w.name}: oracle vs SDPA max err {err}"


def pin_tree_verify(L):
    """Tree-attention verification == torch fp64 SDPA with the tree's boolean mask; the chain mask
    reproduces the causal verify exactly."""
    for k, w in enumerate(_small_cases()):
        if max(w.q_lens) > 8:
            continue
        tm = W.random_tree_masks(300 + k, w.q_lens)
        got, _, _ = oracle_step(w, L, tree_mask=tm)
        ref = sdpa_reference(w, tree_mask=tm)
        err = np.abs(got - ref).max()
        assert err < 1e-12, f"{w.name}: tree oracle vs SDPA max err {err}"
        causal, _, _ = oracle_step(w, L)
        chain, _, _ = oracle_step(w, L, tree_mask=W.chain_masks(w.q_lens))
        assert np.array_equal(causal, chain)
    # a forest where some tokens see no other draft: only their own bit
    w = _small_cases()[2]
    solo = torch.tensor([1 << i for qb in w.q_lens for i in range(int(qb))], dtype=torch.int32)
    got, _, _ = oracle_step(w, L, tree_mask=solo)
    assert np.abs(got - sdpa_reference(w, tree_mask=solo)).max() < 1e-12


def pin_shared_prefix(L):
    """Groups of sequences sharing prompt-prefix blocks: the oracle over the aliased tables == fp64
    SDPA on the gathered keys, and for every row the attention over the group's shared keys merged
    by log-sum-exp with the attention over the sequence's own keys is the whole -- the decomposition
    that the shared-prefix decode computes (the prefix once per group, then the merge)."""
    w = W.shared_prefix_batch(seed=61, B=5, n_groups=2, prefix_tokens=48, suffix=(3, 40), q_max=3, H_q=4, H_kv=2,
                              d=16)
    starts, P = w.notes["group_start"], w.notes["prefix_blocks"]
    for v in range(len(P)):
        for b in range(starts[v], starts[v + 1]):
            assert torch.equal(w.block_tables[b, : P[v]], w.block_tables[starts[v], : P[v]])
    got, kc, vc = oracle_step(w, L)
    assert np.abs(got - sdpa_reference(w)).max() < 1e-12
    G = w.H_q // w.H_kv
    kd = torch.from_numpy(kc.view(np.float16)).double()
    vd = torch.from_numpy(vc.view(np.float16)).double()
    cu = w.cu_seqlens_q.tolist()
    for b in range(w.B):
        v = max(i for i in range(len(P)) if starts[i] <= b)
        n_pre = P[v] * 16
        ctx, qb = w.ctx_lens[b], w.q_lens[b]
        K = gather_contiguous(kd, w.block_tables[b], ctx)
        V = gather_contiguous(vd, w.block_tables[b], ctx)
        for i in range(qb):
            t = cu[b] + i
            last = ctx - qb + i
            for h in range(w.H_q):
                q = w.q[t, h].double().numpy()
                kh, vh = K[h // G].numpy(), V[h // G].numpy()
                parts, lses = [], []
                for lo, hi in ((0, n_pre), (n_pre, last + 1)):
                    o, l_ = oracle.attention_partial(q, kh, vh, lo, hi, w.scale, L=L)
                    parts.append(o)
                    lses.append(l_)
                merged, _ = oracle.lse_merge(np.stack(parts), np.array(lses), L=L)
                assert np.abs(merged - got[t, h]).max() < 1e-13, (b, i, h)


def pin_dense_three_pass(L):
    """Paged oracle == the standard three-pass attention on contiguous data."""
    w = W.random_workload(11, B=2, q_max=5, ctx_max=37, H_kv=2, G=2, d=16, dtype=W.F16, kind="decode")
    got, kc, vc = oracle_step(w, L)
    kc_t = torch.from_numpy(kc.view(np.int16)).view(torch.float16)
    vc_t = torch.from_numpy(vc.view(np.int16)).view(torch.float16)
    cu = w.cu_seqlens_q
    for b in range(w.B):
        ctx, qb = w.ctx_lens[b], w.q_lens[b]
        K = gather_contiguous(kc_t, w.block_tables[b], ctx)
        V = gather_contiguous(vc_t, w.block_tables[b], ctx)
        for h in range(w.H_q):
            g_ = h // (w.H_q // w.H_kv)
            Q = w.q[int(cu[b]) : int(cu[b + 1]), h].double().numpy()
            ref = oracle.dense_attention(Q, K[g_].numpy(), V[g_].numpy(), w.scale, ctx - qb, L=L)
            assert np.abs(got[int(cu[b]) : int(cu[b + 1]), h] - ref).max() < 1e-12


def pin_block_permutation(L):
    """Relabelling physical blocks (pool and table together) leaves the output unchanged."""
    w = W.random_workload(21, B=3, q_max=3, ctx_max=60, H_kv=2, G=2, d=32, dtype=W.BF16, kind="decode")
    base, _, _ = oracle_step(w, L)
    g = torch.Generator().manual_seed(99)
    perm = torch.randperm(w.num_blocks, generator=g)  # new id of old block i is perm[i]
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(w.num_blocks)
    w.key_cache = w.key_cache[inv].contiguous()
    w.value_cache = w.value_cache[inv].contiguous()
    w.block_tables = perm[w.block_tables.long()].to(torch.int32)
    sl = w.slot_mapping.long()
    w.slot_mapping = (perm[sl // 16] * 16 + sl % 16).to(torch.int32)
    again, _, _ = oracle_step(w, L)
    assert np.array_equal(base, again)


def pin_paged_equals_contiguous(L):
    """The same data laid out as one contiguous cache (table = 0..n-1) gives the same output."""
    w = W.random_workload(31, B=2, q_max=4, ctx_max=45, H_kv=1, G=4, d=16, dtype=W.F16, kind="decode")
    base, kc, vc = oracle_step(w, L)
    kc_t = torch.from_numpy(kc.view(np.int16)).view(torch.float16)
    vc_t = torch.from_numpy(vc.view(np.int16)).view(torch.float16)
    cu = w.cu_seqlens_q
    for b in range(w.B):
        ctx = w.ctx_lens[b]
        n = (ctx + 15) // 16
        pages = w.block_tables[b, :n].long()
        kb, vb = kc_t[pages].contiguous(), vc_t[pages].contiguous()
        table = torch.arange(n, dtype=torch.int32).unsqueeze(0)
        qb = w.q[int(cu[b]) : int(cu[b + 1])]
        cu1 = torch.tensor([0, qb.shape[0]], dtype=torch.int32)
        out = oracle.paged_attention(qb, kb, vb, oracle.dtype_code(w.dtype), table, cu1,
                                     torch.tensor([ctx], dtype=torch.int32), w.H_kv, w.scale, L=L)
        assert np.array_equal(out, base[int(cu[b]) : int(cu[b + 1])])


def _one_seq(L, q, k, v, scale, dtype=W.F16):
    """Oracle attention for one decode query over contiguous keys placed in a paged cache."""
    n, d = k.shape
    pages = (n + 15) // 16
    kc = torch.full((pages, 1, 16, d), float("nan"), dtype=dtype)
    vc = torch.full((pages, 1, 16, d), float("nan"), dtype=dtype)
    kc.view(pages * 16, d)[:n] = k.to(dtype)
    vc.view(pages * 16, d)[:n] = v.to(dtype)
    table = torch.arange(pages, dtype=torch.int32).flip(0).unsqueeze(0)  # pages stored back to front
    kc = kc.flip(0).contiguous()
    vc = vc.flip(0).contiguous()
    out = oracle.paged_attention(q.to(dtype).view(1, 1, d), kc, vc, oracle.dtype_code(dtype), table,
                                 torch.tensor([0, 1], dtype=torch.int32), torch.tensor([n], dtype=torch.int32), 1,
                                 scale, L=L)
    return out[0, 0]


def pin_single_key(L):
    g = torch.Generator().manual_seed(3)
    q, k, v = (torch.randn((1, 64), generator=g) for _ in range(3))
    out = _one_seq(L, q[0], k, v, 0.125)
    assert np.array_equal(out, v[0].half().double().numpy())


def pin_equal_scores_mean(L):
    g = torch.Generator().manual_seed(4)
    k = torch.randn((37, 32), generator=g)
    v = torch.randn((37, 32), generator=g)
    out = _one_seq(L, torch.zeros(32), k, v, 0.3)
    ref = v.half().double().mean(0).numpy()
    assert np.abs(out - ref).max() < 1e-14


def pin_two_keys_closed_form(L):
    # q = e0, k0 = a*e0, k1 = b*e0: scores scale*a, scale*b; weight of key 0 = 1/(1+exp(scale*(b-a)))
    d = 16
    q = torch.zeros(d)
    q[0] = 1.0
    a, b, scale = 2.0, -1.5, 0.7
    k = torch.zeros((2, d))
    k[0, 0], k[1, 0] = a, b
    v = torch.zeros((2, d))
    v[0, 1], v[1, 2] = 1.0, 1.0
    out = _one_seq(L, q, k, v, scale)
    w0 = 1.0 / (1.0 + math.exp(scale * (b - a)))
    assert abs(out[1] - w0) < 1e-15 and abs(out[2] - (1 - w0)) < 1e-15 and out[0] == 0.0


def pin_large_scores(L):
    # scores around 1000 (exp would overflow without the max subtracted)
    d = 16
    q = torch.zeros(d)
    q[0] = 1.0
    k = torch.zeros((3, d))
    k[0, 0], k[1, 0], k[2, 0] = 1000.0, 999.0, -1000.0
    v = torch.zeros((3, d))
    v[0, 3], v[1, 4], v[2, 5] = 1.0, 1.0, 1.0
    out = _one_seq(L, q, k, v, 1.0)
    e1 = math.exp(-1.0)
    assert abs(out[3] - 1 / (1 + e1)) < 1e-15 and abs(out[4] - e1 / (1 + e1)) < 1e-15 and out[5] == 0.0


def pin_online_softmax(L):
    """Tiled online softmax (iopencloud section 2.2) == three-pass softmax, for any tile size."""
    g = torch.Generator().manual_seed(8)
    n, d = 53, 24
    q = torch.randn(d, generator=g).double().numpy()
    k = torch.randn((n, d), generator=g).double().numpy()
    v = torch.randn((n, d), generator=g).double().numpy()
    ref = oracle.dense_attention(q[None], k, v, 0.2, 10**9, L=L)[0]
    lib_ref = F.scaled_dot_product_attention(torch.from_numpy(q)[None], torch.from_numpy(k), torch.from_numpy(v),
                                             scale=0.2)[0].numpy()
    assert np.abs(ref - lib_ref).max() < 1e-13
    for block in (1, 2, 5, 16, 53, 64):
        got = oracle.online_softmax(q, k, v, 0.2, block, L=L)
        assert np.abs(got - ref).max() < 1e-13, block


def pin_split_merge(L):
    """Split-KV partials merged by log-sum-exp == unsplit attention; empty splits are ignored."""
    g = torch.Generator().manual_seed(9)
    n, d = 70, 16
    q = torch.randn(d, generator=g).double().numpy()
    k = torch.randn((n, d), generator=g).double().numpy()
    v = torch.randn((n, d), generator=g).double().numpy()
    full, full_lse = oracle.attention_partial(q, k, v, 0, n, 0.25, L=L)
    lib_full = F.scaled_dot_product_attention(torch.from_numpy(q)[None], torch.from_numpy(k), torch.from_numpy(v),
                                              scale=0.25)[0].numpy()
    assert np.abs(full - lib_full).max() < 1e-13
    s = torch.from_numpy(k @ q * 0.25)
    assert abs(full_lse - float(torch.logsumexp(s, 0))) < 1e-12
    bounds = [0, 16, 16, 33, 64, 70]  # includes one empty split
    parts, lses = [], []
    for lo, hi in zip(bounds[:-1], bounds[1:]):
        o, l_ = oracle.attention_partial(q, k, v, lo, hi, 0.25, L=L)
        parts.append(o)
        lses.append(l_)
    assert lses[1] == -math.inf and not np.any(parts[1])
    merged, mlse = oracle.lse_merge(np.stack(parts), np.array(lses), L=L)
    assert np.abs(merged - full).max() < 1e-13 and abs(mlse - full_lse) < 1e-12


def pin_convex_hull(L):
    w = W.random_workload(41, B=3, q_max=2, ctx_max=80, H_kv=2, G=1, d=16, dtype=W.F16, kind="decode")
    out, kc, vc = oracle_step(w, L)
    vc_t = torch.from_numpy(vc.view(np.int16)).view(torch.float16)
    cu = w.cu_seqlens_q
    for b in range(w.B):
        V = gather_contiguous(vc_t, w.block_tables[b], w.ctx_lens[b])
        for t in range(int(cu[b]), int(cu[b + 1])):
            for h in range(w.H_q):
                lo = V[h].min(0).values.numpy()
                hi = V[h].max(0).values.numpy()
                assert np.all(out[t, h] >= lo - 1e-12) and np.all(out[t, h] <= hi + 1e-12)


def pin_causal_rows(L):
    """A fresh prompt: its first query sees key 0 only (output = V_0); row i sees keys 0..i."""
    w = W.build_workload("fresh", q_lens=[20], ctx_lens=[20], H_q=2, H_kv=2, d=16, dtype=W.BF16, seed=5,
                         calls=[W.AttnCall("prefill", 0, 1)], pool_extra=2)
    out, kc, vc = oracle_step(w, L)
    v0 = w.v_new[0].double().numpy()
    assert np.array_equal(out[0], v0)
    kn, vn = w.k_new.double(), w.v_new.double()
    for i in (1, 7, 19):
        for h in range(2):
            ref = F.scaled_dot_product_attention(w.q[i, h].double()[None], kn[: i + 1, h], vn[: i + 1, h],
                                                 scale=w.scale)[0].numpy()
            assert np.abs(out[i, h] - ref).max() < 1e-13


def pin_golden_page_table(L):
    """iopencloud section 3.2 figure: A = [0,1,5,7,8], B = [2,9] in an 11-block pool."""
    pool, tables = {}, {}
    with open(os.path.join(GOLDEN, "page_table_example.txt")) as f:
        for line in f:
            line = line.split("#")[0].split()
            if not line:
                continue
            if line[0] == "slot":
                pool[int(line[1])] = line[2]
            elif line[0] == "table":
                tables[line[1]] = [int(x) for x in line[2:]]
            elif line[0] == "pool_blocks":
                nb = int(line[1])
    assert tables == {"A": [0, 1, 5, 7, 8], "B": [2, 9]} and nb == 11
    # A holds 5 pages (65..80 tokens), B 2 pages (17..32 tokens); take 75 and 20 tokens.
    ctx = {"A": 75, "B": 20}
    H, d = 2, 16
    g = torch.Generator().manual_seed(12)
    kc = torch.full((nb, H, 16, d), float("nan"), dtype=torch.float16)
    vc = torch.full((nb, H, 16, d), float("nan"), dtype=torch.float16)
    k16, v16 = oracle._u16(kc).copy(), oracle._u16(vc).copy()
    seq_k, seq_v = {}, {}
    for name in ("A", "B"):
        n = ctx[name]
        seq_k[name] = torch.randn((n, H, d), generator=g).half()
        seq_v[name] = torch.randn((n, H, d), generator=g).half()
        slots = torch.tensor([tables[name][p // 16] * 16 + p % 16 for p in range(n)], dtype=torch.int32)
        assert oracle.kv_cache_write(seq_k[name], seq_v[name], slots, k16, v16, L=L) == 0
    # pool contents follow the figure: page i of request X sits in the slot labelled Xi; free slots untouched
    kc_after = torch.from_numpy(k16.view(np.int16)).view(torch.float16)
    for slot, label in pool.items():
        if label == "-":
            assert torch.isnan(kc_after[slot]).all()
        else:
            name, page = label[0], int(label[1:]) - 1
            n_in = min(16, ctx[name] - page * 16)
            assert torch.equal(kc_after[slot, :, :n_in], seq_k[name][page * 16 : page * 16 + n_in].permute(1, 0, 2))
    # attention through the tables == attention on each request's contiguous K/V
    q = torch.randn((2, H, d), generator=g).half()
    bt = torch.tensor([tables["A"], tables["B"] + [0, 0, 0]], dtype=torch.int32)
    out = oracle.paged_attention(q, k16, v16, oracle.F16, bt, torch.tensor([0, 1, 2], dtype=torch.int32),
                                 torch.tensor([ctx["A"], ctx["B"]], dtype=torch.int32), H, 0.25, L=L)
    for b, name in enumerate(("A", "B")):
        for h in range(H):
            ref = F.scaled_dot_product_attention(q[b, h].double()[None], seq_k[name][:, h].double(),
                                                 seq_v[name][:, h].double(), scale=0.25)[0].numpy()
            assert np.abs(out[b, h] - ref).max() < 1e-13


def pin_rejects_bad_args(L):
    q = torch.zeros((2, 1, 16), dtype=torch.float16)
    kc = torch.zeros((1, 1, 16, 16), dtype=torch.float16)
    bt = torch.zeros((1, 1), dtype=torch.int32)
    try:
        oracle.paged_attention(q, kc, kc, oracle.F16, bt, torch.tensor([0, 2], dtype=torch.int32),
                               torch.tensor([1], dtype=torch.int32), 1, 1.0, L=L)
    except ValueError:
        return
    raise AssertionError("ctx < q_len must be rejected")


ALL_PINS = [
    pin_f16_decoding,
    pin_bf16_decoding,
    pin_cache_write,
    pin_block_copy,
    pin_block_swap,
    pin_e4m3_codec,
    pin_fp8_write,
    pin_fp8_attention,
    pin_sdpa_library,
    pin_tree_verify,
    pin_shared_prefix,
    pin_dense_three_pass,
    pin_block_permutation,
    pin_paged_equals_contiguous,
    pin_single_key,
    pin_equal_scores_mean,
    pin_two_keys_closed_form,
    pin_large_scores,
    pin_online_softmax,
    pin_split_merge,
    pin_convex_hull,
    pin_causal_rows,
    pin_golden_page_table,
    pin_rejects_bad_args,
]
