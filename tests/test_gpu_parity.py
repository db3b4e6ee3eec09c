"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Tolerances (max-abs error against fp64, N(0,1) inputs): 3e-3 for fp16
outputs, 1.6e-2 for bf16 outputs.  Cache writes and block copies must match
the oracle's caches byte for byte.  Caches are filled with NaN outside every
sequence's context, so any read past a context end shows up as a NaN.

Small seeded cases are checked on every output row; the five full-size
configurations are checked on sampled rows (all rows of the shortest and the
longest sequence of each call, plus random rows), in the same launch
configuration the benchmark times.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_attention_34_b200 as pa
import prefill_schedule_model as S
from oracle_pins import oracle_step
from paged_kv_attention_34_b200 import workloads as W
from paged_kv_attention_34_b200.step import DeviceStep

pytestmark = pytest.mark.gpu

TOL = {torch.float16: 3e-3, torch.bfloat16: 1.6e-2}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pa.lib()


def _u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def sample_rows(w: W.Workload, n_random: int, seed: int = 0) -> np.ndarray:
    rows = set()
    cu = w.cu_seqlens_q.tolist()
    for c in w.calls:
        seqs = list(range(c.seq_lo, c.seq_hi))
        by_ctx = sorted(seqs, key=lambda b: w.ctx_lens[b])
        for b in {by_ctx[0], by_ctx[-1]}:
            toks = range(cu[b], cu[b + 1])
            if len(toks) > 64:  # long prompts: first, last and a spread of tokens
                toks = sorted(set(list(toks[:4]) + list(toks[-4:]) + list(toks[:: max(1, len(toks) // 16)])))
            for t in toks:
                for h in range(w.H_q):
                    rows.add(t * w.H_q + h)
    g = np.random.default_rng(seed)
    rows.update(g.integers(0, w.T * w.H_q, size=n_random).tolist())
    return np.array(sorted(rows), dtype=np.int64)


def run_and_compare(w: W.Workload, rows=None, check_cache=True):
    st = DeviceStep(w)
    out = st.run()
    torch.cuda.synchronize()
    assert st.statuses() == [0] * (1 + len(st.calls)), st.statuses()
    ref, kc_ref, vc_ref = oracle_step(w, oracle.lib(), rows=rows)
    if check_cache:
        # bit-exact caches (compared on the device to keep host memory small)
        dev = st.key_cache.device
        assert torch.equal(st.key_cache.view(torch.int16), torch.from_numpy(kc_ref.view(np.int16)).to(dev))
        assert torch.equal(st.value_cache.view(torch.int16), torch.from_numpy(vc_ref.view(np.int16)).to(dev))
    got = out.double().cpu().numpy().reshape(w.T * w.H_q, w.d)
    if rows is not None:
        got = got[rows]
    else:
        ref = ref.reshape(-1, w.d)
    assert np.isfinite(got).all(), "non-finite output"
    err = np.abs(got - ref).max()
    assert err <= TOL[w.dtype], f"{w.name}: max abs err {err:.3e} > {TOL[w.dtype]}"
    return err


# ---- small seeded sweeps (every row) -----------------------------------------------------

DECODE_CASES = [
    # (B, q_max, ctx_max, H_kv, G, d, dtype)
    (5, 1, 300, 2, 1, 64, W.F16),
    (5, 1, 700, 3, 1, 128, W.F16),
    (4, 4, 500, 2, 4, 128, W.BF16),
    (3, 8, 900, 1, 8, 128, W.BF16),  # 64 rows per CTA
    (3, 8, 400, 2, 8, 64, W.F16),
    (2, 8, 300, 1, 16, 128, W.BF16),  # two row groups per KV head
    (6, 6, 2000, 2, 4, 128, W.BF16),  # many splits, verify-like rows
    (4, 3, 33, 2, 2, 64, W.BF16),     # tiny contexts, partial blocks
]


def _case_id(c):
    return "B{}q{}c{}h{}g{}d{}{}".format(*c[:6], "bf16" if c[6] == W.BF16 else "f16")


@pytest.mark.parametrize("idx", range(len(DECODE_CASES)), ids=lambda i: _case_id(DECODE_CASES[i]))
@pytest.mark.parametrize("seed", [1, 2])
def test_decode_small(idx, seed):
    B, q_max, ctx_max, H_kv, G, d, dt = DECODE_CASES[idx]
    w = W.random_workload(1000 * seed + 17 * idx, B=B, q_max=q_max, ctx_max=ctx_max, H_kv=H_kv, G=G, d=d,
                          dtype=dt, kind="decode")
    run_and_compare(w)


PREFILL_CASES = [
    (3, 200, 300, 2, 1, 128, W.BF16),
    (2, 130, 260, 2, 4, 128, W.BF16),  # chunks with earlier context, GQA
    (3, 90, 90, 2, 1, 64, W.F16),
    (4, 17, 40, 1, 8, 128, W.F16),
]


@pytest.mark.parametrize("idx", range(len(PREFILL_CASES)), ids=lambda i: _case_id(PREFILL_CASES[i]))
def test_prefill_small(idx):
    B, q_max, ctx_max, H_kv, G, d, dt = PREFILL_CASES[idx]
    w = W.random_workload(77 + 31 * idx, B=B, q_max=q_max, ctx_max=ctx_max, H_kv=H_kv, G=G, d=d, dtype=dt,
                          kind="prefill")
    run_and_compare(w)


# The same kinds of small prefill calls with enough items (> 3/4 of the SMs) to stay on the queue
# schedule: the cases above all have few items and take the split one.
QUEUE_PREFILL_CASES = [
    (8, 200, 300, 16, 1, 128, W.BF16),
    (8, 130, 260, 8, 4, 128, W.BF16),  # chunks with earlier context, GQA
    (8, 90, 90, 16, 1, 64, W.F16),
    (16, 17, 40, 8, 8, 128, W.F16),
]


@pytest.mark.parametrize("idx", range(len(QUEUE_PREFILL_CASES)), ids=lambda i: _case_id(QUEUE_PREFILL_CASES[i]))
def test_prefill_small_queue_schedule(idx):
    B, q_max, ctx_max, H_kv, G, d, dt = QUEUE_PREFILL_CASES[idx]
    w = W.random_workload(177 + 31 * idx, B=B, q_max=q_max, ctx_max=ctx_max, H_kv=H_kv, G=G, d=d, dtype=dt,
                          kind="prefill")
    assert not S.takes_split(w.B, max(w.q_lens), w.H_kv, G, _n_ctas())
    run_and_compare(w)


def test_prefill_fresh_prompts_exact_lengths():
    # prompts of 1, 15, 16, 17, 127, 128, 129 tokens with no earlier context
    L = [1, 15, 16, 17, 127, 128, 129]
    w = W.build_workload("fresh", q_lens=L, ctx_lens=L, H_q=4, H_kv=2, d=128, dtype=W.BF16, seed=9,
                         calls=[W.AttnCall("prefill", 0, len(L))], pool_extra=5)
    run_and_compare(w)


# Prefill calls with too few items to keep 3/4 of the SMs busy take the split schedule: items cut
# into pieces on neighbouring CTAs, the pieces' partials merged by the last one to finish.
# (name, q_lens, ctx_lens, H_kv, G, d, dtype)
SPLIT_PREFILL_CASES = [
    ("long_ctx_chunk", [512], [16384 + 37], 2, 4, 128, W.BF16),
    ("few_items", [512, 100], [4000, 2500], 2, 4, 128, W.BF16),
    ("g5_rows125_d64", [300], [9000], 1, 5, 64, W.F16),  # 125 rows per tile: three rows unused
    ("g1_two_tiles_ragged", [200, 3], [20000, 7000], 1, 1, 128, W.F16),
]


def _split_workload(case, seed):
    name, q, c, H_kv, G, d, dt = case
    return W.build_workload(name, q_lens=q, ctx_lens=c, H_q=H_kv * G, H_kv=H_kv, d=d, dtype=dt, seed=seed,
                            calls=[W.AttnCall("prefill", 0, len(q))], pool_extra=3)


def _n_ctas():
    return min(torch.cuda.get_device_properties(0).multi_processor_count, S.MAX_CTAS)


def _prefill_plan(call, w):
    """(T, starts, n_ctas) of the split schedule the prefill call wrote into its workspace."""
    ws = call.ws.cpu()
    T = ws[128:132].view(torch.int32).item()
    tok = 128 // (w.H_q // w.H_kv)
    n_pairs = ((call.max_q_len + tok - 1) // tok + 1) // 2
    off = pa.PA_STATUS_BYTES + (n_pairs * (call.seq_hi - call.seq_lo) * 4 + 255) // 256 * 256
    n_ctas = _n_ctas()
    starts = [tuple(x) for x in ws[off:off + 16 * n_ctas].view(torch.int32).view(-1, 4).tolist()]
    return T, starts, n_ctas


@pytest.mark.parametrize("idx", range(len(SPLIT_PREFILL_CASES)), ids=lambda i: SPLIT_PREFILL_CASES[i][0])
def test_prefill_split_items(idx):
    case = SPLIT_PREFILL_CASES[idx]
    w = _split_workload(case, 300 + idx)
    st = DeviceStep(w)
    call = st.calls[0]
    # the call takes the split schedule, and its plan is the host model's
    q, c = list(w.q_lens), list(w.ctx_lens)
    st.run()
    torch.cuda.synchronize()
    T, starts, n_ctas = _prefill_plan(call, w)
    model = S.plan(q, c, w.H_kv, w.H_q // w.H_kv, n_ctas)
    assert model.mode == S.MODE_WRAP
    assert (T, starts) == (model.T, model.starts)
    rows = sample_rows(w, 1024) if w.T * w.H_q * max(c) > 3e7 else None
    run_and_compare(w, rows=rows)



def test_split_prefill_with_a_dirty_workspace():
    # the merge counters and partials come from the call itself: a workspace full of garbage
    # gives the same bytes as a clean one, call after call
    w = _split_workload(SPLIT_PREFILL_CASES[1], 41)
    st = DeviceStep(w)
    st.copy_blocks()
    st.write()
    call = st.calls[0]
    call.ws.fill_(0x5A)
    call.out.fill_(float("nan"))
    n0 = pa.launch_count()
    st.attend(call)
    o1 = call.out.clone()
    st.attend(call)
    torch.cuda.synchronize()
    assert pa.launch_count() - n0 == 4  # plan + attention kernel per call
    assert pa.read_status(call.ws) == 0
    assert torch.equal(o1.view(torch.int16), call.out.view(torch.int16))
    ref, _, _ = oracle_step(w, oracle.lib())
    got = call.out.double().cpu().numpy().reshape(-1, w.d)
    assert np.abs(got - ref.reshape(-1, w.d)).max() <= TOL[w.dtype]


def test_split_prefill_reports_an_inconsistent_sequence():
    # under the split schedule the plan kernel checks the sequences: one whose context is shorter
    # than its new tokens is reported (PA_ERR_SEQ) and left out of the plan, and the other
    # sequence's rows are still right
    w = _split_workload(("bad_seq", [300, 200], [5000, 4000], 2, 4, 128, W.BF16), 57)
    assert S.takes_split(w.B, max(w.q_lens), w.H_kv, w.H_q // w.H_kv, _n_ctas())
    st = DeviceStep(w)
    st.copy_blocks()
    st.write()
    call = st.calls[0]
    call.ctx[1] = 100  # < q_len 200
    st.attend(call)
    torch.cuda.synchronize()
    assert pa.read_status(call.ws) == -8  # PA_ERR_SEQ
    rows = np.arange(300 * w.H_q, dtype=np.int64)  # every row of sequence 0
    ref, _, _ = oracle_step(w, oracle.lib(), rows=rows)
    got = call.out.double().cpu().numpy().reshape(-1, w.d)[rows]
    assert np.abs(got - ref).max() <= TOL[w.dtype]


# ---- FP8 (E4M3) KV cache ---------------------------------------------------------------------

def _fp8_device_cache(w):
    """The workload's cache (every stored row, then the step's new tokens) written into an FP8 cache on
    the device: (codes K, codes V, scales K, scales V)."""
    NB, H, _, d = w.key_cache.shape
    kc8 = torch.zeros((NB, H, 16, d), dtype=torch.uint8, device="cuda")
    vc8 = torch.zeros((NB, H, d, 16), dtype=torch.uint8, device="cuda")  # transposed within the block
    ks = torch.ones((NB, H, 16), dtype=torch.float32, device="cuda")
    vs = torch.ones_like(ks)
    rows_k = w.key_cache.permute(0, 2, 1, 3).reshape(NB * 16, H, d).contiguous().cuda()
    rows_v = w.value_cache.permute(0, 2, 1, 3).reshape(NB * 16, H, d).contiguous().cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.kv_cache_write_fp8(rows_k, rows_v, torch.arange(NB * 16, dtype=torch.int32, device="cuda"), kc8, vc8, ks, vs,
                          status=status)
    pa.kv_cache_write_fp8(w.k_new.cuda(), w.v_new.cuda(), w.slot_mapping.cuda(), kc8, vc8, ks, vs, status=status)
    torch.cuda.synchronize()
    assert pa.read_status(status) == 0
    return kc8, vc8, ks, vs


def _fp8_decode(w, kc8, vc8, ks, vs):
    call = next(c for c in DeviceStep(w).calls if c.kind == "decode")
    out = pa.paged_attn_decode_fp8(call.q, kc8, vc8, ks, vs, call.bt, call.cu, call.ctx, call.max_ctx, w.scale,
                                   workspace=call.ws)
    torch.cuda.synchronize()
    assert pa.read_status(call.ws) == 0
    return out


FP8_CASES = [
    (4, 1, 300, 2, 1, 128, W.F16),
    (3, 4, 500, 2, 4, 128, W.BF16),
    (3, 8, 400, 2, 8, 64, W.F16),
    (5, 6, 2000, 2, 4, 128, W.BF16),  # several splits
    (4, 3, 33, 2, 2, 64, W.BF16),     # tiny contexts, partial blocks
    # single-token decode with G <= 8 takes the keys-on-M variant
    (6, 1, 700, 2, 8, 128, W.BF16),
    (5, 1, 3000, 1, 4, 64, W.F16),    # several splits
    (4, 1, 40, 4, 2, 128, W.F16),     # tiny contexts
    (3, 1, 17, 2, 1, 64, W.BF16),     # one full block and one key
    (2, 1, 600, 1, 16, 128, W.BF16),  # G 16: the 16-row variant again
]


@pytest.mark.parametrize("idx", range(len(FP8_CASES)), ids=lambda i: _case_id(FP8_CASES[i]))
def test_fp8_cache_and_decode_small(idx):
    B, q_max, ctx_max, H_kv, G, d, dt = FP8_CASES[idx]
    w = W.random_workload(800 + 7 * idx, B=B, q_max=q_max, ctx_max=ctx_max, H_kv=H_kv, G=G, d=d, dtype=dt,
                          kind="decode")
    kc8, vc8, ks, vs = _fp8_device_cache(w)
    # the cache, byte for byte and scale for scale, as the oracle writes it
    NB, H = w.key_cache.shape[:2]
    okc, ovc = np.zeros((NB, H, 16, d), np.uint8), np.zeros((NB, H, d, 16), np.uint8)
    oks, ovs = np.ones((NB, H, 16), np.float32), np.ones((NB, H, 16), np.float32)
    rows_k = w.key_cache.permute(0, 2, 1, 3).reshape(NB * 16, H, d).contiguous()
    rows_v = w.value_cache.permute(0, 2, 1, 3).reshape(NB * 16, H, d).contiguous()
    dtc = oracle.dtype_code(w.dtype)
    assert oracle.kv_cache_write_fp8(rows_k, rows_v, dtc, torch.arange(NB * 16, dtype=torch.int32), okc, ovc, oks,
                                     ovs) == 0
    assert oracle.kv_cache_write_fp8(w.k_new, w.v_new, dtc, w.slot_mapping, okc, ovc, oks, ovs) == 0
    assert np.array_equal(kc8.cpu().numpy(), okc) and np.array_equal(vc8.cpu().numpy(), ovc)
    assert np.array_equal(ks.cpu().numpy().view(np.uint32), oks.view(np.uint32))
    assert np.array_equal(vs.cpu().numpy().view(np.uint32), ovs.view(np.uint32))
    # attention over it
    got = _fp8_decode(w, kc8, vc8, ks, vs).double().cpu().numpy()
    ref = oracle.paged_attention_fp8(w.q, dtc, okc, ovc, oks, ovs, w.block_tables, w.cu_seqlens_q, w.context_lens,
                                     w.H_kv, w.scale)
    assert np.isfinite(got).all()
    err = np.abs(got - ref).max()
    assert err <= TOL[w.dtype], f"max abs err {err:.3e}"


def test_fp8_decode_13b_layer_sampled():
    # the 13B-shaped decode layer (64 sequences, 40 heads, contexts U[128, 4096]) over an FP8 cache
    w = W.config2()
    kc8, vc8, ks, vs = _fp8_device_cache(w)
    out = _fp8_decode(w, kc8, vc8, ks, vs)
    rows = sample_rows(w, 200, seed=6)
    ref = oracle.paged_attention_fp8(w.q, oracle.dtype_code(w.dtype), kc8.cpu().numpy(), vc8.cpu().numpy(),
                                     ks.cpu().numpy(), vs.cpu().numpy(), w.block_tables, w.cu_seqlens_q,
                                     w.context_lens, w.H_kv, w.scale, rows=rows)
    got = out.double().cpu().numpy().reshape(w.T * w.H_q, w.d)[rows]
    assert np.isfinite(got).all()
    err = np.abs(got - ref).max()
    assert err <= TOL[w.dtype], f"max abs err {err:.3e}"


def test_fp8_decode_rejects_missing_scales():
    import ctypes

    w = W.random_workload(5, B=2, q_max=1, ctx_max=40, H_kv=1, G=1, d=64, dtype=W.F16, kind="decode")
    kc8, vc8, ks, vs = _fp8_device_cache(w)
    call = DeviceStep(w).calls[0]
    n0 = pa.launch_count()
    rc = pa.lib().pa_paged_attn_decode_fp8(
        ctypes.c_void_p(call.out.data_ptr()), ctypes.c_void_p(call.q.data_ptr()), ctypes.c_void_p(kc8.data_ptr()),
        ctypes.c_void_p(vc8.data_ptr()), None, ctypes.c_void_p(vs.data_ptr()), kc8.shape[0],
        ctypes.c_void_p(call.bt.data_ptr()), call.bt.shape[1], ctypes.c_void_p(call.cu.data_ptr()),
        ctypes.c_void_p(call.ctx.data_ptr()), call.ctx.shape[0], call.max_ctx, call.q.shape[0], w.H_q, w.H_kv, w.d,
        w.scale, 0, ctypes.c_void_p(call.ws.data_ptr()), call.ws.numel(), None)
    assert rc == -1 and pa.launch_count() == n0


# ---- tree-attention verification ---------------------------------------------------------

def _tree_run(w, tm):
    """Cache write, then the tree-verify decode on the device; returns (output, step)."""
    st = DeviceStep(w)
    st.copy_blocks()
    st.write()
    call = st.calls[0]
    out = pa.paged_attn_decode_tree(call.q, st.key_cache, st.value_cache, call.bt, call.cu, call.ctx, tm.cuda(),
                                    call.max_ctx, w.scale, out=call.out, workspace=call.ws)
    torch.cuda.synchronize()
    assert st.statuses() == [0] * (1 + len(st.calls)), st.statuses()
    return out, st


TREE_CASES = [
    (4, 8, 500, 2, 4, 128, W.BF16),
    (3, 8, 300, 2, 8, 64, W.F16),
    (5, 6, 2000, 2, 4, 128, W.BF16),  # several splits
    (2, 8, 40, 1, 16, 128, W.BF16),   # two row groups, short contexts
    (4, 5, 9, 2, 1, 64, W.F16),       # contexts barely longer than the drafts
]


@pytest.mark.parametrize("idx", range(len(TREE_CASES)), ids=lambda i: _case_id(TREE_CASES[i]))
def test_tree_verify_small(idx):
    B, q_max, ctx_max, H_kv, G, d, dt = TREE_CASES[idx]
    w = W.random_workload(500 + 13 * idx, B=B, q_max=q_max, ctx_max=ctx_max, H_kv=H_kv, G=G, d=d, dtype=dt,
                          kind="decode")
    tm = W.random_tree_masks(600 + idx, w.q_lens)
    out, _ = _tree_run(w, tm)
    ref, _, _ = oracle_step(w, oracle.lib(), tree_mask=tm)
    got = out.double().cpu().numpy()
    assert np.isfinite(got).all()
    err = np.abs(got - ref).max()
    assert err <= TOL[w.dtype], f"max abs err {err:.3e}"


# Every sequence with 16 or more rows per KV head (G x its new tokens): the calls run on the
# tcgen05 rows kernel (rows on the MMA's M side, 64-key tiles, S double-buffered in TMEM).
# (B, q_b of every sequence or None = random 1..8, ctx_max, H_kv, G, d, dtype, tree)
WIDE_CASES = [
    (5, 4, 700, 2, 4, 128, W.BF16, False),    # 16 rows, one warp's worth
    (4, 8, 2000, 1, 8, 64, W.F16, False),     # 64 rows, several splits
    (3, None, 300, 2, 16, 128, W.BF16, False),  # 16..128 rows (G = 16 is wide for any q_b)
    (4, 8, 1500, 2, 2, 128, W.F16, True),     # tree masks, 16 rows, splits
    (3, 6, 60, 2, 4, 64, W.BF16, True),       # tree masks, tiny contexts and partial pages
    (2, 8, 500, 1, 32, 128, W.BF16, False),   # 256 rows: two row groups of 128
    (3, 8, 400, 2, 3, 64, W.F16, False),      # G = 3: 24 rows per CTA
]


def _wide_id(c):
    return "B{}q{}c{}h{}g{}d{}{}{}".format(c[0], c[1] or "r", c[2], c[3], c[4], c[5],
                                          "bf16" if c[6] == W.BF16 else "f16", "tree" if c[7] else "")


@pytest.mark.parametrize("idx", range(len(WIDE_CASES)), ids=lambda i: _wide_id(WIDE_CASES[i]))
def test_decode_wide_rows_tensor_cores(idx):
    B, q, ctx_max, H_kv, G, d, dt, tree = WIDE_CASES[idx]
    g = torch.Generator().manual_seed(900 + idx)
    q_lens = [q if q else int(torch.randint(1, 9, (1,), generator=g)) for _ in range(B)]
    ctx_lens = [int(torch.randint(qb, ctx_max + 1, (1,), generator=g)) for qb in q_lens]
    w = W.build_workload(f"wide{idx}", q_lens=q_lens, ctx_lens=ctx_lens, H_q=H_kv * G, H_kv=H_kv, d=d, dtype=dt,
                         seed=910 + idx, calls=[W.AttnCall("decode", 0, B)], pool_extra=3)
    if tree:
        tm = W.random_tree_masks(920 + idx, w.q_lens)
        out, _ = _tree_run(w, tm)  # checks the status words
        ref, _, _ = oracle_step(w, oracle.lib(), tree_mask=tm)
        got = out.double().cpu().numpy()
        assert np.isfinite(got).all()
        err = np.abs(got - ref).max()
        assert err <= TOL[w.dtype], f"max abs err {err:.3e}"
    else:
        run_and_compare(w)


# Split-KV decode with a workspace that starts as garbage and an output that starts as NaN: every
# sequence has several KV splits, so the order, the partials and the merge all go through the
# workspace; a row the merge misses stays NaN, and a second call on the same (now used) workspace
# must give the same bytes.  (name, q_lens, ctx_lens, H_kv, G, d, dtype, tree)
MERGE_CASES = [
    ("mma_sync_many_splits", [1, 1, 1], [9000, 5000, 300], 2, 1, 128, W.F16, False),
    ("mma_sync_verify_rows", [3, 5], [4000, 7000], 2, 4, 128, W.BF16, False),
    ("tcgen05_rows", [8, 8], [6000, 2500], 2, 4, 128, W.BF16, False),
    ("tcgen05_tree", [8, 8, 8], [3000, 5000, 40], 1, 2, 64, W.F16, True),
]


@pytest.mark.parametrize("idx", range(len(MERGE_CASES)), ids=lambda i: MERGE_CASES[i][0])
def test_split_decode_with_a_dirty_workspace(idx):
    name, q_lens, ctx_lens, H_kv, G, d, dt, tree = MERGE_CASES[idx]
    w = W.build_workload(f"merge{idx}", q_lens=q_lens, ctx_lens=ctx_lens, H_q=H_kv * G, H_kv=H_kv, d=d, dtype=dt,
                         seed=1300 + idx, calls=[W.AttnCall("decode", 0, len(q_lens))], pool_extra=3)
    st = DeviceStep(w)
    st.copy_blocks()
    st.write()
    call = st.calls[0]
    nbytes = pa.decode_workspace_bytes(call.q.shape[0], w.B, w.H_q, w.H_kv, w.d, call.max_ctx)
    assert nbytes > pa.PA_STATUS_BYTES + 256  # the plan splits these contexts
    ws = torch.full((nbytes,), 0x5A, dtype=torch.uint8, device="cuda")
    tm = W.random_tree_masks(1310 + idx, w.q_lens) if tree else None
    outs = []
    for _ in range(2):
        out = torch.full_like(call.q, float("nan"))
        n0 = pa.launch_count()
        if tree:
            pa.paged_attn_decode_tree(call.q, st.key_cache, st.value_cache, call.bt, call.cu, call.ctx, tm.cuda(),
                                      call.max_ctx, w.scale, out=out, workspace=ws)
        else:
            pa.paged_attn_decode(call.q, st.key_cache, st.value_cache, call.bt, call.cu, call.ctx, call.max_ctx,
                                 w.scale, out=out, workspace=ws)
        assert pa.launch_count() - n0 == 3  # order, attention and merge kernels
        torch.cuda.synchronize()
        assert pa.read_status(ws) == 0
        outs.append(out)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    ref, _, _ = oracle_step(w, oracle.lib(), tree_mask=tm) if tree else oracle_step(w, oracle.lib())
    got = outs[0].double().cpu().numpy()
    assert np.isfinite(got).all()
    err = np.abs(got - ref).max()
    assert err <= TOL[w.dtype], f"max abs err {err:.3e}"


def test_tree_chain_mask_is_the_causal_verify():
    # the chain mask takes exactly the decisions of the causal rule: the same bits out
    w = W.random_workload(71, B=5, q_max=8, ctx_max=900, H_kv=2, G=4, d=128, dtype=W.BF16, kind="decode")
    st = DeviceStep(w)
    causal = st.run().clone()
    torch.cuda.synchronize()
    tree, _ = _tree_run(w, W.chain_masks(w.q_lens))
    assert torch.equal(causal.view(torch.int16), tree.view(torch.int16))


def test_tree_verify_full_size_sampled():
    # the benchmark's tree-verify workload (64 x 8 drafts, contexts U[512, 4096], 32/8 heads)
    w = W.tree_verify()
    tm = W.random_tree_masks(34_105, w.q_lens)
    out, _ = _tree_run(w, tm)
    rows = sample_rows(w, 300, seed=5)
    ref, _, _ = oracle_step(w, oracle.lib(), rows=rows, tree_mask=tm)
    got = out.double().cpu().numpy().reshape(w.T * w.H_q, w.d)[rows]
    assert np.isfinite(got).all()
    err = np.abs(got - ref).max()
    assert err <= TOL[w.dtype], f"max abs err {err:.3e}"


def test_tree_verify_rejects_a_missing_mask():
    import ctypes

    w = W.random_workload(3, B=2, q_max=4, ctx_max=50, H_kv=1, G=2, d=64, dtype=W.F16, kind="decode")
    st = DeviceStep(w)
    call = st.calls[0]
    n0 = pa.launch_count()
    rc = pa.lib().pa_paged_attn_decode_tree(
        ctypes.c_void_p(call.out.data_ptr()), ctypes.c_void_p(call.q.data_ptr()),
        ctypes.c_void_p(st.key_cache.data_ptr()), ctypes.c_void_p(st.value_cache.data_ptr()), st.key_cache.shape[0],
        ctypes.c_void_p(call.bt.data_ptr()), call.bt.shape[1], ctypes.c_void_p(call.cu.data_ptr()),
        ctypes.c_void_p(call.ctx.data_ptr()), None, call.ctx.shape[0], call.max_ctx, call.q.shape[0], w.H_q, w.H_kv,
        w.d, w.scale, 0, ctypes.c_void_p(call.ws.data_ptr()), call.ws.numel(), None)
    assert rc == -1 and pa.launch_count() == n0


# ---- the five configurations ----------------------------------------------------------------

def test_config1_tiny_decode_all_rows():
    run_and_compare(W.config1())


def test_config2_13b_decode_sampled():
    w = W.config2()
    run_and_compare(w, rows=sample_rows(w, 512))


def test_config3_prefill_sampled():
    w = W.config3()
    run_and_compare(w, rows=sample_rows(w, 512))


def test_config4_gqa_shared_prefix_sampled():
    w = W.config4()
    run_and_compare(w, rows=sample_rows(w, 256))


def test_config5_mixed_step_sampled():
    w = W.config5()
    run_and_compare(w, rows=sample_rows(w, 1024))


# ---- edge cases and device-side error reporting -------------------------------------------------

def test_empty_batch_launches_nothing():
    dev = "cuda"
    q = torch.empty((0, 4, 64), dtype=torch.float16, device=dev)
    kc = torch.zeros((2, 4, 16, 64), dtype=torch.float16, device=dev)
    n0 = pa.launch_count()
    out = pa.paged_attn_decode(q, kc, kc, torch.zeros((0, 1), dtype=torch.int32, device=dev),
                               torch.zeros(1, dtype=torch.int32, device=dev),
                               torch.zeros(0, dtype=torch.int32, device=dev), 0, 0.125)
    assert out.shape == (0, 4, 64) and pa.launch_count() == n0
    assert pa.read_status(pa.paged_attn_decode.last_workspace) == 0


def test_bad_block_id_is_reported_not_faulted():
    w = W.random_workload(5, B=2, q_max=1, ctx_max=40, H_kv=2, G=1, d=64, dtype=W.F16, kind="decode")
    w.block_tables[1, 0] = w.num_blocks + 3  # out of the pool
    st = DeviceStep(w)
    st.run()
    torch.cuda.synchronize()
    assert st.statuses()[1] == -7  # PA_ERR_BOUNDS
    # sequence 0 is untouched by the bad entry and still exact
    ref, _, _ = oracle_step(W.random_workload(5, B=2, q_max=1, ctx_max=40, H_kv=2, G=1, d=64, dtype=W.F16,
                                              kind="decode"), oracle.lib())
    got = st.out[:1].double().cpu().numpy()
    assert np.abs(got - ref[:1]).max() <= TOL[torch.float16]


def test_bad_slot_is_reported_and_skipped():
    w = W.random_workload(6, B=2, q_max=2, ctx_max=30, H_kv=2, G=1, d=64, dtype=W.F16, kind="decode")
    st = DeviceStep(w)
    before = st.key_cache.clone()
    bad = st.slot_mapping.clone()
    bad[:] = -1
    bad[0] = w.num_blocks * 16 + 5
    pa.kv_cache_write(st.k_new, st.v_new, bad, st.key_cache, st.value_cache, status=st.status)
    assert pa.read_status(st.status) == -7
    assert torch.equal(before.view(torch.int16), st.key_cache.view(torch.int16))


def test_inconsistent_sequence_is_reported():
    w = W.random_workload(7, B=3, q_max=2, ctx_max=30, H_kv=1, G=2, d=128, dtype=W.BF16, kind="decode")
    st = DeviceStep(w)
    st.calls[0].ctx[1] = 0  # ctx < q_len
    st.run()
    torch.cuda.synchronize()
    assert st.statuses()[1] == -8  # PA_ERR_SEQ


def test_bounded_wait_runs_out_and_reports_timeout():
    # the failure path every kernel shares: a wait on a barrier that nothing completes gives up
    # after its limit, records PA_ERR_TIMEOUT (-6) in the status word and returns; the first error
    # sticks, and the context stays usable (a decode right after is correct)
    import time

    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    pa.selftest_wait_timeout(status, 2_000_000)
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert pa.read_status(status) == -6
    status.fill_(-7)
    pa.selftest_wait_timeout(status, 1_000_000)
    assert pa.read_status(status) == -7
    w = W.random_workload(3, B=2, q_max=1, ctx_max=50, H_kv=1, G=2, d=64, dtype=W.F16, kind="decode")
    run_and_compare(w)


_CANARY = 0x7BAD  # an int16 pattern no kernel writes (a large finite fp16 / bf16 value)


def _padded(like, pad=4096):
    """(buffer with `pad` canary elements on each side, a view shaped like `like` inside it)."""
    n = like.numel()
    buf = torch.full((n + 2 * pad,), _CANARY, dtype=torch.int16, device=like.device)
    return buf, buf[pad : pad + n].view(like.dtype).view(like.shape)


def _canaries_intact(buf, n, pad=4096):
    return bool((buf[:pad] == _CANARY).all()) and bool((buf[pad + n :] == _CANARY).all())


def test_outputs_and_workspaces_stay_inside_their_buffers():
    # canary padding around every output and workspace (the pool's compute-sanitizer is closed):
    # decode, prefill, the FP8 decode and the shared-prefix decode write only inside them
    w = W.shared_prefix_batch(seed=90, B=6, n_groups=2, prefix_tokens=64, suffix=(1, 300), q_max=3, H_q=8,
                              H_kv=2, d=128, dtype=W.BF16)
    st = DeviceStep(w)
    st.copy_blocks()
    st.write()
    call = st.calls[0]
    n = call.out.numel()

    def ws_padded(nbytes, pad=4096):
        buf = torch.full((nbytes + 2 * pad,), 0x5A, dtype=torch.uint8, device="cuda")
        return buf, buf[pad : pad + nbytes]

    def ws_intact(buf, nbytes, pad=4096):
        return bool((buf[:pad] == 0x5A).all()) and bool((buf[pad + nbytes :] == 0x5A).all())

    # decode
    ob, out = _padded(call.out)
    wb, ws = ws_padded(call.ws.numel())
    pa.paged_attn_decode(call.q, st.key_cache, st.value_cache, call.bt, call.cu, call.ctx, call.max_ctx, w.scale,
                         out=out, workspace=ws)
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0 and _canaries_intact(ob, n) and ws_intact(wb, call.ws.numel())
    # shared-prefix decode
    starts, P = w.notes["group_start"], w.notes["prefix_blocks"]
    gs = torch.tensor(starts, dtype=torch.int32, device="cuda")
    pb = torch.tensor(P, dtype=torch.int32, device="cuda")
    max_gt = max(sum(w.q_lens[starts[v] : starts[v + 1]]) for v in range(len(P)))
    nbytes = pa.shared_prefix_workspace_bytes(w.T, w.B, w.H_q, w.H_kv, w.d, call.max_ctx, len(P), max(P), max_gt)
    ob, out = _padded(call.out)
    wb, ws = ws_padded(nbytes)
    pa.paged_attn_decode_shared_prefix(call.q, st.key_cache, st.value_cache, call.bt, call.cu, call.ctx, gs, pb,
                                       call.max_ctx, max(P), max_gt, w.scale, out=out, workspace=ws)
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0 and _canaries_intact(ob, n) and ws_intact(wb, nbytes)
    # FP8 decode over the same keys
    kc8, vc8, ks, vs = _fp8_device_cache(w)
    ob, out = _padded(call.out)
    wb, ws = ws_padded(call.ws.numel())
    pa.paged_attn_decode_fp8(call.q, kc8, vc8, ks, vs, call.bt, call.cu, call.ctx, call.max_ctx, w.scale, out=out,
                             workspace=ws)
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0 and _canaries_intact(ob, n) and ws_intact(wb, call.ws.numel())
    # prefill (chunks with earlier context)
    wp = W.random_workload(91, B=3, q_max=150, ctx_max=300, H_kv=2, G=4, d=128, dtype=W.BF16, kind="prefill")
    sp = DeviceStep(wp)
    sp.write()
    pc = sp.calls[0]
    ob, out = _padded(pc.out)
    wb, ws = ws_padded(pc.ws.numel())
    pa.paged_attn_prefill(pc.q, sp.key_cache, sp.value_cache, pc.bt, pc.cu, pc.ctx, pc.max_q_len, pc.max_ctx,
                          wp.scale, out=out, workspace=ws)
    torch.cuda.synchronize()
    assert pa.read_status(ws) == 0 and _canaries_intact(ob, pc.out.numel()) and ws_intact(wb, pc.ws.numel())


def test_block_copy_bitexact_random():
    g = torch.Generator().manual_seed(3)
    NB, H, d = 40, 4, 128
    kc = torch.randn((NB, H, 16, d), generator=g).bfloat16()
    vc = torch.randn((NB, H, 16, d), generator=g).bfloat16()
    pairs = torch.tensor([[3, 10], [3, 11], [17, 2], [39, 0]], dtype=torch.int32)
    k16, v16 = _u16(kc).copy(), _u16(vc).copy()
    assert oracle.kv_block_copy(k16, v16, pairs) == 0
    kd, vd = kc.cuda(), vc.cuda()
    pa.kv_block_copy(kd, vd, pairs.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(_u16(kd), k16) and np.array_equal(_u16(vd), v16)


def _pool(n, H, d, dtype):
    return torch.zeros((n, H, 16, d), dtype=dtype).pin_memory()


def test_block_swap_bitexact_round_trip():
    # swap a request's blocks out to a pinned host pool, reuse the device blocks, swap it back in
    # elsewhere: both directions byte for byte as the oracle (caches hold NaN outside contexts too)
    g = torch.Generator().manual_seed(5)
    NB, HB, H, d = 48, 20, 8, 128
    kc = torch.randn((NB, H, 16, d), generator=g).bfloat16()
    vc = torch.randn((NB, H, 16, d), generator=g).bfloat16()
    kc[5, :, 9:] = float("nan")
    hk, hv = _pool(HB, H, d, torch.bfloat16), _pool(HB, H, d, torch.bfloat16)
    k16, v16 = _u16(kc).copy(), _u16(vc).copy()
    hk16, hv16 = np.zeros((HB, H, 16, d), np.uint16), np.zeros((HB, H, 16, d), np.uint16)
    out_pairs = torch.tensor([[3, 0], [17, 5], [40, 19], [5, 7]], dtype=torch.int32)
    in_pairs = torch.tensor([[10, 0], [11, 5], [12, 19], [47, 7]], dtype=torch.int32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kd, vd = kc.cuda(), vc.cuda()
    assert oracle.kv_block_swap(k16, v16, hk16, hv16, out_pairs, to_host=True) == 0
    pa.kv_block_swap(kd, vd, hk, hv, out_pairs.cuda(), to_host=True, status=status)
    torch.cuda.synchronize()
    assert np.array_equal(_u16(hk), hk16) and np.array_equal(_u16(hv), hv16)
    assert oracle.kv_block_swap(k16, v16, hk16, hv16, in_pairs, to_host=False) == 0
    pa.kv_block_swap(kd, vd, hk, hv, in_pairs.cuda(), to_host=False, status=status)
    torch.cuda.synchronize()
    assert np.array_equal(_u16(kd), k16) and np.array_equal(_u16(vd), v16)
    assert pa.read_status(status) == 0


def test_block_swap_bad_ids_are_reported_and_skipped():
    NB, HB, H, d = 6, 3, 2, 64
    kd = torch.randn((NB, H, 16, d), device="cuda").half()
    vd = torch.randn((NB, H, 16, d), device="cuda").half()
    hk, hv = _pool(HB, H, d, torch.float16), _pool(HB, H, d, torch.float16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pairs = torch.tensor([[NB, 0], [1, HB], [2, 1]], dtype=torch.int32, device="cuda")
    pa.kv_block_swap(kd, vd, hk, hv, pairs, to_host=True, status=status)
    torch.cuda.synchronize()
    assert pa.read_status(status) == -7  # PA_ERR_BOUNDS
    assert torch.equal(hk[1], kd[2].cpu()) and torch.equal(hv[1], vd[2].cpu())
    assert not hk[0].any() and not hk[2].any()


def test_block_swap_refuses_pageable_host_memory():
    import ctypes

    NB, HB, H, d = 4, 2, 2, 64
    kd = torch.zeros((NB, H, 16, d), device="cuda").half()
    host = torch.zeros((HB, H, 16, d)).half()  # pageable
    pairs = torch.tensor([[0, 0]], dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        pa.kv_block_swap(kd, kd.clone(), host, host.clone(), pairs, to_host=True)
    n0 = pa.launch_count()
    rc = pa.lib().pa_kv_block_swap(ctypes.c_void_p(kd.data_ptr()), ctypes.c_void_p(kd.data_ptr()), NB,
                                   ctypes.c_void_p(host.data_ptr()), ctypes.c_void_p(host.data_ptr()), HB, H, d, 0,
                                   ctypes.c_void_p(pairs.data_ptr()), 1, 0, None, None)
    assert rc == -1 and pa.launch_count() == n0


def test_interleaved_calls_on_one_stream_give_each_call_its_result():
    # Every kernel of the library is launched as a programmatic dependent of the kernel before it
    # and waits for it before touching memory.  Calls of two workloads (block copies, cache writes,
    # a decode with several KV splits, a chunked prefill) issued back to back on one stream with no
    # host synchronisation in between must each give their own result.
    wa = W.random_workload(31, B=4, q_max=3, ctx_max=3000, H_kv=2, G=4, d=128, dtype=W.BF16, kind="decode")
    wb = W.random_workload(32, B=3, q_max=150, ctx_max=400, H_kv=2, G=4, d=128, dtype=W.BF16, kind="prefill")
    sa, sb = DeviceStep(wa), DeviceStep(wb)
    torch.cuda.synchronize()
    for _ in range(3):
        sa.run()
        sb.run()
    out_a, out_b = sa.out.clone(), sb.out.clone()
    torch.cuda.synchronize()
    for st, w, out in ((sa, wa, out_a), (sb, wb, out_b)):
        assert st.statuses() == [0] * (1 + len(st.calls)), st.statuses()
        ref, _, _ = oracle_step(w, oracle.lib())
        got = out.double().cpu().numpy()
        assert np.isfinite(got).all()
        err = np.abs(got - ref).max()
        assert err <= TOL[w.dtype], f"{w.name}: max abs err {err:.3e}"


def test_repeat_runs_identical():
    w = W.random_workload(8, B=4, q_max=3, ctx_max=600, H_kv=2, G=4, d=128, dtype=W.BF16, kind="decode")
    st = DeviceStep(w)
    a = st.run().clone()
    b = st.run().clone()
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def _ws_order(ws: torch.Tensor, n: int) -> np.ndarray:
    """The scheduling order the call wrote after the status area of its workspace."""
    return ws[pa.PA_STATUS_BYTES:pa.PA_STATUS_BYTES + 4 * n].cpu().view(torch.int32).numpy()


def test_decode_schedules_longest_sequences_first():
    # decode writes the sequences in non-increasing page count: a permutation of 0..B-1
    w = W.config2(B=48)
    st = DeviceStep(w)
    st.run()
    torch.cuda.synchronize()
    call = st.calls[0]
    B = call.ctx.shape[0]
    order = _ws_order(call.ws, B)
    assert sorted(order.tolist()) == list(range(B))
    pages = np.minimum((call.ctx.cpu().numpy() + 15) // 16, 4095)
    assert np.all(np.diff(pages[order]) <= 0)


def test_prefill_schedules_heaviest_work_first():
    # short prompts take the queue schedule: the (query-tile pair, sequence) entries by
    # non-increasing K/V tiles
    w = W.config3()
    st = DeviceStep(w)
    st.run()
    torch.cuda.synchronize()
    call = next(c for c in st.calls if c.kind == "prefill")
    assert not S.takes_split(w.B, call.max_q_len, w.H_kv, w.H_q // w.H_kv, _n_ctas())
    q = (call.cu[1:] - call.cu[:-1]).cpu().numpy()
    ctx = call.ctx.cpu().numpy()
    B = q.shape[0]
    tok = 128 // (w.H_q // w.H_kv)
    n_pairs = ((call.max_q_len + tok - 1) // tok + 1) // 2
    order = _ws_order(call.ws, n_pairs * B)
    assert sorted(order.tolist()) == list(range(n_pairs * B))

    def tiles(e):
        pair, b = e // B, e % B
        t0 = 2 * pair * tok
        if t0 >= q[b]:
            return 0
        last = min(q[b], t0 + 2 * tok) - 1
        return (ctx[b] - q[b] + last) // 128 + 1

    keys = np.array([min(tiles(int(e)), 4095) for e in order])
    assert np.all(np.diff(keys) <= 0)
    assert keys[0] == max(tiles(e) for e in range(n_pairs * B))


# ---- shared-prefix decode -------------------------------------------------------------------

def _groups_of(w):
    """(group_start, prefix_blocks, max_prefix_blocks, max_group_tokens) from share_prefixes' notes."""
    starts, P = w.notes["group_start"], w.notes["prefix_blocks"]
    tokens = [sum(w.q_lens[starts[v] : starts[v + 1]]) for v in range(len(P))]
    return (torch.tensor(starts, dtype=torch.int32, device="cuda"), torch.tensor(P, dtype=torch.int32, device="cuda"),
            max(P), max(tokens))


def _shared_run(w, groups=None):
    """Block copies and cache write, then the shared-prefix decode; returns (output, status word)."""
    gs, pb, max_pb, max_gt = groups if groups is not None else _groups_of(w)
    st = DeviceStep(w)
    st.copy_blocks()
    st.write()
    call = st.calls[0]
    n_ws = pa.shared_prefix_workspace_bytes(call.q.shape[0], w.B, w.H_q, w.H_kv, w.d, call.max_ctx, pb.shape[0],
                                            max_pb, max_gt)
    ws = torch.zeros(n_ws, dtype=torch.uint8, device="cuda")
    out = pa.paged_attn_decode_shared_prefix(call.q, st.key_cache, st.value_cache, call.bt, call.cu, call.ctx, gs, pb,
                                             call.max_ctx, max_pb, max_gt, w.scale, out=call.out, workspace=ws)
    torch.cuda.synchronize()
    assert st.statuses()[0] == 0
    return out, pa.read_status(ws)


# (B, n_groups, prefix tokens, own suffix range, q_max, H_q, H_kv, d, dtype)
SHARED_CASES = [
    (8, 3, 64, (1, 40), 3, 8, 2, 64, W.F16),          # ragged verify rows, GQA 4
    (6, 2, 256, (16, 300), 1, 4, 4, 128, W.BF16),     # MHA decode
    (16, 1, 2048, (1, 100), 2, 32, 8, 128, W.BF16),   # one group, long prefix (several prefix splits), 2 row groups
    (20, 4, 512, (1, 1000), 1, 16, 2, 128, W.F16),    # long own keys: several splits of their own
    (3, 3, 32, (5, 9), 4, 2, 1, 64, W.BF16),          # one sequence per group
]


def _shared_id(c):
    return "B{}g{}p{}q{}h{}/{}d{}{}".format(c[0], c[1], c[2], c[4], c[5], c[6], c[7], "bf16" if c[8] == W.BF16 else "f16")


@pytest.mark.parametrize("idx", range(len(SHARED_CASES)), ids=lambda i: _shared_id(SHARED_CASES[i]))
def test_shared_prefix_small(idx):
    B, n_groups, pre, suf, q_max, H_q, H_kv, d, dt = SHARED_CASES[idx]
    w = W.shared_prefix_batch(seed=700 + idx, B=B, n_groups=n_groups, prefix_tokens=pre, suffix=suf, q_max=q_max,
                              H_q=H_q, H_kv=H_kv, d=d, dtype=dt)
    out, status = _shared_run(w)
    assert status == 0
    ref, _, _ = oracle_step(w, oracle.lib())
    got = out.double().cpu().numpy()
    assert np.isfinite(got).all()
    err = np.abs(got - ref).max()
    assert err <= TOL[w.dtype], f"max abs err {err:.3e}"


def test_shared_prefix_falls_back_where_tables_differ():
    # one group over sequences that share nothing (each owns its 4 prefix blocks): every member's
    # table differs from the leader's, so each is computed over its own table (same result, status OK)
    w = W.shared_prefix_batch(seed=71, B=5, n_groups=5, prefix_tokens=64, suffix=(1, 60), q_max=2, H_q=4, H_kv=2,
                              d=64, dtype=W.F16)
    groups = (torch.tensor([0, w.B], dtype=torch.int32, device="cuda"),
              torch.tensor([4], dtype=torch.int32, device="cuda"), 4, w.T)
    out, status = _shared_run(w, groups)
    assert status == 0
    ref, _, _ = oracle_step(w, oracle.lib())
    assert np.abs(out.double().cpu().numpy() - ref).max() <= TOL[w.dtype]


def test_shared_prefix_rejects_malformed_groups_and_stays_correct():
    w = W.shared_prefix_batch(seed=72, B=6, n_groups=2, prefix_tokens=64, suffix=(4, 50), q_max=2, H_q=4, H_kv=2,
                              d=64, dtype=W.BF16)
    _, _, max_pb, max_gt = _groups_of(w)
    bad = (torch.tensor([0, 4, 2, 6], dtype=torch.int32, device="cuda"),  # not increasing
           torch.tensor([4, 4, 4], dtype=torch.int32, device="cuda"), max_pb, max_gt)
    out, status = _shared_run(w, bad)
    assert status == -1  # PA_ERR_ARG: every sequence computed alone
    ref, _, _ = oracle_step(w, oracle.lib())
    assert np.abs(out.double().cpu().numpy() - ref).max() <= TOL[w.dtype]


def test_shared_prefix_4_prompts_13b_layer_sampled():
    # 64 requests in 4 groups sharing a 4096-token prompt, own suffixes U[16, 512]; 40/40 heads, d 128
    w = W.shared_prefix_batch()
    out, status = _shared_run(w)
    assert status == 0
    rows = sample_rows(w, 256, seed=8)
    ref, _, _ = oracle_step(w, oracle.lib(), rows=rows)
    got = out.double().cpu().numpy().reshape(w.T * w.H_q, w.d)[rows]
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= TOL[w.dtype]


def test_shared_prefix_on_the_gqa_shared_prefix_config_sampled():
    # the long-context GQA decode (16 sequences sharing 128 blocks = 2048 tokens, one block copy)
    w = W.config4()
    n_shared = w.notes["shared_tokens"] // 16
    groups = (torch.tensor([0, w.B], dtype=torch.int32, device="cuda"),
              torch.tensor([n_shared], dtype=torch.int32, device="cuda"), n_shared, w.T)
    out, status = _shared_run(w, groups)
    assert status == 0
    rows = sample_rows(w, 256, seed=9)
    ref, _, _ = oracle_step(w, oracle.lib(), rows=rows)
    got = out.double().cpu().numpy().reshape(w.T * w.H_q, w.d)[rows]
    assert np.abs(got - ref).max() <= TOL[w.dtype]
