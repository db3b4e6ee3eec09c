"""One step of the hot path on the GPU, through the public binding.

A step, in order: ``kv_block_copy`` (copy-on-write pairs, when the workload
has any), ``kv_cache_write`` of the step's new K/V, then each attention call
of the workload (``paged_attn_prefill`` for prompt chunks,
``paged_attn_decode`` for decode / verify rows).  ``DeviceStep`` uploads a
``workloads.Workload`` once and preallocates outputs and workspaces, so
``run()`` only enqueues library kernels.  Re-running a step rewrites the same
bytes, so it can be timed repeatedly.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import torch

from . import (
    decode_workspace_bytes,
    kv_block_copy,
    kv_cache_write,
    paged_attn_decode,
    paged_attn_prefill,
    prefill_workspace_bytes,
)
from .workloads import Workload


@dataclass
class _Call:
    kind: str
    t0: int
    t1: int
    q: torch.Tensor
    out: torch.Tensor
    cu: torch.Tensor
    ctx: torch.Tensor
    bt: torch.Tensor
    max_q_len: int
    max_ctx: int
    ws: torch.Tensor
    seq_lo: int
    seq_hi: int


class DeviceStep:
    def __init__(self, w: Workload, device="cuda", caches=None):
        self.w = w
        self.device = torch.device(device)
        dev = self.device
        if caches is None:
            self.key_cache = w.key_cache.to(dev)
            self.value_cache = w.value_cache.to(dev)
        else:
            self.key_cache, self.value_cache = caches
        self.q = w.q.to(dev)
        self.out = torch.empty_like(self.q)
        self.k_new = w.k_new.to(dev)
        self.v_new = w.v_new.to(dev)
        self.slot_mapping = w.slot_mapping.to(dev)
        self.pairs = w.copy_pairs.to(dev) if w.copy_pairs is not None else None
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.calls: List[_Call] = []
        for c in w.calls:
            a = w.call_args(c)
            cu = a["cu_seqlens_q"].to(dev)
            ctx = a["context_lens"].to(dev)
            bt = a["block_tables"].to(dev)
            q = self.q[a["t0"] : a["t1"]]
            out = self.out[a["t0"] : a["t1"]]
            T = a["t1"] - a["t0"]
            if c.kind == "decode":
                nbytes = decode_workspace_bytes(T, a["B"], w.H_q, w.H_kv, w.d, a["max_ctx"])
            else:
                nbytes = prefill_workspace_bytes(a["B"], w.H_q, w.H_kv, w.d, a["max_q_len"])
            ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
            self.calls.append(
                _Call(c.kind, a["t0"], a["t1"], q, out, cu, ctx, bt, a["max_q_len"], a["max_ctx"], ws, c.seq_lo,
                      c.seq_hi)
            )

    def copy_blocks(self):
        if self.pairs is not None and self.pairs.shape[0] > 0:
            kv_block_copy(self.key_cache, self.value_cache, self.pairs, status=self.status)

    def write(self):
        kv_cache_write(self.k_new, self.v_new, self.slot_mapping, self.key_cache, self.value_cache,
                       status=self.status)

    def attend(self, call: _Call):
        if call.kind == "decode":
            paged_attn_decode(call.q, self.key_cache, self.value_cache, call.bt, call.cu, call.ctx, call.max_ctx,
                              self.w.scale, out=call.out, workspace=call.ws)
        else:
            paged_attn_prefill(call.q, self.key_cache, self.value_cache, call.bt, call.cu, call.ctx,
                               call.max_q_len, call.max_ctx, self.w.scale, out=call.out, workspace=call.ws)

    def run(self):
        self.copy_blocks()
        self.write()
        for c in self.calls:
            self.attend(c)
        return self.out

    def statuses(self) -> List[int]:
        """Status words of the write/copy calls and of every attention call (synchronises)."""
        from . import read_status

        return [read_status(self.status)] + [read_status(c.ws) for c in self.calls]


# ---- algorithmic work of a step (the roofline numerators) -------------------------------------

def attn_bytes(w: Workload, call_kind: Optional[str] = None) -> int:
    """Algorithmic HBM bytes of the attention calls: each sequence's ctx_b keys of K and V
    (shared physical blocks counted once), Q read once, O written once, the block-table
    entries and context lengths read.  Padding rows of a last partial block and the
    split-KV workspace are implementation traffic and are not counted."""
    esz = 2
    total = 0
    shared_tokens = 0
    if w.shared_blocks:
        shared_tokens = w.shared_blocks * 16
    for c in w.calls:
        if call_kind and c.kind != call_kind:
            continue
        for b in range(c.seq_lo, c.seq_hi):
            ctx = w.ctx_lens[b]
            total += ctx * 2 * w.H_kv * w.d * esz  # K and V rows
            total += w.q_lens[b] * w.H_q * w.d * esz * 2  # Q in, O out
            total += ((ctx + 15) // 16) * 4 + 4 + 4  # table entries, ctx, cu
        if "group_start" in w.notes:  # groups of sequences sharing their first prefix_blocks[v] blocks
            st, P = w.notes["group_start"], w.notes["prefix_blocks"]
            for v in range(len(P)):
                n = len(range(max(st[v], c.seq_lo), min(st[v + 1], c.seq_hi)))
                if n > 1:
                    total -= (n - 1) * P[v] * 16 * 2 * w.H_kv * w.d * esz
        elif shared_tokens:
            n = c.seq_hi - c.seq_lo
            total -= (n - 1) * shared_tokens * 2 * w.H_kv * w.d * esz
    return total


def attn_flops(w: Workload, call_kind: Optional[str] = None) -> int:
    """MMA FLOP of the unmasked (query, key) pairs only: 4 d per pair (Q K^T and P V)."""
    total = 0
    for c in w.calls:
        if call_kind and c.kind != call_kind:
            continue
        for b in range(c.seq_lo, c.seq_hi):
            qb, ctx = w.q_lens[b], w.ctx_lens[b]
            pairs = sum(ctx - qb + i + 1 for i in range(qb))
            total += pairs * w.H_q * 4 * w.d
    return total


def write_bytes(w: Workload) -> int:
    """kv_cache_write: each new token's K and V rows read once and written once, plus its slot."""
    T = w.k_new.shape[0]
    return T * (2 * w.H_kv * w.d * 2 * 2 + 4)


def copy_bytes(w: Workload) -> int:
    if w.copy_pairs is None:
        return 0
    n = w.copy_pairs.shape[0]
    return n * 2 * (w.H_kv * 16 * w.d * 2) * 2 + n * 8
