"""Benchmark of the paged-KV attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline workload (N = 1): the LLaMA-2-13B-shaped decode layer -- 64
sequences, one new token each, 40/40 heads, d 128, fp16, contexts uniform in
[128, 4096], 16-token blocks shuffled over the pool.  One step = the hot path
of a decode iteration: ``kv_cache_write`` of the 64 new K/V rows, then
``paged_attn_decode`` (split-KV kernel + log-sum-exp merge kernel).  ``value``
is the step's algorithmic HBM bytes (every context key's K and V, Q, O, table
entries, the new rows written) over the device time of the step: GB/s.

With N > 1 (torchrun, one process per GPU) every rank runs its own batch of 64
sequences (independent seed): the sequences are independent, so there is no
data-path collective ("weak" scaling); the only collectives are the barriers
and the max-over-ranks of the elapsed time.

The same JSON line carries:
  roofline      decode call (split kernel + merge) vs the measured HBM copy peak
  prefill       causal varlen prefill (8 prompts U[256,2048], 40/40 heads, bf16):
                TFLOP/s of exact causal pairs vs the measured bf16 peak
  legs          the GQA shared-prefix decode step, the mixed continuous-batching step, the
                last 512-token chunk of a 32 K-token prompt (chunked prefill over a long context,
                tensor + HBM roofline), the
                tree-attention verify of speculative drafts (HBM roofline), the FP8 (E4M3) KV
                cache on the 13B decode layer (HBM roofline, speed-up over 16 bits), and
                the preemption swap of KV blocks to a pinned host pool and back (GB/s against
                a plain pinned cudaMemcpyAsync of the same bytes)
  e2e           the same metric with host buffers: every step's inputs go H2D from one pinned
                buffer and its output comes back D2H, all inside the timed region; the copies
                run on a second stream, overlapping the neighbouring steps' kernels (double-
                buffered device inputs and outputs), as a serving loop would
  cpu_baseline  the fp64 CPU oracle, timed on a bounded sample of the same workload
  clocks        SM clock / throttle reasons sampled through NVML during the timed region

``--impl reference`` times the fp64 CPU oracle (the only reference this
method has) on the host cores on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged decode attn HBM GB/s & prefill attn TFLOPS, as % of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# ncu DRAM bytes (read + written) / algorithmic bytes of the 16-bit decode kernel, captured on the
# 13B-shaped decode layer with 16 sequences: (698.58 + 5.11) MB / 696.53 MB
TRAFFIC_RATIO_DECODE_13B = (698.58 + 5.11) / 696.53
HEADLINE = "LLaMA-2-13B-shaped decode layer: B 64, q_len 1, 40/40 heads, d 128, fp16, ctx U[128,4096], block 16"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ---- distributed plumbing (also exercised on CPU with gloo by the tests) --------------------------

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def shard_seed(base: int, rank: int) -> int:
    """Each rank draws its own independent batch of sequences."""
    return base + 1000 * rank


def reduce_max(x: float, device) -> float:
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(x: float, device) -> float:
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier():
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ---- clocks -------------------------------------------------------------------------------------------

class ClockSampler:
    """Samples SM clock and throttle reasons with NVML in a thread (every ~2 ms)."""

    REASONS = {
        "hw_slowdown": 0x8,
        "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80,
        "sw_power_cap": 0x4,
    }

    def __init__(self, device_index: int):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml

            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = device_index
            if vis:
                try:
                    idx = int(vis.split(",")[device_index])
                except ValueError:
                    idx = device_index
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: clocks are reported as unavailable
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or getattr(
                    nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
                r = get(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.nv:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
            time.sleep(0.005)
        return self

    def __exit__(self, *exc):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.nv or not self.samples:
            return None
        s = sorted(self.samples)
        return {"sm_mhz": s[len(s) // 2], "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(s), "source": "NVML"}


# ---- timing helpers ----------------------------------------------------------------------------------

def pctl(xs, q):
    """q-th percentile (0..100) of a list, linear interpolation between order statistics."""
    ys = sorted(xs)
    if not ys:
        return None
    pos = (len(ys) - 1) * q / 100.0
    lo = int(math.floor(pos))
    hi = min(lo + 1, len(ys) - 1)
    return ys[lo] + (ys[hi] - ys[lo]) * (pos - lo)


def stats_ms(xs):
    """mean / p10 / p50 / p90 of per-step durations (ms)."""
    return {"mean": round(sum(xs) / len(xs), 5), "p10": round(pctl(xs, 10), 5), "p50": round(pctl(xs, 50), 5),
            "p90": round(pctl(xs, 90), 5), "n": len(xs)}


def time_calls(fn_list, steps, stream, per_step=None):
    """Run `steps` iterations of the step; per-call CUDA-event durations on `stream`.

    Returns (total_ms, [avg_ms per call]) with the total bracketed by events; when `per_step` is a
    list, it receives, for every step, the list of that step's call durations."""
    import torch

    n = len(fn_list)
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
           for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for s in range(steps):
            for i, fn in enumerate(fn_list):
                evs[s][i][0].record(stream)
                fn()
                evs[s][i][1].record(stream)
        end.record(stream)
    end.synchronize()
    durs = [[evs[s][i][0].elapsed_time(evs[s][i][1]) for i in range(n)] for s in range(steps)]
    if per_step is not None:
        per_step.extend(durs)
    per = [sum(durs[s][i] for s in range(steps)) / steps for i in range(n)]
    return start.elapsed_time(end), per


def time_steps(fn_list, steps, stream):
    """Run `steps` iterations of the step between two CUDA events on `stream`; elapsed ms."""
    import torch

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(steps):
            for fn in fn_list:
                fn()
        end.record(stream)
    end.synchronize()
    return start.elapsed_time(end)


def bench_leg(w, steps, warmup, stream, device):
    """Time one workload's step (copy, write, attention calls) with per-call events."""
    import torch

    from paged_kv_attention_34_b200.step import DeviceStep

    with torch.cuda.stream(stream):
        st = DeviceStep(w, device=device)
    fns = []
    names = []
    if st.pairs is not None:
        fns.append(st.copy_blocks)
        names.append("kv_block_copy")
    fns.append(st.write)
    names.append("kv_cache_write")
    for c in st.calls:
        fns.append(lambda c=c: st.attend(c))
        names.append("paged_attn_" + c.kind)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            for fn in fns:
                fn()
    torch.cuda.synchronize()
    durs = []
    total, per = time_calls(fns, steps, stream, durs)
    stat = st.statuses()
    if any(stat):
        raise RuntimeError(f"{w.name}: device status {stat}")
    st.call_stats = {name: stats_ms([d[i] for d in durs]) for i, name in enumerate(names)}
    st.step_stats = stats_ms([sum(d) for d in durs])
    return st, dict(zip(names, per)), total / steps


# ---- our arm -------------------------------------------------------------------------------------------------

def run_ours(args):
    import torch
    import torch.distributed as dist

    import paged_kv_attention_34_b200 as pa
    from paged_kv_attention_34_b200 import workloads as W
    from paged_kv_attention_34_b200.step import DeviceStep, attn_bytes, attn_flops, copy_bytes, write_bytes

    rank, local_rank, world = dist_env()
    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
    pa.lib()
    peaks, peak_src = load_peaks()
    hbm_peak = float(peaks["hbm_gbs"])
    bf16_peak = float(peaks["bf16_tflops"])
    stream = torch.cuda.Stream(device=device)

    # ---- headline: 13B-shaped decode step ----
    w = W.config2(seed=shard_seed(34_002, rank), B=args.batch)
    with torch.cuda.stream(stream):
        st = DeviceStep(w, device=device)
    call = st.calls[0]
    fns = [st.write, lambda: st.attend(call)]
    step_bytes = attn_bytes(w) + write_bytes(w)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            for fn in fns:
                fn()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        # per-call durations (CUDA events around every call), then the timed steps themselves with
        # events only at the two ends, so the step time carries no per-call event overhead
        durs = []
        _, per = time_calls(fns, args.steps, stream, durs)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        n_launch0 = pa.launch_count()
        total_ms = time_steps(fns, args.steps, stream)
        n_launch = pa.launch_count() - n_launch0
    torch.cuda.synchronize()
    barrier()
    total_ms_max = reduce_max(total_ms, device)
    bytes_all = reduce_sum(float(step_bytes * args.steps), device)
    value = bytes_all / (total_ms_max * 1e-3) / 1e9
    status = st.statuses()
    if any(status):
        raise RuntimeError(f"device status {status}")
    decode_ms = per[1]
    decode_bytes = attn_bytes(w)
    achieved = decode_bytes / (decode_ms * 1e-3) / 1e9

    # ---- e2e through the public API with host buffers ----
    e2e = run_e2e(st, w, args, stream, device, step_bytes)

    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms_max / args.steps, 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16",
        "data": "synthetic: seeded N(0,1) fp16 Q/K/V, uniform context lengths, shuffled 16-token blocks (no dataset)",
        "config": {
            "workload": HEADLINE if args.batch == 64 else HEADLINE.replace("B 64", f"B {args.batch}"),
            "global_batch": args.batch * world,
            "seq_len": "context U[128,4096] (sum %d per rank 0)" % sum(w.ctx_lens),
            "parallelism": f"dp{world} (independent sequences per rank, no data-path collective)",
            "step": f"kv_cache_write({args.batch} new tokens) + paged_attn_decode (split kernel + merge)",
            "l2": "no flush: the KV read per step (%.2f GB) is larger than the 126 MB L2" % (attn_bytes(w) / 1e9),
        },
        "roofline": {
            "kernel": "paged_attn_decode (split-KV kernel + LSE merge kernel, timed together)",
            "bound": "hbm",
            "achieved": round(achieved, 1),
            "peak": hbm_peak,
            "peak_source": f"{peak_src} HBM copy bandwidth",
            "unit": "GB/s",
            "frac": round(achieved / hbm_peak, 4),
            "frac_of_nominal_8TBs": round(achieved / 8000.0, 4),
            # DRAM bytes read + written per launch of the decode kernel: an ncu capture of the same
            # kernel on this workload with 16 sequences measured 1.0092 x its algorithmic bytes (the
            # padding rows of last partial blocks); the same ratio applied to this run's algorithmic
            # bytes.  Only for the captured shape (fp16, 40/40 heads, contexts U[128, 4096]).
            "traffic": round(TRAFFIC_RATIO_DECODE_13B * decode_bytes) if w.name == "cfg2" else None,
            "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum, 16-sequence capture scaled",
            "bytes_per_launch": decode_bytes,
            "avg_launch_ms": round(decode_ms, 5),
        },
        "gpu_launches": n_launch,
        "e2e": e2e,
        "per_call_ms": {"kv_cache_write": round(per[0], 5), "paged_attn_decode": round(per[1], 5)},
        # per-step distributions from the pass with events around every call (the step time above
        # comes from the pass with events only at its ends)
        "step_ms_stats": stats_ms([sum(d) for d in durs]),
        "decode_ms_stats": stats_ms([d[1] for d in durs]),
    }
    clk_sum = clk.summary()
    result["clocks"] = clk_sum if clk_sum else {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                                                 "note": "NVML unavailable"}

    # ---- other legs (rank-local, reported for rank 0) ----
    if not args.no_legs:
        result["prefill"] = leg_prefill(args, stream, device, bf16_peak, peak_src, rank)
        result["legs"] = {
            "gqa_shared_prefix": leg_gqa(args, stream, device, hbm_peak, rank),
            "mixed_step": leg_mixed(args, stream, device, hbm_peak, bf16_peak, rank),
            "long_chunk_prefill": leg_long_chunk(args, stream, device, hbm_peak, bf16_peak, rank),
            "tree_verify": leg_tree(args, stream, device, hbm_peak, rank),
            "fp8_cache": leg_fp8(args, stream, device, hbm_peak, rank),
            "shared_prefix": leg_shared(args, stream, device, hbm_peak, rank),
            "block_swap": leg_swap(args, stream, device, rank),
        }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
        if not args.no_legs:
            result["cpu_baseline"]["per_config"] = cpu_baseline_configs(args.cpu_seconds / 2)
    del st
    if world > 1:
        barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def run_e2e(st, w, args, stream, device, step_bytes):
    """The step with host buffers: H2D of the step inputs (pinned), the calls, D2H of the output.

    The inputs of a step (Q, the new K/V rows, slot mapping, block table, context lengths,
    cu_seqlens) are staged in one pinned host buffer and sent with one copy into one of two device
    buffers, whose views the library calls take; the output goes to one of two device buffers and
    comes back with one copy.  The copies run on a copy stream ordered by events: step k's inputs
    land before its kernels start, step k+1's inputs are copied while step k computes, and step
    k's output is read back while step k+1 computes.  The timed region opens before the first
    input copy and closes after the last output copy.
    """
    import torch
    from paged_kv_attention_34_b200 import kv_cache_write, paged_attn_decode

    call = st.calls[0]
    parts = [("q", w.q), ("k_new", w.k_new), ("v_new", w.v_new), ("slot", w.slot_mapping),
             ("bt", call.bt.cpu()), ("ctx", call.ctx.cpu()), ("cu", call.cu.cpu())]
    offs, off = {}, 0
    for name, t in parts:
        offs[name] = off
        off += (t.numel() * t.element_size() + 255) // 256 * 256
    host_buf = torch.zeros(off, dtype=torch.uint8).pin_memory()
    for name, t in parts:
        n = t.numel() * t.element_size()
        host_buf[offs[name]:offs[name] + n].copy_(t.contiguous().view(-1).view(torch.uint8))
    dev_bufs = [torch.empty(off, dtype=torch.uint8, device=device) for _ in range(2)]
    views = []
    for db in dev_bufs:
        v = {}
        for name, t in parts:
            n = t.numel() * t.element_size()
            v[name] = db[offs[name]:offs[name] + n].view(t.dtype).view(t.shape)
        views.append(v)
    outs = [torch.empty_like(st.out) for _ in range(2)]
    out_host = torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory()
    h2d = off
    d2h = out_host.numel() * out_host.element_size()
    copy = torch.cuda.Stream(device)

    def run(n_steps):
        """n_steps pipelined steps; returns (start, end) events on the compute stream."""
        ev = torch.cuda.Event
        landed = [ev() for _ in range(n_steps)]     # inputs of step k are on the device
        computed = [ev() for _ in range(n_steps)]   # kernels of step k are done
        read = [ev() for _ in range(n_steps)]       # output of step k is on the host
        start, end = ev(enable_timing=True), ev(enable_timing=True)
        start.record(stream)
        copy.wait_event(start)

        def h2d_step(k):
            with torch.cuda.stream(copy):
                if k >= 2:
                    copy.wait_event(computed[k - 2])  # buffer k % 2 is free again
                dev_bufs[k % 2].copy_(host_buf, non_blocking=True)
                landed[k].record(copy)

        h2d_step(0)
        for k in range(n_steps):
            if k + 1 < n_steps:
                h2d_step(k + 1)
            with torch.cuda.stream(stream):
                stream.wait_event(landed[k])
                if k >= 2:
                    stream.wait_event(read[k - 2])  # output buffer k % 2 has been read back
                v = views[k % 2]
                kv_cache_write(v["k_new"], v["v_new"], v["slot"], st.key_cache, st.value_cache, status=st.status)
                paged_attn_decode(v["q"], st.key_cache, st.value_cache, v["bt"], v["cu"], v["ctx"], call.max_ctx,
                                  w.scale, out=outs[k % 2], workspace=call.ws)
                computed[k].record(stream)
            with torch.cuda.stream(copy):
                copy.wait_event(computed[k])
                out_host.copy_(outs[k % 2], non_blocking=True)
                read[k].record(copy)
        stream.wait_event(read[n_steps - 1])
        end.record(stream)
        return start, end

    def serial_step():
        # the same copies and calls one after the other on one stream, no overlap
        dev_bufs[0].copy_(host_buf, non_blocking=True)
        v = views[0]
        kv_cache_write(v["k_new"], v["v_new"], v["slot"], st.key_cache, st.value_cache, status=st.status)
        paged_attn_decode(v["q"], st.key_cache, st.value_cache, v["bt"], v["cu"], v["ctx"], call.max_ctx, w.scale,
                          out=outs[0], workspace=call.ws)
        out_host.copy_(outs[0], non_blocking=True)

    run(args.warmup)
    torch.cuda.synchronize()
    barrier()
    start, end = run(args.steps)
    end.synchronize()
    torch.cuda.synchronize()
    total_ms = reduce_max(start.elapsed_time(end), device)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            serial_step()
    torch.cuda.synchronize()
    barrier()
    serial_ms = reduce_max(time_steps([serial_step], args.steps, stream), device)
    bytes_all = reduce_sum(float(step_bytes * args.steps), device)
    return {"value": round(bytes_all / (total_ms * 1e-3) / 1e9, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(total_ms / args.steps, 6),
            "overlap": "step k+1's H2D and step k-1's D2H run on a copy stream during step k's kernels",
            "serial": {"value": round(bytes_all / (serial_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                       "ms_per_step": round(serial_ms / args.steps, 6),
                       "note": "the same copies and calls in series on one stream"}}


def leg_prefill(args, stream, device, bf16_peak, peak_src, rank):
    from paged_kv_attention_34_b200 import workloads as W
    from paged_kv_attention_34_b200.step import attn_flops, write_bytes

    w = W.config3(seed=shard_seed(34_003, rank))
    st, per, step_ms = bench_leg(w, max(args.steps, 5), args.warmup, stream, device)
    flops = attn_flops(w)
    ms = per["paged_attn_prefill"]
    tf = flops / (ms * 1e-3) / 1e12
    wb = write_bytes(w)
    return {
        "workload": W.CONFIG_NAMES[3],
        "metric": "prefill attn TFLOP/s (exact causal pairs, 4 d FLOP per pair)",
        "value": round(tf, 2),
        "unit": "TFLOP/s",
        "bound": "tensor",
        "peak": bf16_peak,
        "peak_source": f"{peak_src} cuBLAS bf16 burst",
        "frac": round(tf / bf16_peak, 4),
        "frac_of_nominal_2250": round(tf / 2250.0, 4),
        "flop_per_launch": flops,
        "avg_launch_ms": round(ms, 5),
        "kv_cache_write": {"GB/s": round(wb / (per["kv_cache_write"] * 1e-3) / 1e9, 1), "bytes": wb,
                           "avg_launch_ms": round(per["kv_cache_write"], 5)},
        "tokens_per_s": round(w.T / (step_ms * 1e-3), 1),
        "prefill_ms_stats": st.call_stats["paged_attn_prefill"],
    }


LONG_CHUNK = "long-context chunked prefill: the last 512-token chunk of a 32 K-token prompt, 32/8 heads, d 128, bf16"


def leg_long_chunk(args, stream, device, hbm_peak, bf16_peak, rank):
    """Chunked prefill of a long prompt: its last 512-token chunk over the 32 K tokens before it
    (LLaMA-3-8B-shaped attention: 32 query heads, 8 KV heads, d 128, bf16).  Its 64 work items
    (8 query-tile pairs x 8 KV heads) would leave most of the 148 SMs idle, so the call takes the
    split schedule; roofline = tensor time of its FLOP + HBM time of its K/V bytes."""
    from paged_kv_attention_34_b200 import workloads as W
    from paged_kv_attention_34_b200.step import attn_bytes, attn_flops

    w = W.build_workload("long_chunk", q_lens=[512], ctx_lens=[32768], H_q=32, H_kv=8, d=128, dtype=W.BF16,
                         seed=shard_seed(34_006, rank), calls=[W.AttnCall("prefill", 0, 1)])
    st, per, step_ms = bench_leg(w, max(args.steps, 5), args.warmup, stream, device)
    flops, nbytes = attn_flops(w), attn_bytes(w)
    ms = per["paged_attn_prefill"]
    t_roof = flops / (bf16_peak * 1e12) + nbytes / (hbm_peak * 1e9)
    return {"workload": LONG_CHUNK, "TFLOP/s": round(flops / (ms * 1e-3) / 1e12, 2),
            "frac": round(t_roof / (ms * 1e-3), 4), "flop_per_launch": flops, "kv_bytes": nbytes,
            "avg_launch_ms": round(ms, 5), "prefill_ms_stats": st.call_stats["paged_attn_prefill"]}


def leg_gqa(args, stream, device, hbm_peak, rank):
    from paged_kv_attention_34_b200 import workloads as W
    from paged_kv_attention_34_b200.step import attn_bytes

    w = W.config4(seed=shard_seed(34_004, rank))
    st, per, step_ms = bench_leg(w, max(args.steps, 5), args.warmup, stream, device)
    b = attn_bytes(w)
    ms = per["paged_attn_decode"]
    gbs = b / (ms * 1e-3) / 1e9
    return {"workload": W.CONFIG_NAMES[4], "decode_GB/s": round(gbs, 1), "frac": round(gbs / hbm_peak, 4),
            "unique_bytes": b, "decode_ms": round(ms, 5), "step_ms": round(step_ms, 5),
            "per_call_ms": {k: round(v, 5) for k, v in per.items()},
            "decode_ms_stats": st.call_stats["paged_attn_decode"], "step_ms_stats": st.step_stats,
            "note": "shared prefix counted once; its blocks may stay in L2 across sequences"}


def leg_fp8(args, stream, device, hbm_peak, rank):
    """FP8 (E4M3) KV cache on the 13B-shaped decode layer (64 sequences, 40/40 heads, d 128, contexts
    U[128, 4096], fp16 Q): cache written through the FP8 write, then the FP8 decode timed alone and
    beside the 16-bit decode of the same data.  Algorithmic bytes: every context key's K and V codes
    (1 byte per value) and their two row scales, Q, O and the table entries."""
    import torch

    import paged_kv_attention_34_b200 as pa
    from paged_kv_attention_34_b200 import workloads as W
    from paged_kv_attention_34_b200.step import DeviceStep, attn_bytes

    w = W.config2(seed=shard_seed(34_002, rank), fill="zero", B=args.batch)
    with torch.cuda.stream(stream):
        st = DeviceStep(w, device=device)
    call = st.calls[0]
    NB, H, _, d = st.key_cache.shape
    kc8 = torch.zeros((NB, H, 16, d), dtype=torch.uint8, device=device)
    vc8 = torch.zeros((NB, H, d, 16), dtype=torch.uint8, device=device)  # transposed within the block
    ks = torch.ones((NB, H, 16), dtype=torch.float32, device=device)
    vs = torch.ones_like(ks)
    rows_k = st.key_cache.permute(0, 2, 1, 3).reshape(NB * 16, H, d).contiguous()
    rows_v = st.value_cache.permute(0, 2, 1, 3).reshape(NB * 16, H, d).contiguous()
    slots = torch.arange(NB * 16, dtype=torch.int32, device=device)
    with torch.cuda.stream(stream):
        pa.kv_cache_write_fp8(rows_k, rows_v, slots, kc8, vc8, ks, vs)
    del rows_k, rows_v
    torch.cuda.synchronize()

    def fp8():
        pa.paged_attn_decode_fp8(call.q, kc8, vc8, ks, vs, call.bt, call.cu, call.ctx, call.max_ctx, w.scale,
                                 out=call.out, workspace=call.ws)

    def bf():
        st.attend(call)

    steps = max(args.steps, 5)
    ms = {}
    for name, fn in (("fp8", fp8), ("16bit", bf)):
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                fn()
        torch.cuda.synchronize()
        ms[name] = time_steps([fn], steps, stream) / steps
    b16 = attn_bytes(w)
    ctx_tokens = sum(int(c) for c in w.ctx_lens)
    b8 = b16 - ctx_tokens * 2 * H * d * 2 + ctx_tokens * 2 * H * (d + 4)
    gbs = b8 / (ms["fp8"] * 1e-3) / 1e9
    return {"workload": f"FP8 (E4M3) KV cache, 13B-shaped decode layer: B {args.batch}, 40/40 heads, d 128, fp16 Q, "
                        "ctx U[128,4096]",
            "decode_GB/s": round(gbs, 1), "frac": round(gbs / hbm_peak, 4), "bytes": b8,
            "decode_ms": round(ms["fp8"], 5), "decode_16bit_ms": round(ms["16bit"], 5),
            "speedup_vs_16bit": round(ms["16bit"] / ms["fp8"], 3),
            "tokens_per_s": round(w.T / (ms["fp8"] * 1e-3), 1)}


def leg_tree(args, stream, device, hbm_peak, rank):
    """Tree-attention verification: 64 sequences x 8 drafted tokens in a random draft tree,
    contexts U[512, 4096], 32/8 heads, bf16; step = cache write + tree-verify decode."""
    import torch

    from paged_kv_attention_34_b200 import paged_attn_decode_tree
    from paged_kv_attention_34_b200 import workloads as W
    from paged_kv_attention_34_b200.step import DeviceStep, attn_bytes

    w = W.tree_verify(seed=shard_seed(34_105, rank))
    tm = W.random_tree_masks(shard_seed(34_105, rank), w.q_lens).to(device)
    with torch.cuda.stream(stream):
        st = DeviceStep(w, device=device)
    call = st.calls[0]

    def attend():
        paged_attn_decode_tree(call.q, st.key_cache, st.value_cache, call.bt, call.cu, call.ctx, tm, call.max_ctx,
                               w.scale, out=call.out, workspace=call.ws)

    fns = [st.write, attend]
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            for fn in fns:
                fn()
    torch.cuda.synchronize()
    total, per = time_calls(fns, max(args.steps, 5), stream)
    if any(st.statuses()):
        raise RuntimeError(f"device status {st.statuses()}")
    b = attn_bytes(w)
    gbs = b / (per[1] * 1e-3) / 1e9
    return {"workload": "tree-attention verify: 64 sequences x 8 drafts (random draft tree), ctx U[512,4096], "
                        "32/8 heads, d 128, bf16",
            "decode_GB/s": round(gbs, 1), "frac": round(gbs / hbm_peak, 4), "bytes": b,
            "decode_ms": round(per[1], 5), "per_call_ms": {"kv_cache_write": round(per[0], 5),
                                                           "paged_attn_decode_tree": round(per[1], 5)}}


def leg_shared(args, stream, device, hbm_peak, rank):
    """Shared-prefix decode: 64 requests in 4 groups of 16 sharing a 4096-token prompt (256 blocks),
    own suffixes U[16, 512], on the 13B-shaped layer (40/40 heads, d 128, fp16); the shared-prefix
    decode against the plain decode of the same tables.  Algorithmic bytes: every distinct key's K
    and V (each prompt once), Q, O, tables.  Also the long-context GQA config (16 sequences sharing
    2048 tokens of 32768) through both calls."""
    import torch

    from paged_kv_attention_34_b200 import paged_attn_decode, paged_attn_decode_shared_prefix, read_status
    from paged_kv_attention_34_b200 import shared_prefix_workspace_bytes
    from paged_kv_attention_34_b200 import workloads as W
    from paged_kv_attention_34_b200.step import DeviceStep, attn_bytes

    def run(w, starts, P):
        with torch.cuda.stream(stream):
            st = DeviceStep(w, device=device)
            st.copy_blocks()
            st.write()
        call = st.calls[0]
        gs = torch.tensor(starts, dtype=torch.int32, device=device)
        pb = torch.tensor(P, dtype=torch.int32, device=device)
        max_gt = max(sum(w.q_lens[starts[v]:starts[v + 1]]) for v in range(len(P)))
        ws = torch.zeros(shared_prefix_workspace_bytes(w.T, w.B, w.H_q, w.H_kv, w.d, call.max_ctx, len(P), max(P),
                                                       max_gt), dtype=torch.uint8, device=device)
        out2 = torch.empty_like(call.out)

        def shared():
            paged_attn_decode_shared_prefix(call.q, st.key_cache, st.value_cache, call.bt, call.cu, call.ctx, gs, pb,
                                            call.max_ctx, max(P), max_gt, w.scale, out=out2, workspace=ws)

        def plain():
            paged_attn_decode(call.q, st.key_cache, st.value_cache, call.bt, call.cu, call.ctx, call.max_ctx,
                              w.scale, out=call.out, workspace=call.ws)

        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                shared()
                plain()
        torch.cuda.synchronize()
        _, per = time_calls([shared, plain], max(args.steps, 5), stream)
        if any(st.statuses()) or read_status(ws):
            raise RuntimeError("device status")
        dev = (out2.float() - call.out.float()).abs().max().item()
        b = attn_bytes(w)
        return {"shared_ms": round(per[0], 5), "plain_ms": round(per[1], 5),
                "speedup_vs_plain": round(per[1] / per[0], 3), "unique_bytes": b,
                "unique_GB/s": round(b / (per[0] * 1e-3) / 1e9, 1),
                "frac": round(b / (per[0] * 1e-3) / 1e9 / hbm_peak, 4), "max_abs_diff_vs_plain": round(dev, 6)}

    w = W.shared_prefix_batch(seed=shard_seed(34_106, rank), fill="zero")
    res = {"workload": "shared-prefix decode: 64 requests = 4 prompts (4096 tokens) x 16, own suffixes U[16,512], "
                       "40/40 heads, d 128, fp16",
           **run(w, w.notes["group_start"], w.notes["prefix_blocks"])}
    w4 = W.config4(seed=shard_seed(34_004, rank), fill="zero")
    res["gqa_config"] = {"workload": W.CONFIG_NAMES[4],
                         **run(w4, [0, w4.B], [w4.notes["shared_tokens"] // 16])}
    return res


def leg_swap(args, stream, device, rank, n_blocks=512):
    """Preemption swap: n_blocks blocks of the 13B-shaped cache (40 heads, d 128, fp16; 320 KB of
    K+V per block) out to a pinned host pool and back in, each direction timed on its own, against
    one cudaMemcpyAsync of the same number of bytes between pinned host and device memory in the
    same run (the host link's measured copy rate)."""
    import torch

    from paged_kv_attention_34_b200 import kv_block_swap

    g = torch.Generator().manual_seed(shard_seed(34_102, rank))
    NB, H, d = 2 * n_blocks, 40, 128
    kc = torch.randn((NB, H, 16, d), generator=g).half().to(device)
    vc = torch.randn((NB, H, 16, d), generator=g).half().to(device)
    hk = torch.empty((n_blocks, H, 16, d), dtype=torch.float16).pin_memory()
    hv = torch.empty((n_blocks, H, 16, d), dtype=torch.float16).pin_memory()
    perm = torch.randperm(NB, generator=g)[:n_blocks].to(torch.int32)
    pairs = torch.stack([perm, torch.randperm(n_blocks, generator=g).to(torch.int32)], 1).contiguous().to(device)
    nbytes = 2 * n_blocks * H * 16 * d * 2
    dev_flat = torch.empty(nbytes, dtype=torch.uint8, device=device)
    host_flat = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    steps = max(args.steps, 5)
    res = {}
    for name, fn in (("out", lambda: kv_block_swap(kc, vc, hk, hv, pairs, to_host=True, stream=stream)),
                     ("in", lambda: kv_block_swap(kc, vc, hk, hv, pairs, to_host=False, stream=stream)),
                     ("memcpy_d2h", lambda: host_flat.copy_(dev_flat, non_blocking=True)),
                     ("memcpy_h2d", lambda: dev_flat.copy_(host_flat, non_blocking=True))):
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                fn()
        torch.cuda.synchronize()
        ms = time_steps([fn], steps, stream) / steps
        res[name] = round(nbytes / (ms * 1e-3) / 1e9, 2)
    return {"workload": f"swap of {n_blocks} blocks (40 heads, d 128, fp16: {nbytes / 1e6:.0f} MB of K+V) "
                        "to a pinned host pool and back",
            "unit": "GB/s", "out_GB/s": res["out"], "in_GB/s": res["in"],
            "frac_out": round(res["out"] / res["memcpy_d2h"], 4), "frac_in": round(res["in"] / res["memcpy_h2d"], 4),
            "peak_source": "cudaMemcpyAsync of the same bytes, pinned host <-> device, same run",
            "memcpy_GB/s": {"d2h": res["memcpy_d2h"], "h2d": res["memcpy_h2d"]}}


def leg_mixed(args, stream, device, hbm_peak, bf16_peak, rank):
    from paged_kv_attention_34_b200 import workloads as W
    from paged_kv_attention_34_b200.step import attn_bytes, attn_flops, write_bytes

    w = W.config5(seed=shard_seed(34_005, rank))
    st, per, step_ms = bench_leg(w, max(args.steps, 5), args.warmup, stream, device)
    t_roof = {
        "kv_cache_write": write_bytes(w) / (hbm_peak * 1e9),
        "paged_attn_prefill": attn_flops(w, "prefill") / (bf16_peak * 1e12) + attn_bytes(w, "prefill") / (hbm_peak * 1e9),
        "paged_attn_decode": attn_bytes(w, "decode") / (hbm_peak * 1e9),
    }
    meas = {k: per[k] * 1e-3 for k in t_roof}
    return {"workload": W.CONFIG_NAMES[5], "frac": round(sum(t_roof.values()) / sum(meas.values()), 4),
            "per_call_ms": {k: round(v, 5) for k, v in per.items()},
            "per_call_frac": {k: round(t_roof[k] / meas[k], 4) for k in t_roof},
            "tokens_per_s": round(w.T / (step_ms * 1e-3), 1), "step_ms": round(step_ms, 5),
            "step_ms_stats": st.step_stats}


# ---- the CPU oracle ---------------------------------------------------------------------------------------------

def oracle_caches(w):
    """The caches after the step's block copies and cache write, as the oracle computes them."""
    import oracle

    kc = oracle._u16(w.key_cache).copy()
    vc = oracle._u16(w.value_cache).copy()
    if w.copy_pairs is not None:
        oracle.kv_block_copy(kc, vc, w.copy_pairs)
    oracle.kv_cache_write(w.k_new, w.v_new, w.slot_mapping, kc, vc)
    return kc, vc


def oracle_sample_rate(w, caches, n_seq: int, threads: int):
    """Run the fp64 oracle on the first n_seq sequences of a decode workload; returns (GB/s, seconds, bytes)."""
    import numpy as np

    import oracle
    from paged_kv_attention_34_b200.step import attn_bytes
    from paged_kv_attention_34_b200.workloads import AttnCall, Workload

    kc, vc = caches
    cu = w.cu_seqlens_q
    t1 = int(cu[n_seq])
    rows = np.arange(t1 * w.H_q, dtype=np.int64)
    sub = Workload(**{**w.__dict__, "q_lens": w.q_lens[:n_seq], "ctx_lens": w.ctx_lens[:n_seq],
                      "calls": [AttnCall("decode", 0, n_seq)]})
    t0 = time.perf_counter()
    oracle.paged_attention(w.q[:t1], kc, vc, oracle.dtype_code(w.dtype), w.block_tables[:n_seq], cu[: n_seq + 1],
                           w.context_lens[:n_seq], w.H_kv, w.scale, rows=rows, n_threads=threads)
    dt = time.perf_counter() - t0
    b = attn_bytes(sub)
    return b / dt / 1e9, dt, b


def cpu_baseline(w, seconds: float):
    """fp64 oracle on the host cores, on a bounded sample of the headline workload."""
    threads = os.cpu_count() or 1
    caches = oracle_caches(w)
    rate, dt, _ = oracle_sample_rate(w, caches, 2, threads)  # calibration
    n = max(2, min(w.B, int(math.ceil(2 * seconds / max(dt, 1e-3)))))
    rate, dt, b = oracle_sample_rate(w, caches, n, threads)
    return {"value": round(rate, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"first {n} of {w.B} sequences (all 40 heads), {b/1e9:.3f} GB of KV, {dt:.1f} s"}


def row_keys(w):
    """Visible keys of every (token, query head) row of a workload, row index t * H_q + h."""
    import numpy as np

    keys = np.empty(w.T, dtype=np.int64)
    cu = w.cu_seqlens_q.tolist()
    for b in range(w.B):
        qb, ctx = w.q_lens[b], w.ctx_lens[b]
        keys[cu[b]:cu[b + 1]] = ctx - qb + 1 + np.arange(qb)
    return np.repeat(keys, w.H_q)


def oracle_extrapolated(w, seconds: float, threads: int, seed: int):
    """Time the fp64 oracle on a seeded random sample of the workload's query rows, sized to about
    `seconds` of host time, and extrapolate to the whole workload by visible keys (its work per
    row is one dot product and one accumulation per visible key).  Returns (seconds for the
    whole workload, description of the sample)."""
    import numpy as np

    import oracle

    kc, vc = oracle_caches(w)
    keys = row_keys(w)
    order = np.random.default_rng(seed).permutation(keys.shape[0])

    def run(n):
        rows = np.sort(order[:n])
        t0 = time.perf_counter()
        oracle.paged_attention(w.q, kc, vc, oracle.dtype_code(w.dtype), w.block_tables, w.cu_seqlens_q,
                               w.context_lens, w.H_kv, w.scale, rows=rows, n_threads=threads)
        return time.perf_counter() - t0, int(keys[rows].sum())

    n = min(64, keys.shape[0])
    dt, k = run(n)
    n = int(min(keys.shape[0], max(n, n * seconds / max(dt, 1e-3))))
    dt, k = run(n)
    total = float(dt) * float(keys.sum()) / max(k, 1)
    return total, f"{n} of {keys.shape[0]} query rows drawn at random (seed {seed}), {k} visible keys, {dt:.1f} s"


def cpu_baseline_configs(seconds: float):
    """The oracle on the other configurations' workloads (bounded samples, extrapolated): the
    causal varlen prefill (TFLOP/s of exact causal pairs), the long-context GQA decode with a
    shared prefix (GB/s of distinct bytes) and the mixed continuous-batching step (tokens/s of
    the two attention calls)."""
    from paged_kv_attention_34_b200 import workloads as W
    from paged_kv_attention_34_b200.step import attn_bytes, attn_flops

    threads = os.cpu_count() or 1
    res = {}
    w3 = W.config3(seed=shard_seed(34_003, 0))
    t3, smp = oracle_extrapolated(w3, seconds, threads, 3)
    res["cfg3_prefill"] = {"value": round(attn_flops(w3) / t3 / 1e12, 6), "unit": "TFLOP/s", "cores": threads,
                           "kind": "oracle", "sample": smp}
    del w3
    w4 = W.config4(seed=shard_seed(34_004, 0))
    t4, smp = oracle_extrapolated(w4, seconds, threads, 4)
    res["cfg4_gqa_decode"] = {"value": round(attn_bytes(w4) / t4 / 1e9, 4), "unit": "GB/s", "cores": threads,
                              "kind": "oracle", "sample": smp}
    del w4
    w5 = W.config5(seed=shard_seed(34_005, 0))
    t5, smp = oracle_extrapolated(w5, seconds, threads, 5)
    res["cfg5_mixed_step"] = {"value": round(w5.T / t5, 1), "unit": "tokens/s", "cores": threads, "kind": "oracle",
                              "sample": smp, "step_s": round(t5, 3)}
    return res


def run_reference(args):
    """--impl reference: the fp64 oracle on host cores, bounded samples of the headline workload."""
    rank, _, world = dist_env()
    if rank != 0:
        return
    from paged_kv_attention_34_b200 import workloads as W

    w = W.config2(seed=shard_seed(34_002, 0))
    threads = os.cpu_count() or 1
    caches = oracle_caches(w)
    _, dt, _ = oracle_sample_rate(w, caches, 2, threads)
    # each step: a sample sized to about 2 s of host time
    n = max(1, min(w.B, int(round(2 * 2.0 / max(dt, 1e-3)))))
    for _ in range(args.warmup):
        oracle_sample_rate(w, caches, n, threads)
    tot_b, tot_t = 0.0, 0.0
    for _ in range(args.steps):
        _, dt, b = oracle_sample_rate(w, caches, n, threads)
        tot_b += b
        tot_t += dt
    value = tot_b / tot_t / 1e9
    res = {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(tot_t / args.steps * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic: seeded N(0,1) fp16 Q/K/V (same generator as the GPU arm)",
        "config": {"workload": HEADLINE, "global_batch": 64, "seq_len": "context U[128,4096]",
                   "parallelism": "host threads (OpenMP)"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": f"first {n} of 64 sequences per step (all 40 heads)"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(res), flush=True)


def run_one_leg(args):
    """One leg alone on cuda:LOCAL_RANK (for profiling); prints the leg's JSON object."""
    import torch

    import paged_kv_attention_34_b200 as pa

    _, local_rank, _ = dist_env()
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    pa.lib()
    peaks, peak_src = load_peaks()
    stream = torch.cuda.Stream(device=device)
    hbm, bf16 = float(peaks["hbm_gbs"]), float(peaks["bf16_tflops"])
    if args.only == "prefill":
        res = leg_prefill(args, stream, device, bf16, peak_src, 0)
    elif args.only == "gqa":
        res = leg_gqa(args, stream, device, hbm, 0)
    elif args.only == "swap":
        res = leg_swap(args, stream, device, 0)
    elif args.only == "tree":
        res = leg_tree(args, stream, device, hbm, 0)
    elif args.only == "fp8":
        res = leg_fp8(args, stream, device, hbm, 0)
    elif args.only == "shared":
        res = leg_shared(args, stream, device, hbm, 0)
    elif args.only == "long_chunk":
        res = leg_long_chunk(args, stream, device, hbm, bf16, 0)
    else:
        res = leg_mixed(args, stream, device, hbm, bf16, 0)
    print(json.dumps({"leg": args.only, **res}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-legs", action="store_true", help="headline decode step only")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="host time budget of the cpu_baseline sample")
    ap.add_argument("--only", choices=["prefill", "gqa", "mixed", "swap", "tree", "fp8", "shared", "long_chunk"],
                    default=None,
                    help="run one leg alone and print its JSON object (profiling runs)")
    ap.add_argument("--batch", type=int, default=64,
                    help="sequences of the headline decode workload (64 = the 13B-shaped layer; smaller for profiling)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.only:
        run_one_leg(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
