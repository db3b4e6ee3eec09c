"""The N > 1 host logic of bench.py on CPU ranks (gloo, world size 2).

Every rank draws its own batch (independent seed, weak scaling); the only
collectives are barriers, the max over ranks of the elapsed time and the sum
of the processed bytes.  Here two CPU processes check that the shards differ,
that the reductions give the max and the sum, and that the per-rank
algorithmic byte counts add up to the whole-job figure.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    from paged_kv_attention_34_b200 import workloads as W
    from paged_kv_attention_34_b200.step import attn_bytes, write_bytes

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, lr, ws = bench.dist_env()
        assert (r, lr, ws) == (rank, rank, world)
        seed = bench.shard_seed(34_002, rank)
        w = W.config2(seed=seed, B=4, fill="zero")  # a small shard of the headline shape
        b = float(attn_bytes(w) + write_bytes(w))
        elapsed = 1.0 + rank  # rank 1 is the slow one
        mx = bench.reduce_max(elapsed, "cpu")
        tot = bench.reduce_sum(b, "cpu")
        bench.barrier()
        q.put((rank, seed, w.ctx_lens, b, mx, tot))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    (r0, s0, c0, b0, m0, t0), (r1, s1, c1, b1, m1, t1) = res
    assert s0 != s1 and c0 != c1  # independent shards
    assert m0 == m1 == 2.0  # max over ranks
    assert t0 == t1 == pytest.approx(b0 + b1)  # whole-job bytes
