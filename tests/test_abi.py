"""The C-ABI library on the CPU: it builds, loads, exports every declared entry
point, and rejects bad arguments on the host before touching the device.

Only host-side paths run here (no GPU): every call below returns from its
argument checks before any launch; the only CUDA runtime call made is the
block swap's pointer-attribute query of its host pools, which refuses them
cleanly when there is no device.
"""
import ctypes
import os
import re

import numpy as np
import subprocess

import pytest

import paged_kv_attention_34_b200 as pa
from paged_kv_attention_34_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "paged_attn.h")


@pytest.fixture(scope="module")
def L():
    if _build.needs_build():
        _build.build()
    return pa.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ("pa_kv_cache_write", "pa_paged_attn_decode", "pa_paged_attn_prefill", "pa_kv_block_copy"):
        assert n in names


def test_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", pa.LIB_PATH], capture_output=True, text=True, check=True)
    exported = set(re.findall(r"\bT (pa_[a-z_0-9]+)", out.stdout))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(L, n)


def test_version_and_strerror(L):
    assert L.pa_version() == 100
    for code, name in pa.STATUS_NAMES.items():
        assert pa.strerror(code) and pa.strerror(code) != "unknown status", name
    assert pa.strerror(12345) == "unknown status"


def _fake(addr=0x10000):
    return ctypes.c_void_p(addr)


def test_write_rejects_bad_args(L):
    f = L.pa_kv_cache_write
    ok = dict(T=4, NB=8, H=2, d=128, dt=0)

    def call(T=4, NB=8, H=2, d=128, dt=0, kn=_fake(), slot=_fake(), status=None):
        return f(kn, _fake(), slot, T, _fake(), _fake(), NB, H, d, dt, status, None)

    assert call(d=96) == -2
    assert call(d=32) == -2
    assert call(T=-1) == -1
    assert call(NB=0) == -1
    assert call(H=0) == -1
    assert call(dt=7) == -1
    assert call(kn=_fake(0x10008)) == -3  # not 16-byte aligned
    assert call(slot=_fake(0x10002)) == -3
    assert call(T=0) == 0  # nothing to do, nothing launched
    del ok


def test_block_copy_rejects_bad_args(L):
    f = L.pa_kv_block_copy
    assert f(_fake(), _fake(), 8, 2, 80, 0, _fake(), 3, None, None) == -2
    assert f(_fake(), _fake(), 8, 2, 64, 0, _fake(), -1, None, None) == -1
    assert f(_fake(0x10004), _fake(), 8, 2, 64, 0, _fake(), 3, None, None) == -3
    assert f(_fake(), _fake(), 8, 2, 64, 0, _fake(), 0, None, None) == 0


def test_block_swap_rejects_bad_args(L):
    f = L.pa_kv_block_swap

    def call(NB=8, HB=4, H=2, d=64, dt=0, n=3, direction=0, hk=None, hv=None):
        hk = hk if hk is not None else _fake()
        hv = hv if hv is not None else _fake()
        return f(_fake(), _fake(), NB, hk, hv, HB, H, d, dt, _fake(), n, direction, None, None)

    assert call(d=80) == -2
    assert call(n=-1) == -1
    assert call(HB=0) == -1
    assert call(NB=0) == -1
    assert call(direction=2) == -1
    assert call(dt=5) == -1
    assert call(n=0) == 0  # nothing to do, nothing launched
    # host pools that are not page-locked host memory are refused before any launch
    n0 = pa.launch_count()
    host = np.zeros(1 << 16, np.uint8)
    ptr = ctypes.c_void_p(host.ctypes.data)
    assert call(hk=ptr, hv=ptr) == -1
    assert pa.launch_count() == n0


def _decode(L, *, B=2, T=2, H_q=8, H_kv=2, d=128, max_ctx=100, NB=16, ws=_fake(), wsb=1 << 20, q=_fake(),
            scale=0.1, dt=1):
    return L.pa_paged_attn_decode(_fake(), q, _fake(), _fake(), NB, _fake(), 8, _fake(), _fake(), B, max_ctx, T,
                                  H_q, H_kv, d, scale, dt, ws, wsb, None)


def test_decode_rejects_bad_args(L):
    assert _decode(L, H_q=6, H_kv=4) == -2  # H_q % H_kv
    assert _decode(L, d=96) == -2
    assert _decode(L, B=-1) == -1
    assert _decode(L, ws=None) == -4
    assert _decode(L, wsb=16) == -4
    assert _decode(L, ws=_fake(0x10008)) == -3
    assert _decode(L, q=_fake(0x10001)) == -3
    assert _decode(L, scale=float("nan")) == -1
    assert _decode(L, NB=(1 << 31) // 32) == -2  # TMA row coordinate would overflow
    assert _decode(L, dt=3) == -1


def test_noalloc_decode_returns_the_same_codes_as_decode(L):
    """The allocation-free decode runs the same size and shape checks as the regular one, before
    its scratch-size check; none of these calls reaches the device."""
    f = L.pa_paged_attn_decode_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_void_p,
                                          ctypes.c_void_p]

    def noalloc(B=2, T=2, H_q=8, H_kv=2, d=128, max_ctx=100, NB=16, dt=1):
        return f(_fake(), _fake(), _fake(), _fake(), NB, _fake(), 8, _fake(), _fake(), B, max_ctx, T, H_q, H_kv, d,
                 0.1, dt, None, None)

    n0 = pa.launch_count()
    for bad in (dict(d=96), dict(H_q=3, H_kv=2), dict(H_q=6, H_kv=4), dict(B=-1), dict(T=-1), dict(H_kv=0),
                dict(NB=0), dict(dt=3), dict(max_ctx=-1), dict(NB=(1 << 31) // 32)):
        assert noalloc(**bad) == _decode(L, **bad), bad
        assert noalloc(**bad) in (-1, -2), bad
    assert pa.launch_count() == n0


def test_get_status_rejects_null(L):
    assert L.pa_get_status(None) == -1


def test_prefill_rejects_bad_args(L):
    f = L.pa_paged_attn_prefill

    def call(max_q_len=16, H_q=4, H_kv=4, d=64, wsb=256):
        return f(_fake(), _fake(), _fake(), _fake(), 4, _fake(), 4, _fake(), _fake(), 1, max_q_len, 64, 16, H_q,
                 H_kv, d, 0.1, 0, _fake(), wsb, None)

    assert call(max_q_len=0) == -1
    assert call(H_q=5, H_kv=2) == -2
    assert call(d=256) == -2
    assert call(wsb=8) == -4


def test_shared_prefix_rejects_bad_args(L):
    f = L.pa_paged_attn_decode_shared_prefix

    def call(n_groups=2, max_pb=4, max_gt=2, gs=_fake(), pb=_fake(), wsb=1 << 20, B=2, T=2):
        return f(_fake(), _fake(), _fake(), _fake(), 16, _fake(), 8, _fake(), _fake(), B, 100, T, 8, 2, 128, 0.1, 1,
                 gs, pb, n_groups, max_pb, max_gt, _fake(), wsb, None)

    n0 = pa.launch_count()
    assert call(n_groups=0) == -1
    assert call(max_pb=9) == -1     # more prefix blocks than a table holds
    assert call(max_gt=3) == -1     # more new tokens in a group than in the batch
    assert call(gs=None) == -1
    assert call(pb=None) == -1
    assert call(gs=_fake(0x10002)) == -3
    assert call(wsb=64) == -4
    assert call(n_groups=4) == -1   # more groups than B + 1
    assert pa.launch_count() == n0


def test_selftest_wait_timeout_rejects_bad_args(L):
    f = L.pa_selftest_wait_timeout
    n0 = pa.launch_count()
    assert f(None, 1000, None) == -1
    assert f(_fake(0x10002), 1000, None) == -1  # misaligned status word
    assert f(_fake(), 0, None) == -1
    assert f(_fake(), 100_000_001, None) == -1  # more than 0.1 s
    assert pa.launch_count() == n0


def test_workspace_queries(L):
    # one split needs the status word and the sequence order (B int32 in 256-byte units);
    # long contexts need partials
    small = pa.decode_workspace_bytes(3, 3, 4, 4, 64, 50)
    assert small == pa.PA_STATUS_BYTES + 256
    assert pa.decode_workspace_bytes(3, 65, 4, 4, 64, 50) == pa.PA_STATUS_BYTES + 512
    big = pa.decode_workspace_bytes(16, 16, 64, 8, 128, 32768)
    assert big > pa.PA_STATUS_BYTES
    # monotone in T and max_ctx
    assert pa.decode_workspace_bytes(32, 16, 64, 8, 128, 32768) >= big
    assert pa.decode_workspace_bytes(16, 16, 64, 8, 128, 65536) >= big
    assert L.pa_decode_workspace_bytes(1, 1, 6, 4, 128, 10) == 0  # invalid GQA ratio
    assert pa.prefill_workspace_bytes(8, 40, 40, 128, 2048) >= pa.PA_STATUS_BYTES
    # prefill: the split schedule's areas (starts, counters, two fp32 partial slots per CTA for
    # both query tiles) only for calls whose items would keep at most 3/4 of the CTAs busy (the
    # SM count falls back to the B200's 148 without a device: 3/4 of 148 = 111 items)
    queue = pa.prefill_workspace_bytes(8, 40, 40, 128, 2048)  # 8 x 8 pairs x 40 heads = 2560 items
    assert queue == pa.PA_STATUS_BYTES + 256  # the order of 64 entries
    split = pa.prefill_workspace_bytes(1, 32, 8, 128, 512)  # 8 pairs x 8 heads = 64 items
    assert split >= 2 * 160 * 2 * 128 * (128 + 1) * 4
    assert pa.prefill_workspace_bytes(1, 32, 8, 64, 512) < split  # d 64: half the partials
    # 111 items take the split schedule, 112 the queue (G 1: 128 tokens per tile, 256 per pair)
    assert pa.prefill_workspace_bytes(111, 1, 1, 128, 256) >= 2 * 160 * 2 * 128 * 129 * 4
    assert pa.prefill_workspace_bytes(112, 1, 1, 128, 256) == pa.PA_STATUS_BYTES + 512
    assert pa.prefill_workspace_bytes(14, 8, 8, 128, 256) == pa.PA_STATUS_BYTES + 256  # 112 items
    # shared-prefix decode: status, order and per-sequence prefix areas, then every row's partials
    sh = pa.shared_prefix_workspace_bytes(64, 64, 40, 40, 128, 4608, 4, 256, 16)
    assert sh >= pa.PA_STATUS_BYTES + 2 * 256 + 64 * 40 * 129 * 4
    assert pa.shared_prefix_workspace_bytes(64, 64, 40, 40, 128, 4608, 4, 512, 16) >= sh  # longer prefixes
    assert L.pa_shared_prefix_workspace_bytes(64, 64, 40, 40, 128, 4608, 0, 256, 16) == 0  # no group


def test_binding_refuses_cpu_tensors():
    import torch

    q = torch.zeros((1, 1, 64), dtype=torch.float16)
    with pytest.raises(ValueError, match="CUDA"):
        pa.paged_attn_decode(q, q.view(1, 1, 1, 64), q.view(1, 1, 1, 64), torch.zeros((1, 1), dtype=torch.int32),
                             torch.zeros(2, dtype=torch.int32), torch.ones(1, dtype=torch.int32), 1, 0.1)


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(pa, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(pa, "_lib", None)
    with pytest.raises(ImportError, match="no fallback"):
        pa.lib()
