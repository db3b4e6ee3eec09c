"""Loader for the fp64 CPU oracle (``oracle/oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference leg of ``bench.py``.  The product library
never imports it.

``build()`` compiles ``oracle.c`` with gcc (``-O2 -fopenmp``) into
``oracle/liboracle.so``; ``lib()`` loads it (building it first if missing or
older than the source).  The wrappers take torch CPU tensors or numpy arrays
and return numpy float64 arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

F16, BF16 = 0, 1


def build(src: str = _SRC, out: str = _LIB, extra_flags=()) -> str:
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", *extra_flags, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _declare(L):
    c = ctypes
    P = c.c_void_p
    L.oracle_f16_to_f64.restype = c.c_double
    L.oracle_f16_to_f64.argtypes = [c.c_uint16]
    L.oracle_bf16_to_f64.restype = c.c_double
    L.oracle_bf16_to_f64.argtypes = [c.c_uint16]
    L.oracle_kv_cache_write.restype = c.c_int64
    L.oracle_kv_cache_write.argtypes = [P, P, P, c.c_int64, P, P, c.c_int64, c.c_int, c.c_int]
    L.oracle_kv_block_copy.restype = c.c_int64
    L.oracle_kv_block_copy.argtypes = [P, P, c.c_int64, c.c_int, c.c_int, P, c.c_int64]
    L.oracle_e4m3_to_f64.restype = c.c_double
    L.oracle_e4m3_to_f64.argtypes = [c.c_uint8]
    L.oracle_f64_to_e4m3.restype = c.c_uint8
    L.oracle_f64_to_e4m3.argtypes = [c.c_double]
    L.oracle_kv_cache_write_fp8.restype = c.c_int64
    L.oracle_kv_cache_write_fp8.argtypes = [P, P, c.c_int, P, c.c_int64, P, P, P, P, c.c_int64, c.c_int, c.c_int]
    L.oracle_paged_attention_fp8.restype = c.c_int
    L.oracle_paged_attention_fp8.argtypes = [
        P, P, c.c_int, P, P, P, P, P, c.c_int, P, P, c.c_int, c.c_int, c.c_int, c.c_int, c.c_double, P, c.c_int64,
        c.c_int,
    ]
    L.oracle_kv_block_swap.restype = c.c_int64
    L.oracle_kv_block_swap.argtypes = [P, P, c.c_int64, P, P, c.c_int64, c.c_int, c.c_int, P, c.c_int64, c.c_int]
    L.oracle_paged_attention.restype = c.c_int
    L.oracle_paged_attention.argtypes = [
        P, P, P, P, P, c.c_int, P, c.c_int, P, P, c.c_int, c.c_int, c.c_int, c.c_int, c.c_double, P, c.c_int64, c.c_int,
    ]
    L.oracle_paged_attention_tree.restype = c.c_int
    L.oracle_paged_attention_tree.argtypes = [
        P, P, P, P, P, c.c_int, P, c.c_int, P, P, P, c.c_int, c.c_int, c.c_int, c.c_int, c.c_double, P, c.c_int64,
        c.c_int,
    ]
    L.oracle_dense_attention.restype = None
    L.oracle_dense_attention.argtypes = [P, P, P, P, c.c_int, c.c_int, c.c_int, c.c_double, c.c_int64]
    L.oracle_online_softmax.restype = None
    L.oracle_online_softmax.argtypes = [P, P, P, P, c.c_int, c.c_int, c.c_double, c.c_int]
    L.oracle_attention_partial.restype = None
    L.oracle_attention_partial.argtypes = [P, P, P, P, P, c.c_int, c.c_int, c.c_int, c.c_double]
    L.oracle_lse_merge.restype = None
    L.oracle_lse_merge.argtypes = [P, P, P, P, c.c_int, c.c_int]
    return L


def load(path: str):
    """Load an oracle shared object at ``path`` (used for planted-mistake copies too)."""
    return _declare(ctypes.CDLL(path))


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            build()
        _lib = load(_LIB)
    return _lib


# ---- array helpers -------------------------------------------------------------

def _u16(x) -> np.ndarray:
    """Raw 16-bit patterns of a float16/bfloat16 torch tensor or uint16 array (contiguous)."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch

    assert x.dtype in (torch.float16, torch.bfloat16), x.dtype
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _i32(x) -> np.ndarray:
    if isinstance(x, np.ndarray):
        return np.ascontiguousarray(x, dtype=np.int32)
    return np.ascontiguousarray(x.detach().cpu().numpy().astype(np.int32))


def _f64(x) -> np.ndarray:
    if isinstance(x, np.ndarray):
        return np.ascontiguousarray(x, dtype=np.float64)
    return np.ascontiguousarray(x.detach().cpu().double().numpy())


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def dtype_code(torch_dtype) -> int:
    import torch

    return {torch.float16: F16, torch.bfloat16: BF16}[torch_dtype]


# ---- wrappers --------------------------------------------------------------------

def f16_to_f64(bits: int, L=None) -> float:
    return (L or lib()).oracle_f16_to_f64(bits)


def bf16_to_f64(bits: int, L=None) -> float:
    return (L or lib()).oracle_bf16_to_f64(bits)


def kv_cache_write(k_new, v_new, slot_mapping, key_cache: np.ndarray, value_cache: np.ndarray, L=None) -> int:
    """In place on uint16 numpy caches [NB, H_kv, 16, d]; returns the count of out-of-range slots."""
    kn, vn, sm = _u16(k_new), _u16(v_new), _i32(slot_mapping)
    NB, H_kv, _, d = key_cache.shape
    return (L or lib()).oracle_kv_cache_write(
        _p(kn), _p(vn), _p(sm), sm.shape[0], _p(key_cache), _p(value_cache), NB, H_kv, d
    )


def kv_block_copy(key_cache: np.ndarray, value_cache: np.ndarray, pairs, L=None) -> int:
    pr = _i32(pairs).reshape(-1, 2)
    NB, H_kv, _, d = key_cache.shape
    return (L or lib()).oracle_kv_block_copy(_p(key_cache), _p(value_cache), NB, H_kv, d, _p(pr), pr.shape[0])


def e4m3_to_f64(code: int, L=None) -> float:
    return (L or lib()).oracle_e4m3_to_f64(code)


def f64_to_e4m3(x: float, L=None) -> int:
    return (L or lib()).oracle_f64_to_e4m3(float(x))


def kv_cache_write_fp8(k_new, v_new, dtype: int, slot_mapping, key_cache: np.ndarray, value_cache: np.ndarray,
                       key_scale: np.ndarray, value_scale: np.ndarray, L=None) -> int:
    """FP8 cache write: K codes uint8 [NB, H_kv, 16, d], V codes uint8 [NB, H_kv, d, 16] (transposed
    within the block), scales float32 [NB, H_kv, 16]; in place."""
    kn, vn = _u16(k_new), _u16(v_new)
    sm = _i32(slot_mapping)
    NB, H_kv, _, d = key_cache.shape
    assert value_cache.shape == (NB, H_kv, d, 16)
    for a, dt in ((key_cache, np.uint8), (value_cache, np.uint8), (key_scale, np.float32), (value_scale, np.float32)):
        assert a.dtype == dt and a.flags.c_contiguous
    return (L or lib()).oracle_kv_cache_write_fp8(_p(kn), _p(vn), dtype, _p(sm), sm.shape[0], _p(key_cache),
                                                  _p(value_cache), _p(key_scale), _p(value_scale), NB, H_kv, d)


def paged_attention_fp8(q, dtype: int, key_cache: np.ndarray, value_cache: np.ndarray, key_scale: np.ndarray,
                        value_scale: np.ndarray, block_tables, cu_seqlens_q, context_lens, H_kv: int, scale: float,
                        rows: Optional[np.ndarray] = None, n_threads: int = 0, L=None):
    """fp64 attention over the FP8 cache (K and V dequantised exactly: code value x row scale)."""
    qq = _u16(q)
    T, H_q, d = qq.shape
    bt, cu, cl = _i32(block_tables), _i32(cu_seqlens_q), _i32(context_lens)
    B = cl.shape[0]
    if rows is None:
        out = np.empty((T, H_q, d), dtype=np.float64)
        n_rows, r = T * H_q, None
    else:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        n_rows = r.shape[0]
        out = np.empty((n_rows, d), dtype=np.float64)
    rc = (L or lib()).oracle_paged_attention_fp8(
        _p(out), _p(qq), dtype, _p(key_cache), _p(value_cache), _p(key_scale), _p(value_scale), _p(bt), bt.shape[1],
        _p(cu), _p(cl), B, H_q, H_kv, d, float(scale), _p(r), n_rows, n_threads,
    )
    if rc != 0:
        raise ValueError(f"oracle_paged_attention_fp8 rejected its arguments (code {rc})")
    return out


def kv_block_swap(key_cache: np.ndarray, value_cache: np.ndarray, host_key: np.ndarray, host_value: np.ndarray,
                  pairs, to_host: bool, L=None) -> int:
    """Blocks pairs[i, 0] (device caches) <-> pairs[i, 1] (host pool), in place; returns the pairs skipped."""
    pr = _i32(pairs).reshape(-1, 2)
    NB, H_kv, _, d = key_cache.shape
    return (L or lib()).oracle_kv_block_swap(_p(key_cache), _p(value_cache), NB, _p(host_key), _p(host_value),
                                             host_key.shape[0], H_kv, d, _p(pr), pr.shape[0], 1 if to_host else 0)


def paged_attention(
    q,
    key_cache,
    value_cache,
    dtype: int,
    block_tables,
    cu_seqlens_q,
    context_lens,
    H_kv: int,
    scale: float,
    rows: Optional[np.ndarray] = None,
    n_threads: int = 0,
    with_lse: bool = False,
    L=None,
    tree_mask=None,
):
    """fp64 attention over the paged cache.

    q: [T, H_q, d] (16-bit); caches [NB, H_kv, 16, d] (16-bit).  ``rows`` selects
    flattened ``t * H_q + h`` rows; the result is then ``[len(rows), d]``, else
    ``[T, H_q, d]``.  ``tree_mask`` (int32 [T]): tree-attention verification, token t sees the
    cached keys before its sequence's new tokens and new token j when bit j is set; None = causal.
    """
    qq = _u16(q)
    T, H_q, d = qq.shape
    kc, vc = _u16(key_cache), _u16(value_cache)
    bt = _i32(block_tables)
    cu = _i32(cu_seqlens_q)
    cl = _i32(context_lens)
    B = cl.shape[0]
    if rows is None:
        out = np.empty((T, H_q, d), dtype=np.float64)
        n_rows = T * H_q
        r = None
    else:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        n_rows = r.shape[0]
        out = np.empty((n_rows, d), dtype=np.float64)
    lse = np.empty(n_rows, dtype=np.float64) if with_lse else None
    if tree_mask is None:
        rc = (L or lib()).oracle_paged_attention(
            _p(out), _p(lse), _p(qq), _p(kc), _p(vc), dtype, _p(bt), bt.shape[1], _p(cu), _p(cl), B, H_q, H_kv, d,
            float(scale), _p(r), n_rows, n_threads,
        )
    else:
        tm = _i32(tree_mask)
        if tm.shape != (T,):
            raise ValueError("tree_mask must be int32 [T]")
        rc = (L or lib()).oracle_paged_attention_tree(
            _p(out), _p(lse), _p(qq), _p(kc), _p(vc), dtype, _p(bt), bt.shape[1], _p(cu), _p(cl), _p(tm), B, H_q,
            H_kv, d, float(scale), _p(r), n_rows, n_threads,
        )
    if rc != 0:
        raise ValueError(f"oracle_paged_attention rejected its arguments (code {rc})")
    return (out, lse) if with_lse else out


def dense_attention(q, k, v, scale: float, offset: int, L=None) -> np.ndarray:
    q, k, v = _f64(q), _f64(k), _f64(v)
    n_q, d = q.shape
    n_k = k.shape[0]
    out = np.empty((n_q, d), dtype=np.float64)
    (L or lib()).oracle_dense_attention(_p(out), _p(q), _p(k), _p(v), n_q, n_k, d, float(scale), int(offset))
    return out


def online_softmax(q, k, v, scale: float, block: int, L=None) -> np.ndarray:
    q, k, v = _f64(q), _f64(k), _f64(v)
    d = q.shape[-1]
    out = np.empty(d, dtype=np.float64)
    (L or lib()).oracle_online_softmax(_p(out), _p(q), _p(k), _p(v), k.shape[0], d, float(scale), int(block))
    return out


def attention_partial(q, k, v, lo: int, hi: int, scale: float, L=None):
    q, k, v = _f64(q), _f64(k), _f64(v)
    d = q.shape[-1]
    out = np.empty(d, dtype=np.float64)
    lse = np.empty(1, dtype=np.float64)
    (L or lib()).oracle_attention_partial(_p(out), _p(lse), _p(q), _p(k), _p(v), int(lo), int(hi), d, float(scale))
    return out, float(lse[0])


def lse_merge(parts, lses, L=None):
    parts, lses = _f64(parts), _f64(lses)
    n, d = parts.shape
    out = np.empty(d, dtype=np.float64)
    lse = np.empty(1, dtype=np.float64)
    (L or lib()).oracle_lse_merge(_p(out), _p(lse), _p(parts), _p(lses), n, d)
    return out, float(lse[0])
