"""Python binding of libpagedattn (exact attention over a paged KV cache, B200).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libpagedattn.so``, reached through its C ABI
(``include/paged_attn.h``) with ctypes.  Tensors are torch CUDA tensors;
the current torch stream is passed to every call.  There is no fallback: if
the library is not built, or a tensor is not on a CUDA device, the call
raises.

Calls (same names as the C ABI without the ``pa_`` prefix):

* ``kv_cache_write(k_new, v_new, slot_mapping, key_cache, value_cache)``
* ``kv_block_copy(key_cache, value_cache, pairs)``
* ``paged_attn_decode(q, key_cache, value_cache, block_tables, cu_seqlens_q, context_lens, max_ctx, scale)``
* ``paged_attn_prefill(q, key_cache, value_cache, block_tables, cu_seqlens_q, context_lens, max_q_len, max_ctx, scale)``
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpagedattn.so")

PA_F16, PA_BF16 = 0, 1
PA_STATUS_BYTES = 256
STATUS_NAMES = {
    0: "PA_OK",
    -1: "PA_ERR_ARG",
    -2: "PA_ERR_UNSUPPORTED",
    -3: "PA_ERR_ALIGN",
    -4: "PA_ERR_WORKSPACE",
    -5: "PA_ERR_CUDA",
    -6: "PA_ERR_TIMEOUT",
    -7: "PA_ERR_BOUNDS",
    -8: "PA_ERR_SEQ",
    -9: "PA_ERR_TOO_LARGE",
}

_lib = None


class PagedAttnError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)} ({strerror(code)})")


def _declare(L):
    c = ctypes
    P, I, I64, SZ = c.c_void_p, c.c_int, c.c_int64, c.c_size_t
    L.pa_kv_cache_write.restype = I
    L.pa_kv_cache_write.argtypes = [P, P, P, I64, P, P, I64, I, I, I, P, P]
    L.pa_kv_block_copy.restype = I
    L.pa_kv_block_copy.argtypes = [P, P, I64, I, I, I, P, I64, P, P]
    L.pa_kv_block_swap.restype = I
    L.pa_kv_block_swap.argtypes = [P, P, I64, P, P, I64, I, I, I, P, I64, I, P, P]
    L.pa_decode_workspace_bytes.restype = SZ
    L.pa_decode_workspace_bytes.argtypes = [I64, I, I, I, I, I]
    L.pa_paged_attn_decode.restype = I
    L.pa_paged_attn_decode.argtypes = [P, P, P, P, I64, P, I, P, P, I, I, I64, I, I, I, c.c_float, I, P, SZ, P]
    L.pa_kv_cache_write_fp8.restype = I
    L.pa_kv_cache_write_fp8.argtypes = [P, P, P, I64, P, P, P, P, I64, I, I, I, P, P]
    L.pa_paged_attn_decode_fp8.restype = I
    L.pa_paged_attn_decode_fp8.argtypes = [P, P, P, P, P, P, I64, P, I, P, P, I, I, I64, I, I, I, c.c_float, I, P,
                                           SZ, P]
    L.pa_paged_attn_decode_tree.restype = I
    L.pa_paged_attn_decode_tree.argtypes = [P, P, P, P, I64, P, I, P, P, P, I, I, I64, I, I, I, c.c_float, I, P, SZ,
                                            P]
    L.pa_shared_prefix_workspace_bytes.restype = SZ
    L.pa_shared_prefix_workspace_bytes.argtypes = [I64, I, I, I, I, I, I, I, I]
    L.pa_paged_attn_decode_shared_prefix.restype = I
    L.pa_paged_attn_decode_shared_prefix.argtypes = [P, P, P, P, I64, P, I, P, P, I, I, I64, I, I, I, c.c_float, I,
                                                     P, P, I, I, I, P, SZ, P]
    L.pa_prefill_workspace_bytes.restype = SZ
    L.pa_prefill_workspace_bytes.argtypes = [I, I, I, I, I]
    L.pa_paged_attn_prefill.restype = I
    L.pa_paged_attn_prefill.argtypes = [P, P, P, P, I64, P, I, P, P, I, I, I, I64, I, I, I, c.c_float, I, P, SZ, P]
    L.pa_selftest_wait_timeout.restype = I
    L.pa_selftest_wait_timeout.argtypes = [P, c.c_uint64, P]
    L.pa_read_status.restype = I
    L.pa_read_status.argtypes = [P, P, P]
    L.pa_get_status.restype = I
    L.pa_get_status.argtypes = [P]
    L.pa_strerror.restype = c.c_char_p
    L.pa_strerror.argtypes = [I]
    L.pa_launch_count.restype = c.c_uint64
    L.pa_launch_count.argtypes = []
    L.pa_version.restype = I
    L.pa_version.argtypes = []
    return L


def lib():
    """The loaded C library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m paged_kv_attention_34_b200._build` "
                "(or __graft_entry__.build()); there is no fallback implementation"
            )
        _lib = _declare(ctypes.CDLL(LIB_PATH))
    return _lib


def strerror(code: int) -> str:
    return lib().pa_strerror(int(code)).decode()


def launch_count() -> int:
    return int(lib().pa_launch_count())


def _check(rc: int, what: str):
    if rc != 0:
        raise PagedAttnError(rc, what)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return PA_F16
    if t.dtype == torch.bfloat16:
        return PA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; expected float16 or bfloat16")


def _cuda(t: torch.Tensor, name: str, dtype=None, ndim=None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path exists)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    return t


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def kv_cache_write(k_new, v_new, slot_mapping, key_cache, value_cache, status=None, stream=None):
    """Scatter k_new/v_new [T, H_kv, d] into the caches [NB, H_kv, 16, d] at slot_mapping [T] (int32)."""
    _cuda(key_cache, "key_cache", ndim=4)
    dt = key_cache.dtype
    _cuda(value_cache, "value_cache", dt, 4)
    _cuda(k_new, "k_new", dt, 3)
    _cuda(v_new, "v_new", dt, 3)
    _cuda(slot_mapping, "slot_mapping", torch.int32, 1)
    NB, H_kv, bs, d = key_cache.shape
    T = k_new.shape[0]
    if bs != 16 or value_cache.shape != key_cache.shape or k_new.shape != (T, H_kv, d) or v_new.shape != k_new.shape:
        raise ValueError("shape mismatch between k_new/v_new [T,H_kv,d] and caches [NB,H_kv,16,d]")
    if slot_mapping.shape[0] != T:
        raise ValueError("slot_mapping must have T entries")
    if status is not None:
        _cuda(status, "status", torch.int32)
    rc = lib().pa_kv_cache_write(
        _ptr(k_new), _ptr(v_new), _ptr(slot_mapping), T, _ptr(key_cache), _ptr(value_cache), NB, H_kv, d,
        _dtype_code(key_cache), _ptr(status), ctypes.c_void_p(_stream(stream)),
    )
    _check(rc, "pa_kv_cache_write")


def kv_block_copy(key_cache, value_cache, pairs, status=None, stream=None):
    """Copy-on-write: copy block pairs[i,0] to pairs[i,1] in both caches (pairs: int32 [n, 2])."""
    _cuda(key_cache, "key_cache", ndim=4)
    _cuda(value_cache, "value_cache", key_cache.dtype, 4)
    _cuda(pairs, "pairs", torch.int32, 2)
    NB, H_kv, _, d = key_cache.shape
    if status is not None:
        _cuda(status, "status", torch.int32)
    rc = lib().pa_kv_block_copy(
        _ptr(key_cache), _ptr(value_cache), NB, H_kv, d, _dtype_code(key_cache), _ptr(pairs), pairs.shape[0],
        _ptr(status), ctypes.c_void_p(_stream(stream)),
    )
    _check(rc, "pa_kv_block_copy")


PA_SWAP_OUT, PA_SWAP_IN = 0, 1


def kv_block_swap(key_cache, value_cache, host_key, host_value, pairs, to_host: bool, status=None, stream=None):
    """Swap blocks between the device caches and a pinned host pool (pairs: int32 [n, 2] of
    (device block, host block)): device -> host when `to_host`, else host -> device."""
    _cuda(key_cache, "key_cache", ndim=4)
    _cuda(value_cache, "value_cache", key_cache.dtype, 4)
    _cuda(pairs, "pairs", torch.int32, 2)
    NB, H_kv, _, d = key_cache.shape
    for name, t in (("host_key", host_key), ("host_value", host_value)):
        if t.device.type != "cpu" or not t.is_pinned() or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous pinned CPU tensor")
        if t.dtype != key_cache.dtype or t.dim() != 4 or tuple(t.shape[1:]) != (H_kv, 16, d):
            raise ValueError(f"{name} must be [host_blocks, {H_kv}, 16, {d}] {key_cache.dtype}")
    if host_value.shape[0] != host_key.shape[0]:
        raise ValueError("host_key and host_value must hold the same number of blocks")
    if status is not None:
        _cuda(status, "status", torch.int32)
    rc = lib().pa_kv_block_swap(
        _ptr(key_cache), _ptr(value_cache), NB, ctypes.c_void_p(host_key.data_ptr()),
        ctypes.c_void_p(host_value.data_ptr()), host_key.shape[0], H_kv, d, _dtype_code(key_cache), _ptr(pairs),
        pairs.shape[0], PA_SWAP_OUT if to_host else PA_SWAP_IN, _ptr(status), ctypes.c_void_p(_stream(stream)),
    )
    _check(rc, "pa_kv_block_swap")


def decode_workspace_bytes(T: int, B: int, H_q: int, H_kv: int, d: int, max_ctx: int) -> int:
    n = lib().pa_decode_workspace_bytes(T, B, H_q, H_kv, d, max_ctx)
    if n == 0:
        raise ValueError("invalid sizes for pa_decode_workspace_bytes")
    return int(n)


def prefill_workspace_bytes(B: int, H_q: int, H_kv: int, d: int, max_q_len: int) -> int:
    n = lib().pa_prefill_workspace_bytes(B, H_q, H_kv, d, max_q_len)
    if n == 0:
        raise ValueError("invalid sizes for pa_prefill_workspace_bytes")
    return int(n)


def _attn_common(q, key_cache, value_cache, block_tables, cu_seqlens_q, context_lens, out, stream=None):
    _cuda(q, "q", ndim=3)
    dt = q.dtype
    _cuda(key_cache, "key_cache", dt, 4)
    _cuda(value_cache, "value_cache", dt, 4)
    _cuda(block_tables, "block_tables", torch.int32, 2)
    _cuda(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    _cuda(context_lens, "context_lens", torch.int32, 1)
    T, H_q, d = q.shape
    NB, H_kv, bs, dk = key_cache.shape
    if bs != 16 or dk != d or value_cache.shape != key_cache.shape:
        raise ValueError("caches must be [NB, H_kv, 16, d] with d matching q")
    B = context_lens.shape[0]
    if cu_seqlens_q.shape[0] != B + 1 or block_tables.shape[0] != B:
        raise ValueError("cu_seqlens_q must have B+1 entries and block_tables B rows")
    if out is None:
        out = _bind_to_stream(torch.empty_like(q), stream)
    else:
        _cuda(out, "out", dt, 3)
        if out.shape != q.shape:
            raise ValueError("out must have q's shape")
    return out, T, H_q, d, NB, H_kv, B


def _bind_to_stream(t: torch.Tensor, stream) -> torch.Tensor:
    """A tensor allocated here (workspace, output) is used by kernels on `stream`; when that is not
    the current stream, tell the caching allocator, so the memory is not handed out again on the
    current stream while those kernels may still run."""
    if stream is not None and stream != torch.cuda.current_stream(t.device):
        t.record_stream(stream)
    return t


def _workspace(ws, nbytes, device, stream=None):
    if ws is None:
        return _bind_to_stream(torch.empty(nbytes, dtype=torch.uint8, device=device), stream)
    _cuda(ws, "workspace", torch.uint8, 1)
    if ws.numel() < nbytes:
        raise ValueError(f"workspace too small: {ws.numel()} < {nbytes}")
    return ws


def paged_attn_decode(q, key_cache, value_cache, block_tables, cu_seqlens_q, context_lens, max_ctx: int,
                      scale: float, out=None, workspace=None, stream=None):
    """Split-KV decode for 1..8 query tokens per sequence; returns out [T, H_q, d]."""
    out, T, H_q, d, NB, H_kv, B = _attn_common(q, key_cache, value_cache, block_tables, cu_seqlens_q,
                                               context_lens, out, stream)
    nbytes = decode_workspace_bytes(T, B, H_q, H_kv, d, max_ctx)
    ws = _workspace(workspace, nbytes, q.device, stream)
    rc = lib().pa_paged_attn_decode(
        _ptr(out), _ptr(q), _ptr(key_cache), _ptr(value_cache), NB, _ptr(block_tables), block_tables.shape[1],
        _ptr(cu_seqlens_q), _ptr(context_lens), B, int(max_ctx), T, H_q, H_kv, d, float(scale),
        _dtype_code(q), _ptr(ws), ws.numel(), ctypes.c_void_p(_stream(stream)),
    )
    _check(rc, "pa_paged_attn_decode")
    paged_attn_decode.last_workspace = ws
    return out


def _fp8_cache(key_cache, value_cache, key_scale, value_scale):
    _cuda(key_cache, "key_cache", torch.uint8, 4)
    _cuda(value_cache, "value_cache", torch.uint8, 4)
    NB, H_kv, bs, d = key_cache.shape
    if bs != 16 or tuple(value_cache.shape) != (NB, H_kv, d, 16):
        raise ValueError("FP8 caches must be uint8: keys [NB, H_kv, 16, d], values [NB, H_kv, d, 16]")
    for name, t in (("key_scale", key_scale), ("value_scale", value_scale)):
        _cuda(t, name, torch.float32, 3)
        if tuple(t.shape) != (NB, H_kv, 16):
            raise ValueError(f"{name} must be float32 [{NB}, {H_kv}, 16]")
    return NB, H_kv, d


def kv_cache_write_fp8(k_new, v_new, slot_mapping, key_cache, value_cache, key_scale, value_scale, status=None,
                       stream=None):
    """Quantise k_new/v_new [T, H_kv, d] (16-bit) into the FP8 cache (uint8 codes: keys [NB, H_kv, 16, d],
    values transposed within the block [NB, H_kv, d, 16]; float32 row scales [NB, H_kv, 16]) at
    slot_mapping [T]."""
    NB, H_kv, d = _fp8_cache(key_cache, value_cache, key_scale, value_scale)
    _cuda(k_new, "k_new", None, 3)
    _cuda(v_new, "v_new", k_new.dtype, 3)
    _cuda(slot_mapping, "slot_mapping", torch.int32, 1)
    if status is not None:
        _cuda(status, "status", torch.int32)
    rc = lib().pa_kv_cache_write_fp8(
        _ptr(k_new), _ptr(v_new), _ptr(slot_mapping), slot_mapping.shape[0], _ptr(key_cache), _ptr(value_cache),
        _ptr(key_scale), _ptr(value_scale), NB, H_kv, d, _dtype_code(k_new), _ptr(status),
        ctypes.c_void_p(_stream(stream)),
    )
    _check(rc, "pa_kv_cache_write_fp8")


def paged_attn_decode_fp8(q, key_cache, value_cache, key_scale, value_scale, block_tables, cu_seqlens_q,
                          context_lens, max_ctx: int, scale: float, out=None, workspace=None, stream=None):
    """Split-KV decode over the FP8 cache; returns out [T, H_q, d] in q's dtype."""
    NB, H_kv, d = _fp8_cache(key_cache, value_cache, key_scale, value_scale)
    _cuda(q, "q", None, 3)
    T, H_q, dq = q.shape
    if dq != d:
        raise ValueError("q and the caches disagree on d")
    _cuda(block_tables, "block_tables", torch.int32, 2)
    _cuda(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    _cuda(context_lens, "context_lens", torch.int32, 1)
    B = context_lens.shape[0]
    if out is None:
        out = _bind_to_stream(torch.empty_like(q), stream)
    nbytes = decode_workspace_bytes(T, B, H_q, H_kv, d, max_ctx)
    ws = _workspace(workspace, nbytes, q.device, stream)
    rc = lib().pa_paged_attn_decode_fp8(
        _ptr(out), _ptr(q), _ptr(key_cache), _ptr(value_cache), _ptr(key_scale), _ptr(value_scale), NB,
        _ptr(block_tables), block_tables.shape[1], _ptr(cu_seqlens_q), _ptr(context_lens), B, int(max_ctx), T, H_q,
        H_kv, d, float(scale), _dtype_code(q), _ptr(ws), ws.numel(), ctypes.c_void_p(_stream(stream)),
    )
    _check(rc, "pa_paged_attn_decode_fp8")
    paged_attn_decode_fp8.last_workspace = ws
    return out


def paged_attn_decode_tree(q, key_cache, value_cache, block_tables, cu_seqlens_q, context_lens, tree_mask,
                           max_ctx: int, scale: float, out=None, workspace=None, stream=None):
    """Tree-attention verification: decode where token t sees the cached keys before its sequence's
    new tokens and new token j when bit j of tree_mask[t] (int32 [T]) is set; returns out."""
    out, T, H_q, d, NB, H_kv, B = _attn_common(q, key_cache, value_cache, block_tables, cu_seqlens_q,
                                               context_lens, out, stream)
    _cuda(tree_mask, "tree_mask", torch.int32, 1)
    if tree_mask.shape[0] != T:
        raise ValueError(f"tree_mask must be int32 [{T}]")
    nbytes = decode_workspace_bytes(T, B, H_q, H_kv, d, max_ctx)
    ws = _workspace(workspace, nbytes, q.device, stream)
    rc = lib().pa_paged_attn_decode_tree(
        _ptr(out), _ptr(q), _ptr(key_cache), _ptr(value_cache), NB, _ptr(block_tables), block_tables.shape[1],
        _ptr(cu_seqlens_q), _ptr(context_lens), _ptr(tree_mask), B, int(max_ctx), T, H_q, H_kv, d, float(scale),
        _dtype_code(q), _ptr(ws), ws.numel(), ctypes.c_void_p(_stream(stream)),
    )
    _check(rc, "pa_paged_attn_decode_tree")
    paged_attn_decode_tree.last_workspace = ws
    return out


def shared_prefix_workspace_bytes(T: int, B: int, H_q: int, H_kv: int, d: int, max_ctx: int, n_groups: int,
                                  max_prefix_blocks: int, max_group_tokens: int) -> int:
    n = lib().pa_shared_prefix_workspace_bytes(T, B, H_q, H_kv, d, max_ctx, n_groups, max_prefix_blocks,
                                               max_group_tokens)
    if n == 0:
        raise ValueError("invalid sizes for pa_shared_prefix_workspace_bytes")
    return int(n)


def paged_attn_decode_shared_prefix(q, key_cache, value_cache, block_tables, cu_seqlens_q, context_lens,
                                    group_start, prefix_blocks, max_ctx: int, max_prefix_blocks: int,
                                    max_group_tokens: int, scale: float, out=None, workspace=None, stream=None):
    """Decode where groups of consecutive sequences share the first prefix_blocks[v] blocks of their
    tables (group v = sequences group_start[v] .. group_start[v+1]-1, int32 device tensors): the
    shared blocks are read once per group, then merged with each sequence's own keys; returns out."""
    out, T, H_q, d, NB, H_kv, B = _attn_common(q, key_cache, value_cache, block_tables, cu_seqlens_q,
                                               context_lens, out, stream)
    _cuda(group_start, "group_start", torch.int32, 1)
    _cuda(prefix_blocks, "prefix_blocks", torch.int32, 1)
    n_groups = prefix_blocks.shape[0]
    if group_start.shape[0] != n_groups + 1:
        raise ValueError(f"group_start must be int32 [{n_groups + 1}]")
    nbytes = shared_prefix_workspace_bytes(T, B, H_q, H_kv, d, max_ctx, n_groups, max_prefix_blocks,
                                           max_group_tokens)
    ws = _workspace(workspace, nbytes, q.device, stream)
    rc = lib().pa_paged_attn_decode_shared_prefix(
        _ptr(out), _ptr(q), _ptr(key_cache), _ptr(value_cache), NB, _ptr(block_tables), block_tables.shape[1],
        _ptr(cu_seqlens_q), _ptr(context_lens), B, int(max_ctx), T, H_q, H_kv, d, float(scale), _dtype_code(q),
        _ptr(group_start), _ptr(prefix_blocks), n_groups, int(max_prefix_blocks), int(max_group_tokens), _ptr(ws),
        ws.numel(), ctypes.c_void_p(_stream(stream)),
    )
    _check(rc, "pa_paged_attn_decode_shared_prefix")
    paged_attn_decode_shared_prefix.last_workspace = ws
    return out


def paged_attn_prefill(q, key_cache, value_cache, block_tables, cu_seqlens_q, context_lens, max_q_len: int,
                       max_ctx: int, scale: float, out=None, workspace=None, stream=None):
    """Causal varlen prefill over the paged cache; returns out [T, H_q, d]."""
    out, T, H_q, d, NB, H_kv, B = _attn_common(q, key_cache, value_cache, block_tables, cu_seqlens_q,
                                               context_lens, out, stream)
    nbytes = prefill_workspace_bytes(B, H_q, H_kv, d, max_q_len)
    ws = _workspace(workspace, nbytes, q.device, stream)
    rc = lib().pa_paged_attn_prefill(
        _ptr(out), _ptr(q), _ptr(key_cache), _ptr(value_cache), NB, _ptr(block_tables), block_tables.shape[1],
        _ptr(cu_seqlens_q), _ptr(context_lens), B, int(max_q_len), int(max_ctx), T, H_q, H_kv, d, float(scale),
        _dtype_code(q), _ptr(ws), ws.numel(), ctypes.c_void_p(_stream(stream)),
    )
    _check(rc, "pa_paged_attn_prefill")
    paged_attn_prefill.last_workspace = ws
    return out


def selftest_wait_timeout(status: torch.Tensor, timeout_ns: int, stream=None) -> None:
    """Launch the bounded-wait self-test: a wait on a barrier that nothing completes gives up after
    timeout_ns and records PA_ERR_TIMEOUT in status (int32 device tensor)."""
    _cuda(status, "status", torch.int32, None)
    rc = lib().pa_selftest_wait_timeout(_ptr(status), int(timeout_ns), ctypes.c_void_p(_stream(stream)))
    _check(rc, "pa_selftest_wait_timeout")


def read_status(workspace: torch.Tensor, stream=None) -> int:
    """Device status word at the start of a workspace (or a status tensor); synchronises the stream."""
    _cuda(workspace, "workspace")
    val = ctypes.c_int32(0)
    rc = lib().pa_read_status(_ptr(workspace), ctypes.byref(val), ctypes.c_void_p(_stream(stream)))
    _check(rc, "pa_read_status")
    return int(val.value)


def get_status(workspace: torch.Tensor) -> int:
    """Device status word at the start of a workspace (or a status tensor), after waiting for all
    work on the current device.  Raises only if the runtime fails."""
    _cuda(workspace, "workspace")
    rc = int(lib().pa_get_status(_ptr(workspace)))
    if rc == -5:  # the kernels never record PA_ERR_CUDA: this is the runtime failing
        _check(rc, "pa_get_status")
    return rc
