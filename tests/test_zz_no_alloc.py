"""pa_paged_attn_decode_noalloc against pa_paged_attn_decode (GPU).

The allocation-free entry point serves callers that may not allocate device
memory when they call (plugins inside an engine that owns all device memory,
latency-critical code that cannot take cudaMalloc's implicit synchronisation
or a failure mid-step).  Its scratch is a fixed array inside the library.
These tests call it through the C ABI, twice in a row (the second call reuses
the scratch the first one left behind), and compare each output with the
regular entry point's within the decode tolerance of the parity tests.  The
workload needs several KV splits, so the scratch really is used.  The file is
named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import paged_kv_attention_34_b200 as pa
from paged_kv_attention_34_b200 import workloads as W
from paged_kv_attention_34_b200.step import DeviceStep

pytestmark = pytest.mark.gpu

TOL = {torch.float16: 3e-3, torch.bfloat16: 1.6e-2}
SCRATCH_BYTES = 32 << 20  # PA_DECODE_NOALLOC_SCRATCH_BYTES
PA_ERR_TOO_LARGE = -9


def _entry():
    L = pa.lib()
    f = L.pa_paged_attn_decode_noalloc
    c = ctypes
    P, I, I64 = c.c_void_p, c.c_int, c.c_int64
    f.restype = I
    f.argtypes = [P, P, P, P, I64, P, I, P, P, I, I, I64, I, I, I, c.c_float, I, P, P]
    return f


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("dtype", [W.BF16, W.F16])
def test_noalloc_matches_regular_decode_twice(dtype):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = W.random_workload(4242, B=6, q_max=6, ctx_max=2500, H_kv=2, G=4, d=128, dtype=dtype, kind="decode")
    st = DeviceStep(w)
    st.copy_blocks()
    st.write()
    call = st.calls[0]
    T = call.q.shape[0]
    NB, H_kv, _, d = st.key_cache.shape
    need = pa.decode_workspace_bytes(T, call.ctx.shape[0], w.H_q, w.H_kv, d, call.max_ctx)
    assert pa.PA_STATUS_BYTES < need <= SCRATCH_BYTES  # split partials go through the scratch

    ref = pa.paged_attn_decode(call.q, st.key_cache, st.value_cache, call.bt, call.cu, call.ctx, call.max_ctx,
                               w.scale)
    torch.cuda.synchronize()
    assert pa.read_status(pa.paged_attn_decode.last_workspace) == 0

    f = _entry()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    code = 0 if dtype == W.F16 else 1
    for attempt in range(2):
        out = torch.full_like(call.q, float("nan"))
        status = torch.full((1,), 12345, dtype=torch.int32, device=call.q.device)
        rc = f(_p(out), _p(call.q), _p(st.key_cache), _p(st.value_cache), NB, _p(call.bt), call.bt.shape[1],
               _p(call.cu), _p(call.ctx), call.ctx.shape[0], call.max_ctx, T, w.H_q, w.H_kv, d, w.scale, code,
               _p(status), stream)
        assert rc == 0, pa.strerror(rc)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        got = out.double().cpu().numpy()
        assert np.isfinite(got).all()
        err = np.abs(got - ref.double().cpu().numpy()).max()
        assert err <= TOL[dtype], f"call {attempt}: max abs diff {err}"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    f = _entry()
    # 4096 tokens x 64 heads with 32K contexts: far more split partials than the fixed scratch holds
    need = pa.decode_workspace_bytes(4096, 512, 64, 8, 128, 32768)
    assert need > SCRATCH_BYTES
    n0 = pa.launch_count()
    dummy = ctypes.c_void_p(0x10000)
    rc = f(dummy, dummy, dummy, dummy, 1000, dummy, 2048, dummy, dummy, 512, 32768, 4096, 64, 8, 128, 0.088, 1,
           None, None)
    assert rc == PA_ERR_TOO_LARGE
    assert "scratch" in pa.strerror(rc)
    assert pa.launch_count() == n0
