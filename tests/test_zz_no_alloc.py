"""pa_paged_attn_decode_noalloc on the GPU, through the C ABI.

Who needs this entry point: code that may not allocate device memory at the
moment it calls the library -- a plugin inside an inference engine that owns
every byte of device memory through its own pool and forbids raw allocations
while work is being enqueued, or a latency-critical step that cannot accept
cudaMalloc's implicit device synchronisation or an allocation failure in the
middle of a step.  Its scratch (status word, split-KV partials) is a fixed
array inside the library instead of a caller workspace.

What is checked here:
* two calls in a row (the second finds the first call's partials still in the
  scratch) give exactly the bytes of pa_paged_attn_decode -- both run the same
  plan and kernels -- and agree with the fp64 oracle within the decode
  tolerance; the workload needs several KV splits, so the scratch is used;
* a device-detected error (a block id outside the pool, which the kernel skips
  without faulting) reaches the caller's status word, and the next clean call
  reads 0 again (the scratch's status word is cleared per call);
* sizes beyond the fixed scratch are refused before anything is launched
  (every pointer passed is a real device buffer sized for the arguments).

The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import paged_kv_attention_34_b200 as pa
from oracle_pins import oracle_step
from paged_kv_attention_34_b200 import workloads as W
from paged_kv_attention_34_b200.step import DeviceStep

pytestmark = pytest.mark.gpu

TOL = {torch.float16: 3e-3, torch.bfloat16: 1.6e-2}
SCRATCH_BYTES = 32 << 20  # PA_DECODE_NOALLOC_SCRATCH_BYTES
PA_ERR_BOUNDS = -7
PA_ERR_TOO_LARGE = -9


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pa.lib()


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


def _call_noalloc(st, call, w, out, status):
    T = call.q.shape[0]
    NB, H_kv, _, d = st.key_cache.shape
    code = 0 if w.dtype == W.F16 else 1
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return _entry()(_p(out), _p(call.q), _p(st.key_cache), _p(st.value_cache), NB, _p(call.bt), call.bt.shape[1],
                    _p(call.cu), _p(call.ctx), call.ctx.shape[0], call.max_ctx, T, w.H_q, w.H_kv, d, w.scale, code,
                    _p(status), stream)


@pytest.mark.parametrize("dtype", [W.BF16, W.F16])
def test_noalloc_matches_regular_decode_twice(dtype):
    w = W.random_workload(4242, B=6, q_max=6, ctx_max=2500, H_kv=2, G=4, d=128, dtype=dtype, kind="decode")
    st = DeviceStep(w)
    st.copy_blocks()
    st.write()
    call = st.calls[0]
    T = call.q.shape[0]
    need = pa.decode_workspace_bytes(T, call.ctx.shape[0], w.H_q, w.H_kv, w.d, call.max_ctx)
    assert pa.PA_STATUS_BYTES < need <= SCRATCH_BYTES  # split partials go through the scratch

    ref = pa.paged_attn_decode(call.q, st.key_cache, st.value_cache, call.bt, call.cu, call.ctx, call.max_ctx,
                               w.scale)
    torch.cuda.synchronize()
    assert pa.read_status(pa.paged_attn_decode.last_workspace) == 0
    want, _, _ = oracle_step(w, oracle.lib())

    for attempt in range(2):
        out = torch.full_like(call.q, float("nan"))
        status = torch.full((1,), 12345, dtype=torch.int32, device=call.q.device)
        rc = _call_noalloc(st, call, w, out, status)
        assert rc == 0, pa.strerror(rc)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        # the same plan and kernels as the regular entry point: the same bytes
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"call {attempt}: differs from decode"
        got = out.double().cpu().numpy()
        assert np.isfinite(got).all()
        err = np.abs(got - want).max()
        assert err <= TOL[dtype], f"call {attempt}: max abs err {err:.3e} against the oracle"


def test_noalloc_reports_device_status_then_clears_it():
    w = W.random_workload(5, B=2, q_max=1, ctx_max=40, H_kv=2, G=1, d=64, dtype=W.F16, kind="decode")
    st = DeviceStep(w)
    st.copy_blocks()
    st.write()
    call = st.calls[0]
    good_bt = call.bt.clone()
    status = torch.full((1,), 12345, dtype=torch.int32, device=call.q.device)
    out = torch.empty_like(call.q)

    call.bt[1, 0] = w.num_blocks + 3  # outside the pool: the kernel skips it (TMA zero fill), no fault
    assert _call_noalloc(st, call, w, out, status) == 0
    torch.cuda.synchronize()
    assert int(status.item()) == PA_ERR_BOUNDS

    call.bt.copy_(good_bt)
    assert _call_noalloc(st, call, w, out, status) == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    want, _, _ = oracle_step(w, oracle.lib())
    assert np.abs(out.double().cpu().numpy() - want).max() <= TOL[torch.float16]


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # 512 sequences x 8 new tokens x 64 heads with 32K contexts: far more split partials than the
    # fixed scratch holds.  Every buffer is real and sized for these arguments (one pool block that
    # every table entry points at), so nothing here names memory the call does not own.
    B, q_b, H_q, H_kv, d, ctx = 512, 8, 64, 8, 128, 32768
    T, max_blocks = B * q_b, ctx // 16
    need = pa.decode_workspace_bytes(T, B, H_q, H_kv, d, ctx)
    assert need > SCRATCH_BYTES
    dev = "cuda"
    q = torch.zeros((T, H_q, d), dtype=torch.bfloat16, device=dev)
    out = torch.empty_like(q)
    kc = torch.zeros((1, H_kv, 16, d), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    bt = torch.zeros((B, max_blocks), dtype=torch.int32, device=dev)
    cu = torch.arange(0, T + 1, q_b, dtype=torch.int32, device=dev)
    ctx_lens = torch.full((B,), ctx, dtype=torch.int32, device=dev)
    status = torch.full((1,), 12345, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    n0 = pa.launch_count()
    rc = _entry()(_p(out), _p(q), _p(kc), _p(vc), 1, _p(bt), max_blocks, _p(cu), _p(ctx_lens), B, ctx, T, H_q, H_kv,
                  d, 0.088, 1, _p(status), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == PA_ERR_TOO_LARGE
    assert "scratch" in pa.strerror(rc)
    assert pa.launch_count() == n0
    torch.cuda.synchronize()
    assert int(status.item()) == 12345  # nothing was written
