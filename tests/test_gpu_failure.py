"""Failure paths on the GPU without faulting it: undersized workspaces, device allocation
failures inside tq_init (injected on the host), out-of-range slots in device slot arrays
(reported through the context's error word), and pipeline waits that run out (a test limit
of 0 ns on the dequantize kernel), after which the context is still usable."""
import numpy as np
import pytest

import oracle
import parity
import workloads as W

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import ctypes  # noqa: E402

import kv_cache_vector_08_b200 as tq  # noqa: E402

DEV = torch.device("cuda", 0)
TQ_ERR_INVALID_ARG, TQ_ERR_ALLOC, TQ_ERR_WORKSPACE = 1, 4, 5


def _small_cache(d=128, n=512):
    x = torch.tensor(W.round_bf16(W.gaussian((n, d), 3, W.STREAM_KEYS)), dtype=torch.bfloat16, device=DEV)
    ctx = tq.Context(d, 4, 21, tq.MODE_PROD)
    pk = tq.alloc_packed(ctx, n)
    tq.quantize_kv(ctx, x, pk)
    torch.cuda.synchronize()
    return ctx, pk, x


def test_undersized_workspaces_are_rejected():
    ctx, pk, x = _small_cache()
    L = tq.lib()
    q = torch.randn((4, 128), device=DEV)
    need = int(L.tq_attn_logits_workspace_size(ctx.handle, 4))
    small = torch.empty(max(need - 16, 1), dtype=torch.uint8, device=DEV)
    with pytest.raises(tq.TQError) as e:
        tq.attn_logits(ctx, q, pk, 512, workspace=small)
    assert e.value.status == TQ_ERR_WORKSPACE
    # a workspace that is large enough but not 16-byte aligned is refused before any launch
    big = torch.empty(need + 64, dtype=torch.uint8, device=DEV)
    ps0 = pk.struct()
    lg = torch.empty((4, 512), device=DEV)
    st = L.tq_attn_logits(ctx.handle, ctypes.c_void_p(q.data_ptr()), 4, ctypes.byref(ps0), 512,
                          ctypes.c_void_p(lg.data_ptr()), ctypes.c_void_p(big.data_ptr() + 4), need, None)
    assert st == TQ_ERR_INVALID_ARG
    # search
    need = int(L.tq_search_workspace_size(ctx.handle, 4, 512, 10))
    out_s = torch.empty((4, 10), device=DEV)
    out_i = torch.empty((4, 10), dtype=torch.int64, device=DEV)
    small = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
    ps = pk.struct()
    st = L.tq_search_topk(ctx.handle, ctypes.c_void_p(q.data_ptr()), 4, ctypes.byref(ps), 512, 10,
                          ctypes.c_void_p(out_s.data_ptr()), ctypes.c_void_p(out_i.data_ptr()),
                          ctypes.c_void_p(small.data_ptr()), small.numel(), None)
    assert st == TQ_ERR_WORKSPACE
    # decode
    kx, vx = tq.Context(128, 4, 1, tq.MODE_PROD), tq.Context(128, 4, 2, tq.MODE_MSE)
    kc, vc = tq.alloc_packed(kx, 2 * 64), tq.alloc_packed(vx, 2 * 64)
    plan = tq.DecodePlan([kx], [vx], [0, 128], [kc], [vc], 1, 8, 2, 128, 64)
    plan.workspace = plan.workspace[: plan.workspace.numel() - 256]
    with pytest.raises(tq.TQError) as e:
        plan(torch.zeros((1, 8, 128), dtype=torch.bfloat16, device=DEV),
             torch.tensor([64], dtype=torch.int32, device=DEV), 0.1, torch.empty((1, 8, 128), device=DEV))
    assert e.value.status == TQ_ERR_WORKSPACE
    # quantize through the workspace path (fp32 input)
    xf = x.float()
    need = tq.quantize_workspace_size(ctx, 0, 512, 128)
    assert need > 0
    with pytest.raises(tq.TQError) as e:
        tq.quantize_kv(ctx, xf, pk, workspace=torch.empty(need - 256, dtype=torch.uint8, device=DEV))
    assert e.value.status == TQ_ERR_WORKSPACE
    torch.cuda.synchronize()


def test_injected_allocation_failures_leave_nothing_behind():
    L = tq.lib()
    h = ctypes.c_void_p()
    assert L.tq_init(ctypes.byref(h), 1024, 4, 5, 0) == 0      # warm-up cycle (driver pools)
    L.tq_free(h)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for index in range(0, 8):
        L.tq_debug_fail_alloc(index)
        st = L.tq_init(ctypes.byref(h), 1024, 4, 5, 0)
        L.tq_debug_fail_alloc(-1)
        if st == 0:                      # fewer allocations than index + 1: a normal context
            L.tq_free(h)
            break
        assert st == TQ_ERR_ALLOC and not h.value
        assert b"cudaMalloc" in L.tq_last_error()
    else:
        pytest.fail("tq_init made more than 8 allocations")
    torch.cuda.synchronize()
    # every operand of a d = 1024 context is >= 2 MiB, so a leak would show beyond the slack
    assert abs(torch.cuda.mem_get_info()[0] - free0) < (1 << 20)
    ctx = tq.Context(128, 4, 5, tq.MODE_PROD)   # the library still works
    assert ctx.d == 128


def test_out_of_range_slots_are_reported_and_skipped():
    d, n, cap = 128, 300, 1000
    x = W.round_bf16(W.gaussian((n, d), 4, W.STREAM_KEYS))
    slots = np.random.default_rng(2).permutation(cap)[:n].astype(np.int64)
    bad = slots.copy()
    bad[[5, 77]] = [cap, -3]
    for dtype in (torch.bfloat16, torch.float32):            # fused kernel, workspace path
        ctx = tq.Context(d, 4, 33, tq.MODE_PROD)
        pk = tq.alloc_packed(ctx, cap)
        tq.quantize_kv(ctx, torch.tensor(x, dtype=dtype, device=DEV), pk,
                       slots=torch.tensor(bad, device=DEV))
        torch.cuda.synchronize()
        assert ctx.device_error() == 901
        good = np.setdiff1d(np.arange(n), [5, 77])
        rows = torch.tensor(slots[good], device=DEV)
        parity.check_codes(oracle.make_params(d, 4, 33, 0), x[good].astype(np.float64), pk.codes[rows].cpu().numpy(),
                           pk.norm[rows].float().cpu().numpy(), pk.rnorm[rows].float().cpu().numpy(), "good rows")
        # dequantize with a bad gathered slot: that row is zeros, the others are correct
        g = torch.tensor(np.r_[slots[good][:10], cap + 5], device=DEV)
        out = tq.dequantize(ctx, pk, slots=g)
        torch.cuda.synchronize()
        assert ctx.device_error() == 901
        assert (out[-1] == 0).all()
        assert ctx.device_error() == 0        # the word was cleared by the read


def test_expired_pipeline_wait_winds_down_and_the_context_stays_usable():
    """A wait on a barrier that nothing arrives on (injected into the dequantize kernel)
    gives up after a 1 ms limit, the kernel records error 305 and returns; the next call on
    the same context is correct and reports no error."""
    ctx, pk, x = _small_cache(n=40000)
    ref = tq.dequantize(ctx, pk, 40000)
    torch.cuda.synchronize()
    L = tq.lib()
    L.tq_debug_set_wait_limit(1000000)
    L.tq_debug_inject_stall(1)
    try:
        out = torch.full((40000, 128), 3.0, device=DEV)
        tq.dequantize(ctx, pk, 40000, out=out)
        torch.cuda.synchronize()
    finally:
        L.tq_debug_inject_stall(0)
        L.tq_debug_set_wait_limit(2000000000)
    assert ctx.device_error() == 305
    out = tq.dequantize(ctx, pk, 40000)
    torch.cuda.synchronize()
    assert ctx.device_error() == 0
    assert torch.equal(out, ref)
