"""tq_decode_attention_static: decode attention for callers that cannot allocate device
memory (for example a plug-in whose host engine owns all device memory, or a serving loop
that may not call cudaMalloc on the decode path).  Its scratch is a fixed array inside the
library; these checks call it through the C ABI and compare it with tq_decode_attention,
which takes a caller workspace.  Collected last so a failure here never hides another."""
import ctypes
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import kv_cache_vector_08_b200 as tq  # noqa: E402
import parity  # noqa: E402

DEV = torch.device("cuda", 0)
STATIC_BYTES = 8 << 20


def _fn():
    L = tq.lib()
    f = L.tq_decode_attention_static
    P, I, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    PK = ctypes.POINTER(tq._Packed)
    f.restype = I
    f.argtypes = [P, P, P, I, P, I, PK, PK, P, I, I, I, I, I64, ctypes.c_float, P, P]
    return f


def _case(B, Hkv, Hq, D, groups, seq_lens, max_len, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    K = torch.randn((B * Hkv * max_len, D), generator=g, device=DEV).to(torch.bfloat16)
    V = torch.randn((B * Hkv * max_len, D), generator=g, device=DEV).to(torch.bfloat16)
    q = torch.randn((B, Hq, D), generator=g, device=DEV).to(torch.bfloat16)
    kctx, vctx, kc, vc = [], [], [], []
    for gi, (off, w, kb, vb) in enumerate(groups):
        kx = tq.Context(w, kb, 1000 + 2 * gi, tq.MODE_PROD)
        vx = tq.Context(w, vb, 1001 + 2 * gi, tq.MODE_MSE)
        kp = tq.alloc_packed(kx, B * Hkv * max_len)
        vp = tq.alloc_packed(vx, B * Hkv * max_len)
        tq.quantize_kv(kx, K[:, off:off + w], kp)
        tq.quantize_kv(vx, V[:, off:off + w], vp)
        kctx.append(kx); vctx.append(vx); kc.append(kp); vc.append(vp)
    offs = [g_[0] for g_ in groups] + [D]
    seq = torch.tensor(seq_lens, dtype=torch.int32, device=DEV)
    return kctx, vctx, offs, q, kc, vc, seq


def _call_static(plan, q, seq, scale, out):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return _fn()(plan._k, plan._v, plan._off, plan.G, ctypes.c_void_p(q.data_ptr()), 1, plan._kc, plan._vc,
                 ctypes.c_void_p(seq.data_ptr()), plan.B, plan.Hq, plan.Hkv, plan.D, plan.max_len,
                 ctypes.c_float(scale), ctypes.c_void_p(out.data_ptr()), stream)


@pytest.mark.parametrize("groups,B,seq_lens,max_len", [
    (((0, 128, 4, 4),), 1, [4000], 4096),
    (((0, 64, 4, 4), (64, 64, 3, 3)), 3, [1000, 0, 77], 1024),
])
def test_static_scratch_decode_matches_workspace_decode(groups, B, seq_lens, max_len):
    Hkv, Hq, D = 8, 32, 128
    kctx, vctx, offs, q, kc, vc, seq = _case(B, Hkv, Hq, D, groups, seq_lens, max_len, 5)
    assert tq.decode_workspace_size(B, Hq, Hkv, D, len(groups), max_len) <= STATIC_BYTES
    plan = tq.DecodePlan(kctx, vctx, offs, kc, vc, B, Hq, Hkv, D, max_len)
    scale = 1.0 / math.sqrt(D)
    ref = torch.empty((B, Hq, D), dtype=torch.float32, device=DEV)
    plan(q, seq, scale, ref)
    torch.cuda.synchronize()
    for call in range(2):                       # two calls in a row share the array
        out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device=DEV)
        status = _call_static(plan, q, seq, scale, out)
        assert status == 0, tq.lib().tq_last_error()
        torch.cuda.synchronize()
        parity.assert_close(out.cpu().numpy(), ref.cpu().numpy(), "static call %d" % call)


def test_static_scratch_call_allocates_nothing():
    """After a first call (which looks up the array and lets the driver load the kernels),
    a call leaves the device's free memory unchanged."""
    groups = ((0, 128, 4, 4),)
    B, Hkv, Hq, D, max_len = 2, 8, 32, 128, 2048
    kctx, vctx, offs, q, kc, vc, seq = _case(B, Hkv, Hq, D, groups, [2048, 1500], max_len, 7)
    plan = tq.DecodePlan(kctx, vctx, offs, kc, vc, B, Hq, Hkv, D, max_len)
    out = torch.empty((B, Hq, D), dtype=torch.float32, device=DEV)
    assert _call_static(plan, q, seq, 0.1, out) == 0, tq.lib().tq_last_error()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    n0 = tq.launch_count()
    assert _call_static(plan, q, seq, 0.1, out) == 0, tq.lib().tq_last_error()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert tq.launch_count() > n0
    assert free1 == free0, "free device memory changed by %d bytes" % (free0 - free1)


def test_static_scratch_rejects_shapes_above_its_size():
    groups = ((0, 128, 4, 4),)
    B, Hq, Hkv, D, max_len = 512, 64, 8, 128, 16    # prepared queries alone need 32 MiB
    kctx, vctx, offs, q, kc, vc, seq = _case(B, Hkv, Hq, D, groups, [16] * B, max_len, 6)
    assert tq.decode_workspace_size(B, Hq, Hkv, D, 1, max_len) > STATIC_BYTES
    plan = tq.DecodePlan(kctx, vctx, offs, kc, vc, B, Hq, Hkv, D, max_len)
    out = torch.empty((B, Hq, D), dtype=torch.float32, device=DEV)
    torch.cuda.synchronize()
    n0 = tq.launch_count()
    status = _call_static(plan, q, seq, 1.0, out)
    assert status == 5                              # TQ_ERR_WORKSPACE
    assert b"static scratch" in tq.lib().tq_last_error()
    assert tq.launch_count() == n0                  # nothing was launched
    # an invalid shape is reported as such even when it is also too large
    plan.Hq = 63
    assert _call_static(plan, q, seq, 1.0, out) == 1    # TQ_ERR_INVALID_ARG
    assert tq.launch_count() == n0
