"""Python binding of libtq (TurboQuant hot path on B200), argument marshalling only.

Every computation runs in libtq.so's CUDA kernels; PyTorch provides device memory and
streams.  There is no fallback: if libtq.so has not been built this module raises on
first use (build it with ``python -m kv_cache_vector_08_b200.build``).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

__all__ = [
    "MODE_PROD", "MODE_MSE", "TQError", "Context", "Packed", "host_params", "alloc_packed",
    "quantize_kv", "quantize_workspace_size", "channel_perm_by_score", "dequantize", "prepare_queries", "attn_logits", "decode_attention",
    "decode_workspace_size", "search_topk", "launch_count", "lib_path", "lib",
]

MODE_PROD = 0
MODE_MSE = 1
DTYPE_F32, DTYPE_BF16, DTYPE_F16 = 0, 1, 2

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libtq.so")
_lib = None


class TQError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__("libtq status %d: %s" % (status, msg))
        self.status = status


class _Packed(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("norm", ctypes.c_void_p), ("rnorm", ctypes.c_void_p),
                ("cap", ctypes.c_int64)]


class _DecodeOpts(ctypes.Structure):
    _fields_ = [("channel_perm", ctypes.c_void_p), ("block_table", ctypes.c_void_p), ("page_tokens", ctypes.c_int)]


class _Info(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("bits", ctypes.c_int), ("k", ctypes.c_int), ("m", ctypes.c_int),
                ("mode", ctypes.c_int), ("planes", ctypes.c_int), ("d_pad", ctypes.c_int),
                ("code_bytes", ctypes.c_int), ("seed", ctypes.c_uint64)]


def lib_path() -> str:
    return _LIB_PATH


def lib():
    """Load libtq.so (raises if it is missing: there is no other implementation)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError("libtq.so not built at %s; run python -m kv_cache_vector_08_b200.build" % _LIB_PATH)
    L = ctypes.CDLL(_LIB_PATH)
    P, I, I64, U64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t
    F = ctypes.c_float
    PK = ctypes.POINTER(_Packed)
    sig = {
        "tq_init": (I, [ctypes.POINTER(P), I, I, U64, I]),
        "tq_host_params": (I, [I, I, U64, I, P, P, P, P]),
        "tq_free": (None, [P]),
        "tq_get_info": (I, [P, ctypes.POINTER(_Info)]),
        "tq_get_params": (I, [P, P, P, P, P]),
        "tq_quantize_workspace_size": (SZ, [P, I, I64, I64]),
        "tq_quantize_kv": (I, [P, P, I, I64, I64, PK, P, P, SZ, P]),
        "tq_dequantize": (I, [P, PK, P, I64, P, I64, P]),
        "tq_dequantize_qjl": (I, [P, PK, P, I64, P, I64, P]),
        "tq_prepare_queries": (I, [P, P, I64, I64, P, P]),
        "tq_attn_logits_workspace_size": (SZ, [P, I64]),
        "tq_attn_logits": (I, [P, P, I64, PK, I64, P, P, SZ, P]),
        "tq_decode_workspace_size": (SZ, [I, I, I, I, I, I64]),
        "tq_decode_attention": (I, [P, P, P, I, P, I, PK, PK, P, I, I, I, I, I64, F, P, P, SZ, P]),
        "tq_decode_attention_ex": (I, [P, P, P, I, P, I, PK, PK, P, I, I, I, I, I64, F, P, ctypes.POINTER(_DecodeOpts),
                                       P, SZ, P]),
        "tq_channel_perm_by_score": (I, [P, I, I, P]),
        "tq_quantize_cols_workspace_size": (SZ, [P, I64]),
        "tq_quantize_kv_cols": (I, [P, P, I, I64, I64, P, PK, P, P, SZ, P]),
        "tq_search_workspace_size": (SZ, [P, I64, I64, I]),
        "tq_search_topk": (I, [P, P, I64, PK, I64, I, P, P, P, SZ, P]),
        "tq_last_error": (ctypes.c_char_p, []),
        "tq_kernel_launch_count": (U64, []),
        "tq_get_device_error": (I, [P, ctypes.POINTER(I)]),
        "tq_debug_set_wait_limit": (I, [U64]),
        "tq_debug_inject_stall": (I, [I]),
        "tq_debug_fail_alloc": (I, [I]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _check(status: int):
    if status != 0:
        raise TQError(status, lib().tq_last_error().decode())


def launch_count() -> int:
    return int(lib().tq_kernel_launch_count())


def _torch():
    import torch
    return torch


def _stream(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _dtype_code(t) -> int:
    torch = _torch()
    codes = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16, torch.float16: DTYPE_F16}
    if t.dtype not in codes:
        raise TypeError("unsupported dtype %s" % t.dtype)
    return codes[t.dtype]


def _rows(t, d: int):
    """(pointer, n, ld) of a 2-D tensor whose rows are unit-stride with >= d elements."""
    if t.dim() != 2 or t.stride(1) != 1 or t.shape[1] < d:
        raise ValueError("expected a 2-D tensor [n, >=%d] with unit stride along rows" % d)
    return t.shape[0], max(t.stride(0), d)


def host_params(d: int, bits: int, seed: int, mode: int) -> dict:
    """The library's float64 parameters computed on the host (no GPU needed)."""
    k = bits - 1 if mode == MODE_PROD else bits
    Pi = np.zeros((d, d))
    S = np.zeros((d, d)) if mode == MODE_PROD else None
    c = np.zeros(2 ** k) if k >= 1 else np.zeros(1)
    t = np.zeros(max(2 ** k - 1, 1))
    p = lambda a: None if a is None else a.ctypes.data_as(ctypes.c_void_p)
    _check(lib().tq_host_params(d, bits, seed, mode, p(Pi), p(S), p(c), p(t)))
    return dict(Pi=Pi, S=S, centroids=c, boundaries=t[:2 ** k - 1])


class Context:
    """Owns one libtq context (Pi, S, codebook on the current CUDA device)."""

    def __init__(self, d: int, bits: int, seed: int, mode: int = MODE_PROD):
        h = ctypes.c_void_p()
        _check(lib().tq_init(ctypes.byref(h), d, bits, seed, mode))
        self._h = h
        info = _Info()
        _check(lib().tq_get_info(h, ctypes.byref(info)))
        self.d, self.bits, self.k, self.m, self.mode = info.d, info.bits, info.k, info.m, info.mode
        self.planes, self.d_pad, self.code_bytes, self.seed = info.planes, info.d_pad, info.code_bytes, info.seed

    @property
    def handle(self):
        return self._h

    def params(self) -> dict:
        d, K = self.d, 2 ** self.k
        Pi = np.zeros((d, d))
        S = np.zeros((d, d)) if self.mode == MODE_PROD else None
        c = np.zeros(K)
        t = np.zeros(max(K - 1, 1))
        p = lambda a: None if a is None else a.ctypes.data_as(ctypes.c_void_p)
        _check(lib().tq_get_params(self._h, p(Pi), p(S), p(c), p(t)))
        return dict(Pi=Pi, S=S, centroids=c, boundaries=t[:K - 1], mode=self.mode, k=self.k, m=self.m, d=d)

    def device_error(self) -> int:
        """Kernel-side failure code recorded for this context (0 = none); clears it."""
        v = ctypes.c_int(0)
        _check(lib().tq_get_device_error(self._h, ctypes.byref(v)))
        return v.value

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            lib().tq_free(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


@dataclass
class Packed:
    """Caller-owned packed storage: codes [cap, code_bytes] uint8, norm [cap] fp16,
    rnorm [cap] fp16 (prod mode) -- all torch CUDA tensors."""
    codes: object
    norm: object
    rnorm: Optional[object]

    @property
    def cap(self) -> int:
        return self.codes.shape[0]

    def struct(self) -> _Packed:
        return _Packed(self.codes.data_ptr(), self.norm.data_ptr(),
                       0 if self.rnorm is None else self.rnorm.data_ptr(), self.codes.shape[0])


def alloc_packed(ctx: Context, cap: int, device=None) -> Packed:
    torch = _torch()
    device = device or torch.device("cuda", torch.cuda.current_device())
    codes = torch.zeros((cap, ctx.code_bytes), dtype=torch.uint8, device=device)
    norm = torch.zeros(cap, dtype=torch.float16, device=device)
    rnorm = torch.zeros(cap, dtype=torch.float16, device=device) if ctx.mode == MODE_PROD else None
    return Packed(codes, norm, rnorm)


def quantize_workspace_size(ctx: Context, x_dtype: int, n: int, ld: int) -> int:
    return int(lib().tq_quantize_workspace_size(ctx.handle, x_dtype, n, ld))


def quantize_kv(ctx: Context, x, dst: Packed, slots=None, stream=None, workspace=None, cols=None):
    """Quantize rows of x (CUDA tensor [n, >=d], fp32/bf16/fp16) into dst (slot v, or slots[v]).
    cols (CUDA int32 [d]): quantize the columns cols of each row of x instead of its first d.
    A workspace is allocated (torch caching allocator) when the call needs one and none is given."""
    torch = _torch()
    dt = _dtype_code(x)
    ps = dst.struct()
    if cols is not None:
        if x.dim() != 2 or x.stride(1) != 1:
            raise ValueError("expected a 2-D tensor with unit stride along rows")
        n, ld = x.shape[0], x.stride(0)
        need = int(lib().tq_quantize_cols_workspace_size(ctx.handle, n))
        if workspace is None and need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
        _check(lib().tq_quantize_kv_cols(ctx.handle, _ptr(x), dt, n, ld, _ptr(cols), ctypes.byref(ps), _ptr(slots),
                                         _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                         _stream(stream)))
        return
    n, ld = _rows(x, ctx.d)
    need = quantize_workspace_size(ctx, dt, n, ld)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    _check(lib().tq_quantize_kv(ctx.handle, _ptr(x), dt, n, ld, ctypes.byref(ps), _ptr(slots), _ptr(workspace),
                                0 if workspace is None else workspace.numel(), _stream(stream)))


def channel_perm_by_score(score, w0: int) -> np.ndarray:
    """Host permutation putting the w0 highest-scoring channels first (see tq.h)."""
    score = np.ascontiguousarray(score, dtype=np.float32)
    perm = np.zeros(score.shape[0], dtype=np.int32)
    _check(lib().tq_channel_perm_by_score(score.ctypes.data_as(ctypes.c_void_p), score.shape[0], int(w0),
                                          perm.ctypes.data_as(ctypes.c_void_p)))
    return perm


def dequantize(ctx: Context, src: Packed, n: int = None, slots=None, out=None, stream=None, qjl: bool = False):
    """x_hat = norm Pi^T c[idx] of stored vectors (qjl=True, prod mode: plus the QJL term
    norm sqrt(pi/2)/m rnorm S^T (2 s - 1))."""
    torch = _torch()
    if slots is not None:
        n = slots.shape[0]
    if out is None:
        out = torch.empty((n, ctx.d), dtype=torch.float32, device=src.codes.device)
    ps = src.struct()
    fn = lib().tq_dequantize_qjl if qjl else lib().tq_dequantize
    _check(fn(ctx.handle, ctypes.byref(ps), _ptr(slots), n, _ptr(out), out.stride(0), _stream(stream)))
    return out


def prepare_queries(ctx: Context, q, out=None, stream=None):
    torch = _torch()
    nq, ld = _rows(q, ctx.d)
    if out is None:
        out = torch.empty((nq, ctx.d + ctx.m), dtype=torch.float32, device=q.device)
    _check(lib().tq_prepare_queries(ctx.handle, _ptr(q), nq, ld, _ptr(out), _stream(stream)))
    return out


def attn_logits(ctx: Context, q, keys: Packed, n: int, out=None, workspace=None, stream=None):
    torch = _torch()
    q = q.contiguous()
    nq = q.shape[0]
    if out is None:
        out = torch.empty((nq, n), dtype=torch.float32, device=q.device)
    need = int(lib().tq_attn_logits_workspace_size(ctx.handle, nq))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    ps = keys.struct()
    _check(lib().tq_attn_logits(ctx.handle, _ptr(q), nq, ctypes.byref(ps), n, _ptr(out), _ptr(workspace),
                                workspace.numel(), _stream(stream)))
    return out


def decode_workspace_size(B, Hq, Hkv, D, ngroups, max_len) -> int:
    return int(lib().tq_decode_workspace_size(B, Hq, Hkv, D, ngroups, max_len))


class DecodePlan:
    """Pre-marshalled arguments of tq_decode_attention (avoids per-call ctypes setup)."""

    def __init__(self, kctx: Sequence[Context], vctx: Sequence[Context], group_off: Sequence[int],
                 kcache: Sequence[Packed], vcache: Sequence[Packed], B, Hq, Hkv, D, max_len, device=None,
                 channel_perm=None, block_table=None, page_tokens: int = 0):
        torch = _torch()
        # options: channel_perm CUDA int32 [Hkv, D]; block_table CUDA int32 [B, max_len / page_tokens]
        self._opts = None
        if channel_perm is not None or block_table is not None:
            self._opts = _DecodeOpts(0 if channel_perm is None else channel_perm.data_ptr(),
                                     0 if block_table is None else block_table.data_ptr(), int(page_tokens))
            self._keep_opts = (channel_perm, block_table)
        G = len(kctx)
        self.G, self.B, self.Hq, self.Hkv, self.D, self.max_len = G, B, Hq, Hkv, D, max_len
        self._k = (ctypes.c_void_p * G)(*[c.handle.value for c in kctx])
        self._v = (ctypes.c_void_p * G)(*[c.handle.value for c in vctx])
        self._off = (ctypes.c_int * (G + 1))(*list(group_off))
        self._kc = (_Packed * G)(*[p.struct() for p in kcache])
        self._vc = (_Packed * G)(*[p.struct() for p in vcache])
        self._keep = (kctx, vctx, kcache, vcache)
        need = decode_workspace_size(B, Hq, Hkv, D, G, max_len)
        device = device or kcache[0].codes.device
        self.workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=device)

    def __call__(self, q, seq_lens, scale: float, out, stream=None):
        if self._opts is not None:
            _check(lib().tq_decode_attention_ex(self._k, self._v, self._off, self.G, _ptr(q), _dtype_code(q), self._kc,
                                                self._vc, _ptr(seq_lens), self.B, self.Hq, self.Hkv, self.D,
                                                self.max_len, ctypes.c_float(scale), _ptr(out), ctypes.byref(self._opts),
                                                _ptr(self.workspace), self.workspace.numel(), _stream(stream)))
            return out
        _check(lib().tq_decode_attention(self._k, self._v, self._off, self.G, _ptr(q), _dtype_code(q), self._kc,
                                         self._vc, _ptr(seq_lens), self.B, self.Hq, self.Hkv, self.D,
                                         self.max_len, ctypes.c_float(scale), _ptr(out), _ptr(self.workspace),
                                         self.workspace.numel(), _stream(stream)))
        return out


def decode_attention(kctx, vctx, group_off, q, kcache, vcache, seq_lens, Hkv, max_len, scale, out=None,
                     stream=None, channel_perm=None, block_table=None, page_tokens=0):
    """One decode step; q [B, Hq, D] (fp32/bf16 CUDA), seq_lens int32 CUDA [B] -> out fp32 [B, Hq, D].
    Token t of sequence b, kv head h lives in slot (b*Hkv + h)*max_len + t of each cache."""
    torch = _torch()
    B, Hq, D = q.shape
    plan = DecodePlan(kctx, vctx, group_off, kcache, vcache, B, Hq, Hkv, D, max_len, device=q.device,
                      channel_perm=channel_perm, block_table=block_table, page_tokens=page_tokens)
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
    return plan(q.contiguous(), seq_lens, scale, out, stream)


def search_topk(ctx: Context, q, db: Packed, N: int, k: int, stream=None):
    torch = _torch()
    q = q.contiguous()
    nq = q.shape[0]
    scores = torch.empty((nq, k), dtype=torch.float32, device=q.device)
    ids = torch.empty((nq, k), dtype=torch.int64, device=q.device)
    need = int(lib().tq_search_workspace_size(ctx.handle, nq, N, k))
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    ps = db.struct()
    _check(lib().tq_search_topk(ctx.handle, _ptr(q), nq, ctypes.byref(ps), N, k, _ptr(scores), _ptr(ids),
                                _ptr(ws), ws.numel(), _stream(stream)))
    return scores, ids
