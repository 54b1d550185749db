"""exact_tiled_attention_43_b200 -- fused exact attention forward passes for B200 (sm_100a).

Thin Python binding over the C ABI of ``libeta.so`` (declared in ``include/eta.h``).  Every function
here only marshals arguments: it checks dtypes/shapes/devices, allocates outputs with torch (device memory
is torch's job here) and passes raw pointers plus the current CUDA stream to the library, where every step
of the computation runs in hand-written kernels.  There is no fallback: if ``libeta.so`` is missing or the
device is not an sm_100 GPU, calls raise.

Entry points (names follow the C ABI):
  attn_fwd(q, k, v, causal, scale)                     dense [B,H,N,d] softmax attention -> (o, lse)
  attn_fwd_varlen(q, k, v, cu_seqlens, max_len, ...)   packed [T,H,d] sequences          -> (o, lse)
  hstu_fwd_jagged(q, k, v, cu_seqlens, max_len, alpha, inv_n)   HSTU pointwise attention -> o
  attn_decode(q, kcache, vcache, kv_lens, scale)       one-query decode over a KV cache  -> (o, lse)
"""
from __future__ import annotations

import contextlib
import ctypes
import functools
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libeta.so")
_lib = None

ETA_OUT_BF16, ETA_OUT_F32 = 0, 1
ETA_DEV_OK, ETA_DEV_TIMEOUT, ETA_DEV_BAD_KVLEN, ETA_DEV_BAD_CUSEQ, ETA_DEV_BAD_PAGE = 0, 1, 2, 3, 4

# name -> (restype, argtypes); mirrors include/eta.h
_VP, _I, _F, _SZ, _LL = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_longlong
SIGNATURES = {
    "attn_fwd": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _I, _I, _VP]),
    "attn_fwd_varlen": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _I, _I, _VP]),
    "hstu_fwd_jagged": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _F, _VP]),
    "attn_decode_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "attn_decode": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _VP, _SZ, _VP]),
    "attn_decode_noalloc": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _VP]),
    "attn_decode_paged_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "attn_fwd_fp8": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _F, _F, _F, _I, _I, _VP]),
    "attn_decode_paged": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _F, _VP, _SZ, _VP]),
    "eta_status": (_I, [_VP]),
    "eta_strerror": (ctypes.c_char_p, [_I]),
    "eta_set_wait_timeout_ns": (None, [_LL]),
    "eta_selftest_wait_timeout": (_I, [_VP]),
    "eta_prefill_plan": (_I, [_I, _LL, _LL, _I, _I, _I, ctypes.POINTER(ctypes.c_longlong),
                              ctypes.POINTER(ctypes.c_longlong), ctypes.POINTER(ctypes.c_int)]),
    "eta_prefill_sched_group": (_LL, [_LL, _LL, _I, _I]),
}


class EtaError(RuntimeError):
    pass


def lib():
    """Loads libeta.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise EtaError(f"{LIB_PATH} is missing: build it with `python -m exact_tiled_attention_43_b200.build` "
                           "(or __graft_entry__.build()); there is no fallback implementation")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


PLAN_KINDS = {"dense": 0, "varlen": 1, "hstu": 2}


def prefill_plan(kind: str, units: int, rows: int, d: int, causal: bool, sms: int):
    """The work decomposition a prefill call would launch on a GPU with `sms` SMs (host logic, no GPU):
    (work items, items run whole, CTAs of the persistent grid).  kind: "dense", "varlen" or "hstu";
    units = B*H or S*H; rows = N or max_len."""
    items, whole, ctas = ctypes.c_longlong(), ctypes.c_longlong(), ctypes.c_int()
    rc = lib().eta_prefill_plan(PLAN_KINDS[kind], int(units), int(rows), int(d), int(bool(causal)), int(sms),
                                ctypes.byref(items), ctypes.byref(whole), ctypes.byref(ctas))
    _check(rc, "eta_prefill_plan")
    return items.value, whole.value, ctas.value


def prefill_sched_group(units: int, rows: int, d: int, elt_bytes: int = 2) -> int:
    """(batch, head) units a dense prefill launch schedules together so that their K/V stay in L2 (host logic,
    no GPU)."""
    g = int(lib().eta_prefill_sched_group(int(units), int(rows), int(d), int(elt_bytes)))
    _check(g if g < 0 else 0, "eta_prefill_sched_group")
    return g


def strerror(code: int) -> str:
    return lib().eta_strerror(int(code)).decode()


def _check(rc: int, what: str):
    if rc != 0:
        raise EtaError(f"{what} failed: {strerror(rc)} (code {rc})")


def _torch():
    import torch

    return torch


def _stream_ptr(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _need(t, name, dtype, ndim):
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _same_device(ref, *tensors):
    for name, t in tensors:
        if t is not None and t.device != ref.device:
            raise ValueError(f"{name} is on {t.device}, expected {ref.device} (all tensors of a call on one GPU)")


def _check_buf(t, name, shape, dtypes, device):
    """A caller-provided output or workspace: the kernels write exactly `shape` elements of one of `dtypes`
    through its pointer, so anything else is refused before a launch could write past it."""
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} must be one of {dtypes}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _device_ctx(t):
    """Makes t's GPU current for the call, so that the library and the default stream are t's (nothing to
    switch when it is current already, the usual case)."""
    torch = _torch()
    if t.device.index is None or t.device.index == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(t.device)


@functools.lru_cache(maxsize=None)
def default_scale(d: int) -> float:
    """The float32 value of 1/sqrt(d)."""
    import numpy as np

    return float(np.float32(1.0 / math.sqrt(d)))


def attn_fwd(q, k, v, causal: bool = False, scale: float | None = None, out_dtype=None, out=None, lse=None,
             return_lse: bool = True, stream=None):
    """Dense exact attention: q, k, v bf16 [B,H,N,d].  Returns (o [B,H,N,d], lse fp32 [B,H,N] or None)."""
    torch = _torch()
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, torch.bfloat16, 4)
    B, H, N, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape")
    _same_device(q, ("k", k), ("v", v))
    out_dtype = out_dtype or torch.bfloat16
    if out is None:
        out = torch.empty((B, H, N, d), dtype=out_dtype, device=q.device)
    _check_buf(out, "out", (B, H, N, d), (torch.bfloat16, torch.float32), q.device)
    if return_lse and lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if return_lse:
        _check_buf(lse, "lse", (B, H, N), (torch.float32,), q.device)
    scale = default_scale(d) if scale is None else float(scale)
    odt = ETA_OUT_F32 if out.dtype == torch.float32 else ETA_OUT_BF16
    with _device_ctx(q):
        rc = lib().attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse if return_lse else None), B, H, N, d,
                            scale, int(bool(causal)), odt, _stream_ptr(stream))
    _check(rc, "attn_fwd")
    return out, (lse if return_lse else None)


def attn_fwd_fp8(q8, k8, v8, q_descale: float, k_descale: float, v_descale: float, causal: bool = False,
                 scale: float | None = None, out_dtype=None, out=None, lse=None, return_lse: bool = True,
                 stream=None):
    """Exact attention on e4m3 inputs: q8, k8, v8 torch.float8_e4m3fn [B,H,N,128] with per-tensor descale
    factors (Q = q8 * q_descale, ...).  Returns (o [B,H,N,128] bf16 or fp32, lse fp32 [B,H,N] or None)."""
    torch = _torch()
    for t, name in ((q8, "q8"), (k8, "k8"), (v8, "v8")):
        _need(t, name, torch.float8_e4m3fn, 4)
    if k8.shape != q8.shape or v8.shape != q8.shape:
        raise ValueError("q8, k8, v8 must have the same shape")
    B, H, N, d = q8.shape
    _same_device(q8, ("k8", k8), ("v8", v8))
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16 if out_dtype is None else out_dtype, device=q8.device)
    _check_buf(out, "out", (B, H, N, d), (torch.bfloat16, torch.float32), q8.device)
    odt = ETA_OUT_F32 if out.dtype == torch.float32 else ETA_OUT_BF16
    if lse is None and return_lse:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device)
    if not return_lse:
        lse = None
    if lse is not None:
        _check_buf(lse, "lse", (B, H, N), (torch.float32,), q8.device)
    scale = default_scale(d) if scale is None else float(scale)
    with _device_ctx(q8):
        rc = lib().attn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(out), _ptr(lse), B, H, N, d, scale,
                                float(q_descale), float(k_descale), float(v_descale), int(bool(causal)), odt,
                                _stream_ptr(stream))
    _check(rc, "attn_fwd_fp8")
    return out, lse


def attn_fwd_varlen(q, k, v, cu_seqlens, max_len: int, causal: bool = False, scale: float | None = None,
                    out_dtype=None, return_lse: bool = True, stream=None):
    """Packed exact attention: q, k, v bf16 [T,H,d], cu_seqlens int32 [S+1] (device).
    Returns (o [T,H,d], lse fp32 [T,H] or None)."""
    torch = _torch()
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, torch.bfloat16, 3)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    T, H, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape")
    _same_device(q, ("k", k), ("v", v), ("cu_seqlens", cu_seqlens))
    out = torch.empty((T, H, d), dtype=out_dtype or torch.bfloat16, device=q.device)
    lse = torch.empty((T, H), dtype=torch.float32, device=q.device) if return_lse else None
    scale = default_scale(d) if scale is None else float(scale)
    odt = ETA_OUT_F32 if out.dtype == torch.float32 else ETA_OUT_BF16
    with _device_ctx(q):
        rc = lib().attn_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens),
                                   cu_seqlens.numel() - 1, int(max_len), T, H, d, scale, int(bool(causal)), odt,
                                   _stream_ptr(stream))
    _check(rc, "attn_fwd_varlen")
    return out, lse


def hstu_fwd_jagged(q, k, v, cu_seqlens, max_len: int, alpha: float, inv_n: float, out=None, stream=None):
    """HSTU pointwise attention over packed sequences: q, k, v bf16 [T,H,d] -> o bf16 [T,H,d]."""
    torch = _torch()
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, torch.bfloat16, 3)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    T, H, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape")
    _same_device(q, ("k", k), ("v", v), ("cu_seqlens", cu_seqlens))
    if out is None:
        out = torch.empty((T, H, d), dtype=torch.bfloat16, device=q.device)
    _check_buf(out, "out", (T, H, d), (torch.bfloat16,), q.device)
    with _device_ctx(q):
        rc = lib().hstu_fwd_jagged(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(cu_seqlens), cu_seqlens.numel() - 1,
                                   int(max_len), T, H, d, float(alpha), float(inv_n), _stream_ptr(stream))
    _check(rc, "hstu_fwd_jagged")
    return out


def attn_decode_workspace_size(B: int, H: int, Lmax: int, d: int) -> int:
    return int(lib().attn_decode_workspace_size(B, H, Lmax, d))


def attn_decode(q, kcache, vcache, kv_lens, scale: float | None = None, workspace=None, out=None, lse=None,
                stream=None):
    """One decode step: q bf16 [B,H,d], caches bf16 [B,H,Lmax,d], kv_lens int32 [B] (device).
    Returns (o bf16 [B,H,d], lse fp32 [B,H])."""
    torch = _torch()
    _need(q, "q", torch.bfloat16, 3)
    _need(kcache, "kcache", torch.bfloat16, 4)
    _need(vcache, "vcache", torch.bfloat16, 4)
    _need(kv_lens, "kv_lens", torch.int32, 1)
    B, H, Lmax, d = kcache.shape
    if vcache.shape != kcache.shape or q.shape != (B, H, d) or kv_lens.shape != (B,):
        raise ValueError("inconsistent decode shapes")
    _same_device(q, ("kcache", kcache), ("vcache", vcache), ("kv_lens", kv_lens))
    need = attn_decode_workspace_size(B, H, Lmax, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check_buf(workspace, "workspace", None, (workspace.dtype,), q.device)
    if out is None:
        out = torch.empty((B, H, d), dtype=torch.bfloat16, device=q.device)
    _check_buf(out, "out", (B, H, d), (torch.bfloat16,), q.device)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    _check_buf(lse, "lse", (B, H), (torch.float32,), q.device)
    scale = default_scale(d) if scale is None else float(scale)
    with _device_ctx(q):
        rc = lib().attn_decode(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(kv_lens), _ptr(out), _ptr(lse), B, H, Lmax,
                               d, scale, _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _stream_ptr(stream))
    _check(rc, "attn_decode")
    return out, lse


def attn_decode_paged_workspace_size(B: int, Hq: int, max_pages: int, page_size: int, d: int) -> int:
    return int(lib().attn_decode_paged_workspace_size(B, Hq, max_pages, page_size, d))


def attn_decode_paged(q, k_pages, v_pages, block_table, kv_lens, scale: float | None = None, workspace=None,
                      out=None, lse=None, stream=None):
    """Decode step with grouped query heads over a paged cache: q bf16 [B,Hq,d], page pools bf16
    [num_pages,Hkv,page_size,d], block_table int32 [B,max_pages] and kv_lens int32 [B] (device).
    Query head hq reads kv head hq // (Hq // Hkv).  Returns (o bf16 [B,Hq,d], lse fp32 [B,Hq])."""
    torch = _torch()
    _need(q, "q", torch.bfloat16, 3)
    _need(k_pages, "k_pages", torch.bfloat16, 4)
    _need(v_pages, "v_pages", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(kv_lens, "kv_lens", torch.int32, 1)
    num_pages, Hkv, page_size, d = k_pages.shape
    B, Hq, dq = q.shape
    max_pages = block_table.shape[1]
    if v_pages.shape != k_pages.shape or dq != d or block_table.shape[0] != B or kv_lens.shape != (B,):
        raise ValueError("inconsistent paged decode shapes")
    _same_device(q, ("k_pages", k_pages), ("v_pages", v_pages), ("block_table", block_table), ("kv_lens", kv_lens))
    need = attn_decode_paged_workspace_size(B, Hq, max_pages, page_size, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _check_buf(workspace, "workspace", None, (workspace.dtype,), q.device)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q.device)
    _check_buf(out, "out", (B, Hq, d), (torch.bfloat16,), q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _check_buf(lse, "lse", (B, Hq), (torch.float32,), q.device)
    scale = default_scale(d) if scale is None else float(scale)
    with _device_ctx(q):
        rc = lib().attn_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(kv_lens),
                                     _ptr(out), _ptr(lse), B, Hq, Hkv, num_pages, page_size, max_pages, d, scale,
                                     _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _stream_ptr(stream))
    _check(rc, "attn_decode_paged")
    return out, lse


NOALLOC_SCRATCH_BYTES = 8 << 20  # ETA_NOALLOC_SCRATCH_BYTES


def attn_decode_noalloc(q, kcache, vcache, kv_lens, scale: float | None = None, out=None, lse=None, stream=None):
    """attn_decode without a workspace: the library's fixed device scratch (NOALLOC_SCRATCH_BYTES) holds the
    split partials, for callers that cannot allocate device memory at call time.  Calls whose GPU work
    overlaps race on that shared scratch; the first call on a device should precede any stream capture."""
    torch = _torch()
    _need(q, "q", torch.bfloat16, 3)
    _need(kcache, "kcache", torch.bfloat16, 4)
    _need(vcache, "vcache", torch.bfloat16, 4)
    _need(kv_lens, "kv_lens", torch.int32, 1)
    B, H, Lmax, d = kcache.shape
    if vcache.shape != kcache.shape or q.shape != (B, H, d) or kv_lens.shape != (B,):
        raise ValueError("inconsistent decode shapes")
    _same_device(q, ("kcache", kcache), ("vcache", vcache), ("kv_lens", kv_lens))
    if out is None:
        out = torch.empty((B, H, d), dtype=torch.bfloat16, device=q.device)
    _check_buf(out, "out", (B, H, d), (torch.bfloat16,), q.device)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    _check_buf(lse, "lse", (B, H), (torch.float32,), q.device)
    scale = default_scale(d) if scale is None else float(scale)
    with _device_ctx(q):
        rc = lib().attn_decode_noalloc(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(kv_lens), _ptr(out), _ptr(lse), B,
                                       H, Lmax, d, scale, _stream_ptr(stream))
    _check(rc, "attn_decode_noalloc")
    return out, lse


def status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device status word (ETA_DEV_*)."""
    rc = lib().eta_status(_stream_ptr(stream))
    if rc < 0:
        raise EtaError(f"eta_status failed: {strerror(rc)}")
    return rc


def set_wait_timeout_ns(ns: int):
    lib().eta_set_wait_timeout_ns(int(ns))


def selftest_wait_timeout(stream=None):
    _check(lib().eta_selftest_wait_timeout(_stream_ptr(stream)), "eta_selftest_wait_timeout")
