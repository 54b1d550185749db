"""fp64 CPU oracle for exact attention, HSTU pointwise attention and the decode step.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference legs of ``bench.py`` may import this package.  It shares no code with the
CUDA path and the product never calls it.

The arithmetic lives in ``oracle.c`` (plain C, IEEE double, OpenMP over rows), which materialises each
score row in full: it is the textbook definition, not a tiled or online computation.  This module only
marshals numpy/torch arrays into it.  ``build()`` compiles it with gcc.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_lib = None


def _host_tag() -> str:
    """A short tag of this host's CPU (model and feature flags).  The library is built for the host it runs on
    (-march=native), so a copy built on another machine is never loaded here."""
    import hashlib
    import platform

    ident = platform.machine()
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith(("model name", "flags", "Features", "CPU part")):
                    ident += line
                    if line.startswith(("flags", "Features")):
                        break
    except OSError:
        pass
    return hashlib.sha256(ident.encode()).hexdigest()[:12]


_LIB = os.path.join(_HERE, f"liboracle-{_host_tag()}.so")


def build(force: bool = False) -> str:
    """Compile oracle.c into a library for this host (gcc -O3 -march=native, OpenMP).  The arithmetic stays
    strict IEEE double in source order: no -ffast-math, and -ffp-contract=off so that no multiply-add is
    fused, which makes the results identical to any other conforming build."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O3", "-march=native", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        i = ctypes.c_int
        lib.oracle_attn.restype = ctypes.c_int64
        lib.oracle_attn.argtypes = [dp, dp, dp, i, i, i, i, ctypes.c_double, i, ip, i, dp, dp]
        lib.oracle_attn_varlen.restype = ctypes.c_int64
        lib.oracle_attn_varlen.argtypes = [dp, dp, dp, ip, i, i, i, ctypes.c_double, i, dp, dp]
        lib.oracle_hstu_jagged.restype = ctypes.c_int64
        lib.oracle_hstu_jagged.argtypes = [dp, dp, dp, ip, i, i, i, ctypes.c_double, ctypes.c_double, dp]
        lib.oracle_decode.restype = ctypes.c_int64
        lib.oracle_decode.argtypes = [dp, dp, dp, ip, i, i, i, i, ctypes.c_double, dp, dp]
        lib.oracle_decode_paged.restype = ctypes.c_int64
        lib.oracle_decode_paged.argtypes = [dp, dp, dp, ip, ip, i, i, i, i, i, i, ctypes.c_double, dp, dp]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        lib.oracle_set_num_threads.restype = None
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Widen a torch tensor (any float dtype, any device) or array to a C-contiguous float64 array."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x) -> np.ndarray:
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.int32).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _dp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _ip(a):
    if a is None:
        return ctypes.POINTER(ctypes.c_int)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads of later calls (n <= 0: the OpenMP default).  Timing only; results do not depend on it."""
    _load().oracle_set_num_threads(int(n))


def attn(q, k, v, scale: float, causal: bool, rows=None, return_flops: bool = False):
    """Softmax attention of [B,H,N,d] tensors.  Returns (o [B,H,R,d], lse [B,H,R]) as float64 arrays,
    R = N or len(rows).  ``scale`` is used exactly as given (pass the float32 value the GPU uses)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    assert k.shape == (B, H, N, d) and v.shape == (B, H, N, d)
    r = None if rows is None else _i32(rows)
    R = N if r is None else len(r)
    o = np.zeros((B, H, R, d), np.float64)
    lse = np.zeros((B, H, R), np.float64)
    fl = _load().oracle_attn(_dp(q), _dp(k), _dp(v), B, H, N, d, float(scale), int(bool(causal)), _ip(r), R,
                             _dp(o), _dp(lse))
    return (o, lse, int(fl)) if return_flops else (o, lse)


def attn_varlen(q, k, v, cu_seqlens, scale: float, causal: bool, return_flops: bool = False):
    """Packed attention: q,k,v [T,H,d], cu_seqlens int [S+1].  Returns (o [T,H,d], lse [T,H])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    cu = _i32(cu_seqlens)
    T, H, d = q.shape
    S = len(cu) - 1
    assert cu[0] == 0 and cu[-1] == T
    o = np.zeros((T, H, d), np.float64)
    lse = np.zeros((T, H), np.float64)
    fl = _load().oracle_attn_varlen(_dp(q), _dp(k), _dp(v), _ip(cu), S, H, d, float(scale), int(bool(causal)),
                                    _dp(o), _dp(lse))
    return (o, lse, int(fl)) if return_flops else (o, lse)


def hstu_jagged(q, k, v, cu_seqlens, alpha: float, inv_n: float):
    """HSTU pointwise attention over packed sequences.  Returns o [T,H,d] (float64)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    cu = _i32(cu_seqlens)
    T, H, d = q.shape
    S = len(cu) - 1
    assert cu[0] == 0 and cu[-1] == T
    o = np.zeros((T, H, d), np.float64)
    _load().oracle_hstu_jagged(_dp(q), _dp(k), _dp(v), _ip(cu), S, H, d, float(alpha), float(inv_n), _dp(o))
    return o


def decode(q, kcache, vcache, kv_lens, scale: float):
    """Single-query decode: q [B,H,d], caches [B,H,Lmax,d], kv_lens [B].  Returns (o [B,H,d], lse [B,H])."""
    q, kc, vc = _f64(q), _f64(kcache), _f64(vcache)
    lens = _i32(kv_lens)
    B, H, Lmax, d = kc.shape
    assert q.shape == (B, H, d) and vc.shape == kc.shape and lens.shape == (B,)
    assert int(lens.max(initial=0)) <= Lmax and int(lens.min(initial=0)) >= 0
    o = np.zeros((B, H, d), np.float64)
    lse = np.zeros((B, H), np.float64)
    _load().oracle_decode(_dp(q), _dp(kc), _dp(vc), _ip(lens), B, H, Lmax, d, float(scale), _dp(o), _dp(lse))
    return o, lse


def decode_paged(q, k_pages, v_pages, block_table, kv_lens, scale: float):
    """Decode over a paged cache with grouped query heads: q [B,Hq,d], page pools [num_pages,Hkv,page_size,d],
    block_table [B,max_pages], kv_lens [B].  Returns (o [B,Hq,d], lse [B,Hq])."""
    q, kp, vp = _f64(q), _f64(k_pages), _f64(v_pages)
    bt = _i32(block_table)
    lens = _i32(kv_lens)
    num_pages, Hkv, page_size, d = kp.shape
    B, Hq, dq = q.shape
    max_pages = bt.shape[1]
    assert dq == d and vp.shape == kp.shape and bt.shape == (B, max_pages) and lens.shape == (B,)
    assert Hq % Hkv == 0
    assert int(lens.min(initial=0)) >= 0 and int(lens.max(initial=0)) <= max_pages * page_size
    for b in range(B):  # the pages a sequence uses must exist
        used = bt[b, : (int(lens[b]) + page_size - 1) // page_size]
        assert used.size == 0 or (int(used.min()) >= 0 and int(used.max()) < num_pages)
    o = np.zeros((B, Hq, d), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    _load().oracle_decode_paged(_dp(q), _dp(kp), _dp(vp), _ip(bt), _ip(lens), B, Hq, Hkv, page_size, max_pages, d,
                                float(scale), _dp(o), _dp(lse))
    return o, lse
