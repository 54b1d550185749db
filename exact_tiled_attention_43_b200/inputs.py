"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the oracle.

This module holds no attention arithmetic: it only draws random tensors and lengths and lays them out
(dense ``[B,H,N,d]``, packed ``[T,H,d]`` + ``cu_seqlens``, decode caches ``[B,H,Lmax,d]``, page pools
``[num_pages,Hkv,page_size,d]`` + page tables).

Seeds: ``seed = 1000 * config + {0: q, 1: k, 2: v, 3: lengths}``.  Values are iid normal in fp32,
multiplied by ``std`` and rounded to bf16; lengths are inclusive uniform integer draws.  Tensors are
drawn on ``device`` (a CUDA generator for large shapes), so callers that need host copies take them
from the returned tensors.
"""
from __future__ import annotations

import torch

# Config ids follow the workload list: 1 tiny check, 2 prefill d=64, 3 prefill d=128 (+ N sweep),
# 4 HSTU jagged, 5 decode, 6 decode over a paged cache with grouped query heads, 7 prefill on e4m3 inputs.
TINY, PREFILL_D64, PREFILL_D128, HSTU_JAGGED, DECODE, DECODE_PAGED, PREFILL_FP8 = 1, 2, 3, 4, 5, 6, 7


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, seed: int, std: float = 1.0, device="cpu") -> torch.Tensor:
    """iid N(0, std^2) drawn in fp32, rounded to bf16."""
    x = torch.randn(*shape, generator=_gen(device, seed), device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def dense_qkv(config: int, B: int, H: int, N: int, d: int, std: float = 1.0, device="cpu"):
    """Q, K, V as contiguous bf16 ``[B,H,N,d]``."""
    base = 1000 * config
    return tuple(normal_bf16((B, H, N, d), base + i, std, device) for i in range(3))


def uniform_lengths(config: int, S: int, lo: int, hi: int) -> torch.Tensor:
    """S integer lengths drawn uniformly from [lo, hi] (inclusive); int32 on the host."""
    g = _gen("cpu", 1000 * config + 3)
    return torch.randint(lo, hi + 1, (S,), generator=g, dtype=torch.int64).to(torch.int32)


def cu_seqlens(lengths) -> torch.Tensor:
    """Packed offsets [0, L0, L0+L1, ...] as int32 on the host."""
    lengths = torch.as_tensor(lengths, dtype=torch.int64).cpu()
    cu = torch.zeros(lengths.numel() + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(lengths, 0)
    return cu.to(torch.int32)


def jagged_qkv(config: int, T: int, H: int, d: int, std: float = 1.0, device="cpu"):
    """Packed Q, K, V as contiguous bf16 ``[T,H,d]`` (no padding)."""
    base = 1000 * config
    return tuple(normal_bf16((T, H, d), base + i, std, device) for i in range(3))


def decode_inputs(config: int, B: int, H: int, Lmax: int, d: int, lengths, std: float = 1.0, device="cpu",
                  poison_tail: bool = False):
    """One query per (b,h) ``[B,H,d]`` and K/V caches ``[B,H,Lmax,d]``; rows at or beyond ``lengths[b]``
    are filled with NaN when ``poison_tail`` (so any read past a sequence's end shows up)."""
    base = 1000 * config
    q = normal_bf16((B, H, d), base + 0, std, device)
    kc = normal_bf16((B, H, Lmax, d), base + 1, std, device)
    vc = normal_bf16((B, H, Lmax, d), base + 2, std, device)
    lens = torch.as_tensor(lengths, dtype=torch.int32).cpu()
    if poison_tail:
        for b in range(B):
            L = int(lens[b])
            kc[b, :, L:] = float("nan")
            vc[b, :, L:] = float("nan")
    return q, kc, vc, lens


def paged_decode_inputs(config: int, B: int, Hq: int, Hkv: int, d: int, page_size: int, lengths,
                        std: float = 1.0, spare_pages: int = 3, device="cpu", poison_tail: bool = False):
    """Queries ``[B,Hq,d]``, K/V page pools ``[num_pages,Hkv,page_size,d]`` and a page table ``[B,max_pages]``
    (int32).  Each sequence gets ceil(L/page_size) pages; the pool holds them plus ``spare_pages`` unused
    ones, and which physical page backs which logical page is a seeded random permutation (seed + 4).
    Unused table entries are -1.  With ``poison_tail`` every pool row that no sequence reads (the tail of a
    last page, spare pages) is NaN, so any read past a sequence's end shows up."""
    base = 1000 * config
    lens = torch.as_tensor(lengths, dtype=torch.int32).cpu()
    need = [(int(L) + page_size - 1) // page_size for L in lens]
    max_pages = max(1, max(need))
    num_pages = sum(need) + spare_pages
    q = normal_bf16((B, Hq, d), base + 0, std, device)
    kp = normal_bf16((num_pages, Hkv, page_size, d), base + 1, std, device)
    vp = normal_bf16((num_pages, Hkv, page_size, d), base + 2, std, device)
    perm = torch.randperm(num_pages, generator=_gen("cpu", base + 4))
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    used = torch.zeros(num_pages, dtype=torch.bool)
    nxt = 0
    for b in range(B):
        for i in range(need[b]):
            pg = int(perm[nxt])
            nxt += 1
            table[b, i] = pg
            used[pg] = True
    if poison_tail:
        valid = torch.zeros(num_pages, page_size, dtype=torch.bool)
        for b in range(B):
            L = int(lens[b])
            for i in range(need[b]):
                valid[int(table[b, i]), : min(page_size, L - i * page_size)] = True
        mask = (~valid).to(device)[:, None, :, None].expand(num_pages, Hkv, page_size, d)
        kp[mask] = float("nan")
        vp[mask] = float("nan")
    return q, kp, vp, table, lens


def fp8_dense_qkv(config: int, B: int, H: int, N: int, d: int, std: float = 1.0, device="cpu"):
    """Q, K, V as e4m3 (torch.float8_e4m3fn) ``[B,H,N,d]`` with one descale factor per tensor: iid N(0, std^2)
    values x are divided by amax(|x|) / 448 (the e4m3 maximum) and rounded to e4m3; the factor is returned so
    that x ~ x8 * descale.  Returns (q8, k8, v8, (q_descale, k_descale, v_descale))."""
    base = 1000 * config
    out, scales = [], []
    for i in range(3):
        x = torch.randn(B, H, N, d, generator=_gen(device, base + i), device=device, dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        descale = float(x.abs().max()) / 448.0
        out.append((x / descale).to(torch.float8_e4m3fn))
        scales.append(descale)
    return out[0], out[1], out[2], tuple(scales)
