"""attn_fwd_varlen and hstu_fwd_jagged (packed sequences) against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import exact_tiled_attention_43_b200 as eta
import oracle
from exact_tiled_attention_43_b200 import inputs
from parity import check_hstu, check_lse, check_o

pytestmark = pytest.mark.gpu
DEV = "cuda"
EDGE_LENS = [1, 127, 128, 129, 0, 255, 256, 257, 300, 2]


@pytest.mark.parametrize("d", [64, 96, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_varlen_edge_lengths(d, causal):
    cu = inputs.cu_seqlens(EDGE_LENS)
    T, H = int(cu[-1]), 3
    q, k, v = (t.to(DEV) for t in inputs.jagged_qkv(11, T, H, d))
    scale = eta.default_scale(d)
    o, lse = eta.attn_fwd_varlen(q, k, v, cu.to(DEV), max(EDGE_LENS), causal=causal, scale=scale)
    assert eta.status() == 0
    o_ref, lse_ref = oracle.attn_varlen(q, k, v, cu, scale, causal)
    check_o(o, o_ref, f"varlen d={d} causal={causal}")
    check_lse(lse, lse_ref, "varlen lse")


def test_varlen_equals_dense_for_one_sequence():
    q, k, v = (t.to(DEV) for t in inputs.dense_qkv(12, 1, 4, 777, 64))
    od, ld = eta.attn_fwd(q, k, v, causal=True)
    pk = lambda x: x[0].transpose(0, 1).contiguous()
    cu = torch.tensor([0, 777], dtype=torch.int32, device=DEV)
    ov, lv = eta.attn_fwd_varlen(pk(q), pk(k), pk(v), cu, 777, causal=True)
    assert torch.equal(ov, pk(od)) and torch.equal(lv, ld[0].t())


def test_varlen_bad_cu_seqlens_sets_status():
    q, k, v = (t.to(DEV) for t in inputs.jagged_qkv(13, 300, 1, 64))
    cu = torch.tensor([0, 200, 100, 300], dtype=torch.int32, device=DEV)
    eta.attn_fwd_varlen(q, k, v, cu, 300)
    assert eta.status() == eta.ETA_DEV_BAD_CUSEQ
    cu = torch.tensor([0, 300], dtype=torch.int32, device=DEV)
    eta.attn_fwd_varlen(q, k, v, cu, 256)  # a sequence longer than max_len
    assert eta.status() == eta.ETA_DEV_BAD_CUSEQ


@pytest.mark.parametrize("d", [64, 96, 128])
@pytest.mark.parametrize("inv_n", [1.0 / 4096, 1.0])
def test_hstu_edge_lengths(d, inv_n):
    cu = inputs.cu_seqlens(EDGE_LENS)
    T, H = int(cu[-1]), 2
    q, k, v = (t.to(DEV) for t in inputs.jagged_qkv(inputs.HSTU_JAGGED, T, H, d, std=0.5))
    alpha = 1.0 / np.sqrt(d)
    o = eta.hstu_fwd_jagged(q, k, v, cu.to(DEV), max(EDGE_LENS), alpha, inv_n)
    assert eta.status() == 0
    o_ref = oracle.hstu_jagged(q, k, v, cu, alpha, inv_n)
    check_hstu(o, o_ref, f"hstu d={d} inv_n={inv_n}")


def test_hstu_full_config():
    """HSTU jagged: 16 sequences, H=4, d=64, lengths U[256, 4096], N(0, 0.5^2) inputs, alpha = 1/sqrt(d),
    n = 4096 -- every output element compared."""
    lens = inputs.uniform_lengths(inputs.HSTU_JAGGED, 16, 256, 4096)
    cu = inputs.cu_seqlens(lens)
    T = int(cu[-1])
    q, k, v = inputs.jagged_qkv(inputs.HSTU_JAGGED, T, 4, 64, std=0.5, device=DEV)
    o = eta.hstu_fwd_jagged(q, k, v, cu.to(DEV), 4096, 0.125, 1.0 / 4096)
    assert eta.status() == 0
    o_ref = oracle.hstu_jagged(q, k, v, cu, 0.125, 1.0 / 4096)
    check_hstu(o, o_ref, "hstu jagged 16 seqs H4 d64")


@pytest.mark.parametrize("N", [4096, 8192])
def test_hstu_dense_page_shape_sampled(N):
    """HSTU at the page's dense shape (16 sequences x 4 heads, every sequence N long, d = 64, n = N); the GPU
    result of two sequences (first and last) and two heads is compared with the oracle run on them alone."""
    S, H, d = 16, 4, 64
    lens = [N] * S
    cu = inputs.cu_seqlens(lens)
    q, k, v = inputs.jagged_qkv(inputs.HSTU_JAGGED, S * N, H, d, std=0.5, device=DEV)
    o = eta.hstu_fwd_jagged(q, k, v, cu.to(DEV), N, 0.125, 1.0 / N)
    assert eta.status() == 0
    for s in (0, S - 1):
        a, b = s * N, (s + 1) * N
        heads = [0, 3] if N == 4096 else [2]
        sub = lambda x: x[a:b, heads].contiguous()
        o_ref = oracle.hstu_jagged(sub(q), sub(k), sub(v), [0, N], 0.125, 1.0 / N)
        check_hstu(sub(o), o_ref, f"hstu dense N={N} seq={s}")


def _vp(t):
    import ctypes

    return ctypes.c_void_p(t.data_ptr() if t is not None else 0)


SENTINEL = 7.0  # never an attention output here (|o| <= max |v| < 7 for these inputs, HSTU outputs ~1e-2)


@pytest.mark.parametrize("kind,d", [("varlen", 64), ("varlen", 128), ("varlen", 256), ("hstu", 64), ("hstu", 96)])
@pytest.mark.parametrize("tail", ["past_end", "short", "negative_start"])
def test_cu_seqlens_checked_against_T_total(kind, d, tail):
    """The packed kernels read cu_seqlens on the device and check it against the T_total the call was given.
    The q/k/v/o/lse buffers hold T_total rows followed by 64 guard rows; the offset table is broken in one
    of three ways:
      past_end       : the last offset is 100 rows past T_total -> that sequence is skipped;
      short          : the last offset is 60 rows short of T_total -> in bounds, every sequence computed;
      negative_start : the first offset is -5 -> the first sequence is skipped.
    Each records ETA_DEV_BAD_CUSEQ; every computed sequence matches the oracle; skipped sequences, rows past
    the table's end and the guard rows keep their sentinel value."""
    H, T, G = 2, 420, 64
    bounds = {"past_end": [0, 200, T + 100], "short": [0, 200, T - 60], "negative_start": [-5, 200, T]}[tail]
    computed = {"past_end": [(0, 200)], "short": [(0, 200), (200, T - 60)], "negative_start": [(200, T)]}[tail]
    q, k, v = (t.to(DEV) for t in inputs.jagged_qkv(16, T + G, H, d, std=0.5 if kind == "hstu" else 1.0))
    o = torch.full((T + G, H, d), SENTINEL, dtype=torch.bfloat16, device=DEV)
    lse = torch.full((T + G, H), SENTINEL, dtype=torch.float32, device=DEV)
    cu = torch.tensor(bounds, dtype=torch.int32, device=DEV)
    L = eta.lib()
    st = eta._stream_ptr()
    max_len = 320
    scale = eta.default_scale(d)
    if kind == "varlen":
        rc = L.attn_fwd_varlen(_vp(q), _vp(k), _vp(v), _vp(o), _vp(lse), _vp(cu), 2, max_len, T, H, d, scale, 1,
                               eta.ETA_OUT_BF16, st)
    else:
        rc = L.hstu_fwd_jagged(_vp(q), _vp(k), _vp(v), _vp(o), _vp(cu), 2, max_len, T, H, d, 0.125, 1.0 / 256, st)
    assert rc == 0
    assert eta.status() == eta.ETA_DEV_BAD_CUSEQ
    written = torch.zeros(T + G, dtype=torch.bool)
    for a, b in computed:
        written[a:b] = True
        sub = lambda x: x[a:b].contiguous()
        if kind == "varlen":
            o_ref, lse_ref = oracle.attn_varlen(sub(q), sub(k), sub(v), [0, b - a], scale, True)
            check_o(sub(o), o_ref, f"{kind} d={d} {tail} [{a},{b})")
            check_lse(sub(lse), lse_ref, "lse")
        else:
            o_ref = oracle.hstu_jagged(sub(q), sub(k), sub(v), [0, b - a], 0.125, 1.0 / 256)
            check_hstu(sub(o), o_ref, f"{kind} d={d} {tail} [{a},{b})")
    untouched = ~written
    assert torch.all(o.cpu()[untouched] == SENTINEL), "rows outside the computed sequences were written"
    assert torch.all(lse.cpu()[untouched] == SENTINEL), "lse rows outside the computed sequences were written"


@pytest.mark.parametrize("d", [64, 96])
@pytest.mark.parametrize("big_rows", [False, True])
def test_hstu_tanh_on_both_pipes(big_rows, d):
    """At d = 64 and 96 the HSTU tanh of 3 in every 8 pairs runs on the FMA pipe (a polynomial valid for
    |y| <= 1, y = alpha s / 2) when every row of a warp stays in that range, else the warp keeps every tanh on
    the MUFU.  With alpha = 1/8 and N(0, 0.5^2) inputs every warp takes the mixed loop (|y| stays below ~0.7
    at d = 96); with big_rows the query rows 300..599 of the first sequence are scaled by 8 (exact in
    bf16), so |y| reaches ~4 there and those warps -- and the rows of warps straddling the boundary -- take
    the MUFU loop in the same launch."""
    lens = [700, 260]
    cu = inputs.cu_seqlens(lens)
    T, H = int(cu[-1]), 2
    q, k, v = (t.to(DEV) for t in inputs.jagged_qkv(17, T, H, d, std=0.5))
    if big_rows:
        q[300:600] = (q[300:600].float() * 8).to(torch.bfloat16)
    o = eta.hstu_fwd_jagged(q, k, v, cu.to(DEV), max(lens), 0.125, 1.0 / 256)
    assert eta.status() == 0
    o_ref = oracle.hstu_jagged(q, k, v, cu, 0.125, 1.0 / 256)
    check_hstu(o, o_ref, f"hstu tanh pipes d={d} big_rows={big_rows}")
