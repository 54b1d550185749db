"""attn_fwd (dense prefill) against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import exact_tiled_attention_43_b200 as eta
import oracle
from exact_tiled_attention_43_b200 import inputs
from parity import check_lse, check_o

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_tiny_config(causal, out_dtype):
    """B=1, H=2, N=256, d=64, every output element compared."""
    q, k, v = (t.to(DEV) for t in inputs.dense_qkv(inputs.TINY, 1, 2, 256, 64))
    scale = eta.default_scale(64)
    o, lse = eta.attn_fwd(q, k, v, causal=causal, scale=scale, out_dtype=out_dtype)
    assert eta.status() == 0
    o_ref, lse_ref = oracle.attn(q, k, v, scale, causal)
    check_o(o, o_ref, f"tiny causal={causal}")
    check_lse(lse, lse_ref, "tiny lse")


@pytest.mark.parametrize("d", [64, 96, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 17, 127, 128, 129, 255, 256, 257, 700])
def test_ragged_lengths(d, causal, N):
    B, H = 2, 3
    q, k, v = (t.to(DEV) for t in inputs.dense_qkv(7, B, H, N, d))
    scale = eta.default_scale(d)
    o, lse = eta.attn_fwd(q, k, v, causal=causal, scale=scale)
    assert eta.status() == 0
    o_ref, lse_ref = oracle.attn(q, k, v, scale, causal)
    check_o(o, o_ref, f"N={N} d={d} causal={causal}")
    check_lse(lse, lse_ref, "lse")


def test_no_lse_and_custom_scale():
    q, k, v = (t.to(DEV) for t in inputs.dense_qkv(8, 1, 2, 300, 128))
    o, none = eta.attn_fwd(q, k, v, causal=True, scale=0.05, return_lse=False)
    assert none is None
    o_ref, _ = oracle.attn(q, k, v, 0.05, True)
    check_o(o, o_ref, "scale=0.05")


def test_large_score_magnitudes():
    """Scaled scores of order 1e2 exercise the running-max rescale path (and its threshold)."""
    q, k, v = (t.to(DEV) for t in inputs.dense_qkv(9, 1, 2, 640, 64))
    q = (q.float() * 8).to(torch.bfloat16)
    k = (k.float() * 4).to(torch.bfloat16)
    for causal in (False, True):
        o, lse = eta.attn_fwd(q, k, v, causal=causal)
        assert eta.status() == 0
        o_ref, lse_ref = oracle.attn(q, k, v, eta.default_scale(64), causal)
        check_o(o, o_ref, "large scores")
        check_lse(lse, lse_ref, "large scores lse")


def _sampled_rows(N):
    rows = {0, 1, 127, 128, 129, 255, 256, N // 2, N - 129, N - 128, N - 2, N - 1}
    rng = np.random.default_rng(0)
    rows |= set(int(r) for r in rng.integers(0, N, 20))
    return sorted(r for r in rows if 0 <= r < N)


@pytest.mark.parametrize("causal", [False, True])
def test_prefill_d64_full_config(causal):
    """Prefill MHA B=1, H=32, N=4096, d=64 in the benchmark's launch configuration: every output element and
    every lse of all 32 heads compared with the oracle."""
    B, H, N, d = 1, 32, 4096, 64
    q, k, v = inputs.dense_qkv(inputs.PREFILL_D64, B, H, N, d, device=DEV)
    scale = eta.default_scale(d)
    o, lse = eta.attn_fwd(q, k, v, causal=causal, scale=scale)
    assert eta.status() == 0
    o_ref, lse_ref = oracle.attn(q, k, v, scale, causal)
    check_o(o, o_ref, f"B1 H32 N4096 d64 causal={causal}")
    check_lse(lse, lse_ref, "B1 H32 N4096 d64 lse")


def test_prefill_d128_full_config():
    """Prefill MHA B=8, H=32, N=4096, d=128, causal -- the benchmark's headline launch -- with every
    (batch, head), every row and every lse compared with the oracle (one batch index at a time, to bound the
    host memory of the fp64 copies).  At this size the launch takes its 256 units in 16 scheduling groups
    of 16 and its 4096 items from the persistent counter."""
    B, H, N, d = 8, 32, 4096, 128
    q, k, v = inputs.dense_qkv(inputs.PREFILL_D128, B, H, N, d, device=DEV)
    scale = eta.default_scale(d)
    o, lse = eta.attn_fwd(q, k, v, causal=True, scale=scale)
    assert eta.status() == 0
    assert eta.prefill_sched_group(B * H, N, d) == 16
    for b in range(B):
        sl = lambda x: x[b:b + 1]
        o_ref, lse_ref = oracle.attn(sl(q), sl(k), sl(v), scale, True)
        check_o(sl(o), o_ref, f"B8 H32 N4096 d128 b={b}")
        check_lse(sl(lse), lse_ref, f"B8 H32 N4096 d128 lse b={b}")


@pytest.mark.parametrize("causal", [False, True])
def test_grouped_schedule_ragged_last_group(causal):
    """Dense launch whose units do not fit in one scheduling group: B=2, H=40, N=2048, d=128 gives 1 MiB of
    K/V per unit, groups of 32 units -- 32, 32 and a last group of 16 -- and 640 items on the persistent
    grid.  Every row compared."""
    B, H, N, d = 2, 40, 2048, 128
    assert eta.prefill_sched_group(B * H, N, d) == 32
    q, k, v = (t.to(DEV) for t in inputs.dense_qkv(15, B, H, N, d))
    scale = eta.default_scale(d)
    o, lse = eta.attn_fwd(q, k, v, causal=causal, scale=scale)
    assert eta.status() == 0
    o_ref, lse_ref = oracle.attn(q, k, v, scale, causal)
    check_o(o, o_ref, f"grouped causal={causal}")
    check_lse(lse, lse_ref, "grouped lse")


def _sweep_rows(N, n=64):
    """n query rows of an N-row sequence: the first and last rows, the rows on both sides of the first, the
    middle and the last tile boundaries, and seeded random rows up to n."""
    rows = {0, 1, 127, 128, 129, 255, 256, N // 2 - 1, N // 2, N - 129, N - 128, N - 2, N - 1}
    rng = np.random.default_rng(N)
    while len(rows) < n:
        rows.add(int(rng.integers(0, N)))
    return sorted(r for r in rows if 0 <= r < N)


@pytest.mark.parametrize("N", [1024, 8192, 32768])
def test_prefill_d128_sweep(N):
    """N sweep at B=1, H=32, d=128, causal, in the benchmark's launch configuration: 64 rows of every head
    (rows are independent, so a row set checks the launch as a whole), every output element and lse of those
    rows compared with the oracle."""
    q, k, v = inputs.dense_qkv(inputs.PREFILL_D128, 1, 32, N, 128, device=DEV)
    scale = eta.default_scale(128)
    o, lse = eta.attn_fwd(q, k, v, causal=True, scale=scale)
    assert eta.status() == 0
    rows = _sweep_rows(N)
    assert len(rows) == 64
    for h in range(32):
        sl = lambda x: x[:, h:h + 1]
        o_ref, lse_ref = oracle.attn(sl(q), sl(k), sl(v), scale, True, rows=rows)
        check_o(sl(o)[:, :, rows], o_ref, f"sweep N={N} h={h}")
        check_lse(sl(lse)[:, :, rows], lse_ref, "sweep lse")


@pytest.mark.parametrize("d", [64, 96, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_more_items_than_sms(d, causal):
    """B*H*blocks well above the SM count: persistent CTAs take several items each (of unequal work when
    causal), and every output row is compared."""
    B, H, N = 2, 40, 1000  # 80 heads x 4 blocks = 320 items
    q, k, v = (t.to(DEV) for t in inputs.dense_qkv(11, B, H, N, d))
    scale = eta.default_scale(d)
    o, lse = eta.attn_fwd(q, k, v, causal=causal, scale=scale)
    assert eta.status() == 0
    o_ref, lse_ref = oracle.attn(q, k, v, scale, causal)
    check_o(o, o_ref, f"items>SMs d={d} causal={causal}")
    check_lse(lse, lse_ref, "items>SMs lse")


@pytest.mark.parametrize("d", [64, 96, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 32, 1024), (1, 16, 1500), (1, 8, 2048), (3, 1, 700)])
def test_split_all_items(d, causal, shape):
    """Launches too small to fill the GPU split every item (one Q tile, its keys -- up to the diagonal when
    causal -- halved between the warpgroups; a Q tile that sees one key tile stays whole): causal ones with
    no more items than SMs, non-causal ones with at most half as many.  (1,32,1024): 128 items (non-causal:
    whole); (1,16,1500): 96, ragged; (1,8,2048): 64; (3,1,700): 9, ragged.  Every row compared, fp32
    output."""
    B, H, N = shape
    q, k, v = (t.to(DEV) for t in inputs.dense_qkv(14, B, H, N, d))
    scale = eta.default_scale(d)
    o, lse = eta.attn_fwd(q, k, v, causal=causal, scale=scale, out_dtype=torch.float32)
    assert eta.status() == 0
    o_ref, lse_ref = oracle.attn(q, k, v, scale, causal)
    check_o(o, o_ref, f"split all {shape} d={d} causal={causal}")
    check_lse(lse, lse_ref, "split all lse")


def test_repeated_launches_on_two_streams():
    """Hundreds of launches in a row, alternating between two streams, reuse every work-counter slot more
    than once: each result must be bit-identical to the first (an item's arithmetic does not depend on
    which CTA runs it)."""
    q, k, v = (t.to(DEV) for t in inputs.dense_qkv(12, 1, 6, 700, 64))
    ref, ref_lse = eta.attn_fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = []
    for i in range(600):
        s = streams[i % 2]
        with torch.cuda.stream(s):
            o = torch.empty_like(ref)
            lse = torch.empty_like(ref_lse)
            eta.attn_fwd(q, k, v, causal=True, out=o, lse=lse, stream=s)
            if i % 50 == 0:
                outs.append((o, lse))
    torch.cuda.synchronize()
    assert eta.status() == 0
    for o, lse in outs:
        assert torch.equal(o, ref)
        assert torch.equal(lse, ref_lse)


@pytest.mark.parametrize("d", [64, 96, 128])
@pytest.mark.parametrize("shape", [(1, 20, 2000), (1, 160, 200), (2, 74, 1000)])
def test_split_tail_items(d, shape):
    """Non-causal launches whose last wave is at most half full split those items: one Q tile each, keys
    halved between the CTA's two softmax warpgroups and merged in the CTA.  (1,20,2000): 160 items, 12 split
    into halves of 8 key tiles; (1,160,200): 12 split items of 2 key tiles, the second ragged; (2,74,1000):
    592 items = 4 full waves, none split.  Every row compared, in fp32 output."""
    B, H, N = shape
    q, k, v = (t.to(DEV) for t in inputs.dense_qkv(13, B, H, N, d))
    scale = eta.default_scale(d)
    o, lse = eta.attn_fwd(q, k, v, causal=False, scale=scale, out_dtype=torch.float32)
    assert eta.status() == 0
    o_ref, lse_ref = oracle.attn(q, k, v, scale, False)
    check_o(o, o_ref, f"split tail {shape} d={d}")
    check_lse(lse, lse_ref, "split tail lse")


def test_same_buffers_different_shapes_back_to_back():
    """The C ABI caches TMA tensor maps per host thread, keyed by buffer address and shape.  One storage viewed
    as [1, 2, 512, 64] and then as [1, 4, 256, 64] (same base pointers, other sizes) must be mapped afresh each
    time: both results equal the oracle, and repeating the first call after the second gives it again."""
    base = [t.to(DEV) for t in inputs.dense_qkv(18, 1, 2, 512, 64)]
    views_a = [t for t in base]
    views_b = [t.view(1, 4, 256, 64) for t in base]
    for causal in (False, True):
        oa, la = eta.attn_fwd(*views_a, causal=causal)
        ob, lb = eta.attn_fwd(*views_b, causal=causal)
        oa2, la2 = eta.attn_fwd(*views_a, causal=causal)
        assert eta.status() == 0
        ra = oracle.attn(*views_a, eta.default_scale(64), causal)
        rb = oracle.attn(*views_b, eta.default_scale(64), causal)
        check_o(oa, ra[0], "shape A")
        check_lse(la, ra[1], "shape A lse")
        check_o(ob, rb[0], "shape B")
        check_lse(lb, rb[1], "shape B lse")
        assert torch.equal(oa, oa2) and torch.equal(la, la2)
