"""attn_fwd / attn_fwd_varlen at head dimension 256 (the one-Q-tile-per-item kernel) against the fp64 oracle,
through the C ABI."""
import pytest
import torch

import exact_tiled_attention_43_b200 as eta
import oracle
from exact_tiled_attention_43_b200 import inputs
from parity import check_lse, check_o

pytestmark = pytest.mark.gpu
DEV = "cuda"
D = 256


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 17, 64, 65, 127, 128, 129, 300, 700])
def test_d256_ragged_lengths(causal, N):
    q, k, v = (t.to(DEV) for t in inputs.dense_qkv(21, 2, 3, N, D))
    scale = eta.default_scale(D)
    o, lse = eta.attn_fwd(q, k, v, causal=causal, scale=scale)
    o_ref, lse_ref = oracle.attn(q, k, v, scale, causal)
    check_o(o, o_ref, f"d256 N={N} causal={causal}")
    check_lse(lse, lse_ref, "d256 lse")


@pytest.mark.parametrize("causal", [False, True])
def test_d256_fp32_output_and_large_scores(causal):
    """fp32 O, and scores scaled up so that the running-max rescale (of a 256-column O) fires."""
    q, k, v = (t.to(DEV) for t in inputs.dense_qkv(22, 1, 2, 520, D))
    q = (q.float() * 6).to(torch.bfloat16)
    scale = eta.default_scale(D)
    o, lse = eta.attn_fwd(q, k, v, causal=causal, scale=scale, out_dtype=torch.float32)
    o_ref, lse_ref = oracle.attn(q, k, v, scale, causal)
    check_o(o, o_ref, "d256 large scores")
    check_lse(lse, lse_ref, "d256 large scores lse")


@pytest.mark.parametrize("causal", [False, True])
def test_d256_more_items_than_sms(causal):
    """2 x 40 heads x 8 row blocks = 640 work items of unequal work (causal) on the persistent grid."""
    q, k, v = (t.to(DEV) for t in inputs.dense_qkv(23, 2, 40, 1000, D))
    scale = eta.default_scale(D)
    o, lse = eta.attn_fwd(q, k, v, causal=causal, scale=scale)
    o_ref, lse_ref = oracle.attn(q, k, v, scale, causal)
    check_o(o, o_ref, "d256 items > SMs")
    check_lse(lse, lse_ref, "d256 items > SMs lse")


@pytest.mark.parametrize("causal", [False, True])
def test_d256_varlen_edge_lengths(causal):
    lens = [1, 127, 128, 129, 0, 255, 256, 257, 300, 2]
    cu = inputs.cu_seqlens(lens)
    T = int(cu[-1])
    q, k, v = (t.to(DEV) for t in inputs.jagged_qkv(24, T, 3, D))
    scale = eta.default_scale(D)
    o, lse = eta.attn_fwd_varlen(q, k, v, cu.to(DEV), max(lens), causal=causal, scale=scale)
    o_ref, lse_ref = oracle.attn_varlen(q, k, v, cu, scale, causal)
    check_o(o, o_ref, "d256 varlen")
    check_lse(lse, lse_ref, "d256 varlen lse")


def test_d256_benchmark_config():
    """B=4, H=16, N=4096, d=256 causal (the benchmark's d=256 line): every element and lse of every (batch,
    head) compared with the oracle, one batch index at a time."""
    B, H, N = 4, 16, 4096
    q, k, v = inputs.dense_qkv(25, B, H, N, D, device=DEV)
    scale = eta.default_scale(D)
    o, lse = eta.attn_fwd(q, k, v, causal=True, scale=scale)
    assert eta.status() == 0
    for b in range(B):
        sl = lambda x: x[b:b + 1]
        o_ref, lse_ref = oracle.attn(sl(q), sl(k), sl(v), scale, True)
        check_o(sl(o), o_ref, f"d256 config b={b}")
        check_lse(sl(lse), lse_ref, "d256 config lse")
