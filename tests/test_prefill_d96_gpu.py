"""attn_fwd at head dimension 96 (rows of 192 bytes: one full 128-byte swizzle chunk plus a half chunk that
the TMA zero-fills) against the fp64 oracle, through the C ABI.  The shared ragged-length, varlen, HSTU,
split-tail and many-items cases also run at d = 96 (parametrized in the other prefill test files)."""
import pytest
import torch

import exact_tiled_attention_43_b200 as eta
import oracle
from exact_tiled_attention_43_b200 import inputs
from parity import check_lse, check_o

pytestmark = pytest.mark.gpu
DEV = "cuda"
D = 96


@pytest.mark.parametrize("causal", [False, True])
def test_d96_fp32_output_and_large_scores(causal):
    """fp32 O, and scores scaled up so that the running-max rescale of the 96-column O fires."""
    q, k, v = (t.to(DEV) for t in inputs.dense_qkv(26, 1, 2, 520, D))
    q = (q.float() * 6).to(torch.bfloat16)
    scale = eta.default_scale(D)
    o, lse = eta.attn_fwd(q, k, v, causal=causal, scale=scale, out_dtype=torch.float32)
    assert eta.status() == 0
    o_ref, lse_ref = oracle.attn(q, k, v, scale, causal)
    check_o(o, o_ref, "d96 large scores")
    check_lse(lse, lse_ref, "d96 large scores lse")


def test_d96_columns_past_the_head_dim_are_not_read():
    """Rows are packed with no padding, so the half chunk past column 96 of a row lies over the next row
    (for the last row of a head: the next head's first row).  The MMAs read only columns below 96 (Q K^T
    stops after six 16-column steps, P V has N = 96), so NaN in the next head cannot reach this head."""
    q, k, v = (t.to(DEV) for t in inputs.dense_qkv(27, 1, 2, 256, D))
    for t in (q, k, v):
        t[:, 1] = float("nan")
    o, lse = eta.attn_fwd(q, k, v, causal=False)
    assert eta.status() == 0
    o_ref, lse_ref = oracle.attn(q[:, :1], k[:, :1], v[:, :1], eta.default_scale(D), False)
    check_o(o[:, :1], o_ref, "d96 next head NaN")
    check_lse(lse[:, :1], lse_ref, "d96 next head NaN lse")


def test_d96_benchmark_config():
    """B=8, H=32, N=4096, d=96 causal (the benchmark's d=96 line): every element and lse of every (batch,
    head) compared with the oracle, one batch index at a time."""
    B, H, N = 8, 32, 4096
    q, k, v = inputs.dense_qkv(28, B, H, N, D, device=DEV)
    scale = eta.default_scale(D)
    o, lse = eta.attn_fwd(q, k, v, causal=True, scale=scale)
    assert eta.status() == 0
    for b in range(B):
        sl = lambda x: x[b:b + 1]
        o_ref, lse_ref = oracle.attn(sl(q), sl(k), sl(v), scale, True)
        check_o(sl(o), o_ref, f"d96 config b={b}")
        check_lse(sl(lse), lse_ref, "d96 config lse")
