"""attn_fwd_fp8 (e4m3 Q, K, V with per-tensor descales; P rounded to e4m3 for P.V) against the fp64 oracle on the
dequantised inputs, through the C ABI.

Tolerance, derived from the arithmetic: the products q8*k8 and p8*v8 are exact and accumulated in fp32, so the
error is the rounding of P to e4m3 -- at most 2^-4 of P in e4m3's normal range and 2^-10 (in units of the row's
largest P, which is >= 1) in its subnormal range -- giving per output element
    |O - O_ref| <= 2^-4 sum_j p_j |v_j| + 2^-10 sum_j |v_j| / l + (output rounding) + 1e-5,
with p the exact softmax row, l = sum_j e^(s_j - max s) >= 1, and output rounding 2^-8 |O_ref| for bf16.
The first two terms are computed here in fp64 from the dequantised inputs."""
import numpy as np
import pytest
import torch

import exact_tiled_attention_43_b200 as eta
import oracle
from exact_tiled_attention_43_b200 import inputs
from parity import check_lse

pytestmark = pytest.mark.gpu
DEV = "cuda"
D = 128


def _deq(x8, s):
    return x8.to(torch.float64).cpu().numpy() * s


def _fp8_bound(Q, K, V, scale, causal, rows=None):
    """Per element 2^-4 P|V| + 2^-10 sum|V| / l for the selected rows (fp64, textbook softmax)."""
    B, H, N, d = Q.shape
    rows = np.arange(N) if rows is None else np.asarray(rows)
    S = scale * (Q[:, :, rows] @ np.swapaxes(K, -1, -2))
    if causal:
        S = np.where(np.arange(N)[None, None, None, :] <= rows[None, None, :, None], S, -np.inf)
    m = S.max(axis=-1, keepdims=True)
    E = np.exp(S - m)
    l = E.sum(axis=-1, keepdims=True)
    P = E / l
    A = P @ np.abs(V)
    Bs = (E > 0).astype(np.float64) @ np.abs(V)
    return 2.0 ** -4 * A + 2.0 ** -10 * Bs / l


def _check(o, o_ref, bound, out_bf16, what):
    o = o.double().cpu().numpy()
    tol = bound + (2.0 ** -8 * np.abs(o_ref) if out_bf16 else 0.0) + 1e-5
    err = np.abs(o - o_ref)
    assert np.all(np.isfinite(o)), what
    worst = np.unravel_index(int(np.argmax(err - tol)), err.shape)
    assert np.all(err <= tol), f"{what}: err {err[worst]:.3e} > bound {tol[worst]:.3e} at {worst}"


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 17, 128, 129, 300, 700])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_fp8_ragged(causal, N, out_dtype):
    q8, k8, v8, (dq, dk, dv) = inputs.fp8_dense_qkv(inputs.PREFILL_FP8, 2, 3, N, D)
    scale = eta.default_scale(D)
    o, lse = eta.attn_fwd_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), dq, dk, dv, causal=causal, scale=scale,
                              out_dtype=out_dtype)
    Q, K, V = _deq(q8, dq), _deq(k8, dk), _deq(v8, dv)
    o_ref, lse_ref = oracle.attn(Q, K, V, scale, causal)
    _check(o, o_ref, _fp8_bound(Q, K, V, scale, causal), out_dtype == torch.bfloat16, f"fp8 N={N} causal={causal}")
    check_lse(lse, lse_ref, "fp8 lse")


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_more_items_than_sms_and_split_tail(causal):
    """B1 H20 N2000: 160 items on the persistent grid (non-causal: the last 12 split across warpgroups)."""
    q8, k8, v8, (dq, dk, dv) = inputs.fp8_dense_qkv(inputs.PREFILL_FP8, 1, 20, 2000, D)
    scale = eta.default_scale(D)
    o, lse = eta.attn_fwd_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), dq, dk, dv, causal=causal, scale=scale,
                              out_dtype=torch.float32)
    Q, K, V = _deq(q8, dq), _deq(k8, dk), _deq(v8, dv)
    o_ref, lse_ref = oracle.attn(Q, K, V, scale, causal)
    _check(o, o_ref, _fp8_bound(Q, K, V, scale, causal), False, "fp8 items")
    check_lse(lse, lse_ref, "fp8 items lse")


def test_fp8_benchmark_config():
    """B8 H32 N4096 causal (the benchmark's FP8 line): 64 rows (first, last, tile boundaries, seeded random)
    of every (batch, head) compared with the oracle on the dequantised inputs, within the bound derived
    from the e4m3 rounding of P."""
    B, H, N = 8, 32, 4096
    q8, k8, v8, (dq, dk, dv) = inputs.fp8_dense_qkv(inputs.PREFILL_FP8, B, H, N, D, device=DEV)
    scale = eta.default_scale(D)
    o, lse = eta.attn_fwd_fp8(q8, k8, v8, dq, dk, dv, causal=True, scale=scale)
    assert eta.status() == 0
    rng = np.random.default_rng(7)
    rows = {0, 1, 127, 128, 129, 255, 256, 2047, 2048, 4094, 4095}
    while len(rows) < 64:
        rows.add(int(rng.integers(0, N)))
    rows = sorted(rows)
    for b, h in ((b, h) for b in range(B) for h in range(H)):
        sl = lambda x, s: _deq(x[b:b + 1, h:h + 1], s)
        Q, K, V = sl(q8, dq), sl(k8, dk), sl(v8, dv)
        o_ref, lse_ref = oracle.attn(Q, K, V, scale, True, rows=rows)
        _check(o[b:b + 1, h:h + 1, rows], o_ref, _fp8_bound(Q, K, V, scale, True, rows), True, f"fp8 b={b} h={h}")
        check_lse(lse[b:b + 1, h:h + 1, rows], lse_ref, "fp8 config lse")
