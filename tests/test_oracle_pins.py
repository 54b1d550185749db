"""Pins for the fp64 oracle, from what the pages and the mathematics fix (no GPU).

Each test ties the oracle to something other than itself: hand-derived closed forms (tests/golden),
invariants of softmax attention, a separately written tiled online-softmax model (the identity the
pages claim), brute-force small cases, the 4 n^2 d FLOP count, and textbook library routines
(torch's fp64 scaled_dot_product_attention, F.silu, matmul) as cross-checks.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_43_b200 import inputs

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _num(x):
    table = {"ln2": math.log(2), "ln3": math.log(3), "-ln3": -math.log(3), "ln4": math.log(4), "ln5": math.log(5),
             "ln8": math.log(8), "0.75*ln3": 0.75 * math.log(3), "-0.25*ln3": -0.25 * math.log(3)}
    if isinstance(x, list):
        return [_num(e) for e in x]
    return table[x] if isinstance(x, str) else float(x)


def _rand(shape, seed, std=1.0):
    return inputs.normal_bf16(shape, seed, std).double().numpy()


# ----------------------------------------------------------------------------------------------
# attention: closed forms and golden fixtures
# ----------------------------------------------------------------------------------------------
def test_golden_attention_n2():
    g = json.load(open(os.path.join(GOLD, "attn_n2_closed_form.json")))
    q = np.array(_num(g["q"]))[None, None]
    k = np.array(_num(g["k"]))[None, None]
    v = np.array(_num(g["v"]))[None, None]
    for mode, causal in (("noncausal", False), ("causal", True)):
        o, lse = oracle.attn(q, k, v, g["scale"], causal)
        np.testing.assert_allclose(o[0, 0], np.array(_num(g[mode]["o"])), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[0, 0], np.array(_num(g[mode]["lse"])), rtol=0, atol=1e-12)


def test_n2_sigmoid_closed_form():
    # N=2, non-causal: o_i = sigma(s_i1 - s_i0) (v1 - v0) + v0, lse_i = logaddexp(s_i0, s_i1)
    q, k, v = (_rand((1, 1, 2, 8), 7 + i) for i in range(3))
    scale = 0.37
    o, lse = oracle.attn(q, k, v, scale, False)
    for i in range(2):
        s0, s1 = scale * q[0, 0, i] @ k[0, 0, 0], scale * q[0, 0, i] @ k[0, 0, 1]
        sig = 1.0 / (1.0 + math.exp(-(s1 - s0)))
        np.testing.assert_allclose(o[0, 0, i], sig * (v[0, 0, 1] - v[0, 0, 0]) + v[0, 0, 0], atol=1e-13)
        assert abs(lse[0, 0, i] - np.logaddexp(s0, s1)) < 1e-13


def test_probability_rows_via_identity_values():
    # With V = I (d = N) the output row IS the probability row: check it sums to 1, is zero above the
    # diagonal under causal, and that p_ij / p_i0 = exp(s_ij - s_i0).
    N = 12
    q, k = _rand((1, 1, N, N), 11), _rand((1, 1, N, N), 12)
    v = np.eye(N)[None, None]
    scale = 1 / math.sqrt(N)
    for causal in (False, True):
        p, lse = oracle.attn(q, k, v, scale, causal)
        p = p[0, 0]
        np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-12)
        s = scale * q[0, 0] @ k[0, 0].T
        for i in range(N):
            nk = i + 1 if causal else N
            np.testing.assert_allclose(p[i, :nk] / p[i, 0], np.exp(s[i, :nk] - s[i, 0]), rtol=1e-12)
            assert np.all(p[i, nk:] == 0.0)
            assert abs(math.exp(lse[0, 0, i]) - np.exp(s[i, :nk]).sum()) < 1e-10 * np.exp(s[i, :nk]).sum()


def test_zero_query_gives_mean_and_prefix_mean():
    B, H, N, d = 1, 2, 33, 16
    q = np.zeros((B, H, N, d))
    k, v = _rand((B, H, N, d), 21), _rand((B, H, N, d), 22)
    o, lse = oracle.attn(q, k, v, 0.125, False)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(2, keepdims=True), o.shape), atol=1e-13)
    np.testing.assert_allclose(lse, math.log(N), atol=1e-13)
    o, lse = oracle.attn(q, k, v, 0.125, True)
    prefix = np.cumsum(v, 2) / np.arange(1, N + 1)[None, None, :, None]
    np.testing.assert_allclose(o, prefix, atol=1e-13)
    np.testing.assert_allclose(lse, np.broadcast_to(np.log(np.arange(1, N + 1)), lse.shape), atol=1e-13)


def test_causal_row0_and_single_key():
    q, k, v = (_rand((2, 3, 5, 8), 31 + i) for i in range(3))
    o, lse = oracle.attn(q, k, v, 0.3, True)
    np.testing.assert_array_equal(o[:, :, 0], v[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], 0.3 * np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0]), atol=1e-13)
    o1, lse1 = oracle.attn(q[:, :, :1], k[:, :, :1], v[:, :, :1], 0.3, False)
    np.testing.assert_array_equal(o1[:, :, 0], v[:, :, 0])


def test_permutation_invariance_and_equivariance():
    B, H, N, d = 1, 2, 40, 16
    q, k, v = (_rand((B, H, N, d), 41 + i) for i in range(3))
    o, lse = oracle.attn(q, k, v, 0.25, False)
    perm = np.random.default_rng(0).permutation(N)
    o2, lse2 = oracle.attn(q, k[:, :, perm], v[:, :, perm], 0.25, False)
    np.testing.assert_allclose(o2, o, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, atol=1e-13)
    o3, lse3 = oracle.attn(q[:, :, perm], k, v, 0.25, False)
    np.testing.assert_allclose(o3, o[:, :, perm], atol=1e-13)


def test_row_shift_invariance():
    # Adding w to every key shifts row i's scores by scale*q_i.w: o unchanged, lse shifted by that.
    B, H, N, d = 1, 1, 24, 8
    q, k, v = (_rand((B, H, N, d), 51 + i) for i in range(3))
    w = _rand((d,), 54)
    for causal in (False, True):
        o, lse = oracle.attn(q, k, v, 0.5, causal)
        o2, lse2 = oracle.attn(q, k + w, v, 0.5, causal)
        np.testing.assert_allclose(o2, o, atol=1e-12)
        np.testing.assert_allclose(lse2, lse + 0.5 * q[0, 0] @ w, atol=1e-12)


def test_large_scores_do_not_overflow():
    # Scores near 1e3 overflow exp() without the max subtraction.
    q = np.array([[[[1.0], [1.0]]]]) * 1000.0
    k = np.array([[[[1.0], [1.001]]]])
    v = np.array([[[[0.0], [1.0]]]])
    o, lse = oracle.attn(q, k, v, 1.0, False)
    sig = 1 / (1 + math.exp(-1.0))
    np.testing.assert_allclose(o[0, 0, :, 0], [sig, sig], rtol=1e-12)
    assert np.all(np.isfinite(lse)) and abs(lse[0, 0, 0] - (1001 + math.log1p(math.exp(-1)))) < 1e-9


def test_brute_force_tiny_enumeration():
    # N<=4: evaluate the softmax by explicit enumeration with Python floats.
    for N in (1, 2, 3, 4):
        q, k, v = (_rand((1, 1, N, 3), 60 + 3 * N + i) for i in range(3))
        for causal in (False, True):
            o, lse = oracle.attn(q, k, v, 0.7, causal)
            for i in range(N):
                keys = range(i + 1) if causal else range(N)
                e = [math.exp(0.7 * sum(q[0, 0, i, t] * k[0, 0, j, t] for t in range(3))) for j in keys]
                ref = [sum(e[n] * v[0, 0, j, t] for n, j in enumerate(keys)) / sum(e) for t in range(3)]
                np.testing.assert_allclose(o[0, 0, i], ref, rtol=1e-12, atol=1e-14)
                assert abs(lse[0, 0, i] - math.log(sum(e))) < 1e-12


def _online_softmax_model(q, k, v, scale, causal, tile):
    """The pages' online softmax, written separately: per key tile update the running max m, the running
    exp-sum l and rescale the partial output (steps 1-4 of the page's description)."""
    N, d = q.shape
    o = np.zeros((N, d))
    lse = np.zeros(N)
    for i in range(N):
        nk = i + 1 if causal else N
        m, l, acc = -np.inf, 0.0, np.zeros(d)
        for j0 in range(0, nk, tile):
            kb, vb = k[j0:min(nk, j0 + tile)], v[j0:min(nk, j0 + tile)]
            s = scale * (kb @ q[i])
            m_new = max(m, s.max())
            corr = math.exp(m - m_new) if m > -np.inf else 0.0
            p = np.exp(s - m_new)
            l = l * corr + p.sum()
            acc = acc * corr + p @ vb
            m = m_new
        o[i] = acc / l
        lse[i] = m + math.log(l)
    return o, lse


@pytest.mark.parametrize("tile", [1, 7, 64, 128, 200])
@pytest.mark.parametrize("causal", [False, True])
def test_online_softmax_over_any_tiling_equals_global(tile, causal):
    N, d = 200, 16
    q, k, v = (_rand((1, 1, N, d), 70 + i) for i in range(3))
    o, lse = oracle.attn(q, k, v, 0.25, causal)
    om, lsem = _online_softmax_model(q[0, 0], k[0, 0], v[0, 0], 0.25, causal, tile)
    np.testing.assert_allclose(o[0, 0], om, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], lsem, atol=1e-12)


def test_flop_count_is_4n2d():
    B, H, N, d = 1, 2, 48, 16
    q, k, v = (_rand((B, H, N, d), 80 + i) for i in range(3))
    _, _, fl = oracle.attn(q, k, v, 0.25, False, return_flops=True)
    assert fl == 4 * B * H * N * N * d
    _, _, fl = oracle.attn(q, k, v, 0.25, True, return_flops=True)
    assert fl == 2 * B * H * N * (N + 1) * d  # causal: row i touches i+1 keys


def test_library_cross_check_tiny_config():
    # The tiny exact-attention configuration against torch's fp64 CPU scaled_dot_product_attention.
    q, k, v = inputs.dense_qkv(inputs.TINY, 1, 2, 256, 64)
    scale = float(np.float32(1 / math.sqrt(64)))
    for causal in (False, True):
        o, lse = oracle.attn(q, k, v, scale, causal)
        ref = torch.nn.functional.scaled_dot_product_attention(q.double(), k.double(), v.double(),
                                                                is_causal=causal, scale=scale)
        np.testing.assert_allclose(o, ref.numpy(), atol=1e-12)
        s = scale * q.double() @ k.double().transpose(-1, -2)
        if causal:
            s = s.masked_fill(torch.ones(256, 256, dtype=torch.bool).triu(1), float("-inf"))
        np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), atol=1e-12)


@pytest.mark.parametrize("d", [96, 128, 256])
def test_library_cross_check_other_head_dims(d):
    # The head dims the kernels also serve, against torch's fp64 CPU scaled_dot_product_attention (a ragged
    # length, so that no tile boundary is special).
    q, k, v = (inputs.normal_bf16((1, 2, 150, d), 95 + i, 1.0) for i in range(3))
    scale = float(np.float32(1 / math.sqrt(d)))
    for causal in (False, True):
        o, lse = oracle.attn(q, k, v, scale, causal)
        ref = torch.nn.functional.scaled_dot_product_attention(q.double(), k.double(), v.double(),
                                                                is_causal=causal, scale=scale)
        np.testing.assert_allclose(o, ref.numpy(), atol=1e-12)


def test_sampled_rows_match_full():
    B, H, N, d = 1, 3, 70, 8
    q, k, v = (_rand((B, H, N, d), 90 + i) for i in range(3))
    rows = [0, 5, 69, 33]
    for causal in (False, True):
        o, lse = oracle.attn(q, k, v, 0.3, causal)
        os_, lses = oracle.attn(q, k, v, 0.3, causal, rows=rows)
        np.testing.assert_array_equal(os_, o[:, :, rows])
        np.testing.assert_array_equal(lses, lse[:, :, rows])


# ----------------------------------------------------------------------------------------------
# varlen
# ----------------------------------------------------------------------------------------------
def test_varlen_equals_dense_per_sequence():
    lens = [5, 0, 17, 1, 9]
    cu = inputs.cu_seqlens(lens)
    T, H, d = int(cu[-1]), 3, 8
    q, k, v = (_rand((T, H, d), 100 + i) for i in range(3))
    for causal in (False, True):
        o, lse = oracle.attn_varlen(q, k, v, cu, 0.4, causal)
        for s, L in enumerate(lens):
            if L == 0:
                continue
            a, b = int(cu[s]), int(cu[s + 1])
            per = lambda x: np.ascontiguousarray(x[a:b].transpose(1, 0, 2))[None]
            od, lsed = oracle.attn(per(q), per(k), per(v), 0.4, causal)
            np.testing.assert_array_equal(o[a:b], od[0].transpose(1, 0, 2))
            np.testing.assert_array_equal(lse[a:b], lsed[0].T)


# ----------------------------------------------------------------------------------------------
# HSTU
# ----------------------------------------------------------------------------------------------
def test_golden_hstu_l2():
    g = json.load(open(os.path.join(GOLD, "hstu_l2_closed_form.json")))
    q = np.array(_num(g["q"]))[:, None, :]
    k = np.array(_num(g["k"]))[:, None, :]
    v = np.array(_num(g["v"]))[:, None, :]
    o = oracle.hstu_jagged(q, k, v, [0, 2], g["alpha"], g["inv_n"])
    np.testing.assert_allclose(o[:, 0, :], np.array(_num(g["o"])), atol=1e-14)


def _page_hstu_dense(Q, K, V, mask, alpha, n):
    # The page's Python definition, run with torch fp64 library ops on padded [b, heads, s, d].
    x = torch.matmul(Q, K.permute(0, 1, 3, 2))
    x *= alpha
    x = torch.nn.functional.silu(x)
    x *= mask / n
    return torch.matmul(x, V)


def test_hstu_jagged_equals_padded_page_definition():
    lens = [7, 1, 0, 20, 13]
    cu = inputs.cu_seqlens(lens)
    T, H, d = int(cu[-1]), 2, 8
    q, k, v = (inputs.normal_bf16((T, H, d), 200 + i, 0.5).double() for i in range(3))
    alpha, n = 0.125, 16.0
    o = oracle.hstu_jagged(q, k, v, cu, alpha, 1.0 / n)
    Lm = max(lens)
    pad = lambda x: torch.stack([torch.nn.functional.pad(x[int(cu[s]):int(cu[s + 1])], (0, 0, 0, 0, 0, Lm - L))
                                 for s, L in enumerate(lens)]).permute(0, 2, 1, 3)
    Qp, Kp, Vp = pad(q), pad(k), pad(v)
    mask = torch.zeros(len(lens), 1, Lm, Lm, dtype=torch.float64)
    for s, L in enumerate(lens):
        mask[s, 0, :L, :L] = torch.ones(L, L, dtype=torch.float64).tril()
    ref = _page_hstu_dense(Qp, Kp, Vp, mask, alpha, n).permute(0, 2, 1, 3)
    for s, L in enumerate(lens):
        np.testing.assert_allclose(o[int(cu[s]):int(cu[s + 1])], ref[s, :L].numpy(), atol=1e-15, rtol=1e-12)


def test_hstu_zero_query_and_ones_value():
    lens = [9, 4]
    cu = inputs.cu_seqlens(lens)
    T, H, d = 13, 2, 8
    k = inputs.normal_bf16((T, H, d), 300, 0.5).double()
    q = inputs.normal_bf16((T, H, d), 301, 0.5).double()
    o = oracle.hstu_jagged(torch.zeros_like(q), k, k, cu, 0.5, 0.25)
    assert np.all(o == 0.0)
    o = oracle.hstu_jagged(q, k, torch.ones_like(k), cu, 0.5, 0.25)
    for s in range(2):
        a = int(cu[s])
        for i in range(lens[s]):
            x = 0.5 * (q[a + i] * k[a:a + i + 1]).sum(-1)  # [i+1, H]
            ref = 0.25 * torch.nn.functional.silu(x).sum(0)
            np.testing.assert_allclose(o[a + i], ref[:, None].expand(H, d).numpy(), atol=1e-14)


def test_hstu_silu_odd_part_identity():
    # One-token sequences: o = inv_n * silu(alpha q.k) v, and silu(x) - silu(-x) = x.
    T, H, d = 6, 1, 4
    cu = list(range(T + 1))
    q, k, v = (inputs.normal_bf16((T, H, d), 310 + i).double() for i in range(3))
    op = oracle.hstu_jagged(q, k, v, cu, 0.7, 0.5)
    om = oracle.hstu_jagged(-q, k, v, cu, 0.7, 0.5)
    x = 0.7 * (q * k).sum(-1, keepdim=True)
    np.testing.assert_allclose(op - om, (0.5 * x * v).numpy(), atol=1e-14)


def test_hstu_causality_and_linearity_in_inv_n():
    lens = [16]
    T, H, d = 16, 1, 4
    q, k, v = (inputs.normal_bf16((T, H, d), 320 + i).double() for i in range(3))
    o = oracle.hstu_jagged(q, k, v, [0, 16], 1.0, 1.0)
    k2, v2 = k.clone(), v.clone()
    k2[10:] += 3.0
    v2[10:] -= 2.0
    o2 = oracle.hstu_jagged(q, k2, v2, [0, 16], 1.0, 1.0)
    np.testing.assert_array_equal(o2[:10], o[:10])
    o3 = oracle.hstu_jagged(q, k, v, [0, 16], 1.0, 1.0 / 4096)
    np.testing.assert_allclose(o3, o / 4096, rtol=1e-14, atol=0)


# ----------------------------------------------------------------------------------------------
# decode
# ----------------------------------------------------------------------------------------------
def test_golden_decode_l3():
    g = json.load(open(os.path.join(GOLD, "decode_l3_closed_form.json")))
    q = np.array(_num(g["q"])).reshape(1, 1, 1)
    k = np.array(_num(g["k"]) + [np.nan]).reshape(1, 1, 4, 1)
    v = np.array(_num(g["v"]) + [np.nan]).reshape(1, 1, 4, 1)
    o, lse = oracle.decode(q, k, v, [3], 1.0)
    assert abs(o[0, 0, 0] - g["o"]) < 1e-13 and abs(lse[0, 0] - _num(g["lse"])) < 1e-13


def test_decode_equals_prefill_row_and_ignores_tail():
    B, H, Lmax, d = 3, 2, 40, 16
    lens = [40, 17, 1]
    q, kc, vc, lens_t = inputs.decode_inputs(inputs.DECODE, B, H, Lmax, d, lens, poison_tail=True)
    scale = 0.0884
    o, lse = oracle.decode(q, kc, vc, lens_t, scale)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    for b, L in enumerate(lens):
        # place the decode query in the last row of a causal prefill over the first L cache rows
        Q = kc[b:b + 1, :, :L].clone()
        Q[:, :, L - 1] = q[b]
        op, lsep = oracle.attn(Q, kc[b:b + 1, :, :L], vc[b:b + 1, :, :L], scale, True, rows=[L - 1])
        np.testing.assert_allclose(o[b], op[0, :, 0], atol=1e-13)
        np.testing.assert_allclose(lse[b], lsep[0, :, 0], atol=1e-13)
    # a single cached token returns its value
    np.testing.assert_array_equal(o[2], vc[2, :, 0].double().numpy())


def test_decode_split_combine_is_independent_of_split_size():
    # The lse-weighted combine of per-split partial results equals the unsplit result (exact identity).
    B, H, Lmax, d = 1, 1, 300, 8
    q, kc, vc, lens = inputs.decode_inputs(inputs.DECODE, B, H, Lmax, d, [300])
    o, lse = oracle.decode(q, kc, vc, lens, 0.3)
    for chunk in (1, 7, 64, 299, 300):
        parts = []
        for s0 in range(0, 300, chunk):
            s1 = min(300, s0 + chunk)
            op, lp = oracle.decode(q, kc[:, :, s0:s1].contiguous(), vc[:, :, s0:s1].contiguous(),
                                   [s1 - s0], 0.3)
            parts.append((op[0, 0], lp[0, 0]))
        lse_c = np.logaddexp.reduce([lp for _, lp in parts])
        o_c = sum(math.exp(lp - lse_c) * op for op, lp in parts)
        np.testing.assert_allclose(o_c, o[0, 0], atol=1e-13)
        assert abs(lse_c - lse[0, 0]) < 1e-12


def test_decode_empty_cache():
    q, kc, vc, _ = inputs.decode_inputs(inputs.DECODE, 1, 2, 4, 8, [0])
    o, lse = oracle.decode(q, kc, vc, [0], 0.1)
    assert np.all(o == 0.0) and np.all(np.isneginf(lse))


# ----------------------------------------------------------------------------------------------
# decode over a paged cache with grouped query heads
# ----------------------------------------------------------------------------------------------
def _scatter_to_pages(kc, page_size, seed):
    """Cut a contiguous cache [B,Hkv,Lmax,d] into pages scattered over a pool in a seeded random order
    (the inverse of the oracle's gather, written independently): returns pool [num_pages,Hkv,ps,d] and
    the page table [B, max_pages]."""
    B, Hkv, Lmax, d = kc.shape
    max_pages = (Lmax + page_size - 1) // page_size
    num_pages = B * max_pages + 2
    order = np.random.default_rng(seed).permutation(num_pages)
    pool = np.full((num_pages, Hkv, page_size, d), np.nan)
    table = np.zeros((B, max_pages), np.int32)
    for b in range(B):
        for i in range(max_pages):
            phys = int(order[b * max_pages + i])
            table[b, i] = phys
            rows = kc[b, :, i * page_size:(i + 1) * page_size]
            pool[phys, :, :rows.shape[1]] = rows
    return pool, table


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (6, 1)])
@pytest.mark.parametrize("page_size", [16, 64])
def test_paged_decode_equals_contiguous_decode_with_repeated_heads(Hq, Hkv, page_size):
    # GQA: query head hq reads kv head hq // (Hq/Hkv) -- the same as plain multi-head decode with every kv
    # head repeated for its group (torch.repeat_interleave).  Paging changes nothing but where rows live.
    B, Lmax, d = 3, 150, 16
    lens = [150, 33, 1]
    _, kc, vc, lens_t = inputs.decode_inputs(inputs.DECODE_PAGED, B, Hkv, Lmax, d, lens, poison_tail=True)
    q = inputs.normal_bf16((B, Hq, d), 6001)
    kp, table = _scatter_to_pages(kc.double().numpy(), page_size, 1)
    vp, table_v = _scatter_to_pages(vc.double().numpy(), page_size, 1)
    assert np.array_equal(table, table_v)
    o, lse = oracle.decode_paged(q, kp, vp, table, lens_t, 0.25)
    G = Hq // Hkv
    o_ref, lse_ref = oracle.decode(q, kc.repeat_interleave(G, dim=1), vc.repeat_interleave(G, dim=1), lens_t, 0.25)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    np.testing.assert_allclose(o, o_ref, atol=1e-13)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-13)


def test_paged_decode_page_permutation_and_single_token():
    B, Hq, Hkv, d, ps = 2, 4, 2, 8, 16
    q, kp, vp, table, lens = inputs.paged_decode_inputs(inputs.DECODE_PAGED, B, Hq, Hkv, d, ps, [37, 1])
    o, lse = oracle.decode_paged(q, kp, vp, table, lens, 0.5)
    # relabelling the physical pages (and the table with them) changes nothing
    perm = np.random.default_rng(3).permutation(kp.shape[0])
    inv = np.argsort(perm)
    kp2, vp2 = kp[torch.as_tensor(perm)], vp[torch.as_tensor(perm)]
    table2 = np.where(table.numpy() >= 0, inv[np.maximum(table.numpy(), 0)], -1).astype(np.int32)
    o2, lse2 = oracle.decode_paged(q, kp2, vp2, table2, lens, 0.5)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)
    # one cached token: o is that token's value row for the query head's kv head; lse its scaled score
    pg = int(table[1, 0])
    for hq in range(Hq):
        g = hq // (Hq // Hkv)
        np.testing.assert_array_equal(o[1, hq], vp[pg, g, 0].double().numpy())
        s = 0.5 * float((q[1, hq].double() * kp[pg, g, 0].double()).sum())
        assert abs(lse[1, hq] - s) < 1e-12


def test_paged_decode_empty_sequence():
    q, kp, vp, table, lens = inputs.paged_decode_inputs(inputs.DECODE_PAGED, 2, 2, 1, 8, 16, [0, 5])
    o, lse = oracle.decode_paged(q, kp, vp, table, lens, 0.1)
    assert np.all(o[0] == 0.0) and np.all(np.isneginf(lse[0])) and np.all(np.isfinite(lse[1]))
