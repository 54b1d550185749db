"""attn_decode (split-KV decode step) against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import exact_tiled_attention_43_b200 as eta
import oracle
from exact_tiled_attention_43_b200 import inputs
from parity import check_lse, check_o

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("lens,Lmax", [([1, 2, 31, 32, 33], 40), ([300, 0, 17, 299], 300), ([1000, 513, 1], 1024)])
def test_decode_small(d, lens, Lmax):
    B, H = len(lens), 3
    q, kc, vc, kl = inputs.decode_inputs(inputs.DECODE, B, H, Lmax, d, lens, device=DEV, poison_tail=True)
    scale = eta.default_scale(d)
    o, lse = eta.attn_decode(q, kc, vc, kl.to(DEV), scale=scale)
    assert eta.status() == 0
    o_ref, lse_ref = oracle.decode(q, kc, vc, kl, scale)
    check_o(o, o_ref, f"decode d={d} lens={lens}")
    check_lse(lse, lse_ref, "decode lse")
    # a zero-length cache gives o = 0 and lse = -inf
    for b, L in enumerate(lens):
        if L == 0:
            assert torch.all(o[b] == 0) and torch.all(torch.isneginf(lse[b]))


def test_decode_repeatable_and_workspace_reuse():
    lens = [700, 64]
    q, kc, vc, kl = inputs.decode_inputs(inputs.DECODE, 2, 4, 768, 128, lens, device=DEV)
    ws = torch.full((eta.attn_decode_workspace_size(2, 4, 768, 128),), 255, dtype=torch.uint8, device=DEV)
    o1, l1 = eta.attn_decode(q, kc, vc, kl.to(DEV), workspace=ws)
    o2, l2 = eta.attn_decode(q, kc, vc, kl.to(DEV), workspace=ws)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_decode_bad_length_sets_status_and_stays_in_bounds():
    q, kc, vc, kl = inputs.decode_inputs(inputs.DECODE, 2, 2, 64, 64, [64, 10], device=DEV)
    bad = torch.tensor([65, -3], dtype=torch.int32, device=DEV)
    eta.attn_decode(q, kc, vc, bad)
    assert eta.status() == eta.ETA_DEV_BAD_KVLEN
    assert eta.status() == 0  # cleared


def test_decode_full_config():
    """Decode step at the full workload (batch 64, H=32, d=128, lengths U[8192, 32768], Lmax 32768; rows of
    the cache past each length poisoned with NaN): all 32 heads of 10 sequences -- the shortest, the
    longest and 8 drawn at random -- compared with the oracle."""
    B, H, d, Lmax = 64, 32, 128, 32768
    lens = inputs.uniform_lengths(inputs.DECODE, B, 8192, 32768)
    q, kc, vc, kl = inputs.decode_inputs(inputs.DECODE, B, H, Lmax, d, lens, device=DEV)
    for b in range(B):
        kc[b, :, int(lens[b]):] = float("nan")
        vc[b, :, int(lens[b]):] = float("nan")
    scale = eta.default_scale(d)
    o, lse = eta.attn_decode(q, kc, vc, kl.to(DEV), scale=scale)
    assert eta.status() == 0
    rng = np.random.default_rng(5)
    bs = [int(torch.argmin(lens)), int(torch.argmax(lens))]
    for b in rng.permutation(B):
        if len(bs) == 10:
            break
        if int(b) not in bs:
            bs.append(int(b))
    for b in bs:
        L = int(lens[b])
        sub = lambda x: x[b:b + 1, :, :L].contiguous()
        o_ref, lse_ref = oracle.decode(q[b:b + 1], sub(kc), sub(vc), [L], scale)
        check_o(o[b:b + 1], o_ref, f"decode full b={b} L={L}")
        check_lse(lse[b:b + 1], lse_ref, "decode full lse")
    del kc, vc
    torch.cuda.empty_cache()
