"""attn_decode_paged (grouped query heads over a paged KV cache) against the fp64 oracle, through the C ABI."""
import pytest
import torch

import exact_tiled_attention_43_b200 as eta
import oracle
from exact_tiled_attention_43_b200 import inputs
from parity import check_lse, check_o

pytestmark = pytest.mark.gpu
DEV = "cuda"

LENS = [1, 15, 16, 17, 100, 1000, 2500, 0]


def _run(B, Hq, Hkv, d, ps, lens, poison=True, spare=3):
    q, kp, vp, table, kl = inputs.paged_decode_inputs(inputs.DECODE_PAGED, B, Hq, Hkv, d, ps, lens,
                                                      spare_pages=spare, poison_tail=poison)
    scale = eta.default_scale(d)
    o, lse = eta.attn_decode_paged(q.to(DEV), kp.to(DEV), vp.to(DEV), table.to(DEV), kl.to(DEV), scale)
    assert eta.status() == 0
    o_ref, lse_ref = oracle.decode_paged(q, kp, vp, table, kl, scale)
    return o, lse, o_ref, lse_ref


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 2), (32, 8), (16, 1)])
@pytest.mark.parametrize("ps", [16, 64, 256])
def test_paged_decode_parity(d, Hq, Hkv, ps):
    """Ragged lengths (1 row, a page minus/plus one, several splits, empty); rows past each length and spare
    pages hold NaN, so any read past a sequence's end shows up."""
    o, lse, o_ref, lse_ref = _run(len(LENS), Hq, Hkv, d, ps, LENS)
    check_o(o, o_ref, f"paged d={d} Hq={Hq} Hkv={Hkv} ps={ps}")
    check_lse(lse, lse_ref, "paged lse")


def test_paged_decode_long_sequences_many_splits():
    """33k cached rows: 33 splits of 1024 rows each per (sequence, kv head), merged by the combine step."""
    o, lse, o_ref, lse_ref = _run(2, 32, 8, 128, 64, [33000, 20001], poison=False, spare=0)
    check_o(o, o_ref, "paged long")
    check_lse(lse, lse_ref, "paged long lse")


def test_paged_decode_shared_pages_and_bad_entries():
    B, Hq, Hkv, d, ps = 2, 8, 2, 64, 16
    q, kp, vp, table, kl = inputs.paged_decode_inputs(inputs.DECODE_PAGED, B, Hq, Hkv, d, ps, [50, 50])
    q[1] = q[0]
    table[1] = table[0]  # the second sequence reads the first one's pages
    q, kp, vp, table_d, kl_d = q.to(DEV), kp.to(DEV), vp.to(DEV), table.to(DEV), kl.to(DEV)
    o, lse = eta.attn_decode_paged(q, kp, vp, table_d, kl_d)
    assert eta.status() == 0
    assert torch.equal(o[0], o[1]) and torch.equal(lse[0], lse[1])
    # an out-of-range page number is reported (and page 0 read in its place, in bounds)
    bad = table_d.clone()
    bad[0, 1] = kp.shape[0] + 5
    eta.attn_decode_paged(q, kp, vp, bad, kl_d)
    assert eta.status() == eta.ETA_DEV_BAD_PAGE
    # a length past max_pages * page_size is reported and clamped
    long_len = torch.tensor([50, table.shape[1] * ps + 1], dtype=torch.int32, device=DEV)
    eta.attn_decode_paged(q, kp, vp, table_d, long_len)
    assert eta.status() == eta.ETA_DEV_BAD_KVLEN


def test_paged_decode_equals_contiguous_decode():
    """One kv head per query head and pages laid out in order: the paged kernel agrees with the contiguous
    decode kernel within the parity tolerance (they sum in different orders)."""
    B, H, d, ps, L = 3, 4, 128, 64, 1024
    q, kc, vc, lens = inputs.decode_inputs(inputs.DECODE, B, H, L, d, [1024, 500, 3])
    npg = (L + ps - 1) // ps
    kp = kc.view(B, H, npg, ps, d).permute(0, 2, 1, 3, 4).reshape(B * npg, H, ps, d).contiguous()
    vp = vc.view(B, H, npg, ps, d).permute(0, 2, 1, 3, 4).reshape(B * npg, H, ps, d).contiguous()
    table = torch.arange(B * npg, dtype=torch.int32).view(B, npg)
    o1, l1 = eta.attn_decode_paged(q.to(DEV), kp.to(DEV), vp.to(DEV), table.to(DEV), lens.to(DEV))
    o2, l2 = eta.attn_decode(q.to(DEV), kc.to(DEV), vc.to(DEV), lens.to(DEV))
    assert eta.status() == 0
    check_o(o1, o2.double().cpu().numpy(), "paged vs contiguous")
    check_lse(l1, l2.double().cpu().numpy(), "paged vs contiguous lse")
