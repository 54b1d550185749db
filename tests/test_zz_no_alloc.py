"""attn_decode_noalloc: the decode step for callers that cannot allocate device memory at call time (a plugin
inside a host engine that owns all device memory, a latency-critical loop that cannot afford cudaMalloc's
implicit synchronisation).  Its split partials live in the library's fixed device scratch array instead of a
caller workspace.  Checked through the C ABI against attn_decode, on two calls in a row, within the parity
tolerances of the other tests.  This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import exact_tiled_attention_43_b200 as eta
from exact_tiled_attention_43_b200 import build as eta_build
from exact_tiled_attention_43_b200 import inputs
from parity import check_lse, check_o


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_rejects_sizes_beyond_scratch():
    eta_build.build()
    L = eta.lib()
    need = eta.attn_decode_workspace_size(64, 32, 32768, 128)
    assert need > eta.NOALLOC_SCRATCH_BYTES
    a = ctypes.c_void_p(0x10000)  # never dereferenced: the size check comes first
    rc = L.attn_decode_noalloc(a, a, a, a, a, a, 64, 32, 32768, 128, 0.088, ctypes.c_void_p(0))
    assert rc == -5  # ETA_ERR_WORKSPACE


@pytest.mark.gpu
def test_noalloc_matches_attn_decode_two_calls_in_a_row():
    """Each case calls attn_decode_noalloc twice in a row (the second call finds the first one's partials in
    the shared scratch array) and checks both results against attn_decode with a caller workspace and
    against the fp64 oracle.  The last case needs more than 90 % of the scratch array."""
    import oracle

    L = eta.lib()
    dev = "cuda"
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    big_lens = [int(x) for x in torch.randint(1, 513, (31,), generator=torch.Generator().manual_seed(53))]
    cases = [
        dict(B=3, H=4, Lmax=1024, d=128, lens=[1000, 17, 513], seed=51),
        dict(B=2, H=8, Lmax=320, d=64, lens=[1, 320], seed=52),
        dict(B=31, H=32, Lmax=512, d=128, lens=big_lens, seed=53),
    ]
    for c in cases:
        need = eta.attn_decode_workspace_size(c["B"], c["H"], c["Lmax"], c["d"])
        assert need <= eta.NOALLOC_SCRATCH_BYTES
        q, kc, vc, kl = inputs.decode_inputs(c["seed"], c["B"], c["H"], c["Lmax"], c["d"], c["lens"], device=dev,
                                             poison_tail=True)
        kl = kl.to(dev)
        scale = eta.default_scale(c["d"])
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
        o_ref = torch.empty((c["B"], c["H"], c["d"]), dtype=torch.bfloat16, device=dev)
        l_ref = torch.empty((c["B"], c["H"]), dtype=torch.float32, device=dev)
        rc = L.attn_decode(_p(q), _p(kc), _p(vc), _p(kl), _p(o_ref), _p(l_ref), c["B"], c["H"], c["Lmax"], c["d"],
                           scale, _p(ws), ws.numel(), stream)
        assert rc == 0
        outs = []
        for _ in range(2):
            o = torch.full_like(o_ref, float("nan"))
            lse = torch.full_like(l_ref, float("nan"))
            rc = L.attn_decode_noalloc(_p(q), _p(kc), _p(vc), _p(kl), _p(o), _p(lse), c["B"], c["H"], c["Lmax"],
                                       c["d"], scale, stream)
            assert rc == 0
            outs.append((o, lse))
        torch.cuda.synchronize()
        assert eta.status() == 0
        o64, l64 = oracle.decode(q, kc, vc, kl, scale)
        for i, (o, lse) in enumerate(outs):
            check_o(o, o_ref, f"noalloc call {i} vs attn_decode {c['B']}x{c['H']}x{c['Lmax']}")
            check_lse(lse, l_ref, "noalloc lse vs attn_decode")
            check_o(o, o64, f"noalloc call {i} vs oracle")
            check_lse(lse, l64, "noalloc lse vs oracle")
        if c["B"] == 31:
            assert need > 0.9 * eta.NOALLOC_SCRATCH_BYTES
