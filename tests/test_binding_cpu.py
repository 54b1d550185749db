"""The Python binding's argument checks, on CPU: caller-provided outputs and workspaces of the wrong shape,
dtype or layout, and inputs that disagree, are refused before anything reaches the library (a kernel would
write past a short buffer).  The library is replaced by a recorder, so no GPU is involved."""
import contextlib
import ctypes

import pytest
import torch

import exact_tiled_attention_43_b200 as eta


class _Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append((name, args))
            return 0
        return fn


@pytest.fixture
def rec(monkeypatch):
    r = _Recorder()
    monkeypatch.setattr(eta, "lib", lambda: r)

    def need(t, name, dtype, ndim):  # the real check minus "is a CUDA tensor"
        if t.dtype != dtype or t.dim() != ndim or not t.is_contiguous():
            raise ValueError(name)

    monkeypatch.setattr(eta, "_need", need)
    monkeypatch.setattr(eta, "_device_ctx", lambda t: contextlib.nullcontext())
    monkeypatch.setattr(eta, "_stream_ptr", lambda stream=None: ctypes.c_void_p(0))
    return r


def _bf(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_attn_fwd_checks_outputs(rec):
    q = _bf(1, 2, 64, 64)
    eta.attn_fwd(q, q, q)  # allocates its own outputs
    assert rec.calls[-1][0] == "attn_fwd"
    with pytest.raises(ValueError, match="out must have shape"):
        eta.attn_fwd(q, q, q, out=_bf(1, 2, 63, 64))
    with pytest.raises(TypeError, match="out must be one of"):
        eta.attn_fwd(q, q, q, out=torch.zeros(1, 2, 64, 64, dtype=torch.float16))
    with pytest.raises(TypeError, match="lse must be one of"):
        eta.attn_fwd(q, q, q, lse=torch.zeros(1, 2, 64, dtype=torch.float64))
    with pytest.raises(ValueError, match="lse must have shape"):
        eta.attn_fwd(q, q, q, lse=torch.zeros(1, 2, 32, dtype=torch.float32))
    with pytest.raises(ValueError, match="contiguous"):
        eta.attn_fwd(q, q, q, out=_bf(1, 64, 2, 64).transpose(1, 2))
    with pytest.raises(ValueError, match="same shape"):
        eta.attn_fwd(q, _bf(1, 2, 32, 64), q)
    n = len(rec.calls)
    # fp32 output selects the fp32 store; no lse means a NULL pointer
    eta.attn_fwd(q, q, q, out=torch.zeros(1, 2, 64, 64, dtype=torch.float32), return_lse=False)
    name, args = rec.calls[n]
    assert name == "attn_fwd" and args[11] == eta.ETA_OUT_F32 and args[4].value in (None, 0)


def test_packed_calls_check_shapes(rec):
    q = _bf(300, 4, 64)
    cu = torch.tensor([0, 100, 300], dtype=torch.int32)
    eta.attn_fwd_varlen(q, q, q, cu, 200)
    eta.hstu_fwd_jagged(q, q, q, cu, 200, 0.125, 1 / 4096)
    assert [c[0] for c in rec.calls] == ["attn_fwd_varlen", "hstu_fwd_jagged"]
    with pytest.raises(ValueError, match="same shape"):
        eta.attn_fwd_varlen(q, _bf(200, 4, 64), q, cu, 200)
    with pytest.raises(ValueError, match="same shape"):
        eta.hstu_fwd_jagged(q, q, _bf(300, 2, 64), cu, 200, 0.125, 1.0)
    with pytest.raises(ValueError, match="out must have shape"):
        eta.hstu_fwd_jagged(q, q, q, cu, 200, 0.125, 1.0, out=_bf(299, 4, 64))


def test_fp8_output_type_follows_the_buffer(rec):
    q8 = torch.zeros(1, 2, 128, 128, dtype=torch.float8_e4m3fn)
    eta.attn_fwd_fp8(q8, q8, q8, 1.0, 1.0, 1.0, out=torch.zeros(1, 2, 128, 128, dtype=torch.float32))
    assert rec.calls[-1][1][14] == eta.ETA_OUT_F32
    eta.attn_fwd_fp8(q8, q8, q8, 1.0, 1.0, 1.0)
    assert rec.calls[-1][1][14] == eta.ETA_OUT_BF16
    with pytest.raises(ValueError, match="out must have shape"):
        eta.attn_fwd_fp8(q8, q8, q8, 1.0, 1.0, 1.0, out=_bf(1, 2, 128, 64))


def test_decode_calls_check_outputs(rec, monkeypatch):
    monkeypatch.setattr(eta, "attn_decode_workspace_size", lambda *a: 1024)
    monkeypatch.setattr(eta, "attn_decode_paged_workspace_size", lambda *a: 1024)
    q, kc = _bf(2, 4, 128), _bf(2, 4, 512, 128)
    kl = torch.tensor([10, 512], dtype=torch.int32)
    eta.attn_decode(q, kc, kc, kl)
    eta.attn_decode_noalloc(q, kc, kc, kl)
    with pytest.raises(ValueError, match="out must have shape"):
        eta.attn_decode(q, kc, kc, kl, out=_bf(2, 4, 64))
    with pytest.raises(ValueError, match="lse must have shape"):
        eta.attn_decode_noalloc(q, kc, kc, kl, lse=torch.zeros(2, dtype=torch.float32))
    with pytest.raises(ValueError, match="workspace must be contiguous"):
        eta.attn_decode(q, kc, kc, kl, workspace=torch.zeros(2048, dtype=torch.uint8)[::2])
    pages = _bf(16, 2, 64, 128)
    table = torch.zeros(2, 8, dtype=torch.int32)
    eta.attn_decode_paged(q, pages, pages, table, kl)
    with pytest.raises(ValueError, match="out must have shape"):
        eta.attn_decode_paged(q, pages, pages, table, kl, out=_bf(2, 2, 128))
    assert [c[0] for c in rec.calls] == ["attn_decode", "attn_decode_noalloc", "attn_decode_paged"]
