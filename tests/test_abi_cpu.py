"""The C ABI library loads, exports every entry point include/eta.h declares, and rejects bad arguments
on the host before touching any device (no GPU needed)."""
import ctypes
import os
import re

import pytest

import __graft_entry__  # noqa: F401  (makes sure the build entry exists)
import exact_tiled_attention_43_b200 as eta
from exact_tiled_attention_43_b200 import build as eta_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    eta_build.build()
    return eta.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "eta.h")).read()
    return re.findall(r"^ETA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src, flags=re.M)


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/eta.h but not exported by libeta.so"
        assert n in eta.SIGNATURES, f"{n} has no Python binding signature"


def test_strerror_covers_codes(L):
    for c in range(-8, 5):
        assert eta.strerror(c) != "unknown code"
    assert eta.strerror(12345) == "unknown code"


A = ctypes.c_void_p(0x10000)      # a 16-byte aligned, never dereferenced address
MIS = ctypes.c_void_p(0x10008)    # misaligned
NUL = ctypes.c_void_p(0)
S = ctypes.c_void_p(0)


def test_attn_fwd_host_validation(L):
    assert L.attn_fwd(NUL, A, A, A, NUL, 1, 1, 128, 64, 0.125, 0, 0, S) == -1
    for bad_d in (32, 80, 112, 160, 192):
        assert L.attn_fwd(A, A, A, A, NUL, 1, 1, 128, bad_d, 0.125, 0, 0, S) == -2
    assert L.attn_fwd(A, A, A, A, NUL, 0, 1, 128, 64, 0.125, 0, 0, S) == -3
    assert L.attn_fwd(A, A, A, A, NUL, 1, 1, 0, 64, 0.125, 0, 0, S) == -3
    assert L.attn_fwd(A, A, MIS, A, NUL, 1, 1, 128, 64, 0.125, 0, 0, S) == -4
    assert L.attn_fwd(A, A, A, A, NUL, 1, 1, 128, 64, 0.125, 0, 7, S) == -7
    assert L.attn_fwd(A, A, A, A, NUL, 1, 1, 128, 64, float("nan"), 0, 0, S) == -7
    assert L.attn_fwd(A, A, A, A, NUL, 1, 1, 128, 64, -1.0, 0, 0, S) == -7
    assert L.attn_fwd(A, A, A, A, NUL, 1, 1, 128, 64, 0.125, 2, 0, S) == -7
    # valid arguments without a usable GPU: a clean negative code, no crash
    rc = L.attn_fwd(A, A, A, A, NUL, 1, 1, 128, 64, 0.125, 0, 0, S)
    assert rc in (-6, -8)
    # head dim 96: accepted by every prefill mode (past the head-dim check: only the missing GPU stops it)
    assert L.attn_fwd(A, A, A, A, NUL, 1, 1, 128, 96, 0.125, 1, 0, S) in (-6, -8)
    assert L.hstu_fwd_jagged(A, A, A, A, A, 2, 128, 256, 1, 96, 0.125, 1.0, S) in (-6, -8)
    # head dim 256: accepted for softmax attention (dense and packed), not for HSTU
    assert L.attn_fwd(A, A, A, A, NUL, 1, 1, 128, 256, 0.0625, 1, 0, S) in (-6, -8)
    assert L.attn_fwd_varlen(A, A, A, A, NUL, A, 2, 128, 256, 1, 256, 0.0625, 1, 0, S) in (-6, -8)
    assert L.hstu_fwd_jagged(A, A, A, A, A, 2, 128, 256, 1, 256, 0.125, 1.0, S) == -2


def test_varlen_and_hstu_host_validation(L):
    assert L.attn_fwd_varlen(A, A, A, A, NUL, NUL, 2, 128, 256, 1, 64, 0.125, 1, 0, S) == -1
    assert L.attn_fwd_varlen(A, A, A, A, NUL, A, 0, 128, 256, 1, 64, 0.125, 1, 0, S) == -3
    assert L.attn_fwd_varlen(A, A, A, A, NUL, A, 2, 0, 256, 1, 64, 0.125, 1, 0, S) == -3
    assert L.attn_fwd_varlen(A, A, A, A, NUL, A, 2, 128, 0, 1, 64, 0.125, 1, 0, S) == 0  # empty batch: no work
    assert L.hstu_fwd_jagged(A, A, A, A, A, 2, 128, 256, 1, 64, 0.125, 0.0, S) == -7
    assert L.hstu_fwd_jagged(A, A, A, A, A, 2, 128, 256, 1, 64, float("inf"), 1.0, S) == -7
    assert L.hstu_fwd_jagged(A, A, A, MIS, A, 2, 128, 256, 1, 64, 0.125, 1.0, S) == -4
    assert L.hstu_fwd_jagged(A, A, A, A, A, 2, 128, 256, 1, 32, 0.125, 1.0, S) == -2


def test_decode_host_validation(L):
    ws = eta.attn_decode_workspace_size(64, 32, 32768, 128)
    assert ws > 0 and eta.attn_decode_workspace_size(0, 32, 100, 128) == 0
    assert eta.attn_decode_workspace_size(1, 1, 100, 96) == 0
    assert L.attn_decode(A, A, A, A, A, NUL, 64, 32, 32768, 128, 0.088, A, ws - 1, S) == -5
    assert L.attn_decode(A, A, A, NUL, A, NUL, 64, 32, 32768, 128, 0.088, A, ws, S) == -1
    assert L.attn_decode(A, A, A, A, A, NUL, 64, 32, 32768, 100, 0.088, A, ws, S) == -2
    assert L.attn_decode(A, MIS, A, A, A, NUL, 64, 32, 32768, 128, 0.088, A, ws, S) == -4
    assert L.attn_decode(A, A, A, A, A, NUL, 64, 32, 32768, 128, 0.0, A, ws, S) == -7


def test_paged_decode_host_validation(L):
    # B, Hq, Hkv, num_pages, page_size, max_pages, d
    ws = eta.attn_decode_paged_workspace_size(64, 32, 512, 64, 128)
    assert ws > 0 and ws == eta.attn_decode_workspace_size(64, 32, 512 * 64, 128)
    assert eta.attn_decode_paged_workspace_size(64, 32, 512, 48, 128) == 0  # page size not a power of two >= 16
    assert eta.attn_decode_paged_workspace_size(64, 32, 512, 64, 96) == 0

    def call(q=A, kp=A, vp=A, bt=A, kl=A, o=A, B=64, Hq=32, Hkv=8, npg=40000, ps=64, mp=512, d=128, sc=0.088,
             w=A, wsz=ws):
        return L.attn_decode_paged(q, kp, vp, bt, kl, o, NUL, B, Hq, Hkv, npg, ps, mp, d, sc, w, wsz, S)

    assert call(bt=NUL) == -1
    assert call(d=80) == -2
    assert call(Hq=30) == -3          # Hq not a multiple of Hkv
    assert call(Hq=8 * 17) == -3      # more than 16 query heads per kv head
    assert call(ps=48) == -3
    assert call(npg=0) == -3
    assert call(npg=(1 << 31) // 8) == -3  # num_pages * Hkv beyond 32-bit coordinates
    assert call(kp=MIS) == -4
    assert call(sc=float("nan")) == -7
    assert call(wsz=ws - 1) == -5
    rc = call()
    assert rc in (-6, -8)


def test_fp8_host_validation(L):
    # (q, k, v, o, lse, B, H, N, d, scale, q_descale, k_descale, v_descale, causal, o_dtype, stream)
    assert L.attn_fwd_fp8(NUL, A, A, A, NUL, 1, 1, 128, 128, 0.088, 1.0, 1.0, 1.0, 0, 0, S) == -1
    assert L.attn_fwd_fp8(A, A, A, A, NUL, 1, 1, 128, 64, 0.088, 1.0, 1.0, 1.0, 0, 0, S) == -2
    assert L.attn_fwd_fp8(A, A, A, A, NUL, 1, 1, 128, 128, 0.088, 0.0, 1.0, 1.0, 0, 0, S) == -7
    assert L.attn_fwd_fp8(A, A, A, A, NUL, 1, 1, 128, 128, 0.088, 1.0, 1.0, float("inf"), 0, 0, S) == -7
    assert L.attn_fwd_fp8(A, MIS, A, A, NUL, 1, 1, 128, 128, 0.088, 1.0, 1.0, 1.0, 0, 0, S) == -4
    assert L.attn_fwd_fp8(A, A, A, A, NUL, 1, 1, 128, 128, 0.088, 1.0, 1.0, 1.0, 0, 0, S) in (-6, -8)


def test_prefill_plan_split_policy():
    """The host's work decomposition (the same function the launches use), for a 148-SM B200."""
    P = lambda *a: eta.prefill_plan(*a, sms=148)
    # headline: 32 heads x 16 items of 256 rows; non-causal last wave 512 % 148 = 68 <= 74 -> 68 split
    assert P("dense", 32, 4096, 64, False) == (512, 444, 148)
    assert P("dense", 32, 4096, 64, True) == (512, 512, 148)   # causal, several waves: whole
    # d = 64 launches too small to fill the GPU: every item split, one CTA per half
    assert P("dense", 8, 2048, 64, True) == (64, 0, 128)
    assert P("dense", 8, 2048, 64, False) == (64, 0, 128)
    assert P("dense", 32, 1024, 64, True) == (128, 0, 148)
    assert P("dense", 32, 1024, 64, False) == (128, 128, 128)  # 2 x 128 > 148: whole
    # the same small-launch rule at d = 96 and 128; the non-causal last-wave rule still applies
    assert P("dense", 32, 1024, 128, True) == (128, 0, 148)
    assert P("dense", 8, 2048, 128, True) == (64, 0, 128)
    assert P("dense", 8, 2048, 96, True) == (64, 0, 128)
    assert P("dense", 8, 2048, 128, False) == (64, 0, 128)
    assert P("dense", 32, 1024, 128, False) == (128, 128, 128)  # 2 x 128 > 148: whole
    assert P("dense", 74, 1024, 128, True) == (296, 296, 148)  # more items than SMs: whole
    assert P("dense", 20, 2000, 128, False) == (160, 148, 148)  # 160 % 148 = 12 split
    assert P("dense", 148, 4096, 128, False) == (2368, 2368, 148)  # whole waves only
    # one key tile per row block: nothing to split
    assert P("dense", 8, 128, 64, True) == (8, 8, 8)
    # HSTU never splits (and is always causal); d = 256 items are 128 rows, never split
    assert P("hstu", 64, 4096, 64, False) == (1024, 1024, 148)
    assert P("hstu", 4, 1024, 64, True) == (16, 16, 16)
    assert P("dense", 64, 4096, 256, True) == (2048, 2048, 148)
    # packed launches plan on S*H units of max_len rows
    assert P("varlen", 30, 300, 64, True) == (60, 0, 120)
    # size limits: a row-block count past 65535, an item count past the work counter's range
    assert P("dense", 1, 256 * 65535, 64, False)[0] == 65535
    with pytest.raises(eta.EtaError):
        P("dense", 1, 256 * 65535 + 1, 64, False)
    with pytest.raises(eta.EtaError):
        P("dense", 2 ** 31 // 4, 4096, 64, False)
    # rejected like the calls
    with pytest.raises(eta.EtaError):
        P("dense", 1, 128, 80, False)
    with pytest.raises(eta.EtaError):
        P("hstu", 1, 128, 256, True)
    with pytest.raises(eta.EtaError):
        P("dense", 0, 128, 64, False)


def test_prefill_sched_group():
    """Dense launches schedule their (batch, head) units in groups whose K and V (2 * N * d * elt bytes a
    unit) fit in 32 MiB, at least one unit and at most all of them."""
    G = eta.prefill_sched_group
    assert G(32, 4096, 64) == 32        # B1 H32 N4096 d64: 1 MiB a unit, all 32 units in one group
    assert G(256, 4096, 128) == 16      # B8 H32 N4096 d128: 2 MiB a unit
    assert G(256, 4096, 128, 1) == 32   # the same shape in e4m3: 1 MiB a unit
    assert G(64, 4096, 256) == 8        # d = 256: 4 MiB a unit
    assert G(32, 32768, 128) == 2       # N = 32k: 16 MiB a unit
    assert G(32, 65536, 256) == 1       # 64 MiB a unit: one unit per group
    assert G(80, 2048, 128) == 32       # 1 MiB a unit, 80 units: groups of 32, 32, 16
    assert G(5, 1000, 64) == 5          # fewer units than fit
    for bad in ((0, 4096, 64, 2), (1, 0, 64, 2), (1, 4096, 64, 4)):
        with pytest.raises(eta.EtaError):
            G(*bad)


def test_header_is_c99_and_library_links_from_c(tmp_path):
    """The public header compiles as strict C99 and a C program links against libeta.so and gets answers
    from the host-side entry points (no GPU is used)."""
    import shutil
    import subprocess

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    lib_dir = os.path.dirname(eta.LIB_PATH)
    exe = str(tmp_path / "abi_c_check")
    subprocess.check_call([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                           "-I", os.path.join(root, "include"), os.path.join(root, "tests", "abi_c_check.c"),
                           "-o", exe, "-L", lib_dir, "-leta", "-Wl,-rpath," + lib_dir])
    out = subprocess.run([exe], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", (out.returncode, out.stdout, out.stderr)
