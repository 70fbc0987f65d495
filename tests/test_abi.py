"""The C ABI library loads, exports what the header declares, and validates on the host.

These run without a GPU: every call here is rejected by host-side checks
before any CUDA work is enqueued (or fails with ATTN_ERR_CUDA when no device
is present), so no kernel is launched.
"""

import ctypes
import os
import re

import pytest

import attention_online_softmax_fwd_b200 as ab
from attention_online_softmax_fwd_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn_b200.h")

OK, INVALID, UNSUPPORTED, CUDA = 0, 1, 2, 3
FAKE = ctypes.c_void_p(1 << 20)          # 16-byte aligned, never dereferenced on the host


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load_library()


def test_header_and_binding_agree(lib):
    names = declared_functions()
    assert "attn_prefill" in names and "attn_decode_paged" in names
    for name in names:
        assert hasattr(lib, name), f"{name} declared in the header but not exported"
        assert name in binding.SIGNATURES, f"{name} has no binding signature"


def test_status_strings(lib):
    for code, name in binding.STATUS.items():
        assert lib.attn_status_string(code).decode() == name
    assert lib.attn_status_string(99).decode() == "ATTN_ERR_UNKNOWN"
    assert lib.attn_abi_version() == 2


def _prefill(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, B=1, Hq=4, Hkv=2, S=128, D=64, causal=1, scale=0.125)
    a.update(kw)
    return lib.attn_prefill(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["S"],
                            a["D"], a["causal"], a["scale"], None)


@pytest.mark.parametrize("bad", [dict(q=None), dict(o=None), dict(q=ctypes.c_void_p((1 << 20) + 8)),
                                 dict(B=0), dict(S=0), dict(Hq=3), dict(Hkv=0), dict(scale=0.0),
                                 dict(scale=float("nan")), dict(scale=-1.0)])
def test_prefill_rejects_bad_arguments(lib, bad):
    assert _prefill(lib, **bad) == INVALID


def test_prefill_rejects_unsupported_head_dim(lib):
    assert _prefill(lib, D=96) == UNSUPPORTED


def test_prefill_blasst_rejects_bad_lambda(lib):
    for lam in (-0.1, 1.0, 2.0, float("nan")):
        st = lib.attn_prefill_blasst(FAKE, FAKE, FAKE, FAKE, None, 1, 4, 2, 128, 64, 1, 0.125, lam, None, None,
                                     None, None)
        assert st == INVALID


def test_prefill_blasst_rejects_a_misaligned_counter(lib):
    st = lib.attn_prefill_blasst(FAKE, FAKE, FAKE, FAKE, None, 1, 4, 2, 128, 64, 1, 0.125, 0.1, None,
                                 ctypes.c_void_p((1 << 20) + 4), None, None)
    assert st == INVALID


def test_workspace_bytes(lib):
    # a 256 B header (work-ticket counter), fp32 [N][splits][Hq][D] padded to 256 B,
    # then fp32 [N][splits][Hq]
    n, hq, d, mp, ps, sp = 64, 32, 128, 512, 16, 1024
    splits = -(-mp * ps // sp)
    o_bytes = n * splits * hq * d * 4
    want = 256 + -(-o_bytes // 256) * 256 + n * splits * hq * 4
    assert lib.attn_decode_workspace_bytes(n, hq, d, mp, ps, sp) == want
    assert ab.decode_workspace_bytes(n, hq, d, mp, ps, sp) == want
    for bad in [(0, hq, d, mp, ps, sp), (n, hq, 96, mp, ps, sp), (n, hq, d, mp, 24, sp), (n, hq, d, mp, ps, 100),
                (n, hq, d, 0, ps, sp)]:
        assert lib.attn_decode_workspace_bytes(*bad) == 0
        assert lib.attn_decode_blasst_workspace_bytes(*bad) == 0


def test_workspace_bytes_overflow_returns_zero(lib):
    # 2^31 sequences x 2^31 heads x ... does not fit a size_t: 0, never a wrapped small size
    big = 2 ** 31 - 1
    assert lib.attn_decode_workspace_bytes(big, big, 128, 2 ** 20, 256, 64) == 0
    assert lib.attn_decode_blasst_workspace_bytes(big, big, 128, 2 ** 20, 256, 64) == 0


def _blasst_layout(n, hq, d, mp, ps, sp):
    """The tile-skip workspace as the header documents it (chunk choice included)."""
    cap = mp * ps
    c = next((x for x in (256, 192, 128) if sp % x == 0), 64)
    items2 = -(-cap // c)   # the second pass's items (one partial each)
    while c % 128 == 0 and n * hq * -(-cap // c) < 32768:
        c //= 2
    chunks, tiles = -(-cap // c), -(-cap // 64)
    r256 = lambda x: -(-x // 256) * 256
    parts = [n * hq * items2 * d * 4, n * hq * items2 * 4, n * hq * tiles * 64 * 4, n * hq * tiles * 4,
             n * hq * chunks * 4, n * hq * chunks * 4]
    return 256 + sum(r256(x) for x in parts), c


@pytest.mark.parametrize("args", [(64, 32, 128, 512, 16, 256), (1, 32, 128, 2048, 16, 2048),
                                  (8, 16, 64, 40, 64, 320), (3, 8, 128, 10, 16, 64)])
def test_blasst_workspace_bytes(lib, args):
    want, _ = _blasst_layout(*args)
    dense = lib.attn_decode_workspace_bytes(*args)
    assert lib.attn_decode_blasst_workspace_bytes(*args) == max(want, dense)
    assert ab.binding.decode_blasst_workspace_bytes(*args) == max(want, dense)


def _decode(lib, **kw):
    a = dict(q=FAKE, kp=FAKE, vp=FAKE, bt=FAKE, sl=FAKE, N=4, Hq=8, Hkv=2, D=128, ps=16, mp=8, P=64,
             scale=0.09, lam=0.0, split=64, o=FAKE, lse=None, ws=FAKE, wsb=1 << 30)
    a.update(kw)
    return lib.attn_decode_paged(a["q"], a["kp"], a["vp"], a["bt"], a["sl"], a["N"], a["Hq"], a["Hkv"], a["D"],
                                 a["ps"], a["mp"], a["P"], a["scale"], a["lam"], a["split"], a["o"], a["lse"],
                                 a["ws"], a["wsb"], None, a.get("cnt"), None, None)


@pytest.mark.parametrize("bad", [dict(q=None), dict(bt=None), dict(sl=None), dict(ws=None), dict(N=0),
                                 dict(Hq=6, Hkv=4), dict(ps=24), dict(ps=0), dict(split=96), dict(split=0),
                                 dict(mp=0), dict(P=0), dict(lam=1.0), dict(lam=-0.5), dict(wsb=16),
                                 dict(kp=ctypes.c_void_p((1 << 20) + 4)), dict(bt=ctypes.c_void_p((1 << 20) + 2)),
                                 dict(sl=ctypes.c_void_p((1 << 20) + 1)), dict(lse=ctypes.c_void_p((1 << 20) + 2)),
                                 dict(cnt=ctypes.c_void_p((1 << 20) + 4)), dict(N=2 ** 20, Hq=2 ** 12, Hkv=2 ** 10)])
def test_decode_rejects_bad_arguments(lib, bad):
    assert _decode(lib, **bad) == INVALID


def test_decode_skip_path_needs_the_larger_workspace(lib):
    args = (4, 8, 128, 8, 16, 64)
    dense = lib.attn_decode_workspace_bytes(*args)
    skip = lib.attn_decode_blasst_workspace_bytes(*args)
    assert skip > dense > 0
    assert _decode(lib, lam=0.2, wsb=dense) == INVALID
    assert _decode(lib, cnt=FAKE, wsb=dense) == INVALID       # a counter selects the skip path too


@pytest.mark.parametrize("bad", [dict(D=80), dict(Hq=24, Hkv=1), dict(Hq=6, Hkv=2)])
def test_decode_rejects_unsupported(lib, bad):
    assert _decode(lib, **bad) == UNSUPPORTED


def test_valid_arguments_without_a_device_report_cuda_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    assert _prefill(lib) == CUDA
    assert _decode(lib) == CUDA
    assert _decode(lib, lam=0.3) == CUDA
    assert lib.attn_set_library_status(1) == CUDA


@pytest.mark.parametrize("limit", [0, 999, 2_000_000_001])
def test_debug_timeout_rejects_limits_out_of_range(lib, limit):
    st = lib.attn_debug_prefill_timeout(FAKE, FAKE, FAKE, FAKE, None, 1, 2, 1, 128, 128, 1, 0.088, limit, 1,
                                        None, None)
    assert st == INVALID


def test_noalloc_rejects_a_skip_call_beyond_its_scratch(lib):
    # the skip path also keeps the scores: 64 x 32 x 8192 x 4 B alone is 64 MiB
    st = lib.attn_decode_paged_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, 64, 32, 8, 128, 16, 512, 1024, 0.088, 0.3,
                                       2048, FAKE, None, None, None, None)
    assert st == INVALID


def test_binding_fails_loudly_when_library_missing(monkeypatch):
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "lib_path", lambda: "/nonexistent/libattn_b200.so")
    with pytest.raises(binding.AttnError):
        binding.load_library()


def _paged_prefill(lib, **kw):
    a = dict(q=FAKE, kp=FAKE, vp=FAKE, bt=FAKE, sl=FAKE, o=FAKE, lse=None, B=2, Sq=64, Hq=8, Hkv=2, D=128,
             ps=16, mp=16, P=64, scale=0.09)
    a.update(kw)
    return lib.attn_prefill_paged(a["q"], a["kp"], a["vp"], a["bt"], a["sl"], a["o"], a["lse"], a["B"], a["Sq"],
                                  a["Hq"], a["Hkv"], a["D"], a["ps"], a["mp"], a["P"], a["scale"], None, None)


@pytest.mark.parametrize("bad", [dict(q=None), dict(bt=None), dict(sl=None), dict(o=None),
                                 dict(kp=ctypes.c_void_p((1 << 20) + 8)), dict(bt=ctypes.c_void_p((1 << 20) + 2)),
                                 dict(B=0), dict(Sq=0), dict(Hq=6, Hkv=4), dict(ps=24), dict(ps=8), dict(ps=512),
                                 dict(mp=0), dict(P=0), dict(Sq=257, mp=16, ps=16), dict(scale=0.0),
                                 dict(scale=float("inf"))])
def test_prefill_paged_rejects_bad_arguments(lib, bad):
    assert _paged_prefill(lib, **bad) == INVALID


def test_prefill_paged_rejects_unsupported_head_dim(lib):
    assert _paged_prefill(lib, D=96) == UNSUPPORTED


def _append(lib, **kw):
    a = dict(kn=FAKE, vn=FAKE, kp=FAKE, vp=FAKE, bt=FAKE, sp=FAKE, N=4, T=1, Hkv=8, D=128, ps=16, mp=8, P=64)
    a.update(kw)
    return lib.attn_kv_append(a["kn"], a["vn"], a["kp"], a["vp"], a["bt"], a["sp"], a["N"], a["T"], a["Hkv"],
                              a["D"], a["ps"], a["mp"], a["P"], None, None)


@pytest.mark.parametrize("bad", [dict(kn=None), dict(vp=None), dict(bt=None), dict(sp=None),
                                 dict(kn=ctypes.c_void_p((1 << 20) + 8)), dict(sp=ctypes.c_void_p((1 << 20) + 1)),
                                 dict(N=0), dict(T=0), dict(Hkv=0), dict(ps=24), dict(mp=0), dict(P=0)])
def test_kv_append_rejects_bad_arguments(lib, bad):
    assert _append(lib, **bad) == INVALID


def test_kv_append_rejects_unsupported_head_dim(lib):
    assert _append(lib, D=80) == UNSUPPORTED


def _decode_fp8(lib, **kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, ks=0.01, vs=0.02, bt=FAKE, sl=FAKE, N=4, Hq=32, Hkv=8, D=128, ps=16, mp=8,
             P=64, scale=0.09, split=64, o=FAKE, lse=None, ws=FAKE, wsb=1 << 30)
    a.update(kw)
    return lib.attn_decode_paged_fp8(a["q"], a["kc"], a["vc"], a["ks"], a["vs"], a["bt"], a["sl"], a["N"],
                                     a["Hq"], a["Hkv"], a["D"], a["ps"], a["mp"], a["P"], a["scale"], a["split"],
                                     a["o"], a["lse"], a["ws"], a["wsb"], None, None)


@pytest.mark.parametrize("bad", [dict(q=None), dict(kc=None), dict(vc=None), dict(bt=None), dict(sl=None),
                                 dict(ws=None), dict(o=None), dict(N=0), dict(Hq=12, Hkv=8), dict(ps=24),
                                 dict(split=96), dict(mp=0), dict(P=0), dict(wsb=16), dict(ks=0.0),
                                 dict(vs=-1.0), dict(ks=float("nan")), dict(vs=float("inf")), dict(scale=0.0),
                                 dict(kc=ctypes.c_void_p((1 << 20) + 4)), dict(bt=ctypes.c_void_p((1 << 20) + 2))])
def test_decode_fp8_rejects_bad_arguments(lib, bad):
    assert _decode_fp8(lib, **bad) == INVALID


@pytest.mark.parametrize("bad", [dict(D=64), dict(Hq=4, Hkv=2), dict(Hq=12, Hkv=6), dict(Hq=64, Hkv=2), dict(Hq=192, Hkv=12)])
def test_decode_fp8_rejects_unsupported(lib, bad):
    assert _decode_fp8(lib, **bad) == UNSUPPORTED


def test_decode_fp8_valid_arguments_without_a_device_report_cuda_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    assert _decode_fp8(lib) == CUDA


@pytest.mark.parametrize("args,want", [((64, 32, 8, 512, 16, 256), 1),      # 64 x 8 x 32 splits = 16384 triples
                                       ((8, 32, 8, 1024, 16, 2048), 2),     # 8 x 8 x 8 = 512
                                       ((8, 32, 8, 4096, 16, 2048), 1),     # 8 x 8 x 32 = 2048
                                       ((1, 32, 8, 2048, 16, 256), 2),      # one 32K sequence: 1024
                                       ((4, 64, 4, 64, 16, 64), 1),         # Hq / Hkv = 16: one pass always
                                       ((0, 32, 8, 64, 16, 64), 0), ((4, 24, 8, 64, 16, 64), 0),
                                       ((4, 32, 8, 64, 24, 64), 0), ((4, 32, 8, 64, 16, 96), 0),
                                       ((4, 96, 3, 64, 16, 64), 0)])        # Hq / Hkv = 32
def test_decode_skip_passes(lib, args, want):
    assert lib.attn_decode_skip_passes(*args) == want
    assert ab.binding.decode_skip_passes(*args) == want
