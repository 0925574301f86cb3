"""The C ABI library without a GPU: it builds, loads, exports every declared symbol, and rejects
bad arguments on the host (no call here reaches a kernel or needs a CUDA device)."""
import ctypes
import os
import re

import pytest

import hadamard_bit_quant_hbl_b200 as hbl
from hadamard_bit_quant_hbl_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    _build.build()
    return hbl.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "hbl.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hbl_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("hbl_pack_weights", "hbl_norm_fht_quant", "hbl_ternary_gemm", "hbl_forward"):
        assert name in syms


def test_every_declared_symbol_is_exported(L):
    for name in declared_symbols():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_status_strings(L):
    for s in range(5):
        assert hbl.hbl_status_string(s).startswith("HBL_")
    assert "unknown" in hbl.hbl_status_string(99)


def test_sizes(L):
    K, N = 4096, 2560
    r = lambda v: (v + 255) // 256 * 256  # noqa: E731
    assert hbl.hbl_packed_weights_bytes(K, N) == r(N * K // 4) + r(N * K) + r(4 * N)  # N a multiple of 128
    assert hbl.hbl_packed_weights_bytes(K, 520) == r(640 * K // 4) + r(520 * K) + r(4 * 520)
    assert hbl.hbl_packed_weights_bytes(0, N) == 0
    assert hbl.hbl_forward_workspace(100, 4096, hbl.HBL_Q_A4_ABSMEAN) == r(100 * 4096) + r(400)
    assert hbl.hbl_pack_weights_workspace(K, N) >= 8 * 593


FAKE = 1 << 20  # a 256-byte aligned non-null address; never dereferenced on these paths


def test_norm_fht_quant_rejects_bad_arguments(L):
    f = L.hbl_norm_fht_quant
    ok = dict(X=FAKE, gain=None, M=4, K=1024, hb=0, q=1, en=1e-6, eq=0.0, fmt=0, codes=FAKE, sx=FAKE, s=None)

    def call(**kw):
        a = {**ok, **kw}
        return f(a["X"], a["gain"], a["M"], a["K"], a["hb"], a["q"], a["en"], a["eq"], a["fmt"], a["codes"], a["sx"],
                 a["s"])

    assert call(X=None) == hbl.HBL_EINVAL
    assert call(codes=None) == hbl.HBL_EINVAL
    assert call(M=0) == hbl.HBL_EINVAL
    assert call(K=1000) == hbl.HBL_EINVAL          # not a multiple of 256
    assert call(K=65536) == hbl.HBL_EINVAL         # above the limit
    assert call(X=FAKE + 2) == hbl.HBL_EINVAL      # misaligned
    assert call(q=7) == hbl.HBL_EUNSUPPORTED
    assert call(fmt=5) == hbl.HBL_EINVAL
    assert call(en=-1.0) == hbl.HBL_EINVAL
    assert call(K=768, hb=0) == hbl.HBL_EUNSUPPORTED   # full transform needs a power of two
    assert call(K=768, hb=384) == hbl.HBL_EUNSUPPORTED  # block not a power of two
    assert call(K=1024, hb=128) == hbl.HBL_EUNSUPPORTED  # block below 256
    assert call(K=1280, hb=512) == hbl.HBL_EUNSUPPORTED  # block does not divide K


def test_gemm_and_forward_reject_bad_arguments(L):
    g = L.hbl_ternary_gemm
    nbytes = hbl.hbl_packed_weights_bytes(1024, 64)
    assert g(None, 0, 4, FAKE, FAKE, nbytes, 1.0, 4, 64, 1024, FAKE, 0, None, None) == hbl.HBL_EINVAL
    assert g(FAKE, 0, 4, FAKE, FAKE, nbytes, 1.0, 4, 60, 1024, FAKE, 0, None, None) == hbl.HBL_EINVAL  # N % 8
    assert g(FAKE, 0, 3, FAKE, FAKE, nbytes, 1.0, 4, 64, 1024, FAKE, 0, None, None) == hbl.HBL_EUNSUPPORTED
    assert g(FAKE, 0, 4, FAKE, FAKE, nbytes - 1, 1.0, 4, 64, 1024, FAKE, 0, None, None) == hbl.HBL_EINVAL
    assert g(FAKE, 0, 4, FAKE, FAKE + 16, nbytes, 1.0, 4, 64, 1024, FAKE, 0, None, None) == hbl.HBL_EINVAL
    assert g(FAKE, 0, 4, FAKE, FAKE, nbytes, 1.0, 4, 64, 1024, FAKE, 9, None, None) == hbl.HBL_EINVAL
    fw = L.hbl_forward
    ws = hbl.hbl_forward_workspace(4, 1024, 1)
    assert fw(FAKE, None, FAKE, nbytes, 1.0, 4, 1024, 64, 0, 1, 1e-6, 0.0, FAKE, ws - 1, FAKE, 0, None) == \
        hbl.HBL_EINVAL
    assert fw(FAKE, None, FAKE, nbytes, 1.0, 4, 1024, 64, 0, 1, 1e-6, 0.0, None, ws, FAKE, 0, None) == hbl.HBL_EINVAL


def test_forward_decode_rejects_bad_arguments(L):
    # every call below has at least one invalid argument, so none reaches a kernel
    fd = L.hbl_forward_decode
    nb = lambda K, N: hbl.hbl_packed_weights_bytes(K, N)  # noqa: E731
    ok = dict(X=FAKE, gain=None, packed=FAKE, pb=nb(1024, 64), alpha=1.0, K=1024, N=64, hb=0, quant=1,
              en=1e-6, eq=0.0, Y=FAKE, od=0)

    def call(**kw):
        a = dict(ok, **kw)
        return fd(a["X"], a["gain"], a["packed"], a["pb"], a["alpha"], a["K"], a["N"], a["hb"], a["quant"],
                  a["en"], a["eq"], a["Y"], a["od"], None)

    assert call(X=None) == hbl.HBL_EINVAL
    assert call(Y=None, quant=9) == hbl.HBL_EINVAL
    assert call(N=60, quant=9) == hbl.HBL_EINVAL                       # N % 8
    assert call(pb=nb(1024, 64) - 1, quant=9) == hbl.HBL_EINVAL       # blob too small
    assert call(K=16384, pb=nb(16384, 64)) == hbl.HBL_EUNSUPPORTED     # wider than one launch takes
    assert call(K=3072, pb=nb(3072, 64)) == hbl.HBL_EUNSUPPORTED       # not a power of two
    assert call(hb=128) == hbl.HBL_EUNSUPPORTED                         # transform block below 256
    assert call(quant=9) == hbl.HBL_EUNSUPPORTED
    assert call(en=-1.0) == hbl.HBL_EINVAL
    assert call(X=FAKE + 2) == hbl.HBL_EINVAL                           # misaligned
    assert call(od=7) == hbl.HBL_EINVAL


def test_pack_rejects_bad_arguments(L):
    alpha = ctypes.c_float(0)
    nbytes = hbl.hbl_packed_weights_bytes(512, 64)
    ws = hbl.hbl_pack_weights_workspace(512, 64)
    p = L.hbl_pack_weights
    assert p(None, 512, 64, 0.0, FAKE, nbytes, ctypes.byref(alpha), FAKE, ws, None) == hbl.HBL_EINVAL
    assert p(FAKE, 500, 64, 0.0, FAKE, nbytes, ctypes.byref(alpha), FAKE, ws, None) == hbl.HBL_EINVAL
    assert p(FAKE, 512, 64, -1.0, FAKE, nbytes, ctypes.byref(alpha), FAKE, ws, None) == hbl.HBL_EINVAL
    assert p(FAKE, 512, 64, 0.0, FAKE, nbytes, None, FAKE, ws, None) == hbl.HBL_EINVAL
    assert p(FAKE, 512, 64, 0.0, FAKE, nbytes, ctypes.byref(alpha), FAKE, ws - 8, None) == hbl.HBL_EINVAL
    assert L.hbl_pack_ternary(FAKE, 512, 63, FAKE, nbytes, None) == hbl.HBL_EINVAL


def test_selftest_timeout_rejects_limits_outside_range(L):
    # checked on the host before any launch
    assert L.hbl_selftest_timeout(0, None) == hbl.HBL_EINVAL
    assert L.hbl_selftest_timeout(1001, None) == hbl.HBL_EINVAL


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(hbl, "_lib", None)
    monkeypatch.setattr(hbl, "library_path", str(tmp_path / "nope.so"))
    with pytest.raises(ImportError):
        hbl.lib()


def test_pack_weights_rotated_rejects_bad_arguments(L):
    f = hbl.lib().hbl_pack_weights_rotated
    alpha = ctypes.c_float(0.0)
    ws = hbl.hbl_pack_weights_rotated_workspace(4096, 64)
    assert ws >= 4096 * 64 * 4
    # NULL pointers, a bad K, a negative or unsupported block: refused on the host
    assert f(None, 4096, 64, 0, 0.0, None, 0, ctypes.byref(alpha), None, 0, None) == hbl.HBL_EINVAL
    assert f(FAKE, 4000, 64, 0, 0.0, FAKE, 1 << 30, ctypes.byref(alpha), FAKE, 1 << 30, None) == hbl.HBL_EINVAL
    assert f(FAKE, 4096, 64, -1, 0.0, FAKE, 1 << 30, ctypes.byref(alpha), FAKE, 1 << 30, None) == hbl.HBL_EINVAL
    assert f(FAKE, 4096, 64, 0, 0.0, FAKE, 1 << 30, ctypes.byref(alpha), FAKE, 16, None) == hbl.HBL_EINVAL
    assert f(FAKE, 4096, 64, 96, 0.0, FAKE, 1 << 30, ctypes.byref(alpha), FAKE, 1 << 30, None) == hbl.HBL_EUNSUPPORTED


def test_qkv_quant_rejects_bad_arguments(L):
    f = hbl.lib().hbl_qkv_quant
    big = 1 << 30
    assert hbl.hbl_qkv_codes_bytes(10, 4, 128, 3) == 10 * 4 * 48
    assert f(None, 512, None, 10000.0, 1, 4, 128, 3, FAKE, big, FAKE, None) == hbl.HBL_EINVAL
    assert f(FAKE, 512, None, 10000.0, 1, 4, 96, 3, FAKE, big, FAKE, None) == hbl.HBL_EUNSUPPORTED
    assert f(FAKE, 512, None, 10000.0, 1, 4, 128, 5, FAKE, big, FAKE, None) == hbl.HBL_EUNSUPPORTED
    assert f(FAKE, 500, None, 10000.0, 1, 4, 128, 3, FAKE, big, FAKE, None) == hbl.HBL_EINVAL  # stride < H*D
    assert f(FAKE, 516, None, 10000.0, 1, 4, 128, 3, FAKE, big, FAKE, None) == hbl.HBL_EINVAL  # stride % 8
    assert f(FAKE, 512, FAKE, 0.5, 1, 4, 128, 3, FAKE, big, FAKE, None) == hbl.HBL_EINVAL      # theta
    assert f(FAKE, 512, None, 10000.0, 1, 4, 128, 3, FAKE, 100, FAKE, None) == hbl.HBL_EINVAL  # codes too small
    d = hbl.lib().hbl_qkv_dequant
    assert d(None, FAKE, 1, 4, 128, 3, FAKE, None) == hbl.HBL_EINVAL
    assert d(FAKE, FAKE, 1, 4, 100, 3, FAKE, None) == hbl.HBL_EUNSUPPORTED


def test_binding_forward_decode_takes_one_token():
    import torch

    X = torch.zeros((2, 1024), dtype=torch.bfloat16)  # host tensor: rejected before any library call
    with pytest.raises(ValueError):
        hbl.hbl_forward_decode(X, torch.zeros(16, dtype=torch.uint8), 1.0, 64)
