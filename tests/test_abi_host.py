"""Host-only checks of libswa.so: it loads, exports every symbol include/swa.h
declares, and rejects bad arguments with status codes before any launch.
No GPU is touched (every call here returns before the first CUDA call)."""
import ctypes
import os
import re

import pytest

import sliding_window_attention_fwd_b200 as swa
from sliding_window_attention_fwd_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "swa.h")

OK, ARG, ALIGN, UNSUP = 0, -1, -2, -3


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"SWA_API\s+[\w\s\*]+?\b(swa_\w+)\s*\(", text)


def test_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 11
    lib = ctypes.CDLL(swa.library_path())
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings_and_version():
    assert swa.swa_status_string(0) == "ok"
    assert "aligned" in swa.swa_status_string(ALIGN)
    assert swa.swa_version() >= 100


L = binding._lib
A = 0x10000  # fake, 16-byte aligned addresses: validation never dereferences them


def fwd(*, q=A, k=A, v=A, out=A, lse=None, B=1, H=4, Hkv=2, N=64, D=128, L_=8, R=8, d=1,
        bs=0, G=None, ng=0, scale=0.0, f32=False):
    fn = L.swa_forward_f32 if f32 else L.swa_forward_ex
    return fn(q, k, v, out, lse, B, H, Hkv, N, D, L_, R, d, bs, G, ng, scale, None)


@pytest.mark.parametrize("kw,code", [
    (dict(H=4, Hkv=3), ARG),
    (dict(d=0), ARG),
    (dict(bs=-1), ARG),
    (dict(ng=2, G=None), ARG),
    (dict(ng=100, G=A, N=64), ARG),
    (dict(q=None), ARG),
    (dict(B=-1), ARG),
    (dict(q=A + 8), ALIGN),
    (dict(out=A + 2), ALIGN),
    (dict(lse=A + 2), ALIGN),
    (dict(D=96), UNSUP),
    (dict(D=256), UNSUP),
    (dict(bs=32), UNSUP),
    (dict(B=0), OK),
    (dict(N=0), OK),
])
def test_forward_validation(kw, code):
    assert fwd(**kw) == code


def test_f32_validation():
    assert fwd(D=96, f32=True, B=0) == OK   # D=96 is supported by the fp32 path
    assert fwd(D=80, f32=True) == UNSUP
    assert fwd(H=3, Hkv=2, f32=True) == ARG


def test_decode_validation():
    dec = lambda **kw: L.swa_decode_ex(kw.get("q", A), A, A, A, None, kw.get("pos", A),
                                       kw.get("B", 2), kw.get("H", 32), kw.get("Hkv", 8),
                                       kw.get("D", 128), kw.get("W", 64), 0.0, None)
    assert dec(H=32, Hkv=3) == ARG
    assert dec(W=0) == ARG
    assert dec(pos=A + 4) == ALIGN
    assert dec(D=96) == UNSUP
    assert dec(H=32, Hkv=2) == UNSUP     # GQA group of 16 heads > 8
    assert dec(B=0) == OK


def test_selftest_rejects_bad_limit():
    assert L.swa_selftest_timeout(0, None) == ARG
