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


def declared_parameter_counts():
    """{name: number of parameters} of every SWA_API function in the header."""
    text = open(HEADER).read()
    out = {}
    for m in re.finditer(r"SWA_API\s+[\w\s\*]+?\b(swa_\w+)\s*\(([^)]*)\)", text):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argtypes_match_the_header():
    """Each ctypes prototype of the binding has as many arguments as the
    header declares (a missing or extra one would shift every later
    argument)."""
    counts = declared_parameter_counts()
    checked = 0
    for name, n in counts.items():
        fn = getattr(binding._lib, name)
        if fn.argtypes is None:
            continue
        assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)
        checked += 1
    assert checked >= 15


def test_status_strings_and_version():
    assert swa.swa_status_string(0) == "ok"
    assert "aligned" in swa.swa_status_string(ALIGN)
    assert swa.swa_version() >= 100


L = binding._lib
A = 0x10000  # fake, 16-byte aligned addresses: validation never dereferences them


def fwd(*, q=A, k=A, v=A, out=A, lse=None, B=1, H=4, Hkv=2, N=64, D=128, L_=8, R=8, d=1,
        bs=0, G=None, ng=0, scale=0.0, f32=False, dtype=None):
    """swa_forward_ex over a parameter block (swa_forward_f32 for f32=True)."""
    if f32:
        return L.swa_forward_f32(q, k, v, out, lse, B, H, Hkv, N, D, L_, R, d, bs, G, ng, scale,
                                 None)
    prm = binding.SwaParams(q, k, v, out, lse, B, H, Hkv, N, D, L_, R, d, bs, G, ng, scale,
                            binding.SWA_DTYPE_BF16 if dtype is None else dtype)
    return L.swa_forward_ex(ctypes.c_void_p(ctypes.addressof(prm)), None)


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
    # global query rows run in the fused kernel, which serves any GQA group
    # (B = 0 keeps the call on the host)
    (dict(H=32, Hkv=2, ng=1, G=A, B=0), OK),
    (dict(H=32, Hkv=2, B=0), OK),
    (dict(B=0), OK),
    (dict(N=0), OK),
])
def test_forward_validation(kw, code):
    assert fwd(**kw) == code


def test_forward_ex_parameter_block():
    # the dtype field selects the path; NULL and unknown dtypes are rejected
    assert L.swa_forward_ex(None, None) == ARG
    assert fwd(dtype=7) == ARG
    assert fwd(dtype=binding.SWA_DTYPE_F32, D=96, B=0) == OK   # fp32 path serves D=96
    assert fwd(dtype=binding.SWA_DTYPE_BF16, D=96) == UNSUP    # the bf16 kernel does not
    assert fwd(dtype=binding.SWA_DTYPE_F32, D=80) == UNSUP
    assert fwd(dtype=binding.SWA_DTYPE_F32, bs=32, B=0) == OK  # any block size in fp32
    # plain swa_forward (flat arguments) validates the same way
    assert L.swa_forward(A, A, A, A, None, 1, 4, 3, 64, 128, 8, 8, 1, None, 0, 0.0, None) == ARG
    assert L.swa_forward(A, A, A, A, None, 0, 4, 2, 64, 128, 8, 8, 1, None, 0, 0.0, None) == OK


def test_params_struct_layout_matches_the_header():
    """Field offsets of the ctypes mirror equal the C struct's (compiled
    with gcc against include/swa.h)."""
    import shutil
    import subprocess
    import tempfile
    if shutil.which("gcc") is None:
        pytest.skip("needs gcc")
    fields = [f[0] for f in binding.SwaParams._fields_]
    prog = "#include <stdio.h>\n#include <stddef.h>\n#include \"swa.h\"\nint main(void){\n"
    prog += "".join(f'printf("%zu\\n", offsetof(swa_params, {f}));\n' for f in fields)
    prog += 'printf("%zu\\n", sizeof(swa_params)); return 0; }\n'
    with tempfile.TemporaryDirectory() as d:
        src, exe = os.path.join(d, "o.c"), os.path.join(d, "o")
        open(src, "w").write(prog)
        subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), src, "-o", exe],
                       check=True, capture_output=True)
        got = [int(x) for x in subprocess.run([exe], check=True, capture_output=True,
                                              text=True).stdout.split()]
    want = [getattr(binding.SwaParams, f).offset for f in fields] + [
        ctypes.sizeof(binding.SwaParams)]
    assert got == want


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


def test_paged_validation():
    def pg(**kw):
        return L.swa_decode_paged(kw.get("q", A), A, A, A, kw.get("lse", None), kw.get("tab", A),
                                  kw.get("pos", A), kw.get("B", 2), kw.get("H", 32),
                                  kw.get("Hkv", 8), kw.get("D", 128), kw.get("ps", 256),
                                  kw.get("npages", 16), kw.get("maxp", 8), kw.get("W", 4096),
                                  0.0, None)
    assert pg(H=32, Hkv=3) == ARG
    assert pg(ps=0) == ARG
    assert pg(npages=0) == ARG
    assert pg(tab=None) == ARG
    assert pg(tab=A + 2) == ALIGN
    assert pg(pos=A + 4) == ALIGN
    assert pg(ps=96) == UNSUP       # pages must hold whole 64-row boxes
    assert pg(H=32, Hkv=2) == UNSUP  # GQA group of 16
    assert pg(D=96) == UNSUP
    assert pg(B=0) == OK


def test_append_validation():
    def ap(**kw):
        return L.swa_append(kw.get("q", A), A, A, A, A, A, None, kw.get("pos", A), kw.get("B", 2),
                            kw.get("C", 16), kw.get("H", 32), kw.get("Hkv", 8), kw.get("D", 128),
                            kw.get("W", 4096), 0.0, None)
    assert ap(C=-1) == ARG
    assert ap(W=0) == ARG
    assert ap(pos=None) == ARG
    assert ap(q=A + 8) == ALIGN
    assert ap(W=100) == UNSUP       # ring slots of a 64-row box must not wrap
    assert ap(C=70000) == UNSUP
    assert ap(C=0) == OK
    assert ap(B=0) == OK


@pytest.mark.parametrize("pos,W,ps", [(0, 1, 64), (5000, 4096, 256), (4095, 4096, 256),
                                      (131071, 4096, 64), (10, 4096, 128), (256, 1, 256)])
def test_paged_window_is_exactly_the_pages_of_the_key_set(pos, W, ps):
    """Pages below first hold no position of the decode's key set (the oracle's
    key list for the causal window), page first and last hold its ends."""
    import oracle
    first, last = swa.swa_paged_window(pos, W, ps)
    lo = max(0, pos - W + 1)
    if pos < 20000:
        keys = oracle.key_set(pos, pos + 1, W - 1, 0)
        assert min(keys) == lo and max(keys) == pos
    assert first == lo // ps and last == pos // ps
    assert first * ps <= lo < (first + 1) * ps


def test_paged_window_rejects_bad_arguments():
    with pytest.raises(swa.SwaError):
        swa.swa_paged_window(-1, 10, 64)
    with pytest.raises(swa.SwaError):
        swa.swa_paged_window(5, 0, 64)


def test_layers_validation_names_the_bad_layer():
    """An invalid layer anywhere in the schedule stops it before any launch."""
    from sliding_window_attention_fwd_b200.binding import SwaLayer
    good = SwaLayer(A, A, A, A, None, 8, 8, 1, 0, None, 0, 0.0)
    bad_d = SwaLayer(A, A, A, A, None, 8, 8, 0, 0, None, 0, 0.0)      # dilation 0
    bad_al = SwaLayer(A, A, A + 8, A, None, 8, 8, 1, 0, None, 0, 0.0)  # misaligned v
    for layers, code, idx in [([good, good, bad_d], ARG, 2), ([good, bad_al, good], ALIGN, 1),
                              ([bad_d], ARG, 0)]:
        arr = (SwaLayer * len(layers))(*layers)
        bad = ctypes.c_int(-7)
        st = L.swa_forward_layers(ctypes.cast(arr, ctypes.c_void_p), len(layers), 1, 4, 2, 64, 128,
                                  ctypes.byref(bad), None)
        assert st == code and bad.value == idx
    bad = ctypes.c_int(-7)
    assert L.swa_forward_layers(None, 0, 1, 4, 2, 64, 128, ctypes.byref(bad), None) == OK
    assert L.swa_forward_layers(None, 2, 1, 4, 2, 64, 128, ctypes.byref(bad), None) == ARG


def test_workspace_allocator_arguments():
    """Both callbacks or neither; restoring the default touches no GPU (no
    workspace exists in this process)."""
    from sliding_window_attention_fwd_b200 import binding as b
    alloc = b._ALLOC_FN(lambda n, u: None)
    free = b._FREE_FN(lambda p, u: None)
    assert L.swa_set_workspace_allocator(alloc, b._FREE_FN(), None) == ARG
    assert L.swa_set_workspace_allocator(b._ALLOC_FN(), free, None) == ARG
    assert L.swa_set_workspace_allocator(b._ALLOC_FN(), b._FREE_FN(), None) == OK
    with pytest.raises(ValueError):
        swa.swa_set_workspace_allocator(lambda n: 0)
    swa.swa_set_workspace_allocator()


def test_forward_host_validation():
    """Host and device buffers both required; lse both or neither; B = 0 is a
    no-op before any CUDA call."""
    def fh(**kw):
        a = [kw.get(n, A) for n in ("qh", "kh", "vh", "oh")] + [kw.get("lh", None)]
        a += [kw.get(n, A) for n in ("qd", "kd", "vd", "od")] + [kw.get("ld", None)]
        return L.swa_forward_host(*a, kw.get("B", 1), 4, 2, 64, 128, 8, 0, 1, 0, None, 0, 0.0,
                                  None)
    assert fh(qh=None) == ARG
    assert fh(oh=None) == ARG
    assert fh(qd=None) == ARG
    assert fh(lh=A) == ARG          # lse on the host but not on the device
    assert fh(qd=A + 8) == ALIGN
    assert fh(B=0) == OK
    assert fh(B=0, lh=A, ld=A) == OK
