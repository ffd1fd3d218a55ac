"""Argument marshalling of the Python binding, checked on the host: the C
entry points are replaced by recorders, the CUDA placement check by a no-op,
and every binding function must hand the library the tensors' pointers and
the sizes in the order include/swa.h declares them."""
import contextlib
import ctypes

import pytest
import torch

from sliding_window_attention_fwd_b200 import binding as b

BF = torch.bfloat16


class Recorder:
    def __init__(self):
        self.calls = {}

    def __getattr__(self, name):
        if not name.startswith("swa_"):
            raise AttributeError(name)

        def fn(*args):
            self.calls[name] = args
            return 0
        return fn


@pytest.fixture
def lib(monkeypatch):
    rec = Recorder()
    monkeypatch.setattr(b, "_lib", rec)
    monkeypatch.setattr(b, "_placed", lambda ref, **kw: None)
    monkeypatch.setattr(b, "_stream", lambda s: "STREAM")
    monkeypatch.setattr(b.torch.cuda, "device", lambda d: contextlib.nullcontext())
    return rec


def ptr(x):
    return None if x is None else x.value


def z(*shape, dtype=BF):
    return torch.zeros(shape, dtype=dtype)


def unpack(args):
    return [a.value if isinstance(a, ctypes.c_void_p) else a for a in args]


def test_forward_ex(lib):
    q, k, v = z(2, 50, 8, 64), z(2, 50, 2, 64), z(2, 50, 2, 64)
    out, lse = z(2, 50, 8, 64), z(2, 8, 50, dtype=torch.float32)
    G = torch.tensor([0, 7], dtype=torch.int32)
    seen = {}

    def rec(pp, stream):  # read the parameter block while the call lasts
        prm = ctypes.cast(pp, ctypes.POINTER(b.SwaParams))[0]
        seen["p"] = [getattr(prm, f[0]) for f in b.SwaParams._fields_]
        seen["stream"] = stream
        return 0
    lib.swa_forward_ex = rec
    b.swa_forward_ex(q, k, v, out, lse, 11, 3, 2, 64, G, 0.25)
    assert seen["p"] == [q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                         2, 8, 2, 50, 64, 11, 3, 2, 64, G.data_ptr(), 2, 0.25,
                         b.SWA_DTYPE_BF16]
    assert seen["stream"] == "STREAM"
    qf, kf, vf = (t.float() for t in (q, k, v))
    outf = b.swa_forward_ex(qf, kf, vf, None, None, 1, 1)
    assert seen["p"][3] == outf.data_ptr() and seen["p"][-1] == b.SWA_DTYPE_F32


def test_forward_plain_and_f32(lib):
    q, k, v = z(1, 30, 4, 128), z(1, 30, 4, 128), z(1, 30, 4, 128)
    out = b.swa_forward(q, k, v, None, None, 5, 0, 1)
    got = unpack(lib.calls["swa_forward"])
    assert got == [q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), None,
                   1, 4, 4, 30, 128, 5, 0, 1, None, 0, 0.0, "STREAM"]
    qf, kf, vf = (t.float() for t in (q, k, v))
    outf = b.swa_forward_f32(qf, kf, vf, None, None, 2, 2, 3, 0)
    got = unpack(lib.calls["swa_forward_f32"])
    assert got == [qf.data_ptr(), kf.data_ptr(), vf.data_ptr(), outf.data_ptr(), None,
                   1, 4, 4, 30, 128, 2, 2, 3, 0, None, 0, 0.0, "STREAM"]


def test_backward(lib):
    q, k, v = z(1, 20, 4, 64), z(1, 20, 2, 64), z(1, 20, 2, 64)
    out, do, lse = z(1, 20, 4, 64), z(1, 20, 4, 64), z(1, 4, 20, dtype=torch.float32)
    dq, dk, dv = b.swa_backward(q, k, v, out, do, lse, 6, 0, 1, 0, None, 0.5)
    got = unpack(lib.calls["swa_backward"])
    assert got == [q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), do.data_ptr(),
                   lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                   1, 4, 2, 20, 64, 6, 0, 1, 0, None, 0, 0.5, "STREAM"]
    assert dq.shape == q.shape and dk.shape == k.shape and dv.shape == v.shape


def test_decodes(lib):
    q, kr, vr = z(3, 8, 128), z(3, 512, 2, 128), z(3, 512, 2, 128)
    pos = torch.zeros(3, dtype=torch.int64)
    out = b.swa_decode(q, kr, vr, pos)
    assert unpack(lib.calls["swa_decode"]) == [q.data_ptr(), kr.data_ptr(), vr.data_ptr(),
                                                out.data_ptr(), pos.data_ptr(), 3, 8, 2, 128,
                                                512, "STREAM"]
    lse = z(3, 8, dtype=torch.float32)
    out = b.swa_decode_ex(q, kr, vr, pos, None, lse, 0.1)
    got = unpack(lib.calls["swa_decode_ex"])
    assert got[:6] == [q.data_ptr(), kr.data_ptr(), vr.data_ptr(), out.data_ptr(),
                       lse.data_ptr(), pos.data_ptr()]
    assert got[6:11] == [3, 8, 2, 128, 512] and got[11] == pytest.approx(0.1)
    out = z(3, 8, 128)
    b.swa_decode_noalloc(q, kr, vr, pos, out)
    assert unpack(lib.calls["swa_decode_noalloc"]) == [q.data_ptr(), kr.data_ptr(),
                                                        vr.data_ptr(), out.data_ptr(),
                                                        pos.data_ptr(), 3, 8, 2, 128, 512,
                                                        "STREAM"]


def test_paged_decode(lib):
    q, kp, vp = z(2, 8, 64), z(5 * 64, 1, 64), z(5 * 64, 1, 64)
    table = torch.zeros(2, 3, dtype=torch.int32)
    pos = torch.zeros(2, dtype=torch.int64)
    out = b.swa_decode_paged(q, kp, vp, table, pos, 64, 100)
    got = unpack(lib.calls["swa_decode_paged"])
    assert got == [q.data_ptr(), kp.data_ptr(), vp.data_ptr(), out.data_ptr(), None,
                   table.data_ptr(), pos.data_ptr(), 2, 8, 1, 64, 64, 5, 3, 100, 0.0, "STREAM"]


def test_append(lib):
    B, C, H, Hkv, D, W = 2, 16, 8, 2, 64, 128
    q, kn, vn = z(B, C, H, D), z(B, C, Hkv, D), z(B, C, Hkv, D)
    kr, vr = z(B, W, Hkv, D), z(B, W, Hkv, D)
    pos0 = torch.zeros(B, dtype=torch.int64)
    lse = z(B, H, C, dtype=torch.float32)
    out = b.swa_append(q, kn, vn, kr, vr, pos0, None, lse)
    got = unpack(lib.calls["swa_append"])
    assert got == [q.data_ptr(), kn.data_ptr(), vn.data_ptr(), kr.data_ptr(), vr.data_ptr(),
                   out.data_ptr(), lse.data_ptr(), pos0.data_ptr(), B, C, H, Hkv, D, W, 0.0,
                   "STREAM"]


def test_layers(lib):
    layers = []
    for i in range(3):
        layers.append(dict(q=z(1, 40, 4, 64), k=z(1, 40, 2, 64), v=z(1, 40, 2, 64),
                           win_left=10 + i, win_right=0, dilation=i + 1))
    outs = b.swa_forward_layers(layers)
    got = lib.calls["swa_forward_layers"]
    arr = ctypes.cast(got[0], ctypes.POINTER(b.SwaLayer))
    assert got[1:7] == (3, 1, 4, 2, 40, 64)
    for i, (L, o) in enumerate(zip(layers, outs)):
        rec = arr[i]
        assert (rec.q, rec.k, rec.v, rec.out) == (L["q"].data_ptr(), L["k"].data_ptr(),
                                                  L["v"].data_ptr(), o.data_ptr())
        assert (rec.win_left, rec.win_right, rec.dilation, rec.n_global) == (10 + i, 0, i + 1, 0)
