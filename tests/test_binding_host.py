"""Host-side checks of the Python binding: the library receives bare
pointers, so a buffer of the wrong shape must be rejected before any call.
CPU tensors with the right shapes get as far as the CUDA-tensor check, which
shows the shape checks accepted them."""
import pytest
import torch

from sliding_window_attention_fwd_b200 import binding as b

BF = torch.bfloat16
F32 = torch.float32
CUDA_ONLY = "must be a contiguous CUDA tensor"


def t(*shape, dtype=BF):
    return torch.zeros(shape, dtype=dtype)


def fwd_args(B=2, N=40, H=4, Hkv=2, D=64):
    return t(B, N, H, D), t(B, N, Hkv, D), t(B, N, Hkv, D)


def test_forward_accepts_matching_buffers():
    q, k, v = fwd_args()
    with pytest.raises(ValueError, match=CUDA_ONLY):
        b.swa_forward(q, k, v, out=t(2, 40, 4, 64), lse=t(2, 4, 40, dtype=F32))


@pytest.mark.parametrize("out,lse", [
    (t(2, 40, 4, 32), None),                 # head dim
    (t(2, 39, 4, 64), None),                 # sequence
    (t(2, 40, 2, 64), None),                 # heads (kv count instead of q count)
    (None, t(2, 40, 4, dtype=F32)),          # lse as [B, N, H]
    (None, t(2, 4, 41, dtype=F32)),
])
def test_forward_rejects_wrong_buffers(out, lse):
    q, k, v = fwd_args()
    with pytest.raises(ValueError, match="expected shape"):
        b.swa_forward_ex(q, k, v, out=out, lse=lse)


def test_f32_forward_checks_the_same_shapes():
    q, k, v = (x.float() for x in fwd_args())
    with pytest.raises(ValueError, match="expected shape"):
        b.swa_forward_f32(q, k, v, out=t(2, 40, 4, 64, dtype=F32), lse=t(2, 40, 4, dtype=F32))


def test_backward_needs_forward_outputs_and_matching_gradients():
    q, k, v = fwd_args()
    out, lse, dout = t(2, 40, 4, 64), t(2, 4, 40, dtype=F32), t(2, 40, 4, 64)
    with pytest.raises(ValueError, match="required"):
        b.swa_backward(q, k, v, None, dout, lse)
    with pytest.raises(ValueError, match="required"):
        b.swa_backward(q, k, v, out, dout, None)
    with pytest.raises(ValueError, match="expected shape"):
        b.swa_backward(q, k, v, out, t(2, 40, 2, 64), lse)
    with pytest.raises(ValueError, match="expected shape"):
        b.swa_backward(q, k, v, out, dout, lse, dk=t(2, 40, 4, 64))
    with pytest.raises(ValueError, match=CUDA_ONLY):
        b.swa_backward(q, k, v, out, dout, lse, dq=t(2, 40, 4, 64), dk=t(2, 40, 2, 64),
                       dv=t(2, 40, 2, 64))


def dec_args(B=3, H=8, Hkv=2, D=128, W=256):
    return t(B, H, D), t(B, W, Hkv, D), t(B, W, Hkv, D), torch.zeros(B, dtype=torch.int64)


def test_decode_buffers():
    q, kr, vr, pos = dec_args()
    with pytest.raises(ValueError, match=CUDA_ONLY):
        b.swa_decode_ex(q, kr, vr, pos, out=t(3, 8, 128), lse=t(3, 8, dtype=F32))
    with pytest.raises(ValueError, match="expected shape"):
        b.swa_decode(q, kr, vr, pos, out=t(3, 2, 128))
    with pytest.raises(ValueError, match="expected shape"):
        b.swa_decode_ex(q, kr, vr, pos, lse=t(8, 3, dtype=F32))
    with pytest.raises(ValueError, match="out is required"):
        b.swa_decode_noalloc(q, kr, vr, pos, None)


def test_paged_decode_buffers():
    q = t(3, 8, 128)
    kp = vp = t(4 * 64, 2, 128)
    table = torch.zeros(3, 4, dtype=torch.int32)
    pos = torch.zeros(3, dtype=torch.int64)
    with pytest.raises(ValueError, match=CUDA_ONLY):
        b.swa_decode_paged(q, kp, vp, table, pos, 64, 128, out=t(3, 8, 128),
                           lse=t(3, 8, dtype=F32))
    with pytest.raises(ValueError, match="expected shape"):
        b.swa_decode_paged(q, kp, vp, table, pos, 64, 128, lse=t(3, 8, 1, dtype=F32)[..., 0]
                           .reshape(8, 3))


def test_append_buffers():
    B, C, H, Hkv, D, W = 2, 16, 8, 2, 64, 128
    q, kn, vn = t(B, C, H, D), t(B, C, Hkv, D), t(B, C, Hkv, D)
    kr, vr = t(B, W, Hkv, D), t(B, W, Hkv, D)
    pos0 = torch.zeros(B, dtype=torch.int64)
    with pytest.raises(ValueError, match=CUDA_ONLY):
        b.swa_append(q, kn, vn, kr, vr, pos0, out=t(B, C, H, D), lse=t(B, H, C, dtype=F32))
    with pytest.raises(ValueError, match="expected shape"):
        b.swa_append(q, kn, vn, kr, vr, pos0, lse=t(B, C, H, dtype=F32))
    with pytest.raises(ValueError, match="expected shape"):
        b.swa_append(q, kn, vn, kr, vr, pos0, out=t(B, C, Hkv, D))


def _maps_after(code):
    """Runs `code` in a fresh interpreter and returns the shared objects it
    has mapped afterwards (from /proc/self/maps)."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    prog = (f"import sys; sys.path.insert(0, {root!r})\n{code}\n"
            "print('\\n'.join(sorted({l.split()[-1] for l in open('/proc/self/maps') "
            "if l.strip().endswith('.so')})))")
    res = subprocess.run([sys.executable, "-c", prog], capture_output=True, text=True,
                         timeout=300, env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert res.returncode == 0, res.stderr
    return res.stdout.split()


def test_package_import_maps_no_library():
    # the seeded generator and the build module serve processes that never
    # run the CUDA path (the oracle's timing arm, the build check)
    maps = _maps_after("import sliding_window_attention_fwd_b200 as s\n"
                       "from sliding_window_attention_fwd_b200 import inputs, build\n"
                       "inputs.normal((2, 3), 1, 0)")
    assert not any(m.endswith("libswa.so") for m in maps)


def test_first_binding_use_loads_library():
    maps = _maps_after("import sliding_window_attention_fwd_b200 as s\n"
                       "assert s.swa_version() > 0")
    assert any(m.endswith("sliding_window_attention_fwd_b200/libswa.so") for m in maps)
