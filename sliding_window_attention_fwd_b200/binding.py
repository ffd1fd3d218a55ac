"""ctypes marshalling between torch tensors and the C ABI of libswa.so."""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libswa.so")

if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"libswa.so not found at {_LIB_PATH}: build it with "
        "`python -m sliding_window_attention_fwd_b200.build` (nvcc, sm_100a)")

_lib = ctypes.CDLL(_LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float

_lib.swa_forward.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _I, _F, _P]
_lib.swa_forward_ex.argtypes = [_P, _P]
_lib.swa_forward_host.argtypes = [_P] * 10 + [_I] * 9 + [_P, _I, _F, _P]
_lib.swa_forward_host.restype = _I
_lib.swa_forward_f32.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _P, _I,
                                 _F, _P]
_lib.swa_decode.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]
_lib.swa_decode_ex.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]
_lib.swa_decode_noalloc.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]
_lib.swa_decode_noalloc.restype = _I
_lib.swa_decode_noalloc_scratch_bytes.argtypes = []
_lib.swa_decode_noalloc_scratch_bytes.restype = ctypes.c_size_t
_lib.swa_decode_paged.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I,
                                  _F, _P]
_lib.swa_paged_window.argtypes = [ctypes.c_int64, _I, _I, _P, _P]
_lib.swa_append.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]


SWA_DTYPE_BF16 = 0
SWA_DTYPE_F32 = 1


class SwaParams(ctypes.Structure):
    """struct swa_params of include/swa.h."""
    _fields_ = [("q", _P), ("k", _P), ("v", _P), ("out", _P), ("lse", _P),
                ("B", _I), ("H", _I), ("Hkv", _I), ("N", _I), ("D", _I),
                ("win_left", _I), ("win_right", _I), ("dilation", _I), ("dilation_block", _I),
                ("global_idx", _P), ("n_global", _I), ("scale", _F), ("dtype", _I)]


class SwaLayer(ctypes.Structure):
    """struct swa_layer of include/swa.h."""
    _fields_ = [("q", _P), ("k", _P), ("v", _P), ("out", _P), ("lse", _P),
                ("win_left", _I), ("win_right", _I), ("dilation", _I), ("dilation_block", _I),
                ("global_idx", _P), ("n_global", _I), ("scale", _F)]


_lib.swa_forward_layers.argtypes = [_P, _I, _I, _I, _I, _I, _I, _P, _P]
_lib.swa_backward.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I,
                              _I, _P, _I, _F, _P]
_lib.swa_device_error.argtypes = [_P]
_lib.swa_selftest_timeout.argtypes = [_I, _P]
_lib.swa_schedule.argtypes = [_I, _I, _I, _I, _I, _P, _I]
_ALLOC_FN = ctypes.CFUNCTYPE(ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p)
_FREE_FN = ctypes.CFUNCTYPE(None, ctypes.c_void_p, ctypes.c_void_p)
_lib.swa_set_workspace_allocator.argtypes = [_ALLOC_FN, _FREE_FN, _P]
_lib.swa_set_workspace_allocator.restype = _I
_lib.swa_release.argtypes = []
_lib.swa_status_string.argtypes = [_I]
_lib.swa_status_string.restype = ctypes.c_char_p
_lib.swa_version.argtypes = []
for _fn in ("swa_forward", "swa_forward_ex", "swa_forward_f32", "swa_decode", "swa_decode_ex",
            "swa_decode_paged", "swa_paged_window", "swa_append", "swa_forward_layers",
            "swa_backward",
            "swa_device_error", "swa_selftest_timeout", "swa_schedule", "swa_release",
            "swa_version"):
    getattr(_lib, _fn).restype = _I


class SwaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {swa_status_string(status)} ({status})")


def library_path() -> str:
    return _LIB_PATH


def swa_status_string(status: int) -> str:
    return _lib.swa_status_string(int(status)).decode()


def swa_version() -> int:
    return _lib.swa_version()


def _check(status: int, where: str) -> None:
    if status != 0:
        raise SwaError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _need(t, name, dtype, ndim, shape=None):
    """Checks dtype, rank and (if given) the exact shape.  The library
    receives bare pointers, so a buffer of the wrong size must be caught
    here."""
    if t.dtype != dtype:
        raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name}: expected {ndim} dims, got shape {tuple(t.shape)}")
    if shape is not None and tuple(t.shape) != tuple(int(x) for x in shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")


def _placed(ref, **tensors):
    """Every given tensor (None skipped) must be a contiguous CUDA tensor on
    ref's device, where the call then runs."""
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name}: must be a contiguous CUDA tensor")
        if t.device != ref.device:
            raise ValueError(f"{name}: on {t.device}, expected {ref.device} like the queries")


def _fwd_common(q, k, v, out, lse, global_idx, dtype):
    _need(q, "q", dtype, 4)
    _need(k, "k", dtype, 4)
    _need(v, "v", dtype, 4)
    B, N, H, D = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, N, Hkv, D) or v.shape != k.shape:
        raise ValueError("k and v must be [B, N, Hkv, D] matching q [B, N, H, D]")
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", dtype, 4, (B, N, H, D))
    if lse is not None:
        _need(lse, "lse", torch.float32, 3, (B, H, N))
    ng = 0
    if global_idx is not None and global_idx.numel() > 0:
        _need(global_idx, "global_idx", torch.int32, 1)
        ng = global_idx.numel()
    else:
        global_idx = None
    _placed(q, q=q, k=k, v=v, out=out, lse=lse, global_idx=global_idx)
    return B, N, H, Hkv, D, out, global_idx, ng


def swa_forward(q, k, v, out=None, lse=None, win_left=-1, win_right=-1, dilation=1,
                global_idx=None, scale=0.0, stream=None):
    """bf16 SWA forward (C: swa_forward).  Returns out."""
    B, N, H, Hkv, D, out, gi, ng = _fwd_common(q, k, v, out, lse, global_idx, torch.bfloat16)
    with torch.cuda.device(q.device):
        _check(_lib.swa_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Hkv, N, D,
                                int(win_left), int(win_right), int(dilation), _ptr(gi), ng,
                                float(scale), _stream(stream)), "swa_forward")
    return out


def swa_forward_ex(q, k, v, out=None, lse=None, win_left=-1, win_right=-1, dilation=1,
                   dilation_block=0, global_idx=None, scale=0.0, stream=None):
    """SWA forward with block-level dilation over a parameter block (C:
    swa_forward_ex).  bf16 tensors take the tcgen05 kernel, fp32 tensors the
    FFMA path (the block's dtype follows q)."""
    dt = torch.float32 if q.dtype == torch.float32 else torch.bfloat16
    B, N, H, Hkv, D, out, gi, ng = _fwd_common(q, k, v, out, lse, global_idx, dt)
    prm = SwaParams(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                    None if lse is None else lse.data_ptr(), B, H, Hkv, N, D, int(win_left),
                    int(win_right), int(dilation), int(dilation_block),
                    None if gi is None else gi.data_ptr(), ng, float(scale),
                    SWA_DTYPE_F32 if dt == torch.float32 else SWA_DTYPE_BF16)
    with torch.cuda.device(q.device):
        _check(_lib.swa_forward_ex(ctypes.c_void_p(ctypes.addressof(prm)), _stream(stream)),
               "swa_forward_ex")
    return out


def swa_forward_host(q_host, k_host, v_host, q_dev, k_dev, v_dev, out_host=None, out_dev=None,
                     lse_host=None, lse_dev=None, win_left=-1, win_right=-1, dilation=1,
                     dilation_block=0, global_idx=None, scale=0.0, stream=None):
    """The bf16 forward for host-resident inputs and outputs (C:
    swa_forward_host): q/k/v are copied from the (pinned) host tensors into
    the given device tensors, the forward runs, out (and lse) come back into
    out_host / lse_host, the copies overlapping the kernels chunk by chunk.
    Asynchronous on `stream`; returns out_host."""
    for name, h, dv in (("q", q_host, q_dev), ("k", k_host, k_dev), ("v", v_host, v_dev)):
        if h.is_cuda or not h.is_contiguous() or h.shape != dv.shape or h.dtype != dv.dtype:
            raise ValueError(f"{name}_host: a contiguous host tensor shaped like {name}_dev")
    if out_dev is None:
        out_dev = torch.empty_like(q_dev)
    if out_host is None:
        out_host = torch.empty(q_host.shape, dtype=q_host.dtype, pin_memory=True)
    if (lse_host is None) != (lse_dev is None):
        raise ValueError("give both lse_host and lse_dev, or neither")
    B, N, H, Hkv, D, out_dev, gi, ng = _fwd_common(q_dev, k_dev, v_dev, out_dev, lse_dev,
                                                    global_idx, torch.bfloat16)
    if out_host.is_cuda or not out_host.is_contiguous() or out_host.shape != out_dev.shape:
        raise ValueError("out_host: a contiguous host tensor shaped like out")
    if lse_host is not None and (lse_host.is_cuda or not lse_host.is_contiguous()
                                 or lse_host.shape != lse_dev.shape):
        raise ValueError("lse_host: a contiguous host tensor shaped like lse")
    with torch.cuda.device(q_dev.device):
        _check(_lib.swa_forward_host(_ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(out_host),
                                     _ptr(lse_host), _ptr(q_dev), _ptr(k_dev), _ptr(v_dev),
                                     _ptr(out_dev), _ptr(lse_dev), B, H, Hkv, N, D,
                                     int(win_left), int(win_right), int(dilation),
                                     int(dilation_block), _ptr(gi), ng, float(scale),
                                     _stream(stream)), "swa_forward_host")
    return out_host


def swa_forward_layers(layers, stream=None):
    """A per-layer window schedule (C: swa_forward_layers).  `layers` is a list
    of dicts with q, k, v (bf16 [B, N, H|Hkv, D], the same shapes in every
    layer), and optionally out, lse, win_left, win_right, dilation,
    dilation_block, global_idx, scale.  Returns the list of outputs."""
    if not layers:
        return []
    arr = (SwaLayer * len(layers))()
    outs, keep = [], []
    shape = None
    for i, L in enumerate(layers):
        B, N, H, Hkv, D, out, gi, ng = _fwd_common(L["q"], L["k"], L["v"], L.get("out"),
                                                    L.get("lse"), L.get("global_idx"),
                                                    torch.bfloat16)
        if shape is None:
            shape = (B, N, H, Hkv, D)
            dev0 = L["q"].device
        elif shape != (B, N, H, Hkv, D):
            raise ValueError(f"layer {i}: shapes differ from layer 0")
        elif L["q"].device != dev0:
            raise ValueError(f"layer {i}: on {L['q'].device}, layer 0 on {dev0}")
        outs.append(out)
        keep.append(gi)
        arr[i] = SwaLayer(L["q"].data_ptr(), L["k"].data_ptr(), L["v"].data_ptr(), out.data_ptr(),
                          None if L.get("lse") is None else L["lse"].data_ptr(),
                          int(L.get("win_left", -1)), int(L.get("win_right", -1)),
                          int(L.get("dilation", 1)), int(L.get("dilation_block", 0)),
                          None if gi is None else gi.data_ptr(), ng, float(L.get("scale", 0.0)))
    B, N, H, Hkv, D = shape
    bad = ctypes.c_int(-1)
    with torch.cuda.device(dev0):
        st = _lib.swa_forward_layers(ctypes.cast(arr, _P), len(layers), B, H, Hkv, N, D,
                                     ctypes.byref(bad), _stream(stream))
    _check(st, f"swa_forward_layers (layer {bad.value})")
    return outs


def swa_backward(q, k, v, out, dout, lse, win_left=-1, win_right=-1, dilation=1,
                 dilation_block=0, global_idx=None, scale=0.0, dq=None, dk=None, dv=None,
                 stream=None):
    """Gradients (dq, dk, dv) of swa_forward_ex (C: swa_backward); out and lse
    are the forward's outputs for the same arguments."""
    if out is None or lse is None:
        raise ValueError("out and lse (from the forward) are required")
    _need(dout, "dout", torch.bfloat16, 4, q.shape)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, n, ref in ((dq, "dq", q), (dk, "dk", k), (dv, "dv", v)):
        _need(t, n, torch.bfloat16, 4, ref.shape)
    B, N, H, Hkv, D, out, gi, ng = _fwd_common(q, k, v, out, lse, global_idx, torch.bfloat16)
    _placed(q, dout=dout, dq=dq, dk=dk, dv=dv)
    with torch.cuda.device(q.device):
        _check(_lib.swa_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse),
                                 _ptr(dq), _ptr(dk), _ptr(dv), B, H, Hkv, N, D, int(win_left),
                                 int(win_right), int(dilation), int(dilation_block), _ptr(gi),
                                 ng, float(scale), _stream(stream)), "swa_backward")
    return dq, dk, dv


def swa_forward_f32(q, k, v, out=None, lse=None, win_left=-1, win_right=-1, dilation=1,
                    dilation_block=0, global_idx=None, scale=0.0, stream=None):
    """fp32 SWA forward on CUDA cores (C: swa_forward_f32)."""
    B, N, H, Hkv, D, out, gi, ng = _fwd_common(q, k, v, out, lse, global_idx, torch.float32)
    with torch.cuda.device(q.device):
        _check(_lib.swa_forward_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Hkv,
                                    N, D, int(win_left), int(win_right), int(dilation),
                                    int(dilation_block), _ptr(gi), ng, float(scale),
                                    _stream(stream)), "swa_forward_f32")
    return out


def _dec_common(q, k_ring, v_ring, out, pos):
    _need(q, "q", torch.bfloat16, 3)
    _need(k_ring, "k_ring", torch.bfloat16, 4)
    _need(v_ring, "v_ring", torch.bfloat16, 4)
    _need(pos, "pos", torch.int64, 1)
    B, H, D = q.shape
    W, Hkv = k_ring.shape[1], k_ring.shape[2]
    if k_ring.shape != (B, W, Hkv, D) or v_ring.shape != k_ring.shape or pos.shape != (B,):
        raise ValueError("k_ring/v_ring must be [B, W, Hkv, D] and pos [B]")
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, 3, (B, H, D))
    return B, H, Hkv, D, W, out


def swa_decode(q, k_ring, v_ring, pos, out=None, stream=None):
    """Ring-buffer decode (C: swa_decode).  Returns out [B, H, D]."""
    B, H, Hkv, D, W, out = _dec_common(q, k_ring, v_ring, out, pos)
    _placed(q, q=q, k_ring=k_ring, v_ring=v_ring, pos=pos, out=out)
    with torch.cuda.device(q.device):
        _check(_lib.swa_decode(_ptr(q), _ptr(k_ring), _ptr(v_ring), _ptr(out), _ptr(pos), B, H,
                               Hkv, D, W, _stream(stream)), "swa_decode")
    return out


def swa_decode_ex(q, k_ring, v_ring, pos, out=None, lse=None, scale=0.0, stream=None):
    """Ring-buffer decode that also writes lse [B, H] (C: swa_decode_ex)."""
    B, H, Hkv, D, W, out = _dec_common(q, k_ring, v_ring, out, pos)
    if lse is not None:
        _need(lse, "lse", torch.float32, 2, (B, H))
    _placed(q, q=q, k_ring=k_ring, v_ring=v_ring, pos=pos, out=out, lse=lse)
    with torch.cuda.device(q.device):
        _check(_lib.swa_decode_ex(_ptr(q), _ptr(k_ring), _ptr(v_ring), _ptr(out), _ptr(lse),
                                  _ptr(pos), B, H, Hkv, D, W, float(scale), _stream(stream)),
               "swa_decode_ex")
    return out


def swa_decode_noalloc(q, k_ring, v_ring, pos, out, stream=None):
    """swa_decode without any device allocation by the library (C:
    swa_decode_noalloc): for callers whose device memory is a fixed pool, or
    whose hot loop cannot take a cudaMalloc.  Its split partials live in a
    fixed array inside the library, shared by all calls on a device, so calls
    must not overlap on the GPU.  `out` must be given (nothing is allocated
    here either)."""
    if out is None:
        raise ValueError("out is required (nothing is allocated here)")
    B, H, Hkv, D, W, out = _dec_common(q, k_ring, v_ring, out, pos)
    _placed(q, q=q, k_ring=k_ring, v_ring=v_ring, pos=pos, out=out)
    with torch.cuda.device(q.device):
        _check(_lib.swa_decode_noalloc(_ptr(q), _ptr(k_ring), _ptr(v_ring), _ptr(out),
                                       _ptr(pos), B, H, Hkv, D, W, _stream(stream)),
               "swa_decode_noalloc")
    return out


def swa_decode_noalloc_scratch_bytes() -> int:
    """Bytes of the fixed device array swa_decode_noalloc uses (per GPU)."""
    return int(_lib.swa_decode_noalloc_scratch_bytes())


def swa_decode_paged(q, k_pages, v_pages, block_table, pos, page_size, W, out=None, lse=None,
                     scale=0.0, stream=None):
    """Decode over a paged KV cache (C: swa_decode_paged).  q [B, H, D];
    k_pages/v_pages [num_pages * page_size, Hkv, D]; block_table [B, max_pages]
    int32; pos [B] int64.  Returns out [B, H, D]."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_pages, "k_pages", torch.bfloat16, 3)
    _need(v_pages, "v_pages", torch.bfloat16, 3)
    _need(block_table, "block_table", torch.int32, 2)
    _need(pos, "pos", torch.int64, 1)
    B, H, D = q.shape
    rows, Hkv = k_pages.shape[0], k_pages.shape[1]
    if (k_pages.shape[2] != D or v_pages.shape != k_pages.shape or pos.shape != (B,)
            or block_table.shape[0] != B or rows % int(page_size) != 0):
        raise ValueError("k_pages/v_pages [num_pages * page_size, Hkv, D], block_table [B, *], "
                         "pos [B]")
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, 3, (B, H, D))
    if lse is not None:
        _need(lse, "lse", torch.float32, 2, (B, H))
    _placed(q, q=q, k_pages=k_pages, v_pages=v_pages, block_table=block_table, pos=pos, out=out,
            lse=lse)
    with torch.cuda.device(q.device):
        _check(_lib.swa_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(out), _ptr(lse),
                                     _ptr(block_table), _ptr(pos), B, H, Hkv, D, int(page_size),
                                     rows // int(page_size), block_table.shape[1], int(W),
                                     float(scale), _stream(stream)), "swa_decode_paged")
    return out


def swa_paged_window(pos: int, W: int, page_size: int):
    """Host-only: (first_page, last_page) of the logical pages a decode at
    `pos` reads; pages below first_page can be released (C: swa_paged_window)."""
    first, last = ctypes.c_int64(), ctypes.c_int64()
    _check(_lib.swa_paged_window(int(pos), int(W), int(page_size), ctypes.byref(first),
                                 ctypes.byref(last)), "swa_paged_window")
    return first.value, last.value


def swa_append(q, k_new, v_new, k_ring, v_ring, pos0, out=None, lse=None, scale=0.0,
               stream=None):
    """A chunk of C tokens enters the ring cache (C: swa_append).  q [B, C, H, D];
    k_new/v_new [B, C, Hkv, D]; k_ring/v_ring [B, W, Hkv, D] (updated in place);
    pos0 [B] int64.  Returns out [B, C, H, D]."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k_new, "k_new", torch.bfloat16, 4)
    _need(v_new, "v_new", torch.bfloat16, 4)
    _need(k_ring, "k_ring", torch.bfloat16, 4)
    _need(v_ring, "v_ring", torch.bfloat16, 4)
    _need(pos0, "pos0", torch.int64, 1)
    B, C, H, D = q.shape
    W, Hkv = k_ring.shape[1], k_ring.shape[2]
    if (k_new.shape != (B, C, Hkv, D) or v_new.shape != k_new.shape
            or k_ring.shape != (B, W, Hkv, D) or v_ring.shape != k_ring.shape
            or pos0.shape != (B,)):
        raise ValueError("k_new/v_new [B, C, Hkv, D], k_ring/v_ring [B, W, Hkv, D], pos0 [B]")
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, 4, (B, C, H, D))
    if lse is not None:
        _need(lse, "lse", torch.float32, 3, (B, H, C))
    _placed(q, q=q, k_new=k_new, v_new=v_new, k_ring=k_ring, v_ring=v_ring, pos0=pos0, out=out,
            lse=lse)
    with torch.cuda.device(q.device):
        _check(_lib.swa_append(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_ring), _ptr(v_ring),
                               _ptr(out), _ptr(lse), _ptr(pos0), B, C, H, Hkv, D, W,
                               float(scale), _stream(stream)), "swa_append")
    return out


def swa_device_error(stream=None) -> int:
    """Synchronises the stream; returns 0 or the (negative) status of a device timeout."""
    return _lib.swa_device_error(_stream(stream))


def swa_selftest_timeout(limit_us: int, stream=None) -> None:
    _check(_lib.swa_selftest_timeout(int(limit_us), _stream(stream)), "swa_selftest_timeout")


def swa_schedule(N, win_left, win_right, dilation=1, dilation_block=0):
    """Host-only scheduler query: list of (class, q_tile, first_row, kv_begin, kv_end, n_edge)."""
    n = _lib.swa_schedule(int(N), int(win_left), int(win_right), int(dilation),
                          int(dilation_block), None, 0)
    if n < 0:
        raise SwaError(n, "swa_schedule")
    buf = (ctypes.c_int32 * (6 * max(n, 1)))()
    n2 = _lib.swa_schedule(int(N), int(win_left), int(win_right), int(dilation),
                           int(dilation_block), ctypes.cast(buf, ctypes.c_void_p), n)
    if n2 < 0:
        raise SwaError(n2, "swa_schedule")
    return [tuple(buf[6 * t: 6 * t + 6]) for t in range(n)]


def swa_release() -> None:
    _check(_lib.swa_release(), "swa_release")


_allocator_keep = None  # the installed callbacks must outlive every library call


def swa_set_workspace_allocator(alloc=None, free=None) -> None:
    """Routes the library-owned workspaces through the caller's allocator
    (C: swa_set_workspace_allocator): alloc(nbytes) -> device pointer as an
    int (0 when out of memory), free(ptr).  No arguments: back to cudaMalloc
    / cudaFree.  Existing workspaces are released first."""
    global _allocator_keep
    if (alloc is None) != (free is None):
        raise ValueError("give both alloc and free, or neither")
    if alloc is None:
        _check(_lib.swa_set_workspace_allocator(_ALLOC_FN(), _FREE_FN(), None),
               "swa_set_workspace_allocator")
        _allocator_keep = None
        return

    def _a(nbytes, _user):
        try:
            return int(alloc(int(nbytes)) or 0) or None
        except Exception:  # an allocator error is an allocation failure
            return None

    def _f(ptr, _user):
        try:
            free(int(ptr))
        except Exception:
            pass

    keep = (_ALLOC_FN(_a), _FREE_FN(_f))
    _check(_lib.swa_set_workspace_allocator(keep[0], keep[1], None),
           "swa_set_workspace_allocator")
    _allocator_keep = keep
