"""fp64 CPU oracle for sliding-window attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (``sliding_window_attention_fwd_b200``) never imports it, and it
imports nothing from the product.

The arithmetic lives in ``swa_oracle.c`` (plain C, fp64, one query at a time
over an explicit key list); this module only builds/loads it and marshals
numpy arrays.  Every function states the page passage it follows in the C
source.  ``block-level dilation`` (``dilation_block > 1``) is parity
unpinned by any printed value: it is pinned only by its reductions to
block-diagonal attention and to a block-aligned band (see tests).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "swa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile swa_oracle.c into liboracle.so (gcc, -O2) if stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(
            ["gcc", "-O2", "-shared", "-fPIC", "-o", _LIB, _SRC, "-lpthread", "-lm"]
        )
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_key_set.argtypes = [I, I, I, I, I, I, P, I, P]
        lib.oracle_key_set.restype = I
        lib.oracle_forward.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, I, I, P, I,
                                       ctypes.c_double, P, ctypes.c_int64, I]
        lib.oracle_forward.restype = None
        lib.oracle_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, ctypes.c_double, I]
        lib.oracle_decode.restype = None
        lib.oracle_decode_paged.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I,
                                            ctypes.c_double, I]
        lib.oracle_decode_paged.restype = None
        lib.oracle_append.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I,
                                      ctypes.c_double, I]
        lib.oracle_append.restype = None
        lib.oracle_backward.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, P, I,
                                        ctypes.c_double, I]
        lib.oracle_backward.restype = None
        _lib = lib
    return _lib


def _f32(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor (possibly bf16) -> exact fp32 numpy
        a = a.detach().to("cpu").float().numpy()
    return np.ascontiguousarray(a, dtype=np.float32)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def key_set(i, N, win_left, win_right, dilation=1, dilation_block=0, global_idx=()):
    """K(i): sorted unique key indices query i attends to."""
    lib = _load()
    G = np.ascontiguousarray(np.asarray(global_idx, dtype=np.int32))
    buf = np.zeros(N + len(G) + 1, dtype=np.int32)
    n = lib.oracle_key_set(int(i), int(N), int(win_left), int(win_right), int(dilation),
                           int(dilation_block), _ptr(G), len(G), _ptr(buf))
    return buf[:n].copy()


def forward(q, k, v, win_left, win_right, dilation=1, dilation_block=0, global_idx=(),
            scale=None, rows=None, threads=None):
    """fp64 SWA forward.

    q [B,N,H,D], k/v [B,N,Hkv,D].  Returns (out, lse): with ``rows=None`` out is
    [B,N,H,D] and lse [B,H,N]; with ``rows`` an int array of (b,h,i) triples,
    out is [len(rows),D] and lse [len(rows)].  ``scale`` None or <= 0 means
    1/sqrt(D).
    """
    lib = _load()
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, N, H, D = q.shape
    Hkv = k.shape[2]
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(D)
    G = np.ascontiguousarray(np.asarray(global_idx, dtype=np.int32))
    if rows is None:
        out = np.zeros((B, N, H, D), dtype=np.float64)
        lse = np.zeros((B, H, N), dtype=np.float64)
        rp, nr = None, 0
    else:
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
        out = np.zeros((rows.shape[0], D), dtype=np.float64)
        lse = np.zeros((rows.shape[0],), dtype=np.float64)
        rp, nr = _ptr(rows), rows.shape[0]
    lib.oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Hkv, N, D,
                       int(win_left), int(win_right), int(dilation), int(dilation_block),
                       _ptr(G), len(G), float(scale), rp, nr,
                       int(threads or default_threads()))
    return out, lse


def decode(q, k_ring, v_ring, pos, scale=None, threads=None):
    """fp64 ring-buffer decode.  q [B,H,D], k_ring/v_ring [B,W,Hkv,D], pos [B].

    Returns (out [B,H,D], lse [B,H]).
    """
    lib = _load()
    q, kr, vr = _f32(q), _f32(k_ring), _f32(v_ring)
    if hasattr(pos, "detach"):
        pos = pos.detach().cpu().numpy()
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64))
    B, H, D = q.shape
    W, Hkv = kr.shape[1], kr.shape[2]
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(D)
    out = np.zeros((B, H, D), dtype=np.float64)
    lse = np.zeros((B, H), dtype=np.float64)
    lib.oracle_decode(_ptr(q), _ptr(kr), _ptr(vr), _ptr(pos), _ptr(out), _ptr(lse),
                      B, H, Hkv, D, W, float(scale), int(threads or default_threads()))
    return out, lse


def _i64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.int64))


def decode_paged(q, k_pages, v_pages, block_table, pos, page_size, W, scale=None, threads=None):
    """fp64 paged decode.  q [B,H,D]; k_pages/v_pages [rows,Hkv,D] with rows a
    multiple of page_size; block_table [B,max_pages] int32 (logical page ->
    physical page); pos [B].  Returns (out [B,H,D], lse [B,H])."""
    lib = _load()
    q, kp, vp = _f32(q), _f32(k_pages), _f32(v_pages)
    if hasattr(block_table, "detach"):
        block_table = block_table.detach().cpu().numpy()
    table = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32))
    pos = _i64(pos)
    B, H, D = q.shape
    Hkv = kp.shape[1]
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(D)
    out = np.zeros((B, H, D), dtype=np.float64)
    lse = np.zeros((B, H), dtype=np.float64)
    lib.oracle_decode_paged(_ptr(q), _ptr(kp), _ptr(vp), _ptr(table), _ptr(pos), _ptr(out),
                            _ptr(lse), B, H, Hkv, D, int(page_size), table.shape[1], int(W),
                            float(scale), int(threads or default_threads()))
    return out, lse


def append(q, k_ring, v_ring, k_new, v_new, pos0, scale=None, threads=None):
    """fp64 chunked append.  q [B,C,H,D]; k_ring/v_ring [B,W,Hkv,D] (the cache
    before the chunk); k_new/v_new [B,C,Hkv,D]; pos0 [B] = position of the
    chunk's first token.  Returns (out [B,C,H,D], lse [B,H,C])."""
    lib = _load()
    q, kr, vr, kn, vn = _f32(q), _f32(k_ring), _f32(v_ring), _f32(k_new), _f32(v_new)
    pos0 = _i64(pos0)
    B, C, H, D = q.shape
    W, Hkv = kr.shape[1], kr.shape[2]
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(D)
    out = np.zeros((B, C, H, D), dtype=np.float64)
    lse = np.zeros((B, H, C), dtype=np.float64)
    lib.oracle_append(_ptr(q), _ptr(kr), _ptr(vr), _ptr(kn), _ptr(vn), _ptr(pos0), _ptr(out),
                      _ptr(lse), B, C, H, Hkv, D, W, float(scale),
                      int(threads or default_threads()))
    return out, lse


def backward(q, k, v, dout, win_left, win_right, dilation=1, dilation_block=0, global_idx=(),
             scale=None, threads=None):
    """fp64 gradients (dq [B,N,H,D], dk, dv [B,N,Hkv,D]) of the forward for an
    upstream gradient dout [B,N,H,D]."""
    lib = _load()
    q, k, v, do = _f32(q), _f32(k), _f32(v), _f32(dout)
    B, N, H, D = q.shape
    Hkv = k.shape[2]
    G = np.ascontiguousarray(np.asarray(global_idx, dtype=np.int32))
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(D)
    dq = np.zeros((B, N, H, D), dtype=np.float64)
    dk = np.zeros((B, N, Hkv, D), dtype=np.float64)
    dv = np.zeros((B, N, Hkv, D), dtype=np.float64)
    lib.oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv), B, H,
                        Hkv, N, D, int(win_left), int(win_right), int(dilation),
                        int(dilation_block), _ptr(G), len(G), float(scale),
                        int(threads or default_threads()))
    return dq, dk, dv
