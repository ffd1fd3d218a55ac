"""Planted mistakes: each mutant of the oracle's C source must fail a pin.

The mutants are built from a text copy of oracle/swa_oracle.c in a temporary
directory; the committed oracle is never modified.  Each models a plausible
slip: the exclusive window end of page "别再只加Mask了" §2.2, a causal clip
that drops the current token, a missing softmax scale, a wrong GQA head map,
no de-duplication of band and global keys, and a max that is not subtracted
consistently.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle
from test_oracle_pins import CASES, _brute, _rand

SRC = os.path.join(os.path.dirname(oracle.__file__), "swa_oracle.c")

MUTANTS = {
    "exclusive_end": ("k <= kmax", "k < kmax"),
    "causal_drops_self": ("keys[t] <= i", "keys[t] < i"),
    "no_scale": ("s[t] = scale * acc;", "s[t] = acc;"),
    "gqa_modulo": ("int g = h / grp;", "int g = h % J->Hkv;"),
    "no_dedup": ("if (u == 0 || keys[t] != keys[u - 1]) keys[u++] = keys[t];",
                 "keys[u++] = keys[t];"),
    "lse_without_max": ("*lse = m + log(l);", "*lse = log(l);"),
}


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, name
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / f"{name}.so"
    subprocess.check_call(["gcc", "-O2", "-shared", "-fPIC", "-o", str(so), str(path),
                           "-lpthread", "-lm"])
    lib = ctypes.CDLL(str(so))
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.oracle_forward.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, I, I, P, I,
                                   ctypes.c_double, P, ctypes.c_int64, I]
    return lib


def _run(lib, q, k, v, L, R, d, bs, G):
    B, N, H, D = q.shape
    Hkv = k.shape[2]
    G = np.ascontiguousarray(np.asarray(G, dtype=np.int32))
    out = np.zeros((B, N, H, D))
    lse = np.zeros((B, H, N))
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    lib.oracle_forward(p(q), p(k), p(v), p(out), p(lse), B, H, Hkv, N, D, L, R, d, bs,
                       p(G), len(G), 1.0 / np.sqrt(D), None, 0, 1)
    return out, lse


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    lib = _build_mutant(tmp_path, name, *MUTANTS[name])
    caught = False
    for N, H, Hkv, D, L, R, d, bs, G in CASES:
        q = _rand((2, N, H, D), 1)
        k = _rand((2, N, Hkv, D), 2)
        v = _rand((2, N, Hkv, D), 3)
        o1, l1 = _run(lib, q, k, v, L, R, d, bs, G)
        o2, l2 = _brute(q, k, v, L, R, d, bs, G)
        if not (np.allclose(o1, o2, atol=1e-12) and np.allclose(l1, l2, atol=1e-12)):
            caught = True
            break
    assert caught, f"mutant {name} passed every brute-force pin"
