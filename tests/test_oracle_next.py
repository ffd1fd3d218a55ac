"""Pins of the oracle's paged decode and chunked append (no GPU).

Both are exact attention over the same key set as the ring decode, only the
storage differs, so each is pinned by reductions and invariants that do not
retype its code:
  * paged decode equals causal windowed attention (the forward oracle) on the
    contiguous sequence, whatever the physical page order; pages that left the
    window are never read (filled with NaN here); a one-key window returns the
    value row itself;
  * chunked append equals the forward oracle on the contiguous sequence
    (history + chunk), also when the history is shorter than the window and
    when the chunk wraps the ring; it equals C single-token decodes with the
    ring updated between them.
Planted mistakes in a copy of the C source must each fail one of these.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "swa_oracle.c")


def _seq(rng, B, N, H, Hkv, D):
    q = rng.standard_normal((B, N, H, D)).astype(np.float32)
    k = rng.standard_normal((B, N, Hkv, D)).astype(np.float32)
    v = rng.standard_normal((B, N, Hkv, D)).astype(np.float32)
    return q, k, v


def _pages_from_seq(rng, k, v, ps, max_pages, n_phys, evict_before=None):
    """Scatter each sequence's tokens into randomly chosen physical pages."""
    B, N, Hkv, D = k.shape
    kp = np.full((n_phys * ps, Hkv, D), np.nan, dtype=np.float32)
    vp = np.full((n_phys * ps, Hkv, D), np.nan, dtype=np.float32)
    perm = rng.permutation(n_phys)
    table = np.full((B, max_pages), -1, dtype=np.int32)
    nxt = 0
    for b in range(B):
        for lp in range((N + ps - 1) // ps):
            phys = int(perm[nxt]); nxt += 1
            table[b, lp] = phys
            lo, hi = lp * ps, min(N, lp * ps + ps)
            if evict_before is not None and hi <= evict_before[b]:
                continue  # evicted page: left as NaN, must never be read
            kp[phys * ps:phys * ps + hi - lo] = k[b, lo:hi]
            vp[phys * ps:phys * ps + hi - lo] = v[b, lo:hi]
    return kp, vp, table


def _forward_rows(q, k, v, W, rows):
    o, l = oracle.forward(q, k, v, W - 1, 0, 1, 0, [], 0.0, rows=np.asarray(rows, np.int64))
    return o, l


@pytest.mark.parametrize("W,ps,N", [(100, 64, 300), (256, 128, 300), (64, 64, 64), (500, 64, 130)])
def test_paged_equals_forward_any_page_order(W, ps, N):
    rng = np.random.default_rng(W + ps + N)
    B, H, Hkv, D = 2, 4, 2, 32
    q, k, v = _seq(rng, B, N, H, Hkv, D)
    pos = np.array([N - 1, N // 2 + 3])
    first = np.maximum(0, pos - W + 1)
    kp, vp, table = _pages_from_seq(rng, k, v, ps, (N + ps - 1) // ps + 1, 2 * ((N + ps - 1) // ps) + 2,
                                    evict_before=(first // ps) * ps)
    qd = np.stack([q[b, pos[b]] for b in range(B)])
    o, l = oracle.decode_paged(qd, kp, vp, table, pos, ps, W)
    rows = [(b, h, pos[b]) for b in range(B) for h in range(H)]
    ro, rl = _forward_rows(q, k, v, W, rows)
    assert np.isfinite(o).all()
    np.testing.assert_allclose(o.reshape(B * H, D), ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l.reshape(B * H), rl, rtol=0, atol=1e-12)


def test_paged_single_key_window_returns_value_row():
    rng = np.random.default_rng(3)
    B, N, H, Hkv, D, ps = 1, 200, 2, 1, 16, 64
    q, k, v = _seq(rng, B, N, H, Hkv, D)
    pos = np.array([137])
    kp, vp, table = _pages_from_seq(rng, k, v, ps, 4, 6, evict_before=np.array([128]))
    o, l = oracle.decode_paged(q[:, 137], kp, vp, table, pos, ps, 1)
    for h in range(H):
        np.testing.assert_allclose(o[0, h], v[0, 137, 0], rtol=0, atol=1e-12)
        s = float(np.dot(q[0, 137, h].astype(np.float64), k[0, 137, 0].astype(np.float64))) / 4.0
        assert abs(l[0, h] - s) < 1e-12


def _ring_from_seq(k, v, pos0, W):
    """The ring as it stands before position pos0: slot t % W holds token t."""
    B, N, Hkv, D = k.shape
    kr = np.zeros((B, W, Hkv, D), np.float32)
    vr = np.zeros((B, W, Hkv, D), np.float32)
    for b in range(B):
        for t in range(max(0, pos0[b] - W), pos0[b]):
            kr[b, t % W] = k[b, t]
            vr[b, t % W] = v[b, t]
    return kr, vr


@pytest.mark.parametrize("W,C,p0", [(64, 16, 200), (64, 16, 10), (128, 40, 250), (32, 70, 100),
                                    (64, 1, 63)])
def test_append_equals_forward_on_contiguous_sequence(W, C, p0):
    rng = np.random.default_rng(W * 7 + C + p0)
    B, H, Hkv, D = 2, 4, 2, 32
    pos0 = np.array([p0, p0 + 5])
    N = int(pos0.max()) + C
    q, k, v = _seq(rng, B, N, H, Hkv, D)
    kr, vr = _ring_from_seq(k, v, pos0, W)
    qc = np.stack([q[b, pos0[b]:pos0[b] + C] for b in range(B)])
    kn = np.stack([k[b, pos0[b]:pos0[b] + C] for b in range(B)])
    vn = np.stack([v[b, pos0[b]:pos0[b] + C] for b in range(B)])
    o, l = oracle.append(qc, kr, vr, kn, vn, pos0)
    rows = [(b, h, pos0[b] + c) for b in range(B) for c in range(C) for h in range(H)]
    ro, rl = _forward_rows(q, k, v, W, rows)
    np.testing.assert_allclose(o.reshape(B * C * H, D), ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l.transpose(0, 2, 1).reshape(B * C * H), rl, rtol=0, atol=1e-12)


def test_append_equals_token_by_token_decode():
    rng = np.random.default_rng(11)
    B, C, H, Hkv, D, W = 2, 9, 4, 2, 16, 24
    pos0 = np.array([30, 5])
    N = int(pos0.max()) + C
    q, k, v = _seq(rng, B, N, H, Hkv, D)
    kr, vr = _ring_from_seq(k, v, pos0, W)
    qc = np.stack([q[b, pos0[b]:pos0[b] + C] for b in range(B)])
    kn = np.stack([k[b, pos0[b]:pos0[b] + C] for b in range(B)])
    vn = np.stack([v[b, pos0[b]:pos0[b] + C] for b in range(B)])
    o, l = oracle.append(qc, kr, vr, kn, vn, pos0)
    kr2, vr2 = kr.copy(), vr.copy()
    for c in range(C):
        for b in range(B):
            kr2[b, (pos0[b] + c) % W] = kn[b, c]
            vr2[b, (pos0[b] + c) % W] = vn[b, c]
        od, ld = oracle.decode(qc[:, c], kr2, vr2, pos0 + c)
        np.testing.assert_allclose(o[:, c], od, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l[:, :, c], ld, rtol=0, atol=1e-12)


# ------------------------------------------------------------ planted mistakes
MUTANTS = {
    "paged_row_in_page": ("keys[nk++] = (int)(page * J->ps + t % J->ps);",
                          "keys[nk++] = (int)(page * J->ps + (t + 1) % J->ps);"),
    "paged_window_one_short": ("for (int64_t t = first; t <= p; ++t) {\n      int64_t page",
                               "for (int64_t t = first + 1; t <= p; ++t) {\n      int64_t page"),
    "append_first_new_from_ring": ("if (t >= J->pos0[b]) {", "if (t > J->pos0[b]) {"),
    "append_slot_from_position": ("long row = ((long)b * J->W + t % J->W) * J->Hkv + kvh;",
                                  "long row = ((long)b * J->W + (t + 1) % J->W) * J->Hkv + kvh;"),
}


def _mutant_lib(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, name
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / f"{name}.so"
    subprocess.check_call(["gcc", "-O2", "-shared", "-fPIC", "-o", str(so), str(path),
                           "-lpthread", "-lm"])
    return ctypes.CDLL(str(so))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(tmp_path, name, monkeypatch):
    lib = _mutant_lib(tmp_path, name)
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.oracle_forward.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, I, I, P, I,
                                   ctypes.c_double, P, ctypes.c_int64, I]
    lib.oracle_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, ctypes.c_double, I]
    lib.oracle_decode_paged.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I,
                                        ctypes.c_double, I]
    lib.oracle_append.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, ctypes.c_double, I]
    monkeypatch.setattr(oracle, "_lib", lib)
    failed = False
    tests = [lambda: test_paged_equals_forward_any_page_order(100, 64, 300),
             lambda: test_append_equals_forward_on_contiguous_sequence(64, 16, 200)]
    for t in tests:
        try:
            t()
        except AssertionError:
            failed = True
    assert failed, f"mutant {name} passed every pin"


try:
    from hypothesis import given, settings, strategies as st
except ImportError:  # pragma: no cover - hypothesis is part of the test image
    given = None


if given is not None:
    @settings(max_examples=40, deadline=None, derandomize=True)
    @given(data=st.data())
    def test_paged_equals_forward_random(data):
        """Paged decode = the forward oracle's causal window, over random
        windows, page sizes, positions, GQA groups and page orders."""
        B = data.draw(st.integers(1, 3), "B")
        Hkv = data.draw(st.integers(1, 2), "Hkv")
        H = Hkv * data.draw(st.sampled_from([1, 2, 4]), "group")
        D = data.draw(st.sampled_from([8, 16]), "D")
        N = data.draw(st.integers(1, 260), "N")
        W = data.draw(st.integers(1, 300), "W")
        ps = data.draw(st.sampled_from([8, 64, 96]), "page_size")
        pos = np.array([data.draw(st.integers(0, N - 1), f"pos{b}") for b in range(B)])
        rng = np.random.default_rng(data.draw(st.integers(0, 10_000), "seed"))
        q, k, v = _seq(rng, B, N, H, Hkv, D)
        first = np.maximum(0, pos - W + 1)
        n_lp = (N + ps - 1) // ps
        kp, vp, table = _pages_from_seq(rng, k, v, ps, n_lp, B * n_lp,
                                        evict_before=(first // ps) * ps)
        qd = np.stack([q[b, pos[b]] for b in range(B)])
        o, l = oracle.decode_paged(qd, kp, vp, table, pos, ps, W)
        rows = [(b, h, pos[b]) for b in range(B) for h in range(H)]
        ro, rl = _forward_rows(q, k, v, W, rows)
        assert np.isfinite(o).all()
        np.testing.assert_allclose(o.reshape(B * H, D), ro, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l.reshape(B * H), rl, rtol=0, atol=1e-12)

    @settings(max_examples=40, deadline=None, derandomize=True)
    @given(data=st.data())
    def test_append_equals_forward_random(data):
        """Chunked append = the forward oracle on history + chunk, over random
        windows, chunk lengths (also longer than the ring), start positions
        (also inside the first window) and GQA groups."""
        B = data.draw(st.integers(1, 2), "B")
        Hkv = data.draw(st.integers(1, 2), "Hkv")
        H = Hkv * data.draw(st.sampled_from([1, 3, 4]), "group")
        D = data.draw(st.sampled_from([8, 16]), "D")
        W = data.draw(st.integers(1, 96), "W")
        C = data.draw(st.integers(1, 80), "C")
        pos0 = np.array([data.draw(st.integers(0, 300), f"pos0_{b}") for b in range(B)])
        rng = np.random.default_rng(data.draw(st.integers(0, 10_000), "seed"))
        N = int(pos0.max()) + C
        q, k, v = _seq(rng, B, N, H, Hkv, D)
        kr, vr = _ring_from_seq(k, v, pos0, W)
        qc = np.stack([q[b, pos0[b]:pos0[b] + C] for b in range(B)])
        kn = np.stack([k[b, pos0[b]:pos0[b] + C] for b in range(B)])
        vn = np.stack([v[b, pos0[b]:pos0[b] + C] for b in range(B)])
        o, l = oracle.append(qc, kr, vr, kn, vn, pos0)
        rows = [(b, h, pos0[b] + c) for b in range(B) for c in range(C) for h in range(H)]
        ro, rl = _forward_rows(q, k, v, W, rows)
        np.testing.assert_allclose(o.reshape(B * C * H, D), ro, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l.transpose(0, 2, 1).reshape(B * C * H), rl, rtol=0,
                                   atol=1e-12)
