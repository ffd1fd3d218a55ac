"""Pins for the fp64 oracle: each checks it against something other than itself.

The pins are chosen so that a plausible mistake in the oracle (a dropped
term, an exclusive bound, a wrong sign, a transposed operand, a wrong GQA
head, a double-counted key) fails at least one of them:

* worked index examples printed on the pages (tests/golden/*.txt);
* brute-force O(N^2) attention with a dense band mask, the way the pages'
  mask pseudo-code builds it (page "滑动窗口注意力", "掩码实现");
* textbook full attention when the window covers the sequence;
* closed forms (zero query -> uniform weights, lse = ln |K(i)|; one-key
  window -> out = v_i);
* invariants (one-hot values expose the weight vector, convex hull,
  causality, residue-class identity for dilation, block-diagonal reduction,
  GQA head mapping, ring rotation, decode = causal forward).
"""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(path):
    out = []
    for line in open(path):
        line = line.strip()
        if line and not line.startswith("#"):
            out.append([int(t) for t in line.split()])
    return out


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape).astype(np.float32)


# ---------------------------------------------------------------- golden pins
def test_dilated_worked_example():
    N, i = 100, 50
    for row in _rows(os.path.join(GOLDEN, "dilated_window_example.txt")):
        w, d, offs = row[0], row[1], row[2:]
        ks = oracle.key_set(i, N, w, w, dilation=d)
        assert list(ks - i) == offs, (w, d)


def test_causal_demo_window():
    for n, W, qi, *keys in _rows(os.path.join(GOLDEN, "causal_demo_window.txt")):
        assert list(oracle.key_set(qi, n, W - 1, 0)) == keys


def test_bidirectional_truncated_window():
    for N, W, qi, first, last in _rows(os.path.join(GOLDEN, "bidirectional_window.txt")):
        half = (W - 1) // 2
        ks = oracle.key_set(qi, N, half, half)
        assert list(ks) == list(range(first, last + 1))


def test_receptive_fields_the_pages_print():
    """Span of the key set after stacking layers: each layer's keys come from
    the oracle's key sets, composed layer by layer (for the causal stacks the
    reach of a contiguous band only depends on its first key)."""
    for W, d, layers, span, tol in _rows(os.path.join(GOLDEN, "receptive_field.txt")):
        if layers == 1:
            w = (W - 1) // 2
            ks = oracle.key_set(1000, 4000, w, w, dilation=d)
            assert len(ks) == W and ks.max() - ks.min() + 1 == span
            continue
        N = layers * W + 10
        i = N - 1
        first = i
        for _ in range(layers):
            ks = oracle.key_set(first, N, W - 1, 0, dilation=d)
            assert list(ks) == list(range(ks.min(), first + 1))  # contiguous, causal
            first = int(ks.min())
        reach = i - first + 1
        assert reach == layers * (W - 1) + 1
        assert abs(reach - span) <= tol


# ------------------------------------------------------- brute force with mask
def _brute(q, k, v, L, R, d=1, bs=0, G=(), scale=None):
    """Dense scores, then a band mask built pair by pair, then softmax."""
    B, N, H, D = q.shape
    Hkv = k.shape[2]
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    if bs and bs > 1:
        bi, bj = i // bs, j // bs
        diff = bj - bi
        lo, hi = -(L // bs) * d, (R // bs) * d
    else:
        diff = j - i
        lo, hi = -L * d, R * d
    allowed = diff % d == 0
    if L >= 0:
        allowed &= diff >= lo
    if R >= 0:
        allowed &= diff <= hi
    G = np.asarray(G, dtype=np.int64)
    if len(G):
        isg = np.zeros(N, dtype=bool)
        isg[G] = True
        allowed |= isg[None, :] | isg[:, None]
    if R == 0:
        allowed &= j <= i
    out = np.zeros((B, N, H, D))
    lse = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            g = h // (H // Hkv)
            s = scale * (q[b, :, h, :].astype(np.float64) @ k[b, :, g, :].astype(np.float64).T)
            s = np.where(allowed, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            p = np.exp(s - m)
            l = p.sum(axis=1, keepdims=True)
            out[b, :, h, :] = (p / l) @ v[b, :, g, :].astype(np.float64)
            lse[b, h, :] = (m + np.log(l))[:, 0]
    return out, lse


CASES = [
    # (N, H, Hkv, D, L, R, d, bs, G)
    (37, 2, 2, 8, 3, 3, 1, 0, ()),          # bidirectional band
    (41, 4, 2, 4, 6, 0, 1, 0, ()),          # causal band, GQA
    (50, 2, 1, 8, 2, 2, 2, 0, ()),          # dilated d=2
    (53, 2, 2, 8, 3, 3, 4, 0, ()),          # dilated d=4, N mod d != 0
    (47, 2, 2, 4, 5, 5, 1, 0, (0, 13, 40)),  # band + globals
    (44, 2, 2, 4, 4, 0, 1, 0, (0, 7, 30)),   # causal + globals
    (64, 2, 2, 4, 16, 16, 2, 4, ()),        # block-level dilation
    (61, 2, 2, 4, 8, 0, 2, 4, (5,)),        # block-level, causal, global, ragged
    (30, 2, 2, 4, -1, 2, 1, 0, ()),         # unbounded left
    (30, 2, 2, 4, 3, -1, 3, 0, ()),         # unbounded right, dilated
]


@pytest.mark.parametrize("case", CASES)
def test_bruteforce_mask(case):
    N, H, Hkv, D, L, R, d, bs, G = case
    q = _rand((2, N, H, D), 1)
    k = _rand((2, N, Hkv, D), 2)
    v = _rand((2, N, Hkv, D), 3)
    o1, l1 = oracle.forward(q, k, v, L, R, d, bs, G, threads=2)
    o2, l2 = _brute(q, k, v, L, R, d, bs, G)
    np.testing.assert_allclose(o1, o2, atol=1e-12, rtol=0)
    np.testing.assert_allclose(l1, l2, atol=1e-12, rtol=0)


try:
    from hypothesis import given, settings, strategies as st
except ImportError:  # pragma: no cover - hypothesis is part of the test image
    given = None


if given is not None:
    @settings(max_examples=80, deadline=None, derandomize=True)
    @given(data=st.data())
    def test_bruteforce_mask_random(data):
        """The same brute-force pin over randomly drawn problems: any window
        kind, dilation, block size, GQA group, global set and scale."""
        N = data.draw(st.integers(1, 70), "N")
        Hkv = data.draw(st.integers(1, 2), "Hkv")
        H = Hkv * data.draw(st.sampled_from([1, 2, 3]), "group")
        D = data.draw(st.sampled_from([4, 8]), "D")
        L = data.draw(st.integers(-1, 24), "L")
        R = data.draw(st.integers(-1, 24), "R")
        d = data.draw(st.integers(1, 5), "d")
        bs = data.draw(st.sampled_from([0, 2, 4, 8]), "bs")
        G = sorted(set(data.draw(st.lists(st.integers(0, N - 1), max_size=4), "G")))
        scale = data.draw(st.sampled_from([None, 0.37]), "scale")
        seed = data.draw(st.integers(0, 10_000), "seed")
        q = _rand((1, N, H, D), seed)
        k = _rand((1, N, Hkv, D), seed + 1)
        v = _rand((1, N, Hkv, D), seed + 2)
        o1, l1 = oracle.forward(q, k, v, L, R, d, bs, G, scale, threads=2)
        o2, l2 = _brute(q, k, v, L, R, d, bs, G, scale)
        np.testing.assert_allclose(o1, o2, atol=1e-12, rtol=0)
        np.testing.assert_allclose(l1, l2, atol=1e-12, rtol=0)


def test_wide_window_is_full_attention():
    N, D = 29, 8
    q, k, v = _rand((1, N, 1, D), 4), _rand((1, N, 1, D), 5), _rand((1, N, 1, D), 6)
    o, lse = oracle.forward(q, k, v, 2 * N, 2 * N)
    s = (q[0, :, 0].astype(np.float64) @ k[0, :, 0].astype(np.float64).T) / np.sqrt(D)
    w = np.exp(s - s.max(1, keepdims=True))
    w /= w.sum(1, keepdims=True)
    np.testing.assert_allclose(o[0, :, 0], w @ v[0, :, 0].astype(np.float64), atol=1e-12)


# ------------------------------------------------------------- closed forms
def test_zero_query_uniform_weights():
    N, D, L, R = 40, 4, 5, 7
    q = np.zeros((1, N, 1, D), np.float32)
    k, v = _rand((1, N, 1, D), 7), _rand((1, N, 1, D), 8)
    o, lse = oracle.forward(q, k, v, L, R)
    for i in range(N):
        lo, hi = max(0, i - L), min(N - 1, i + R)
        assert lse[0, 0, i] == pytest.approx(np.log(hi - lo + 1), abs=1e-13)
        np.testing.assert_allclose(o[0, i, 0], v[0, lo:hi + 1, 0].astype(np.float64).mean(0),
                                   atol=1e-12)


def test_single_key_window():
    N, D = 16, 8
    q, k, v = _rand((1, N, 2, D), 9), _rand((1, N, 2, D), 10), _rand((1, N, 2, D), 11)
    scale = 0.37
    o, lse = oracle.forward(q, k, v, 0, 0, scale=scale)
    np.testing.assert_allclose(o, v.astype(np.float64), atol=1e-14)
    ref = scale * np.einsum("bnhd,bnhd->bhn", q.astype(np.float64), k.astype(np.float64))
    np.testing.assert_allclose(lse, ref, atol=1e-12)


# --------------------------------------------------------------- invariants
def test_onehot_values_expose_weights():
    """v_j = e_j: out_i is the weight vector; it sums to 1 on exactly K(i)."""
    N = 24
    D = N
    q, k = _rand((1, N, 1, D), 12), _rand((1, N, 1, D), 13)
    v = np.eye(N, dtype=np.float32)[None, :, None, :]
    G = (3, 17)
    o, _ = oracle.forward(q, k, v, 2, 3, 2, 0, G)
    for i in range(N):
        w = o[0, i, 0]
        assert w.sum() == pytest.approx(1.0, abs=1e-12)
        support = set(np.nonzero(w > 0)[0].tolist())
        assert support == set(oracle.key_set(i, N, 2, 3, 2, 0, G).tolist())


def test_convex_hull():
    N, D = 33, 6
    q, k, v = _rand((1, N, 1, D), 14), _rand((1, N, 1, D), 15), _rand((1, N, 1, D), 16)
    o, _ = oracle.forward(q, k, v, 4, 4, 2)
    for i in range(N):
        ks = oracle.key_set(i, N, 4, 4, 2)
        vv = v[0, ks, 0].astype(np.float64)
        assert np.all(o[0, i, 0] >= vv.min(0) - 1e-12)
        assert np.all(o[0, i, 0] <= vv.max(0) + 1e-12)


def test_causality():
    N, D, L = 30, 4, 9
    q, k, v = _rand((1, N, 1, D), 17), _rand((1, N, 1, D), 18), _rand((1, N, 1, D), 19)
    o1, l1 = oracle.forward(q, k, v, L, 0)
    cut = 17
    k2, v2 = k.copy(), v.copy()
    k2[:, cut + 1:] += 5.0
    v2[:, cut + 1:] -= 3.0
    o2, l2 = oracle.forward(q, k2, v2, L, 0)
    np.testing.assert_array_equal(o1[:, :cut + 1], o2[:, :cut + 1])
    np.testing.assert_array_equal(l1[:, :, :cut + 1], l2[:, :, :cut + 1])
    assert not np.allclose(o1[:, cut + 1:], o2[:, cut + 1:])


def test_residue_class_identity():
    """Token-level dilation d equals d independent plain bands on x[r::d]."""
    N, D, d, L, R = 43, 4, 3, 4, 2
    q, k, v = _rand((1, N, 2, D), 20), _rand((1, N, 2, D), 21), _rand((1, N, 2, D), 22)
    o, lse = oracle.forward(q, k, v, L, R, d)
    for r in range(d):
        o_r, l_r = oracle.forward(q[:, r::d], k[:, r::d], v[:, r::d], L, R, 1)
        np.testing.assert_allclose(o[:, r::d], o_r, atol=1e-13)
        np.testing.assert_allclose(lse[:, :, r::d], l_r, atol=1e-13)


def test_block_level_reduces_to_block_diagonal():
    """win < block and d = 1: each 64-token block attends only to itself, which
    is the non-overlapping block attention of page "别再只加Mask了", §2.1."""
    bs, nb, D = 8, 5, 4
    N = bs * nb
    q, k, v = _rand((1, N, 1, D), 23), _rand((1, N, 1, D), 24), _rand((1, N, 1, D), 25)
    o, _ = oracle.forward(q, k, v, bs - 1, bs - 1, 1, bs)
    qb = q[0, :, 0].reshape(nb, bs, D).astype(np.float64)
    kb = k[0, :, 0].reshape(nb, bs, D).astype(np.float64)
    vb = v[0, :, 0].reshape(nb, bs, D).astype(np.float64)
    s = np.einsum("nqd,nkd->nqk", qb, kb) / np.sqrt(D)
    w = np.exp(s - s.max(-1, keepdims=True))
    w /= w.sum(-1, keepdims=True)
    ref = np.einsum("nqk,nkd->nqd", w, vb).reshape(N, D)
    np.testing.assert_allclose(o[0, :, 0], ref, atol=1e-12)


def test_block_level_dilation_blocks():
    """Config-4 reading: L=R=128, Bs=64, d=4 -> blocks b-8, b-4, b, b+4, b+8."""
    N = 64 * 32
    i = 64 * 16 + 5
    ks = oracle.key_set(i, N, 128, 128, 4, 64)
    blocks = sorted(set((ks // 64).tolist()))
    assert blocks == [8, 12, 16, 20, 24]
    assert len(ks) == 320


def test_globals_all_and_none():
    N, D = 20, 4
    q, k, v = _rand((1, N, 1, D), 26), _rand((1, N, 1, D), 27), _rand((1, N, 1, D), 28)
    o_all, _ = oracle.forward(q, k, v, 1, 1, global_idx=range(N))
    o_full, _ = oracle.forward(q, k, v, -1, -1)
    np.testing.assert_allclose(o_all, o_full, atol=1e-13)
    o_none, _ = oracle.forward(q, k, v, 1, 1, global_idx=())
    o_band, _ = _brute(q, k, v, 1, 1)
    np.testing.assert_allclose(o_none, o_band, atol=1e-12)


def test_gqa_head_mapping():
    """Query head h reads kv head h // (H/Hkv): equal to repeating kv heads."""
    N, D, H, Hkv = 18, 4, 6, 2
    q = _rand((1, N, H, D), 29)
    k, v = _rand((1, N, Hkv, D), 30), _rand((1, N, Hkv, D), 31)
    o1, l1 = oracle.forward(q, k, v, 3, 3)
    kr, vr = np.repeat(k, H // Hkv, axis=2), np.repeat(v, H // Hkv, axis=2)
    o2, l2 = oracle.forward(q, kr, vr, 3, 3)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_rows_subset_matches_full():
    N, D = 25, 4
    q, k, v = _rand((2, N, 3, D), 32), _rand((2, N, 3, D), 33), _rand((2, N, 3, D), 34)
    o, lse = oracle.forward(q, k, v, 3, 5, 2, 0, (4,))
    rows = np.array([[1, 2, 7], [0, 0, 0], [1, 1, 24]])
    o2, l2 = oracle.forward(q, k, v, 3, 5, 2, 0, (4,), rows=rows)
    for t, (b, h, i) in enumerate(rows):
        np.testing.assert_array_equal(o2[t], o[b, i, h])
        assert l2[t] == lse[b, h, i]


# ---------------------------------------------------------------- ring decode
def _derotate(kr, pos, W):
    """Linear sequence of the positions max(0,pos-W+1)..pos from the ring."""
    first = max(0, pos - W + 1)
    return np.stack([kr[t % W] for t in range(first, pos + 1)])


@pytest.mark.parametrize("pos", [3, 15, 16, 40, 1000])
def test_decode_is_causal_forward(pos):
    W, H, Hkv, D = 16, 4, 2, 8
    q = _rand((1, H, D), 35)
    kr, vr = _rand((1, W, Hkv, D), 36), _rand((1, W, Hkv, D), 37)
    o, lse = oracle.decode(q, kr, vr, [pos])
    ks, vs = _derotate(kr[0], pos, W), _derotate(vr[0], pos, W)
    n = ks.shape[0]
    qs = np.zeros((1, n, H, D), np.float32)
    qs[0, -1] = q[0]
    of, lf = oracle.forward(qs, ks[None], vs[None], W - 1, 0)
    np.testing.assert_allclose(o[0], of[0, -1], atol=1e-13)
    np.testing.assert_allclose(lse[0], lf[0, :, -1], atol=1e-13)


def test_decode_rotation_invariance():
    W, H, Hkv, D, pos = 12, 2, 1, 4, 30
    q = _rand((1, H, D), 38)
    kr, vr = _rand((1, W, Hkv, D), 39), _rand((1, W, Hkv, D), 40)
    o1, l1 = oracle.decode(q, kr, vr, [pos])
    shift = 5  # same tokens, written 5 positions later into the ring
    kr2, vr2 = np.roll(kr, shift, axis=1), np.roll(vr, shift, axis=1)
    o2, l2 = oracle.decode(q, kr2, vr2, [pos + shift])
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)
