"""Pins of the oracle's backward pass (no GPU).

The pages print no backward pass; the oracle writes out the derivative of
the forward definition.  It is pinned by things other than itself:
  * central finite differences of the (separately pinned) forward oracle's
    loss  L = sum(out * dout)  for band, causal, dilated, block-dilated and
    global-token windows;
  * closed forms that hold for any window: sum_j dK_j = 0 and
    sum_j dV_j = sum over the group's query rows of dout (softmax rows sum to
    one, and the rows of dS sum to zero);
  * full attention (window wider than the sequence) equals torch autograd of
    textbook softmax attention in fp64, and so does dense attention with the
    key-set mask over randomly drawn windows;
Planted mistakes in a copy of the C source each fail one of them.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "swa_oracle.c")

CASES = [  # (N, L, R, d, bs, G)
    (24, 3, 2, 1, 0, []),
    (24, 5, 0, 1, 0, []),
    (30, 2, 2, 3, 0, []),
    (32, 8, 8, 2, 4, []),
    (24, 2, 2, 1, 0, [0, 13]),
    (24, 4, 0, 1, 0, [0, 7]),
]


def _rand(rng, B, N, H, Hkv, D):
    f = lambda *s: rng.standard_normal(s).astype(np.float32)
    return f(B, N, H, D), f(B, N, Hkv, D), f(B, N, Hkv, D), f(B, N, H, D)


def _loss(q, k, v, do, L, R, d, bs, G):
    out, _ = oracle.forward(q, k, v, L, R, d, bs, G, 0.0)
    return float((out * do.astype(np.float64)).sum())


@pytest.mark.parametrize("case", CASES)
def test_backward_matches_finite_differences(case):
    N, L, R, d, bs, G = case
    rng = np.random.default_rng(N + L + 7 * d)
    B, H, Hkv, D = 1, 2, 1, 8
    q, k, v, do = _rand(rng, B, N, H, Hkv, D)
    dq, dk, dv = oracle.backward(q, k, v, do, L, R, d, bs, G)
    eps = 2.0 ** -7
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, s)) for s in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            ap = dict(args, **{name: xp})
            am = dict(args, **{name: xm})
            num = (_loss(ap["q"], ap["k"], ap["v"], do, L, R, d, bs, G)
                   - _loss(am["q"], am["k"], am["v"], do, L, R, d, bs, G)) / (
                       float(xp[idx]) - float(xm[idx]))
            assert abs(num - g[idx]) <= 2e-4 + 2e-3 * abs(num), (case, name, idx, num, g[idx])


@pytest.mark.parametrize("case", CASES)
def test_backward_closed_forms(case):
    N, L, R, d, bs, G = case
    rng = np.random.default_rng(3 * N + L)
    B, H, Hkv, D = 2, 4, 2, 16
    q, k, v, do = _rand(rng, B, N, H, Hkv, D)
    dq, dk, dv = oracle.backward(q, k, v, do, L, R, d, bs, G)
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-11)
    grp = H // Hkv
    dsum = do.astype(np.float64).reshape(B, N, Hkv, grp, D).sum(axis=(1, 3))
    np.testing.assert_allclose(dv.sum(axis=1), dsum, rtol=0, atol=1e-10)


def test_full_window_equals_autograd_softmax_attention():
    rng = np.random.default_rng(5)
    B, N, H, Hkv, D = 1, 16, 4, 2, 8
    q, k, v, do = _rand(rng, B, N, H, Hkv, D)
    dq, dk, dv = oracle.backward(q, k, v, do, 2 * N, 2 * N)
    tq, tk, tv = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
    kk = tk.repeat_interleave(H // Hkv, dim=2)
    vv = tv.repeat_interleave(H // Hkv, dim=2)
    s = torch.einsum("bihd,bjhd->bhij", tq, kk) / np.sqrt(D)
    out = torch.einsum("bhij,bjhd->bihd", torch.softmax(s, -1), vv)
    (out * torch.tensor(do, dtype=torch.float64)).sum().backward()
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=0, atol=1e-12)


def _allowed(N, L, R, d, bs, G):
    """Pair-wise key-set predicate written from the definition (band, then
    globals, then the causal cut), independent of the oracle's index lists."""
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    if bs > 1:
        diff, lo, hi = j // bs - i // bs, -(L // bs) * d, (R // bs) * d
    else:
        diff, lo, hi = j - i, -L * d, R * d
    ok = diff % d == 0
    if L >= 0:
        ok &= diff >= lo
    if R >= 0:
        ok &= diff <= hi
    isg = np.zeros(N, dtype=bool)
    isg[list(G)] = True
    ok |= isg[None, :] | isg[:, None]
    if R == 0:
        ok &= j <= i
    return ok


try:
    from hypothesis import given, settings, strategies as st
except ImportError:  # pragma: no cover - hypothesis is part of the test image
    given = None


if given is not None:
    @settings(max_examples=40, deadline=None, derandomize=True)
    @given(data=st.data())
    def test_masked_autograd_random(data):
        """Over randomly drawn windows (band, causal, dilated, block-dilated,
        global tokens, GQA) the oracle's gradients equal torch autograd of
        dense fp64 attention with the key-set mask."""
        N = data.draw(st.integers(1, 40), "N")
        Hkv = data.draw(st.integers(1, 2), "Hkv")
        H = Hkv * data.draw(st.sampled_from([1, 2, 3]), "group")
        D = data.draw(st.sampled_from([4, 8]), "D")
        L = data.draw(st.integers(-1, 12), "L")
        R = data.draw(st.integers(-1, 12), "R")
        d = data.draw(st.integers(1, 4), "d")
        bs = data.draw(st.sampled_from([0, 2, 4]), "bs")
        G = sorted(set(data.draw(st.lists(st.integers(0, N - 1), max_size=3), "G")))
        rng = np.random.default_rng(data.draw(st.integers(0, 10_000), "seed"))
        q, k, v, do = _rand(rng, 1, N, H, Hkv, D)
        dq, dk, dv = oracle.backward(q, k, v, do, L, R, d, bs, G)
        tq, tk, tv = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
        kk = tk.repeat_interleave(H // Hkv, dim=2)
        vv = tv.repeat_interleave(H // Hkv, dim=2)
        s = torch.einsum("bihd,bjhd->bhij", tq, kk) / np.sqrt(D)
        mask = torch.tensor(_allowed(N, L, R, d, bs, G))
        s = torch.where(mask, s, torch.tensor(float("-inf"), dtype=torch.float64))
        out = torch.einsum("bhij,bjhd->bihd", torch.softmax(s, -1), vv)
        (out * torch.tensor(do, dtype=torch.float64)).sum().backward()
        np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=0, atol=1e-11)


MUTANTS = {
    "no_rowsum_term": ("double ds = s[t] * (dp[t] - Di);", "double ds = s[t] * dp[t];"),
    "dq_without_scale": ("dqi[c] += J->scale * ds * (double)kr[c];",
                         "dqi[c] += ds * (double)kr[c];"),
    "dv_from_dp": ("dvr[c] += s[t] * (double)doi[c];", "dvr[c] += dp[t] * (double)doi[c];"),
    "dk_from_key": ("dkr[c] += J->scale * ds * (double)qi[c];",
                    "dkr[c] += J->scale * ds * (double)kr[c];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(tmp_path, name, monkeypatch):
    old, new = MUTANTS[name]
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
    lib.oracle_backward.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, P, I,
                                    ctypes.c_double, I]
    monkeypatch.setattr(oracle, "_lib", lib)
    failed = False
    for t in (lambda: test_backward_matches_finite_differences(CASES[0]),
              lambda: test_backward_closed_forms(CASES[1]),
              test_full_window_equals_autograd_softmax_attention):
        try:
            t()
        except AssertionError:
            failed = True
    assert failed, f"mutant {name} passed every pin"
