"""Backward parity: swa_backward (C ABI) against the fp64 oracle's gradients,
on every element, for causal GQA, token and block dilation, global tokens
and full causal attention.  The GPU takes out and lse from its own forward,
as a training step would.

Tolerance (derived, not fitted): inputs, out, dout and the results are bf16,
so each term of the gradient sums carries a relative rounding error of about
2^-8 (the D_i = dout . out term included); sums of many such terms with
mixed signs stay well inside 2e-2 of the largest gradient entry (max abs)
and 1e-2 of the mean magnitude (mean abs)."""
import numpy as np
import pytest
import torch

import oracle
from sliding_window_attention_fwd_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def swa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import sliding_window_attention_fwd_b200 as m
    return m


def rel_check(got, ref, what):
    err = np.abs(got - ref)
    scale_max = max(np.abs(ref).max(), 1e-6)
    scale_mean = max(np.abs(ref).mean(), 1e-6)
    assert err.max() <= 2e-2 * scale_max, f"{what}: max abs {err.max():.3e} vs {scale_max:.3e}"
    assert err.mean() <= 1e-2 * scale_mean, f"{what}: mean abs {err.mean():.3e} vs {scale_mean:.3e}"


@pytest.mark.parametrize("B,N,H,Hkv,D,L,R,d,bs,G", [
    (1, 300, 4, 2, 128, 64, 0, 1, 0, None),
    (2, 257, 2, 2, 64, 32, 32, 2, 0, None),
    (1, 320, 2, 1, 64, 128, 128, 2, 64, None),
    (1, 300, 4, 4, 128, 50, 50, 1, 0, [0, 150]),
    (1, 200, 8, 1, 128, -1, 0, 1, 0, None),
])
def test_backward_matches_oracle(swa, B, N, H, Hkv, D, L, R, d, bs, G):
    seed = N + H + D
    q = inputs.normal((B, N, H, D), seed, 0)
    k = inputs.normal((B, N, Hkv, D), seed, 1)
    v = inputs.normal((B, N, Hkv, D), seed, 2)
    do = inputs.normal((B, N, H, D), seed, 3)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    gi = torch.tensor(G, dtype=torch.int32, device="cuda") if G else None
    lse = torch.empty(B, H, N, device="cuda")
    out = swa.swa_forward_ex(qd, kd, vd, None, lse, L, R, d, bs, gi)
    dq, dk, dv = swa.swa_backward(qd, kd, vd, out, dod, lse, L, R, d, bs, gi)
    torch.cuda.synchronize()
    assert swa.swa_device_error() == 0
    rq, rk, rv = oracle.backward(q, k, v, do, L, R, d, bs, G or [])
    rel_check(dq.float().cpu().numpy(), rq, "dq")
    rel_check(dk.float().cpu().numpy(), rk, "dk")
    rel_check(dv.float().cpu().numpy(), rv, "dv")
    # the closed forms hold on the GPU too (up to bf16 rounding of each row)
    assert np.abs(dk.float().sum(1).cpu().numpy()).max() <= 2e-2 * N * max(np.abs(rk).max(), 1e-6)


def test_backward_twice_gives_identical_results(swa):
    """The fp32 accumulators are cleared on every call (atomics sum in a
    different order, so compare two runs within rounding, not bitwise)."""
    B, N, H, Hkv, D = 1, 200, 4, 2, 128
    q, k, v, do = (inputs.normal(s, 77, t).cuda() for t, s in
                   enumerate([(B, N, H, D), (B, N, Hkv, D), (B, N, Hkv, D), (B, N, H, D)]))
    lse = torch.empty(B, H, N, device="cuda")
    out = swa.swa_forward(q, k, v, None, lse, 100, 0)
    a = swa.swa_backward(q, k, v, out, do, lse, 100, 0)
    a = [t.clone() for t in a]
    b = swa.swa_backward(q, k, v, out, do, lse, 100, 0)
    for x, y in zip(a, b):
        assert (x.float() - y.float()).abs().max().item() <= 1e-2 * x.float().abs().max().item()
