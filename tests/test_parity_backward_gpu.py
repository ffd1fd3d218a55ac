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
    # band problems run on the tensor-core kernels: several query and key
    # tiles, ragged tails, every window kind
    (1, 1000, 8, 2, 128, 300, 0, 1, 0, None),    # causal, GQA 4, ragged
    (2, 700, 4, 4, 64, 100, 100, 1, 0, None),    # bidirectional, D = 64
    (1, 1100, 4, 1, 64, 90, 90, 3, 0, None),     # token dilation 3, GQA 4
    (1, 900, 2, 2, 128, 200, 0, 2, 64, None),    # block dilation, causal
    (1, 129, 2, 1, 128, -1, -1, 1, 0, None),     # full bidirectional, tile + 1
    (1, 2048, 8, 2, 128, 600, 0, 1, 0, None),    # many interior tiles
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


def test_backward_full_size_properties(swa):
    """Mistral-shaped prefill (B1 N8192 H32/8 D128, causal W=4096): closed
    forms that hold at any size.  Softmax is shift invariant, so every row's
    dS sums to zero and sum_j dK_j = 0 per (batch, kv head); every row's P
    sums to one, so sum_j dV_j = sum over the group's heads of sum_i dO_i.
    Both are compared against the scale of the summed terms (bf16 rounding
    of each row of dK / dV)."""
    cfg = inputs.CONFIGS["mistral_causal_prefill"]
    q, k, v, _ = inputs.forward_inputs(cfg, device="cuda")
    do = inputs.normal((cfg.B, cfg.N, cfg.H, cfg.D), cfg.seed, 9, torch.bfloat16, "cuda")
    lse = torch.empty(cfg.B, cfg.H, cfg.N, device="cuda")
    out = swa.swa_forward(q, k, v, None, lse, cfg.win_left, cfg.win_right)
    dq, dk, dv = swa.swa_backward(q, k, v, out, do, lse, cfg.win_left, cfg.win_right)
    torch.cuda.synchronize()
    assert swa.swa_device_error() == 0
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    grp = cfg.H // cfg.Hkv
    sum_do = do.float().view(cfg.B, cfg.N, cfg.Hkv, grp, cfg.D).sum(dim=(1, 3))
    sum_dv = dv.float().sum(1)
    tol_v = 2e-2 * dv.float().abs().amax() * cfg.N ** 0.5 + 1e-3 * sum_do.abs().amax()
    assert (sum_dv - sum_do).abs().max().item() <= tol_v.item()
    sum_dk = dk.float().sum(1)
    tol_k = 2e-2 * dk.float().abs().amax() * cfg.N ** 0.5
    assert sum_dk.abs().max().item() <= tol_k.item()
