"""Parity of paged decode and chunked ring append: the CUDA path (C ABI)
against the fp64 oracle on every element, plus the ring contents after an
append (bit-exact copies).  Covers partial windows (pos < W - 1), chunks that
wrap the ring or are longer than it, every GQA ratio the kernels take, both
head sizes, and the full-size workloads."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import BF16_MAX_ABS, BF16_MEAN_ABS, LSE_ABS, check_guards, compare, guarded
from sliding_window_attention_fwd_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def swa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import sliding_window_attention_fwd_b200 as m
    return m


# ---------------------------------------------------------------- paged decode
def run_paged(swa, q, kp, vp, table, pos, ps, W):
    B, H, D = q.shape
    obuf, out = guarded((B, H, D), torch.bfloat16)
    lbuf, lse = guarded((B, H), torch.float32)
    swa.swa_decode_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), pos.cuda(), ps, W, out=out,
                         lse=lse)
    torch.cuda.synchronize()
    assert swa.swa_device_error() == 0
    check_guards(obuf)
    check_guards(lbuf)
    return out.float().cpu().numpy(), lse.cpu().numpy()


def check_paged(swa, q, kp, vp, table, pos, ps, W):
    out, lse = run_paged(swa, q, kp, vp, table, pos, ps, W)
    ro, rl = oracle.decode_paged(q, kp, vp, table, pos, ps, W)
    compare(out, ro, BF16_MAX_ABS, BF16_MEAN_ABS, what="paged out")
    compare(lse, rl, LSE_ABS, what="paged lse")


@pytest.mark.parametrize("name", ["small_paged", "paged_decode"])
def test_paged_configs(swa, name):
    cfg = inputs.PAGED_CONFIGS[name]
    q, kp, vp, table, pos = inputs.paged_inputs(cfg)
    check_paged(swa, q, kp, vp, table, pos, cfg.page_size, cfg.W)


@pytest.mark.parametrize("B,H,Hkv,D,W,ps,lo,hi", [
    (3, 8, 8, 128, 100, 64, 0, 400),     # MHA, window shorter than a page
    (2, 16, 2, 64, 1000, 128, 0, 3000),  # GQA 8
    (4, 6, 3, 128, 777, 64, 700, 900),   # GQA 2, windows straddling pages
    (2, 4, 4, 64, 64, 64, 60, 70),       # window of exactly one box
    (2, 8, 2, 128, 4096, 256, 0, 200),   # partial window (pos < W - 1)
])
def test_paged_shapes(swa, B, H, Hkv, D, W, ps, lo, hi):
    cfg = inputs.PagedConfig("t", B=B, H=H, Hkv=Hkv, D=D, W=W, page_size=ps, pos_lo=lo,
                             pos_hi=hi, seed=B * 100 + W)
    q, kp, vp, table, pos = inputs.paged_inputs(cfg)
    check_paged(swa, q, kp, vp, table, pos, ps, W)


def test_paged_equals_ring_decode_on_the_same_tokens(swa):
    """The same cache contents stored as a ring and as pages give the same
    output (up to the order of the fp32 sums)."""
    B, H, Hkv, D, W, ps = 3, 8, 2, 128, 512, 64
    q = inputs.normal((B, H, D), 31, 0)
    kr = inputs.normal((B, W, Hkv, D), 31, 1)
    vr = inputs.normal((B, W, Hkv, D), 31, 2)
    pos = torch.tensor([1000, 511, 2047], dtype=torch.int64)
    # page the ring's contents by position: position t is ring slot t % W
    npg = W // ps + 1
    table = torch.full((B, int(pos.max()) // ps + 1), -1, dtype=torch.int32)
    kp = torch.zeros((B * npg * ps, Hkv, D), dtype=torch.bfloat16)
    vp = torch.zeros_like(kp)
    nxt = 0
    for b in range(B):
        p = int(pos[b])
        for lp in range(max(0, p - W + 1) // ps, p // ps + 1):
            table[b, lp] = nxt
            for r in range(ps):
                t = lp * ps + r
                if max(0, p - W + 1) <= t <= p:
                    kp[nxt * ps + r] = kr[b, t % W]
                    vp[nxt * ps + r] = vr[b, t % W]
            nxt += 1
    out_p, lse_p = run_paged(swa, q, kp, vp, table, pos, ps, W)
    out_r = swa.swa_decode(q.cuda(), kr.cuda(), vr.cuda(), pos.cuda()).float().cpu().numpy()
    assert np.abs(out_p - out_r).max() <= 2 * 2 ** -8 * max(1.0, np.abs(out_r).max())


# ------------------------------------------------------------- chunked append
def run_append(swa, q, kn, vn, kr, vr, pos0):
    B, C, H, D = q.shape
    obuf, out = guarded((B, C, H, D), torch.bfloat16)
    lbuf, lse = guarded((B, H, C), torch.float32)
    krd, vrd = kr.cuda().clone(), vr.cuda().clone()
    swa.swa_append(q.cuda(), kn.cuda(), vn.cuda(), krd, vrd, pos0.cuda(), out=out, lse=lse)
    torch.cuda.synchronize()
    assert swa.swa_device_error() == 0
    check_guards(obuf)
    check_guards(lbuf)
    return out.float().cpu().numpy(), lse.cpu().numpy(), krd.cpu(), vrd.cpu()


def check_append(swa, q, kn, vn, kr, vr, pos0):
    out, lse, kr2, vr2 = run_append(swa, q, kn, vn, kr, vr, pos0)
    ro, rl = oracle.append(q, kr, vr, kn, vn, pos0)
    compare(out, ro, BF16_MAX_ABS, BF16_MEAN_ABS, what="append out")
    compare(lse, rl, LSE_ABS, what="append lse")
    # the ring afterwards: slot (pos0 + c) % W holds token c (the last W stay)
    B, C = q.shape[:2]
    W = kr.shape[1]
    ek, ev = kr.clone(), vr.clone()
    for b in range(B):
        for c in range(max(0, C - W), C):
            ek[b, (int(pos0[b]) + c) % W] = kn[b, c]
            ev[b, (int(pos0[b]) + c) % W] = vn[b, c]
    assert torch.equal(kr2, ek) and torch.equal(vr2, ev)


@pytest.mark.parametrize("name", ["small_append", "ring_append"])
def test_append_configs(swa, name):
    cfg = inputs.APPEND_CONFIGS[name]
    check_append(swa, *inputs.append_inputs(cfg))


@pytest.mark.parametrize("B,C,H,Hkv,D,W,pos0", [
    (5, 1, 8, 2, 128, 64, [0, 5, 63, 64, 1000]),   # C = 1: a decode step
    (2, 200, 4, 2, 128, 128, [0, 300]),            # chunk longer than the ring
    (2, 17, 4, 4, 64, 192, [190, 400]),            # MHA, chunk wraps the ring
    (2, 9, 16, 2, 128, 64, [60, 2]),               # GQA 8
    (3, 64, 8, 4, 64, 256, [255, 256, 1]),         # GQA 2, D = 64
    (2, 40, 4, 4, 64, 128, [100, 3]),              # MHA, D = 64, tensor-core path
    (1, 33, 2, 2, 128, 64, [70]),                  # MHA, D = 128, tensor-core path
    (2, 130, 6, 2, 128, 192, [5, 1000]),           # GQA 3, two query tiles
    # ring read in place (W % 64 == 0): the window's oldest slot at every
    # offset class within a 64-row box (0, 1, 2, 63), windows that start
    # inside the chunk (C > W), positions below W
    (3, 100, 4, 2, 128, 64, [62, 63, 65]),
    (2, 150, 4, 4, 64, 128, [129, 64]),
    # four heads per CTA (two stacked per tile, GQA 4 and 8) with split key
    # walks, one at D = 64, one with positions below W
    (2, 64, 16, 4, 128, 1024, [5000, 700]),
    (1, 48, 16, 2, 128, 2048, [3000]),
    (2, 50, 8, 2, 128, 1024, [1500, 20]),
    (2, 64, 8, 2, 64, 512, [600, 511]),
    # two-part key walks merged in pairs (clusters of two CTAs): the chunk
    # stored from inside the launch (GQA 2 at D = 128, GQA 4 stacked at
    # D = 64, MHA at D = 64 with two CTAs per SM) or by the store kernel
    # (GQA 8: a kv head's heads span two items); small positions leave the
    # second part empty
    (16, 100, 8, 4, 128, 512, [5, 3000, 700, 511, 512, 513, 9000, 64] * 2),
    (16, 64, 16, 4, 64, 256, [300, 2, 255, 256, 1000, 77, 63, 4000] * 2),
    (8, 40, 16, 16, 64, 256, [1, 260, 5000, 255, 128, 129, 64, 700]),
    (8, 64, 32, 4, 128, 512, [600, 3, 511, 512, 2000, 100, 64, 65]),
])
def test_append_shapes(swa, B, C, H, Hkv, D, W, pos0):
    q = inputs.normal((B, C, H, D), C + W, 0)
    kn = inputs.normal((B, C, Hkv, D), C + W, 1)
    vn = inputs.normal((B, C, Hkv, D), C + W, 2)
    kr = inputs.normal((B, W, Hkv, D), C + W, 3)
    vr = inputs.normal((B, W, Hkv, D), C + W, 4)
    check_append(swa, q, kn, vn, kr, vr, torch.tensor(pos0, dtype=torch.int64))


def test_append_then_decode_sees_the_chunk(swa):
    """After an append, a ring decode at the chunk's last position equals the
    append's own output for that token."""
    B, C, H, Hkv, D, W = 2, 12, 8, 2, 128, 128
    q = inputs.normal((B, C, H, D), 41, 0)
    kn = inputs.normal((B, C, Hkv, D), 41, 1)
    vn = inputs.normal((B, C, Hkv, D), 41, 2)
    kr = inputs.normal((B, W, Hkv, D), 41, 3)
    vr = inputs.normal((B, W, Hkv, D), 41, 4)
    pos0 = torch.tensor([500, 7], dtype=torch.int64)
    out, _, kr2, vr2 = run_append(swa, q, kn, vn, kr, vr, pos0)
    last = (pos0 + C - 1)
    od = swa.swa_decode(q[:, C - 1].contiguous().cuda(), kr2.cuda(), vr2.cuda(), last.cuda())
    np.testing.assert_allclose(od.float().cpu().numpy(), out[:, C - 1], rtol=0, atol=2e-2)
