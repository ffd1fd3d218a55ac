"""Ring-buffer decode parity: the CUDA path (C ABI) against the fp64 oracle,
on every element, including the full 64-sequence workload; plus partial
caches (pos < W - 1), other GQA ratios and head sizes."""
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


def run_decode(swa, q, kr, vr, pos):
    B, H, D = q.shape
    obuf, out = guarded((B, H, D), torch.bfloat16)
    lbuf, lse = guarded((B, H), torch.float32)
    swa.swa_decode_ex(q.cuda(), kr.cuda(), vr.cuda(), pos.cuda(), out, lse)
    torch.cuda.synchronize()
    assert swa.swa_device_error() == 0
    check_guards(obuf)
    check_guards(lbuf)
    return out.float().cpu().numpy(), lse.cpu().numpy()


def check(swa, q, kr, vr, pos):
    out, lse = run_decode(swa, q, kr, vr, pos)
    ref_o, ref_l = oracle.decode(q, kr, vr, pos)
    compare(out, ref_o, BF16_MAX_ABS, BF16_MEAN_ABS, what="decode out")
    compare(lse, ref_l, LSE_ABS, what="decode lse")


def test_ring_decode_full_workload(swa):
    q, kr, vr, pos = inputs.decode_inputs(inputs.DECODE_CONFIGS["ring_decode"])
    check(swa, q, kr, vr, pos)


def test_ring_decode_partial_cache(swa):
    q, kr, vr, pos = inputs.decode_inputs(inputs.DECODE_CONFIGS["small_ring_partial"])
    pos[0] = 0          # only slot 0 valid
    pos[1] = 63         # exactly one stage
    pos[2] = 511        # W - 1: first full ring
    check(swa, q, kr, vr, pos)


@pytest.mark.parametrize("B,H,Hkv,D,W", [(3, 8, 8, 128, 300), (2, 16, 2, 64, 1000),
                                         (4, 6, 2, 128, 777), (1, 2, 1, 64, 64),
                                         (3, 16, 2, 128, 2500), (2, 4, 4, 128, 4096)])
def test_ring_decode_shapes(swa, B, H, Hkv, D, W):
    q = inputs.normal((B, H, D), 9, 0)
    kr = inputs.normal((B, W, Hkv, D), 9, 1)
    vr = inputs.normal((B, W, Hkv, D), 9, 2)
    pos = inputs.uniform_int(B, 0, 3 * W, 9, 3)
    check(swa, q, kr, vr, pos)


def test_ring_decode_wrapped_equals_forward(swa):
    """A wrapped ring gives the same row as the causal forward kernel over the
    de-rotated window (both on the GPU, through the C ABI)."""
    W, H, Hkv, D, p = 256, 4, 1, 128, 1000
    seq = inputs.normal((1, p + 1, Hkv, D), 13, 1)
    vseq = inputs.normal((1, p + 1, Hkv, D), 13, 2)
    qs = inputs.normal((1, p + 1, H, D), 13, 0)
    kr = torch.zeros(1, W, Hkv, D, dtype=torch.bfloat16)
    vr = torch.zeros_like(kr)
    for t in range(p + 1):           # stream the tokens through the ring
        kr[0, t % W] = seq[0, t]
        vr[0, t % W] = vseq[0, t]
    out_d, lse_d = run_decode(swa, qs[:, p].contiguous(), kr, vr, torch.tensor([p]))
    out_f = swa.swa_forward(qs.cuda(), seq.cuda(), vseq.cuda(), win_left=W - 1, win_right=0)
    torch.cuda.synchronize()
    np.testing.assert_allclose(out_d[0], out_f[0, p].float().cpu().numpy(), atol=2e-2)


def test_workspace_reuse_across_sizes(swa):
    """Calls with fewer and then more query sets reuse one workspace: the
    split counters of the big call must still start at zero afterwards."""
    big = inputs.decode_inputs(inputs.DECODE_CONFIGS["ring_decode"])
    small = inputs.decode_inputs(inputs.DECODE_CONFIGS["small_ring_partial"])
    check(swa, *big)
    check(swa, *small)
    q = inputs.normal((2, 8, 128), 17, 0)
    kr = inputs.normal((2, 2048, 4, 128), 17, 1)
    vr = inputs.normal((2, 2048, 4, 128), 17, 2)
    check(swa, q, kr, vr, torch.tensor([5000, 100], dtype=torch.int64))
    check(swa, *big)


def test_ring_decode_parts_of_a_short_cache(swa):
    """A long ring holding few tokens: parts of the ring past the filled slots
    are empty and must not contribute (D = 128, GQA 4, positions below one
    part, at a part boundary and past the first part)."""
    B, H, Hkv, D, W = 4, 8, 2, 128, 4096
    q = inputs.normal((B, H, D), 21, 0)
    kr = inputs.normal((B, W, Hkv, D), 21, 1)
    vr = inputs.normal((B, W, Hkv, D), 21, 2)
    check(swa, q, kr, vr, torch.tensor([10, 1023, 1024, 2900], dtype=torch.int64))
