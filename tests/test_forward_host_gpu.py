"""swa_forward_host: the forward for inputs and outputs in page-locked host
memory, with the copies in, the kernels and the copies out overlapped chunk
by chunk.  Its host results must equal, bit for bit, those of swa_forward on
the same inputs already on the device (the same kernels compute every query
tile), and the oracle's on sampled rows; chunked windows (causal,
right-bounded) and the one-chunk cases (globals, dilation, unbounded right)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import BF16_MAX_ABS, BF16_MEAN_ABS, LSE_ABS, compare, sample_rows
from sliding_window_attention_fwd_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def swa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import sliding_window_attention_fwd_b200 as m
    return m


@pytest.mark.parametrize("B,N,H,Hkv,D,L,R,d,bs,G,with_lse", [
    (1, 3000, 8, 2, 128, 700, 0, 1, 0, None, True),     # causal, 3 chunks, ragged
    (2, 2500, 4, 4, 64, 300, 100, 1, 0, None, True),    # right-bounded band, B = 2
    (1, 4096, 4, 1, 128, 4095, 0, 1, 0, None, False),   # 4 chunks, no lse
    (1, 9000, 4, 1, 64, 1500, 0, 1, 0, None, True),     # 6 chunks: short, 2048s, ragged
    (1, 1500, 2, 2, 64, 40, 40, 1, 0, [0, 700], True),  # globals: one chunk
    (1, 1200, 2, 1, 128, 30, 30, 3, 0, None, True),     # dilation: one chunk
    (1, 1100, 2, 2, 64, 128, 0, 2, 64, None, True),     # block dilation: one chunk
    (1, 1300, 2, 2, 128, 50, -1, 1, 0, None, True),     # unbounded right: one chunk
])
def test_forward_host_matches_device_forward(swa, B, N, H, Hkv, D, L, R, d, bs, G, with_lse):
    seed = N + D
    q = inputs.normal((B, N, H, D), seed, 0)
    k = inputs.normal((B, N, Hkv, D), seed, 1)
    v = inputs.normal((B, N, Hkv, D), seed, 2)
    Gd = torch.tensor(G, dtype=torch.int32, device="cuda") if G else None
    # reference: everything already on the device
    lse_ref = torch.empty(B, H, N, device="cuda")
    out_ref = swa.swa_forward_ex(q.cuda(), k.cuda(), v.cuda(), None, lse_ref, L, R, d, bs, Gd)
    # host inputs and outputs
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    qd, kd, vd = (torch.empty(t.shape, dtype=t.dtype, device="cuda") for t in (q, k, v))
    oh = torch.full(q.shape, float("nan"), dtype=q.dtype).pin_memory()
    lh = torch.full((B, H, N), float("nan")).pin_memory() if with_lse else None
    ld = torch.empty(B, H, N, device="cuda") if with_lse else None
    swa.swa_forward_host(qh, kh, vh, qd, kd, vd, out_host=oh, lse_host=lh, lse_dev=ld,
                         win_left=L, win_right=R, dilation=d, dilation_block=bs, global_idx=Gd)
    torch.cuda.current_stream().synchronize()
    assert swa.swa_device_error() == 0
    assert torch.equal(oh, out_ref.cpu())
    if with_lse:
        assert torch.equal(lh, lse_ref.cpu())
    rows = sample_rows(B, H, N, 200, seed=3, extra_i=[0, 1023, 1024, 2047, 2048, N - 1])
    ro, rl = oracle.forward(q, k, v, L, R, d, bs, G or [], rows=rows)
    got = oh.float().numpy()[rows[:, 0], rows[:, 2], rows[:, 1]]
    compare(got, ro, BF16_MAX_ABS, BF16_MEAN_ABS)
    if with_lse:
        compare(lh.numpy()[rows[:, 0], rows[:, 1], rows[:, 2]], rl, LSE_ABS, what="lse")
