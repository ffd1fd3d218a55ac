"""Per-layer window schedules (swa_forward_layers): every layer of a hybrid
schedule -- plain causal windows, growing dilation, a full causal "global"
layer and attention-sink tokens -- matches the fp64 oracle for that layer,
and the schedule gives bit-identical results to one swa_forward_ex call per
layer."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import BF16_MAX_ABS, BF16_MEAN_ABS, LSE_ABS, compare
from sliding_window_attention_fwd_b200 import inputs

pytestmark = pytest.mark.gpu

SCHEDULE = [  # (win_left, win_right, dilation, dilation_block, global_idx)
    (255, 0, 1, 0, []),          # lower layers: plain causal window
    (127, 0, 2, 0, []),          # middle layers: dilation grows
    (63, 0, 4, 0, []),
    (-1, 0, 1, 0, []),           # every few layers: a global (full causal) layer
    (255, 0, 1, 0, [0, 1, 2, 3]),  # attention sinks: the first tokens stay visible
    (128, 128, 2, 64, []),       # block-level dilation, bidirectional
]


@pytest.fixture(scope="module")
def swa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import sliding_window_attention_fwd_b200 as m
    return m


@pytest.mark.parametrize("B,N,H,Hkv,D", [(1, 1000, 4, 2, 128), (2, 700, 4, 4, 64)])
def test_schedule_matches_oracle_and_single_calls(swa, B, N, H, Hkv, D):
    layers, cpu = [], []
    for li, (L, R, d, bs, G) in enumerate(SCHEDULE):
        q = inputs.normal((B, N, H, D), 60 + li, 0)
        k = inputs.normal((B, N, Hkv, D), 60 + li, 1)
        v = inputs.normal((B, N, Hkv, D), 60 + li, 2)
        lse = torch.empty(B, H, N, device="cuda")
        g = torch.tensor(G, dtype=torch.int32, device="cuda") if G else None
        layers.append(dict(q=q.cuda(), k=k.cuda(), v=v.cuda(), lse=lse, win_left=L, win_right=R,
                           dilation=d, dilation_block=bs, global_idx=g))
        cpu.append((q, k, v))
    outs = swa.swa_forward_layers(layers)
    torch.cuda.synchronize()
    assert swa.swa_device_error() == 0
    for li, ((L, R, d, bs, G), (q, k, v), lay, out) in enumerate(zip(SCHEDULE, cpu, layers, outs)):
        ro, rl = oracle.forward(q, k, v, L, R, d, bs, G, 0.0)
        compare(out.float().cpu().numpy(), ro, BF16_MAX_ABS, BF16_MEAN_ABS, what=f"layer {li} out")
        compare(lay["lse"].cpu().numpy(), rl, LSE_ABS, what=f"layer {li} lse")
        single = swa.swa_forward_ex(lay["q"], lay["k"], lay["v"], None, None, L, R, d, bs,
                                    lay["global_idx"])
        torch.cuda.synchronize()
        assert torch.equal(single, out), f"layer {li}: schedule and single call differ"
