"""swa_decode_noalloc: decode for callers that must not have the library
allocate device memory (a serving engine whose device memory is one
pre-sized pool, or a hot loop that cannot take a cudaMalloc).

Its split partials live in a fixed array compiled into the library instead
of a cudaMalloc'd workspace.  This file is collected last on purpose.  The
tests call the entry point through the C ABI twice in a row (the array keeps
the first call's leftovers, so the second call also checks that the part
that must start at zero is cleared) and compare each result with the
ordinary swa_decode on the same inputs and with the fp64 oracle, within the
bf16 tolerance the other tests use; the device's free memory must not move
across the calls.  They pass alone in a fresh process and after the other
tests.  (The size limit is checked on the host, with no GPU visible, in
tests/test_noalloc_host.py.)
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import BF16_MAX_ABS, BF16_MEAN_ABS, compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def swa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import sliding_window_attention_fwd_b200 as m
    return m


def test_decode_noalloc_matches_decode_twice(swa):
    from sliding_window_attention_fwd_b200 import inputs

    cfg = inputs.DECODE_CONFIGS["ring_decode"]
    hq, hk, hv, hpos = inputs.decode_inputs(cfg)
    q, kr, vr, pos = hq.cuda(), hk.cuda(), hv.cuda(), hpos.cuda()
    ref = swa.swa_decode(q, kr, vr, pos)
    outs = [torch.full_like(q, float("nan")) for _ in range(3)]
    swa.swa_decode_noalloc(q, kr, vr, pos, outs[2])  # first call on the device: address look-up
    torch.cuda.synchronize()
    # free device memory read right around the two calls only (the error
    # checks below may make torch's caching allocator grow)
    free0 = torch.cuda.mem_get_info()[0]
    for call in range(2):
        swa.swa_decode_noalloc(q, kr, vr, pos, outs[call])
        torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    assert free1 == free0, "device memory changed across the calls"
    assert swa.swa_device_error() == 0
    for call in range(2):
        err = (outs[call].float() - ref.float()).abs().max().item()
        assert np.isfinite(err) and err <= BF16_MAX_ABS, f"call {call}: max abs diff {err}"
    ref_o, _ = oracle.decode(hq, hk, hv, hpos)
    compare(outs[1].float().cpu().numpy(), ref_o, BF16_MAX_ABS, BF16_MEAN_ABS)


@pytest.mark.parametrize("B,H,Hkv,D,W,pos", [
    (5, 8, 2, 64, 1000, [0, 10, 999, 1500, 123456]),   # one chunk: no partials
    (3, 2, 2, 128, 2100, [2099, 5000, 40]),             # GQA group 1, 3 chunks
    (4, 4, 2, 64, 1500, [1499, 3000, 1100, 7]),         # group 2
    (2, 16, 2, 128, 3000, [2999, 100000]),              # group 8
    (3, 12, 4, 128, 1100, [1099, 2000, 1050]),          # group 3 (padded to 4)
])
def test_decode_noalloc_groups(swa, B, H, Hkv, D, W, pos):
    """Every GQA group size the entry point dispatches to, split over several
    key chunks (W > 1024), reusing the array the previous problem left."""
    from sliding_window_attention_fwd_b200 import inputs
    hq = inputs.normal((B, H, D), 21 + H, 0)
    hk = inputs.normal((B, W, Hkv, D), 21 + H, 1)
    hv = inputs.normal((B, W, Hkv, D), 21 + H, 2)
    hpos = torch.tensor(pos, dtype=torch.int64)
    q, k, v, p = hq.cuda(), hk.cuda(), hv.cuda(), hpos.cuda()
    ref = swa.swa_decode(q, k, v, p)
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        swa.swa_decode_noalloc(q, k, v, p, out)
        torch.cuda.synchronize()
        assert swa.swa_device_error() == 0
        assert (out.float() - ref.float()).abs().max().item() <= BF16_MAX_ABS
    ref_o, _ = oracle.decode(hq, hk, hv, hpos)
    compare(out.float().cpu().numpy(), ref_o, BF16_MAX_ABS, BF16_MEAN_ABS)
