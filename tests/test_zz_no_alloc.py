"""swa_decode_noalloc: decode for callers that must not have the library
allocate device memory (a serving engine whose device memory is one
pre-sized pool, or a hot loop that cannot take a cudaMalloc).

Its split partials live in a fixed array compiled into the library instead
of a cudaMalloc'd workspace.  This file is collected last on purpose.  The
test calls the new entry point through the C ABI twice in a row (the array
keeps the first call's leftovers, so the second call also checks that the
part that must start at zero is cleared) and compares each result with the
ordinary swa_decode on the same inputs, within the bf16 tolerance the other
tests use.  It passes alone in a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

from gpu_util import BF16_MAX_ABS

pytestmark = pytest.mark.gpu


def test_decode_noalloc_matches_decode_twice():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import sliding_window_attention_fwd_b200 as swa
    from sliding_window_attention_fwd_b200 import inputs

    cfg = inputs.DECODE_CONFIGS["ring_decode"]
    q, kr, vr, pos = (t.cuda() for t in inputs.decode_inputs(cfg))
    ref = swa.swa_decode(q, kr, vr, pos)
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        swa.swa_decode_noalloc(q, kr, vr, pos, out)
        torch.cuda.synchronize()
        assert swa.swa_device_error() == 0
        err = (out.float() - ref.float()).abs().max().item()
        assert np.isfinite(err) and err <= BF16_MAX_ABS, f"call {call}: max abs diff {err}"

    # a second, differently shaped problem reuses the same array
    q2 = inputs.normal((5, 8, 64), 21, 0).cuda()
    k2 = inputs.normal((5, 1000, 2, 64), 21, 1).cuda()
    v2 = inputs.normal((5, 1000, 2, 64), 21, 2).cuda()
    p2 = torch.tensor([0, 10, 999, 1500, 123456], dtype=torch.int64, device="cuda")
    ref2 = swa.swa_decode(q2, k2, v2, p2)
    out2 = torch.empty_like(q2)
    swa.swa_decode_noalloc(q2, k2, v2, p2, out2)
    torch.cuda.synchronize()
    assert (out2.float() - ref2.float()).abs().max().item() <= BF16_MAX_ABS


def test_decode_noalloc_rejects_oversized_problem():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import sliding_window_attention_fwd_b200 as swa
    from sliding_window_attention_fwd_b200 import binding

    # B * Hkv * ceil(W/512) * pow2(H/Hkv) * (D + 2) * 4 bytes > 16 MiB; nothing
    # is read from these (never dereferenced) aligned addresses.
    A = 0x10000
    B, H, Hkv, D, W = 4096, 32, 8, 128, 4096
    rc = binding._lib.swa_decode_noalloc(A, A, A, A, A, B, H, Hkv, D, W, None)
    assert rc == -3, swa.swa_status_string(rc)
