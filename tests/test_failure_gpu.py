"""Failure detection without faulting the GPU.

* A device wait that nothing will satisfy gives up after its bound, records
  an error word, and the host reads it as SWA_ERR_TIMEOUT; the context stays
  usable afterwards.
* The same inside the production kernels: a test-only build of the library
  (SWA_TEST_WITHHOLD_TILE) never loads one K/V tile, and lowers the bound on
  every wait to 5 ms.  The fused forward, the tensor-core decode, the
  split-KV row kernel and the append's two-part clusters (whose CTAs also
  wait on each other) must then time out, leave their abort path
  (in-flight copies drained, TMEM released, both CTAs of a cluster meeting
  before they exit) and return; a problem that needs no withheld tile still
  gives the oracle's result, so the context and the SM resources (TMEM) are
  intact.
* A workspace allocation that fails (injected through the caller-allocator
  hook, on the host) is reported as SWA_ERR_NOMEM before any launch, and a
  counting allocator shows which calls allocate at all.
No test faults, traps or hangs a GPU: every wait is bounded and returns.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gpu_util import BF16_MAX_ABS, BF16_MEAN_ABS, LSE_ABS, build_test_library, compare
from sliding_window_attention_fwd_b200 import inputs

pytestmark = pytest.mark.gpu

TIMEOUT, NOMEM = -5, -6


@pytest.fixture(scope="module")
def swa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import sliding_window_attention_fwd_b200 as m
    return m


def test_bounded_wait_reports_timeout(swa):
    assert swa.swa_device_error() == 0
    swa.swa_selftest_timeout(2000)  # 2 ms bound on a wait nobody satisfies
    assert swa.swa_device_error() == TIMEOUT
    assert swa.swa_device_error() == 0  # cleared
    # the context still works
    q = torch.randn(1, 64, 2, 64, device="cuda").to(torch.bfloat16)
    out = swa.swa_forward(q, q[:, :, :1].contiguous(), q[:, :, :1].contiguous(), win_left=8,
                          win_right=8)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()


@pytest.fixture(scope="module")
def withheld_lib(tmp_path_factory, swa):
    d = tmp_path_factory.mktemp("withheld")
    path = build_test_library(str(d), ["SWA_TEST_WITHHOLD_TILE=1",
                                       "SWA_WAIT_LIMIT_NS=5000000ull"])
    lib = ctypes.CDLL(path)
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.swa_forward.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, I, P, I, F, P]
    lib.swa_decode.argtypes = [P, P, P, P, P, I, I, I, I, I, P]
    lib.swa_append.argtypes = [P] * 8 + [I] * 6 + [F, P]
    lib.swa_device_error.argtypes = [P]
    return lib


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_forward_abort_path(withheld_lib):
    lib = withheld_lib
    # N = 512, causal 300: query tiles 1-3 walk two or more key tiles, so
    # they wait for the withheld second tile and give up
    B, N, H, Hkv, D, L = 1, 512, 2, 1, 128, 300
    q = inputs.normal((B, N, H, D), 41, 0).cuda()
    k = inputs.normal((B, N, Hkv, D), 41, 1).cuda()
    v = inputs.normal((B, N, Hkv, D), 41, 2).cuda()
    out = torch.empty_like(q)
    lse = torch.empty(B, H, N, device="cuda")
    rc = lib.swa_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                         lse.data_ptr(), B, H, Hkv, N, D, L, 0, 1, None, 0, 0.0, _stream())
    assert rc == 0
    assert lib.swa_device_error(_stream()) == TIMEOUT
    assert lib.swa_device_error(_stream()) == 0
    # one key tile per query tile: nothing is withheld, the result is exact
    N2 = 128
    q2, k2, v2 = (t[:, :N2].contiguous() for t in (q, k, v))
    out2 = torch.empty_like(q2)
    lse2 = torch.empty(B, H, N2, device="cuda")
    rc = lib.swa_forward(q2.data_ptr(), k2.data_ptr(), v2.data_ptr(), out2.data_ptr(),
                         lse2.data_ptr(), B, H, Hkv, N2, D, 60, 0, 1, None, 0, 0.0, _stream())
    assert rc == 0
    assert lib.swa_device_error(_stream()) == 0
    ref_o, ref_l = oracle.forward(q2.cpu(), k2.cpu(), v2.cpu(), 60, 0)
    compare(out2.float().cpu().numpy(), ref_o, BF16_MAX_ABS, BF16_MEAN_ABS)
    compare(lse2.cpu().numpy(), ref_l, LSE_ABS, what="lse")


@pytest.mark.parametrize("D", [128, 64])
def test_decode_abort_path(withheld_lib, D):
    """D = 128: the tensor-core decode (K tile 1 of every part withheld);
    D = 64: the split-KV row kernel (its 64-row stage 1 withheld)."""
    lib = withheld_lib
    B, H, Hkv, W = 2, 8, 2, 4096  # 1024 keys per CTA: 8 tiles / 16 stages
    q = inputs.normal((B, H, D), 43, 0).cuda()
    kr = inputs.normal((B, W, Hkv, D), 43, 1).cuda()
    vr = inputs.normal((B, W, Hkv, D), 43, 2).cuda()
    pos = torch.tensor([5000, 9000], dtype=torch.int64, device="cuda")
    out = torch.empty_like(q)
    rc = lib.swa_decode(q.data_ptr(), kr.data_ptr(), vr.data_ptr(), out.data_ptr(),
                        pos.data_ptr(), B, H, Hkv, D, W, _stream())
    assert rc == 0
    assert lib.swa_device_error(_stream()) == TIMEOUT
    # a 64-slot ring is one stage per CTA: nothing withheld
    W2 = 64
    kr2, vr2 = kr[:, :W2].contiguous(), vr[:, :W2].contiguous()
    out2 = torch.empty_like(q)
    rc = lib.swa_decode(q.data_ptr(), kr2.data_ptr(), vr2.data_ptr(), out2.data_ptr(),
                        pos.data_ptr(), B, H, Hkv, D, W2, _stream())
    assert rc == 0
    assert lib.swa_device_error(_stream()) == 0
    ref, _ = oracle.decode(q.cpu(), kr2.cpu(), vr2.cpu(), pos.cpu())
    compare(out2.float().cpu().numpy(), ref, BF16_MAX_ABS, BF16_MEAN_ABS)


def test_append_pair_abort_path(withheld_lib, swa):
    """A chunked append whose key walks are split in two parts merged on chip
    (64 work items: clusters of two CTAs): every part waits for its withheld
    second K tile, gives up, and both CTAs of each cluster still meet and
    exit.  Then the regular library's append on the same shapes equals the
    oracle."""
    lib = withheld_lib
    B, C, H, Hkv, D, W = 8, 64, 32, 8, 128, 1024  # four heads per CTA, 2 parts of ~5 tiles
    q = inputs.normal((B, C, H, D), 47, 0).cuda()
    kn = inputs.normal((B, C, Hkv, D), 47, 1).cuda()
    vn = inputs.normal((B, C, Hkv, D), 47, 2).cuda()
    kr = inputs.normal((B, W, Hkv, D), 47, 3)
    vr = inputs.normal((B, W, Hkv, D), 47, 4)
    pos0 = torch.tensor([5000, 1024, 2000, 3000, 4000, 6000, 7000, 1100], dtype=torch.int64)
    krd, vrd, posd = kr.cuda(), vr.cuda(), pos0.cuda()
    out = torch.empty_like(q)
    lse = torch.empty(B, H, C, device="cuda")
    rc = lib.swa_append(q.data_ptr(), kn.data_ptr(), vn.data_ptr(), krd.data_ptr(),
                        vrd.data_ptr(), out.data_ptr(), lse.data_ptr(), posd.data_ptr(), B, C, H,
                        Hkv, D, W, 0.0, _stream())
    assert rc == 0
    assert lib.swa_device_error(_stream()) == TIMEOUT
    assert lib.swa_device_error(_stream()) == 0
    # the context and the SMs are intact: the regular library's append
    krd, vrd = kr.cuda(), vr.cuda()
    lse2 = torch.empty(B, H, C, device="cuda")
    out2 = swa.swa_append(q, kn, vn, krd, vrd, posd, lse=lse2)
    torch.cuda.synchronize()
    assert swa.swa_device_error() == 0
    ro, rl = oracle.append(q.cpu(), kr, vr, kn.cpu(), vn.cpu(), pos0)
    compare(out2.float().cpu().numpy(), ro, BF16_MAX_ABS, BF16_MEAN_ABS)
    compare(lse2.cpu().numpy(), rl, LSE_ABS, what="lse")


def test_allocation_failure_reports_nomem(swa):
    cfg = inputs.DECODE_CONFIGS["ring_decode"]
    q, kr, vr, pos = (t.cuda() for t in inputs.decode_inputs(cfg))
    calls = []
    swa.swa_set_workspace_allocator(lambda n: calls.append(n) or 0, lambda p: None)
    try:
        out = torch.full_like(q, float("nan"))
        with pytest.raises(swa.SwaError) as ei:
            swa.swa_decode(q, kr, vr, pos, out)
        assert ei.value.status == NOMEM
        torch.cuda.synchronize()
        assert calls, "the workspace allocator was not asked"
        assert torch.isnan(out.float()).all(), "a kernel ran although allocation failed"
        assert swa.swa_device_error() == 0
    finally:
        swa.swa_set_workspace_allocator()


def test_counting_allocator(swa):
    """Workspaces come from the caller's allocator; the forward (with global
    tokens too) asks it for nothing; restoring the default gives every block
    back."""
    live, log = {}, []

    def alloc(n):
        p = torch.cuda.caching_allocator_alloc(n)
        live[p] = n
        log.append(n)
        return p

    def free(p):
        torch.cuda.caching_allocator_delete(p)
        del live[p]

    cfg = inputs.DECODE_CONFIGS["ring_decode"]
    hq, hk, hv, hpos = inputs.decode_inputs(cfg)
    q, kr, vr, pos = hq.cuda(), hk.cuda(), hv.cuda(), hpos.cuda()
    swa.swa_set_workspace_allocator(alloc, free)
    try:
        out = swa.swa_decode(q, kr, vr, pos)
        torch.cuda.synchronize()
        assert log, "decode took its split workspace from the allocator"
        ref, _ = oracle.decode(hq, hk, hv, hpos)
        compare(out.float().cpu().numpy(), ref, BF16_MAX_ABS, BF16_MEAN_ABS)
        n0 = len(log)
        fc = inputs.CONFIGS["small_global"]
        fq, fk, fv, G = inputs.forward_inputs(fc, device="cuda")
        swa.swa_forward(fq, fk, fv, None, None, fc.win_left, fc.win_right, fc.dilation, G.cuda())
        torch.cuda.synchronize()
        assert len(log) == n0, "the forward allocated"
    finally:
        swa.swa_set_workspace_allocator()
    assert not live, "blocks left with the caller's allocator"
    assert swa.swa_device_error() == 0
