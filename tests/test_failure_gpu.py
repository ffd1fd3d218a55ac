"""Failure detection without faulting the GPU: a device wait that nothing
will satisfy gives up after its bound, records an error word, and the host
reads it as SWA_ERR_TIMEOUT; the context stays usable afterwards."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import sliding_window_attention_fwd_b200 as swa

    assert swa.swa_device_error() == 0
    swa.swa_selftest_timeout(2000)  # 2 ms bound on a wait nobody satisfies
    assert swa.swa_device_error() == -5
    assert swa.swa_device_error() == 0  # cleared
    # the context still works
    q = torch.randn(1, 64, 2, 64, device="cuda").to(torch.bfloat16)
    out = swa.swa_forward(q, q[:, :, :1].contiguous(), q[:, :, :1].contiguous(), win_left=8,
                          win_right=8)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
