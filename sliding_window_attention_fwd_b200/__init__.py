"""Sliding-window attention for NVIDIA B200 (sm_100a).

Python binding of ``libswa.so``: argument marshalling only.  Every step of
the computation runs in the library's CUDA kernels; there is no CPU or
PyTorch fallback.  If the library is missing the import fails with a clear
message (build it with ``python -m sliding_window_attention_fwd_b200.build``).

The functions carry the C ABI names (see ``include/swa.h``); tensors are
torch CUDA tensors, shapes and sizes are taken from them.
"""
from .binding import (  # noqa: F401
    SwaError,
    library_path,
    swa_append,
    swa_backward,
    swa_decode,
    swa_decode_ex,
    swa_decode_noalloc,
    swa_decode_noalloc_scratch_bytes,
    swa_decode_paged,
    swa_device_error,
    swa_forward,
    swa_forward_ex,
    swa_forward_f32,
    swa_forward_layers,
    swa_paged_window,
    swa_release,
    swa_schedule,
    swa_selftest_timeout,
    swa_status_string,
    swa_version,
)
