"""Sliding-window attention for NVIDIA B200 (sm_100a).

Python binding of ``libswa.so``: argument marshalling only.  Every step of
the computation runs in the library's CUDA kernels; there is no CPU or
PyTorch fallback.

The functions carry the C ABI names (see ``include/swa.h``); tensors are
torch CUDA tensors, shapes and sizes are taken from them.  The library is
loaded on first use of one of them (``sliding_window_attention_fwd_b200.
binding``): importing the package, or its ``build`` and ``inputs``
modules, maps nothing, so the library can be built from a clean tree and
the seeded input generator serves processes that never touch the GPU path.
If the library is missing, that first use fails with ImportError and a
clear message (build it with ``python -m sliding_window_attention_fwd_b200.build``).
"""

_EXPORTS = (
    "SwaError",
    "library_path",
    "swa_append",
    "swa_backward",
    "swa_decode",
    "swa_decode_ex",
    "swa_decode_noalloc",
    "swa_decode_noalloc_scratch_bytes",
    "swa_decode_paged",
    "swa_device_error",
    "swa_forward",
    "swa_forward_ex",
    "swa_forward_f32",
    "swa_forward_host",
    "swa_forward_layers",
    "swa_paged_window",
    "swa_release",
    "swa_schedule",
    "swa_selftest_timeout",
    "swa_set_workspace_allocator",
    "swa_status_string",
    "swa_version",
)

__all__ = list(_EXPORTS)


def __getattr__(name):
    if name in _EXPORTS:
        from . import binding

        return getattr(binding, name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")


def __dir__():
    return sorted(set(globals()) | set(_EXPORTS))
