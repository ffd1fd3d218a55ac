"""Helpers shared by the GPU parity tests (tolerances, guard bands, sampling)."""
import numpy as np
import torch

# Tolerances against the fp64 oracle on identical inputs.
F32_MAX_ABS = 1e-4
BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
LSE_ABS = 1e-3

GUARD = 64  # elements of sentinel before and after each output


def guarded(shape, dtype, device="cuda"):
    """Output tensor inside a larger buffer whose margins hold a NaN sentinel."""
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * GUARD,), float("nan"), dtype=dtype, device=device)
    return buf, buf[GUARD:GUARD + n].view(*shape)


def check_guards(buf):
    head = buf[:GUARD].float()
    tail = buf[-GUARD:].float()
    assert torch.isnan(head).all() and torch.isnan(tail).all(), "write outside the output"


def compare(out, ref, max_abs, mean_abs=None, what="out"):
    out = np.asarray(out, dtype=np.float64)
    err = np.abs(out - ref)
    assert np.isfinite(out).all(), f"{what}: non-finite values"
    assert err.max() <= max_abs, f"{what}: max abs err {err.max():.3e} > {max_abs}"
    if mean_abs is not None:
        assert err.mean() <= mean_abs, f"{what}: mean abs err {err.mean():.3e} > {mean_abs}"
    return float(err.max()), float(err.mean())


def sample_rows(B, H, N, n, seed, extra_i=()):
    """n random (b, h, i) triples plus every (b=0, h=0, i) in extra_i."""
    rng = np.random.default_rng(seed)
    rows = np.stack([rng.integers(0, B, n), rng.integers(0, H, n), rng.integers(0, N, n)], 1)
    extra = [[0, 0, i] for i in extra_i if 0 <= i < N] + [[B - 1, H - 1, i] for i in extra_i
                                                           if 0 <= i < N]
    if extra:
        rows = np.concatenate([rows, np.array(extra)], 0)
    return rows.astype(np.int64)


def build_test_library(out_dir, defines):
    """Compiles libswa's sources with extra preprocessor definitions (a
    test-only build, e.g. a failure-injection switch) into out_dir and
    returns the path of the shared library.  Each source compiles in its own
    nvcc process, in parallel."""
    import glob
    import os
    import subprocess

    from sliding_window_attention_fwd_b200 import build as b

    flags = [f for f in b.NVCC_FLAGS if f != "-shared"]
    objs, procs = [], []
    for src in b.sources():
        obj = os.path.join(out_dir, os.path.basename(src) + ".o")
        objs.append(obj)
        procs.append(subprocess.Popen(
            ["nvcc", *flags, *(f"-D{d}" for d in defines), "-I", b.INCLUDE, "-I", b.CSRC, "-c",
             src, "-o", obj], stdout=subprocess.PIPE, stderr=subprocess.STDOUT))
    for pr in procs:
        out, _ = pr.communicate()
        assert pr.returncode == 0, out.decode()[-2000:]
    lib = os.path.join(out_dir, "libswa_test.so")
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", lib,
                    *objs], check=True, capture_output=True)
    assert glob.glob(lib)
    return lib
