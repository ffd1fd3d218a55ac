"""The size limit of swa_decode_noalloc, checked on the host.

The entry point keeps its split partials in a fixed device array and must
refuse, before any CUDA call, a problem whose partials would not fit.  The
check runs in a child process that sees no GPU: a problem the library
accepts then fails at its first CUDA call (SWA_ERR_CUDA), one it refuses
returns SWA_ERR_UNSUPPORTED, and no kernel can ever be launched on the
placeholder addresses passed here, whatever the library does."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
sys.path.insert(0, ROOT)
from sliding_window_attention_fwd_b200 import binding
L = binding._lib
A = 0x10000  # placeholder, 16-byte aligned: never dereferenced on the host
cap = binding.swa_decode_noalloc_scratch_bytes()

def need(S, nsplit, nq, D):
    # the bound stated in include/swa.h
    return ((S * 4 + 255) // 256) * 256 + S * nsplit * nq * (D + 2) * 4

def call(B, H, Hkv, D, W):
    return L.swa_decode_noalloc(A, A, A, A, A, B, H, Hkv, D, W, None)

res = [cap]
for H, Hkv, D, W in [(8, 1, 128, 2048), (32, 8, 128, 4096), (2, 2, 64, 1025)]:
    nq = 1
    while nq < H // Hkv:
        nq *= 2
    nsplit = -(-W // 1024)
    B = 1
    while need((B + 1) * Hkv, nsplit, nq, D) <= cap:
        B += 1
    res += [call(B, H, Hkv, D, W), call(B + 1, H, Hkv, D, W)]
res.append(call(10**6, 32, 8, 128, 1024))   # one chunk per set: no partials at all
print(" ".join(str(x) for x in res))
"""


def test_noalloc_size_limit_is_the_documented_bound():
    env = {**os.environ, "CUDA_VISIBLE_DEVICES": ""}
    out = subprocess.run([sys.executable, "-c", CHILD.replace("ROOT", repr(ROOT))],
                         capture_output=True, text=True, timeout=300, env=env, check=True)
    vals = [int(x) for x in out.stdout.split()]
    assert vals[0] == 16 << 20
    for fits, over in zip(vals[1:7:2], vals[2:7:2]):
        assert fits == -4, "a problem within the bound must pass the size check"
        assert over == -3, "a problem one batch over the bound must be refused"
    assert vals[7] == -4
