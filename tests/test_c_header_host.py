"""The boundary is a C ABI: include/swa.h must compile as strict C99 and a
plain C program must link against libswa.so and call it with bare pointers
and sizes.  Only host-side entry points are called here (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

from sliding_window_attention_fwd_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")

PROGRAM = r"""
#include <stdio.h>
#include "swa.h"

int main(void) {
  static int32_t tiles[6 * 4096];
  int n = swa_schedule(%(N)d, %(L)d, %(R)d, %(d)d, %(bs)d, tiles, 4096);
  int64_t first = -1, last = -1;
  int st = swa_paged_window(%(pos)d, %(W)d, %(ps)d, &first, &last);
  int bad = swa_paged_window(-1, %(W)d, %(ps)d, &first, &last);
  printf("%%d %%d %%d %%lld %%lld %%d\n", swa_version(), n, st, (long long)first,
         (long long)last, bad);
  if (n > 0)
    printf("%%d %%d %%d %%d %%d %%d\n", tiles[0], tiles[1], tiles[2], tiles[3], tiles[4],
           tiles[5]);
  printf("%%s\n", swa_status_string(SWA_ERR_UNSUPPORTED));
  /* the parameter-block forward, validated on the host: B = 0 is a no-op */
  swa_params p = {0};
  p.q = p.k = p.v = (const void*)tiles;
  p.out = (void*)tiles;
  p.H = 4; p.Hkv = 2; p.N = 64; p.D = 128; p.dilation = 1;
  p.dtype = SWA_DTYPE_BF16;
  int ok0 = swa_forward_ex(&p, NULL);
  p.dtype = 9;
  int bad_dtype = swa_forward_ex(&p, NULL);
  printf("%%d %%d\n", ok0, bad_dtype);
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("case", [
    dict(N=1000, L=100, R=0, d=1, bs=0, pos=5000, W=4096, ps=256),
    dict(N=16384, L=128, R=128, d=4, bs=0, pos=100, W=4096, ps=64),
    dict(N=4096, L=256, R=256, d=2, bs=64, pos=4095, W=4096, ps=512),
])
def test_header_is_c99_and_links(tmp_path, case):
    src = tmp_path / "use_swa.c"
    exe = tmp_path / "use_swa"
    src.write_text(PROGRAM % case)
    libdir = os.path.dirname(binding.library_path())
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", INCLUDE,
                    str(src), "-L", libdir, "-lswa", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                   check=True, capture_output=True)
    lines = subprocess.run([str(exe)], check=True, capture_output=True,
                           text=True).stdout.splitlines()
    version, n, st, first, last, bad = (int(x) for x in lines[0].split())
    assert version == binding.swa_version()
    sched = binding.swa_schedule(case["N"], case["L"], case["R"], case["d"], case["bs"])
    assert n == len(sched)
    assert tuple(int(x) for x in lines[1].split()) == sched[0]
    assert st == 0
    lo = max(0, case["pos"] - case["W"] + 1)
    assert (first, last) == (lo // case["ps"], case["pos"] // case["ps"])
    assert bad == -1  # SWA_ERR_ARG
    assert lines[2] == binding.swa_status_string(-3)
    assert lines[3].split() == ["0", "-1"]  # SWA_OK, SWA_ERR_ARG
