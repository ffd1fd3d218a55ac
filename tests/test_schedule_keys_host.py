"""The key-stationary side of the band-aware scheduler (the backward's
walk): for every key row, the query rows whose window holds it form the
interval [query_lo, query_hi] the scheduler computes; the query tiles it
lists for a 128-key tile are exactly those holding such rows; and its
interior tiles are exactly those where every (query, key) pair is inside
the window.  The scheduler's header is compiled as plain C++ (g++) into a
small driver; the truth is the oracle's explicit key lists.  No GPU."""
import os
import shutil
import subprocess

import pytest

import oracle
from test_schedule_host import CASES, TILE, classes

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "sliding_window_attention_fwd_b200", "csrc")

DRIVER = r"""
#include <cstdio>
#include <cstdlib>
#include "swa_sched.cuh"
using namespace swa;
int main(int argc, char** argv) {
  const int N = atoi(argv[1]), L = atoi(argv[2]), R = atoi(argv[3]), d = atoi(argv[4]),
            bs = atoi(argv[5]);
  const Geometry g = make_geometry(N, L, R, d, bs);
  for (int c = 0; c < g.nclass; ++c) {
    const int Mv = class_valid_rows(g, c);
    printf("class %d %d\n", c, Mv);
    for (int j = 0; j < Mv; ++j) {
      int lo = query_lo(g, j), hi = query_hi(g, j, Mv);
      if (lo < 0) lo = 0;
      if (hi > Mv - 1) hi = Mv - 1;
      printf("key %d %d %d\n", j, lo, hi);
    }
    for (int kt = 0; kt * 128 < Mv; ++kt) {
      const TileRange r = qtile_range_keys(g, Mv, kt * 128);
      int ilo, ihi;
      interior_qtiles_keys(g, Mv, kt * 128, &ilo, &ihi);
      printf("tile %d %d %d %d %d\n", kt, r.kv_begin, r.kv_end, ilo, ihi);
    }
  }
  return 0;
}
"""


@pytest.fixture(scope="module")
def driver(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("needs g++")
    d = tmp_path_factory.mktemp("sched")
    src, exe = d / "drv.cpp", d / "drv"
    src.write_text(DRIVER)
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", CSRC, str(src), "-o", str(exe)],
                   check=True, capture_output=True)
    return str(exe)


def parse(out):
    res, cur = {}, None
    for ln in out.splitlines():
        f = ln.split()
        if f[0] == "class":
            cur = res.setdefault(int(f[1]), {"Mv": int(f[2]), "key": {}, "tile": {}})
        elif f[0] == "key":
            cur["key"][int(f[1])] = (int(f[2]), int(f[3]))
        else:
            cur["tile"][int(f[1])] = tuple(int(x) for x in f[2:])
    return res


def check(driver, case):
    N, L, R, d, bs = case
    out = subprocess.run([driver, *(str(x) for x in case)], check=True, capture_output=True,
                         text=True).stdout
    got = parse(out)
    cls = classes(N, d, bs)
    assert sorted(got) == list(range(len(cls)))
    for c, rows in enumerate(cls):
        Mv = len(rows)
        assert got[c]["Mv"] == Mv
        virt = {p: m for m, p in enumerate(rows)}
        # queries (virtual rows) that see each key (virtual row)
        seen_by = {j: set() for j in range(Mv)}
        for m in range(Mv):
            for kp in oracle.key_set(rows[m], N, L, R, d, bs):
                seen_by[virt[int(kp)]].add(m)
        for j in range(Mv):
            lo, hi = got[c]["key"][j]
            assert seen_by[j] == set(range(lo, hi + 1)), (c, j)
        for kt, (qb, qe, ilo, ihi) in got[c]["tile"].items():
            keys = range(kt * TILE, min(kt * TILE + TILE, Mv))
            need = {m // TILE for j in keys for m in seen_by[j]}
            if need:
                assert (qb, qe - 1) == (min(need), max(need)), (c, kt)
            full = set()
            for qt in range(qb, qe):
                qrows = range(qt * TILE, qt * TILE + TILE)
                if qt * TILE + TILE <= Mv and kt * TILE + TILE <= Mv and all(
                        set(qrows) <= seen_by[j] for j in keys):
                    full.add(qt)
            assert set(range(ilo, ihi + 1)) & set(range(qb, qe)) == full, (c, kt)


@pytest.mark.parametrize("case", [c for c in CASES if c[0] <= 2100])
def test_key_stationary_bounds(driver, case):
    check(driver, case)


@pytest.mark.parametrize("case", [
    (1000, 300, 300, 1, 64), (900, 63, 0, 1, 64), (640, 200, 70, 3, 64), (777, 5, 9, 2, 0),
    (500, -1, -1, 1, 0), (400, -1, 0, 3, 64),
])
def test_key_stationary_more(driver, case):
    check(driver, case)
