// swa_sched.cuh -- band-aware tile scheduler for the fused forward kernel.
//
// The rows of one problem are split into residue classes so that inside a
// class the key set of every row is a contiguous interval of the class's
// own ("virtual") row order:
//
//   token-level dilation d: class c holds positions c, c+d, c+2d, ...
//     (the dilated window j = i + k*d of page "空洞滑窗机制" §二.1 keeps
//     i and j in the same class, and inside it becomes a plain band
//     [m - L, m + R] of virtual rows);
//   block-level dilation with Bs-token blocks: class c holds the blocks
//     c, c+d, c+2d, ... (page "空洞滑窗机制" §四: skip whole 64-token
//     blocks), inside which a row of virtual block u sees the blocks
//     [u - L/Bs, u + R/Bs].
//
// With the interval [lo(m), hi(m)] monotone in the virtual row m, the key
// tiles a 128-row query tile needs are exactly those meeting
// [lo(first row), hi(last row)] (the per-query start/end range of the
// sparse_pattern array on page "大模型窗口扩展技术" §6, lifted to tiles), and
// a tile needs no element mask when it lies inside every row's interval.
// Tiles outside the band are never visited: the work is O(n * w).
#pragma once

#include <cstdint>

#if defined(__CUDACC__)
#define SWA_HD __host__ __device__ __forceinline__
#else
#define SWA_HD inline
#endif

namespace swa {

constexpr int kTileM = 128;  // query rows per tile
constexpr int kTileN = 128;  // keys per tile
constexpr int kBlockRows = 64;  // rows per TMA box (one dilation block)

struct Geometry {
  int N;         // sequence length
  int d;         // dilation (>= 1)
  int bs;        // 0/1: token-level; > 1: block size of block-level dilation
  int L, R;      // window half-widths in steps (< 0: unbounded)
  int nclass;    // residue classes
};

SWA_HD Geometry make_geometry(int N, int L, int R, int d, int bs) {
  Geometry g;
  g.N = N;
  g.d = d;
  g.bs = bs > 1 ? bs : 0;
  g.L = L;
  g.R = R;
  if (g.bs) {
    int nb = (N + g.bs - 1) / g.bs;
    g.nclass = nb < d ? nb : d;
  } else {
    g.nclass = N < d ? N : d;
  }
  return g;
}

// Number of virtual rows of class c (including the padding rows of a
// partial final block in block mode).
SWA_HD int class_rows(const Geometry& g, int c) {
  if (g.bs) {
    int nb = (g.N + g.bs - 1) / g.bs;
    int nu = (nb - c + g.d - 1) / g.d;
    return nu * g.bs;
  }
  return (g.N - c + g.d - 1) / g.d;
}

// Number of valid virtual rows of class c: rows past the sequence end only
// exist in the last block of block mode, and they come last in the class.
SWA_HD int class_valid_rows(const Geometry& g, int c) {
  int M = class_rows(g, c);
  if (g.bs) {
    int nb = (g.N + g.bs - 1) / g.bs;
    int nu = M / g.bs;
    int last_block = c + (nu - 1) * g.d;
    if (last_block == nb - 1 && (g.N % g.bs) != 0) M -= g.bs - g.N % g.bs;
  }
  return M;
}

// Physical position of virtual row m of class c.
SWA_HD int64_t phys_row(const Geometry& g, int c, int m) {
  if (g.bs) return (int64_t)(c + (int64_t)(m / g.bs) * g.d) * g.bs + (m % g.bs);
  return (int64_t)c + (int64_t)m * g.d;
}

// Key interval [lo, hi] of virtual row m, in virtual rows of its class,
// before clipping to [0, Mv-1].  win_right == 0 is causal: hi = m.
SWA_HD int key_lo(const Geometry& g, int m) {
  if (g.L < 0) return 0;
  if (g.bs) return (m / g.bs - g.L / g.bs) * g.bs;
  return m - g.L;
}
SWA_HD int key_hi(const Geometry& g, int m, int Mv) {
  if (g.R < 0) return Mv - 1;
  if (g.R == 0) return m;
  if (g.bs) return (m / g.bs + g.R / g.bs + 1) * g.bs - 1;
  return m + g.R;
}

// First and last query row (virtual rows of the class, before clipping to
// [0, Mv-1]) whose key interval [key_lo, key_hi] contains key row j: the
// transpose of key_lo / key_hi (both are monotone in the row, so the rows
// that see a key form one interval).  The backward walks it key-stationary.
SWA_HD int query_lo(const Geometry& g, int j) {
  if (g.R < 0) return 0;
  if (g.R == 0) return j;
  if (g.bs) return (j / g.bs - g.R / g.bs) * g.bs;
  return j - g.R;
}
SWA_HD int query_hi(const Geometry& g, int j, int Mv) {
  if (g.L < 0) return Mv - 1;
  if (g.bs) return (j / g.bs + g.L / g.bs + 1) * g.bs - 1;
  return j + g.L;
}

struct TileRange {
  int kv_begin, kv_end;  // kv tiles [begin, end) of the class
};

// KV tiles needed by the query rows [m0, m1] of a class whose keys are its
// Mv valid rows.
SWA_HD TileRange tile_range_rows(const Geometry& g, int Mv, int m0, int m1) {
  int lo = key_lo(g, m0);
  if (lo < 0) lo = 0;
  int hi = key_hi(g, m1, Mv);
  if (hi > Mv - 1) hi = Mv - 1;
  TileRange r;
  r.kv_begin = lo / kTileN;
  r.kv_end = hi / kTileN + 1;
  if (r.kv_end < r.kv_begin) r.kv_end = r.kv_begin;
  return r;
}

// KV tiles needed by query tile qt of a class with Mv valid rows.
SWA_HD TileRange tile_range(const Geometry& g, int Mv, int qt) {
  int m0 = qt * kTileM;
  int m1 = m0 + kTileM - 1;
  if (m1 > Mv - 1) m1 = Mv - 1;
  return tile_range_rows(g, Mv, m0, m1);
}

// KV tiles [*lo, *hi] of the 128 query rows [m0, m0 + 127] whose every
// (row, key) pair is inside the window and in range, so they need no
// element mask (empty when *lo > *hi).  Key bounds are monotone in the row,
// so the keys every row sees are [key_lo(last row), key_hi(first row)], and
// those tiles form one contiguous run.
SWA_HD void interior_tiles_rows(const Geometry& g, int Mv, int m0, int* lo, int* hi) {
  const int m1 = m0 + kTileM - 1;
  *lo = 1;
  *hi = 0;
  if (m1 > Mv - 1) return;
  int a = key_lo(g, m1);
  if (a < 0) a = 0;
  int b = key_hi(g, m0, Mv);
  if (b > Mv - 1) b = Mv - 1;
  *lo = (a + kTileN - 1) / kTileN;
  *hi = (b + 1) / kTileN - 1;
}

// The same for query tile qt of a class with Mv valid rows.
SWA_HD void interior_tiles(const Geometry& g, int Mv, int qt, int* lo, int* hi) {
  interior_tiles_rows(g, Mv, qt * kTileM, lo, hi);
}

// Query tiles that see any key of the 128 key rows [j0, j0 + 127] of a
// class with Mv valid rows (the key-stationary walk of the backward).
SWA_HD TileRange qtile_range_keys(const Geometry& g, int Mv, int j0) {
  int j1 = j0 + kTileN - 1;
  if (j1 > Mv - 1) j1 = Mv - 1;
  int lo = query_lo(g, j0);
  if (lo < 0) lo = 0;
  int hi = query_hi(g, j1, Mv);
  if (hi > Mv - 1) hi = Mv - 1;
  TileRange r;
  r.kv_begin = lo / kTileM;
  r.kv_end = hi / kTileM + 1;
  if (r.kv_end < r.kv_begin) r.kv_end = r.kv_begin;
  return r;
}

// Query tiles [*lo, *hi] in which every (query, key) pair with a key of
// [j0, j0 + 127] is inside the window and in range (no element mask).
SWA_HD void interior_qtiles_keys(const Geometry& g, int Mv, int j0, int* lo, int* hi) {
  const int j1 = j0 + kTileN - 1;
  *lo = 1;
  *hi = 0;
  if (j1 > Mv - 1) return;
  int a = query_lo(g, j1);
  if (a < 0) a = 0;
  int b = query_hi(g, j0, Mv);
  if (b > Mv - 1) b = Mv - 1;
  *lo = (a + kTileM - 1) / kTileM;
  *hi = (b + 1) / kTileM - 1;
}

}  // namespace swa
