// swa_fwd_sm100.cu -- fused bf16 sliding-window attention forward for B200.
//
// A CTA computes the same 128-row query tile of one (batch, residue class)
// for NSLOT (1 or 2) query heads.  Only the key tiles the band-aware
// scheduler lists are visited (page "别再只加Mask了", §1: out-of-window
// pairs are skipped, not masked; "空洞滑窗机制" §四: dilation handled on
// dense tiles of whole blocks), followed, when global tokens exist, by
// tiles of gathered global keys (aiqz.cc page, "全局注意力token").
//
// Two query heads per CTA let the tensor core alternate between them:
// while one softmax warpgroup turns S into P for head 0, the MMAs of head 1
// run, and the other way round.  The two heads share a kv head (GQA: one
// K/V stream; the kernel can also stream two kv heads, NSTREAM = 2).
// Without such a pair a CTA takes one head; at D = 64 two of those CTAs
// share an SM and alternate the same way.
//
// Warp roles (warpgroup 0 = warps 0-3; warpgroup 1 + s = softmax of slot s):
//   warp 0     producer: TMA loads of the Q tiles once and of the K/V tiles
//              into a shared-memory ring (128-byte swizzle); global keys are
//              gathered with plain 16-byte loads into the same layout;
//   warp 1 + s MMA issuer of slot s (warp 1 also owns the 512 TMEM columns):
//                S_s  = Q_s K^T     tcgen05.mma, operands in smem, fp32 in
//                                   TMEM, in two 64-key halves
//                O_s += P_s V       tcgen05.mma, P (bf16) read from TMEM where
//                                   it overwrote S_s, V from smem
//              Tile j's P is kept in the columns of its early half (j & 1);
//              the early half of tile j+1 goes to the other columns as soon
//              as the softmax has read them, so it is ready when the softmax
//              finishes tile j, and only the late half waits for PV(j).  PV
//              itself is issued in two key halves: the early half's share as
//              soon as its P is written, so only a quarter-tile of PV sits
//              between the end of tile j's softmax and S of tile j+1's late
//              half.  One issuer per slot, each on its own SM sub-partition:
//              a single issuer sharing a sub-partition with two busy softmax
//              warps gets too few issue slots to keep the tensor core fed;
//   softmax    thread t of warpgroup 1+s owns query row t of slot s: row max
//              and row sum are thread-local tree reductions, no shuffles.
//              Element masks only on tiles the scheduler marks as edges.
//              Scores are read from TMEM 64 columns at a time and turned into
//              P against the current running max while the half's max is
//              found (the max changes rarely); a max that grows by more than
//              2^8 is adopted before the next tile by rescaling O and l, one
//              that jumps by more than 2^64 at once (the half is redone), and
//              the final O / l is exact either way.  With two slots the
//              producer/issuer warpgroup gives registers to the softmax
//              warpgroups (setmaxnreg), which then run without spills.
// Per row: out = O / l (bf16), lse = m + ln l (fp32).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "swa_internal.h"
#include "swa_ptx.cuh"
#include "swa_sched.cuh"

namespace swa {
namespace {

constexpr int kMaxClasses = 8;   // residue classes per launch (tensor maps in params)
constexpr int kChunkBytes = kTileM * 128;  // one 64-column slice of a 128-row tile
constexpr float kRescaleThreshold = 8.0f;  // log2 units
struct FwdParams {
  CUtensorMap tmQ[kMaxClasses];
  CUtensorMap tmK[kMaxClasses];
  CUtensorMap tmV[kMaxClasses];
  CUtensorMap tmKf;  // K and V over the whole sequence (rows in position order):
  CUtensorMap tmVf;  // the keys of the global query rows
  uint16_t* out;
  float* lse;
  const int32_t* G;
  const uint16_t* q_raw;
  const uint16_t* k_raw;
  const uint16_t* v_raw;
  int* err;
  int n_global;
  int B, H, Hkv, N;
  int L, R, d, bs;
  int class0, nclass;
  // Global query rows: the first n_gitems CTAs of the grid each take up to
  // 128 global rows (a "global tile") of one (batch, head pair), n_gq_tiles
  // tiles per pair, and attend every key of the sequence (causal: up to the
  // row).  The band CTAs leave those rows to them.
  int n_gitems, n_gq_tiles;
  int qtile_prefix[kMaxClasses + 1];
  int qt_base;  // first query tile of the launch (a row-range launch of one class)
  int Mv[kMaxClasses];
  float scale_log2;
  // Query window (chunked append; pos0 == NULL otherwise): the Mq query
  // rows are local rows 0..Mq-1 of q / out / lse ([B, Mq, H, D] /
  // [B, H, Mq]) and sit at virtual rows q0.. of the key sequence, whose
  // row v holds position pos0[b] - (win - 1) + v; rows of negative
  // positions (v < win - 1 - pos0[b]) are masked.
  const int64_t* pos0;
  int q0, Mq, win;
  // In place (win % 64 == 0): the keys are read from the ring (tmK[0],
  // tmV[0]: [B, win, Hkv, D]) and the chunk (tmKf, tmVf: [B, Mq, Hkv, D])
  // without a staged copy.  Per batch, with s_first = (pos0 - win + 1) mod
  // win the slot of the window's oldest position and hs = s_first mod 64,
  // virtual key row v < cs reads ring slot (s_first - hs + v) mod win and
  // row v >= cs chunk row v - cs, where cs = the multiple of 64 at or above
  // hs + win - 1: every 64-row box then lies inside one source without
  // wrapping.  The history sits at rows [hs, hs + win - 1), the rows
  // [hs + win - 1, cs) between it and the chunk are masked, and chunk row c
  // (virtual row cs + c) sees rows [hs + c, cs + c].
  int inplace;
  // Stacked heads (query window, two slots, Mq <= 64, GQA group a multiple
  // of 4): a slot's 128-row tile holds two heads of the group, rows 0-63
  // the first one's tokens and rows 64-127 the second one's, so the four
  // heads of a CTA share one key walk with no empty query rows.
  int stack;
  // Split key walks (query window): each item's key tiles are cut into
  // nsplit contiguous parts, one CTA each, which write O / l (fp32) and
  // lse to part_o [nsplit, B, H, Mq, D] and part_lse [nsplit, B, H, Mq];
  // a merge kernel combines them.  nsplit == 1: the output is written
  // directly.
  int nsplit;
  float* part_o;
  float* part_lse;
  // Paired parts (nsplit == 2, launched as clusters of two CTAs whose rank
  // is the part): the two parts merge through distributed shared memory and
  // write out / lse themselves, with no partials and no merge kernel.
  // ring_store (paired, in place, one query tile, every head of the kv head
  // in one item, so the cluster holds every reader of the kv head's ring
  // rows): once both parts' MMAs are done, the chunk's keys (part 0) and
  // values (part 1) enter their ring slots (pos0 + c) % win.
  int pair;
  int ring_store;
  uint4* k_ring;
  uint4* v_ring;
  const uint4* kn_raw;
  const uint4* vn_raw;
};

template <int D, int NSLOT, int NSTREAM>
struct Cfg {
  static constexpr int kTile = D / 64 * kChunkBytes;        // 128 rows x D bf16
  static constexpr int kStageBytes = 2 * NSTREAM * kTile;   // K and V of every stream
  static constexpr int kQBytes = NSLOT * kTile;
  // one head at D = 64 is small enough for two CTAs per SM (shared memory,
  // TMEM and, with the register split below, registers), so one CTA's fill
  // and drain overlap the other's tiles
  static constexpr int kMinBlocks = (NSLOT == 1 && D == 64) ? 2 : 1;
  static constexpr int kBudget = kMinBlocks == 2 ? 96 * 1024 : 224 * 1024;
  // TMEM: S/P of slot s at [128 s, 128 s + 128), O of slot s at kOcol + D s
  static constexpr uint32_t kOcol = 128u * NSLOT;
  static constexpr uint32_t kTmemCols = kOcol + NSLOT * D <= 256 ? 256u : 512u;
  static constexpr int kFit = (kBudget - kQBytes) / kStageBytes;
  static constexpr int kStages = kFit > 4 ? 4 : kFit;
  static_assert(kStages >= 2, "K/V ring needs two stages");
  static constexpr int kThreads = 128 * (1 + NSLOT);
  static constexpr int kQ = 0;
  static constexpr int kRing = kQ + kQBytes;
  static constexpr int kBar = kRing + kStages * kStageBytes;
  // full_q, full_k[S], empty_k[S], full_v[S], empty_v[S],
  // se_full[2], sl_full[2], l_free[2], p_full[2], o_done[2], o_final[2],
  // pe_full[2], oe_done[2], peer_free, xfer
  static constexpr int kNumBars = 1 + 4 * kStages + 18;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kTotal = kMisc + 16;
  static constexpr int kAlloc = kTotal + 1024;  // slack for 1024-byte alignment
  static_assert(kAlloc <= 232448, "shared memory budget");
  // paired parts: the half of O the other part writes (fp32, NSLOT x 128
  // rows of D / 2) and its (m, l) per row land in the ring
  static constexpr int kRxO = NSLOT * 128 * (D / 2) * 4;
  static_assert(kRxO + NSLOT * 128 * 8 <= kStages * kStageBytes, "pair exchange area");
};

// KIND (compile-time, so each form carries only its own code): 0 band (and
// token/block dilation) only; 1 the query window of a chunked append; 2 the
// band plus global tokens (global-key tiles and global query rows).
template <int D, int NSLOT, int NSTREAM, int KIND>
__global__ void __launch_bounds__(Cfg<D, NSLOT, NSTREAM>::kThreads,
                                  Cfg<D, NSLOT, NSTREAM>::kMinBlocks)
    swa_fwd_sm100_kernel(const __grid_constant__ FwdParams p) {
  using C = Cfg<D, NSLOT, NSTREAM>;
  constexpr int kStages = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBar);
  uint64_t* full_q = bars;
  uint64_t* full_k = bars + 1;
  uint64_t* empty_k = full_k + kStages;
  uint64_t* full_v = empty_k + kStages;
  uint64_t* empty_v = full_v + kStages;
  uint64_t* se_full = empty_v + kStages;  // [slot]: early half of S ready
  uint64_t* sl_full = se_full + 2;        // [slot]: late half of S ready
  uint64_t* l_free = sl_full + 2;         // [slot]: late half of S read out
  uint64_t* p_full = l_free + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* o_final = o_done + 2;
  uint64_t* pe_full = o_final + 2;  // [slot]: P of the early half written
  uint64_t* oe_done = pe_full + 2;  // [slot]: PV of the early half done
  // paired parts: the other part's MMAs are done (its ring may be
  // written); the other part's half of O and (m, l) have landed here
  uint64_t* peer_free = oe_done + 2;
  uint64_t* xfer = peer_free + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMisc + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  // ---- work item: the global tiles first (each walks the whole sequence),
  // then (class, q tile, batch, head pair) with heavy (late) tiles first
  constexpr bool qwin = KIND == 1;
  const bool stack = qwin && NSLOT == 2 && p.stack;
  const int npair = stack ? p.H / (2 * NSLOT) : (p.H + NSLOT - 1) / NSLOT;
  int x = blockIdx.x;
  constexpr bool glob = KIND == 2;
  const bool gitem = glob && x < p.n_gitems;
  if (glob && !gitem) x -= p.n_gitems;
  int sp = 0;  // part of a split key walk
  if (qwin) {
    sp = x % p.nsplit;
    x /= p.nsplit;
  }
  const int hp = x % npair;
  x /= npair;
  const int b = x % p.B;
  x /= p.B;
  int cl = 0, qt = 0, gq0 = 0, gcnt = 0;
  if (gitem) {
    gq0 = x * kTileM;  // first global row of this tile
    gcnt = min(kTileM, p.n_global - gq0);
  } else {
    const int jt = p.qtile_prefix[p.nclass] - 1 - x;
    while (cl + 1 < p.nclass && p.qtile_prefix[cl + 1] <= jt) ++cl;
    qt = jt - p.qtile_prefix[cl] + p.qt_base;
  }
  const int c = p.class0 + cl;
  const int grp = p.H / p.Hkv;
  int head[NSLOT], kvh[NSLOT];
  bool slot_ok[NSLOT];
#pragma unroll
  for (int s = 0; s < NSLOT; ++s) {
    // stacked: slot s holds heads head[s] (rows 0-63) and head[s] + 1
    head[s] = stack ? hp * 2 * NSLOT + 2 * s : hp * NSLOT + s;
    slot_ok[s] = head[s] < p.H;
    if (!slot_ok[s]) head[s] = p.H - 1;
    kvh[s] = head[s] / grp;
  }
  // in-place query window: per-batch key layout (see FwdParams::inplace)
  const bool inplace = qwin && p.inplace;
  int ip_hs = 0, ip_cs = 0, ip_base = 0;
  if (inplace) {
    const int W = p.win;
    long long sf = (p.pos0[b] - W + 1) % W;
    if (sf < 0) sf += W;
    ip_hs = (int)sf & 63;
    ip_cs = ip_hs <= 1 ? W : W + 64;
    ip_base = (int)sf - ip_hs;  // ring slot of virtual row 0, a multiple of 64
  }
  const Geometry g = inplace ? make_geometry(ip_cs + p.Mq, ip_cs - ip_hs, 0, 1, 0)
                             : make_geometry(p.N, p.L, p.R, p.d, p.bs);
  // a global tile's keys are the physical rows of the sequence
  const int Mv = gitem ? p.N : (inplace ? ip_cs + p.Mq : p.Mv[cl]);
  const int Mq = qwin ? p.Mq : Mv;           // query rows (local; stacked: tokens)
  const int q0 = qwin ? (inplace ? ip_cs : p.q0) : 0;  // virtual row of local query row 0
  const int qm0 = q0 + qt * kTileM;
  const int qm1 = q0 + min(qt * kTileM + kTileM - 1, Mq - 1);
  TileRange tr;
  if (gitem) {
    // every key tile (causal: up to the tile's last, i.e. largest, global row)
    int last = __ldg(p.G + gq0 + gcnt - 1);
    last = last < 0 ? 0 : (last >= p.N ? p.N - 1 : last);
    tr.kv_begin = 0;
    tr.kv_end = p.R == 0 ? last / kTileN + 1 : (p.N + kTileN - 1) / kTileN;
  } else {
    tr = tile_range_rows(g, Mv, qm0, qm1);
    if (qwin && p.nsplit > 1) {
      // this CTA's part of the key walk
      const int n = tr.kv_end - tr.kv_begin;
      const int part = (n + p.nsplit - 1) / p.nsplit;
      const int a = tr.kv_begin + sp * part;
      tr.kv_begin = min(a, tr.kv_end);
      tr.kv_end = min(a + part, tr.kv_end);
    }
  }
  int lo_b = 0;  // first key row holding a real position (query window only)
  if (qwin) {
    const long long pb = p.pos0[b];
    const long long lb = (long long)(p.win - 1) - pb + ip_hs;
    lo_b = lb <= ip_hs ? ip_hs : (lb > Mv ? Mv : (int)lb);
  }
  // in place: the masked rows between the history and the chunk
  const int gap_lo = inplace ? ip_hs + p.win - 1 : 0, gap_hi = inplace ? ip_cs : 0;
  const int n_band = tr.kv_end - tr.kv_begin;
  int n_gtiles = (!glob || gitem) ? 0 : (p.n_global + kTileN - 1) / kTileN;
  if (n_gtiles > 0 && p.d == 1 && p.bs <= 1 && p.L >= 0) {
    // token-level band: a global key g joins row i unless i - L <= g <= i +
    // R (in the band) or, causal, g > i.  If no row of the tile [qm0, qm1]
    // takes any global key (the smallest one lies inside or right of every
    // row's band, the largest inside or left of it), the global-key tiles
    // would be fully masked: skip them (attention sinks near the start of
    // the sequence, seen by the first W rows through the band anyway).
    const int qr0 = qt * kTileM, qr1 = min(qt * kTileM + kTileM - 1, Mv - 1);
    int g_first = __ldg(p.G), g_last = __ldg(p.G + p.n_global - 1);
    g_first = g_first < 0 ? 0 : (g_first >= p.N ? p.N - 1 : g_first);
    g_last = g_last < 0 ? 0 : (g_last >= p.N ? p.N - 1 : g_last);
    const bool left = g_first < qr1 - p.L;
    const bool right = p.R > 0 && g_last > qr0 + p.R;  // causal (R == 0) takes none right
    if (!left && !right) n_gtiles = 0;
  }
  const int n_tiles = n_band + n_gtiles;
  const bool block_mode = p.bs > 1;
  const int map_idx = block_mode ? 0 : cl;

  // virtual row -> TMA row coordinate of a 64-row box
  auto box_row = [&](int vrow) -> int {
    return block_mode ? (c + p.d * (vrow / kBlockRows)) * kBlockRows : vrow;
  };
  const CUtensorMap* mapK = gitem ? &p.tmKf : &p.tmK[map_idx];
  const CUtensorMap* mapV = gitem ? &p.tmVf : &p.tmV[map_idx];
  // the source of a 64-row key box at virtual row vrow (a multiple of 64):
  // its tensor map and row coordinate
  auto kv_box = [&](int kv, int vrow, int* row) -> const CUtensorMap* {
    if (inplace) {
      if (vrow < ip_cs) {
        *row = (ip_base + vrow) % p.win;
        return kv ? &p.tmV[0] : &p.tmK[0];
      }
      *row = vrow - ip_cs;
      return kv ? &p.tmVf : &p.tmKf;
    }
    *row = gitem ? vrow : box_row(vrow);
    return kv ? mapV : mapK;
  };
  // TMA loads (one thread): the Q tiles, and K or V of band tile it
  auto load_q = [&]() {
    prefetch_tensormap(&p.tmQ[map_idx]);
    mbar_arrive_expect_tx(full_q, C::kQBytes);
    for (int s = 0; s < NSLOT; ++s)
      for (int cc = 0; cc < D / 64; ++cc)
        for (int hh = 0; hh < 2; ++hh)
          tma_load_4d(smem + C::kQ + s * C::kTile + cc * kChunkBytes + hh * (kChunkBytes / 2),
                      &p.tmQ[map_idx], full_q, cc * 64, head[s] + (stack ? hh : 0),
                      stack ? 0 : box_row(qt * kTileM + hh * 64), b);
  };
  auto load_kv = [&](int it, int kv) {
    const int st = it % kStages;
    uint64_t* ful = kv ? &full_v[st] : &full_k[st];
    uint8_t* dst = smem + C::kRing + st * C::kStageBytes + kv * NSTREAM * C::kTile;
    const int t = tr.kv_begin + it;
    mbar_arrive_expect_tx(ful, NSTREAM * C::kTile);
    for (int hh = 0; hh < 2; ++hh) {
      int row;
      const CUtensorMap* m = kv_box(kv, t * kTileN + hh * 64, &row);
      for (int s = 0; s < NSTREAM; ++s)
        for (int cc = 0; cc < D / 64; ++cc)
          tma_load_4d(dst + s * C::kTile + cc * kChunkBytes + hh * (kChunkBytes / 2), m, ful,
                      cc * 64, kvh[s], row, b);
    }
  };
#ifdef SWA_TEST_WITHHOLD_TILE
  // failure-detection test build only: this K tile is never loaded, so the
  // MMA issuer's bounded wait for it runs out
  auto withheld = [](int it, int kv) { return kv == 0 && it == SWA_TEST_WITHHOLD_TILE; };
#else
  auto withheld = [](int, int) { return false; };
#endif
  // Thread 0 loads Q and the first K tile as soon as the barriers exist
  // (before TMEM allocation and the block barrier), the producer warp the
  // rest of the first ring pass after the block barrier: with every CTA of
  // a wave starting at once, a smaller first burst lands Q and K(0) sooner
  // (measured: append 57.3 -> 55.4 us, token / block dilation 152 -> 148 /
  // 154 -> 150 us, prefill within noise).  With global tokens the whole
  // first ring pass goes early (there one K tile only measured 2 % slower).
  const int n_early_k = gitem ? 0 : min(KIND == 2 ? kStages : 1, n_band);
  const int n_early_v = gitem ? 0 : min(KIND == 2 ? kStages : 0, n_band);

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(full_q, 1);
    // every issuing slot releases each K/V stage once
    int n_issuers = 0;
    for (int s = 0; s < NSLOT; ++s) n_issuers += slot_ok[s] ? 1 : 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_k[s], 1);
      mbar_init(&empty_k[s], n_issuers);
      mbar_init(&full_v[s], 1);
      mbar_init(&empty_v[s], n_issuers);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&se_full[s], 1);
      mbar_init(&sl_full[s], 1);
      mbar_init(&l_free[s], 128);
      mbar_init(&p_full[s], 128);
      mbar_init(&o_done[s], 1);
      mbar_init(&o_final[s], 1);
      mbar_init(&pe_full[s], 128);
      mbar_init(&oe_done[s], 1);
    }
    mbar_init(peer_free, 128 * NSLOT);
    mbar_init(xfer, 128 * NSLOT);
    fence_mbar_init();
    // (an empty part of a split key walk loads nothing: no copy may still
    // be landing in shared memory when the CTA exits)
    if (!gitem && n_tiles > 0) {
      prefetch_tensormap(mapK);
      prefetch_tensormap(mapV);
      if (inplace) {
        prefetch_tensormap(&p.tmKf);
        prefetch_tensormap(&p.tmVf);
      }
      load_q();
      for (int it = 0; it < n_early_k || it < n_early_v; ++it)
        for (int kv = 0; kv < 2; ++kv)
          if (it < (kv ? n_early_v : n_early_k) && !withheld(it, kv)) load_kv(it, kv);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // paired parts: this CTA's barriers exist (the other part waits for this
  // arrival before its first access to them)
  const bool pair = qwin && p.pair;
  if (pair) cluster_arrive_relaxed();
  const uint32_t tmem = *tmem_holder;
  // TMEM columns: slot s has S/P at [128 s, 128 s + 128) and O at 256 + 128 s.
  const uint32_t q_addr = smem_u32(smem + C::kQ);
  const uint32_t ring_addr = smem_u32(smem + C::kRing);

  if (warp < 4) {
    // producer and issuers need few registers: hand the rest to the softmax
    // warpgroups (two slots: 128 x 56 + 256 x 208 = 60416 <= 384 x 168
    // launched; one slot, two CTAs per SM: 128 x 56 + 128 x 200 = 256 x 128)
    if (NSLOT == 2 || C::kMinBlocks == 2)
      asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
    if (warp == 0) {
      // =========================== producer ===========================
      if (gitem) {
        // gather the tile's global query rows (zeros past the last) with
        // plain 16-byte loads into the swizzled layout of a TMA box
        if (lane == 0) {
          prefetch_tensormap(mapK);
          prefetch_tensormap(mapV);
        }
        constexpr int kC16 = D / 8;  // 16-byte chunks per row
        for (int s = 0; s < NSLOT; ++s) {
          for (int idx = lane; idx < kTileM * kC16; idx += 32) {
            const int row = idx / kC16, c16 = idx % kC16;
            uint4 val = make_uint4(0u, 0u, 0u, 0u);
            if (row < gcnt) {
              int gv = __ldg(p.G + gq0 + row);
              gv = gv < 0 ? 0 : (gv >= p.N ? p.N - 1 : gv);
              val = __ldg(reinterpret_cast<const uint4*>(
                  p.q_raw + (((size_t)b * p.N + gv) * p.H + head[s]) * D + c16 * 8));
            }
            uint8_t* d8 = smem + C::kQ + s * C::kTile + (c16 / 8) * kChunkBytes + row * 128 +
                          (((c16 % 8) ^ (row % 8)) * 16);
            *reinterpret_cast<uint4*>(d8) = val;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(full_q);
      }
      // last tiles whose loads were issued (the first n_early_k / n_early_v
      // already are)
      int last_k = n_early_k - 1, last_v = n_early_v - 1;
      for (int it = min(n_early_k, n_early_v); it < n_tiles; ++it) {
        const int st = it % kStages;
        const uint32_t ph = (uint32_t)(it / kStages) & 1u;
        for (int kv = 0; kv < 2; ++kv) {  // 0: K, 1: V
          if (it < (kv ? n_early_v : n_early_k)) continue;
          uint64_t* emp = kv ? &empty_v[st] : &empty_k[st];
          uint64_t* ful = kv ? &full_v[st] : &full_k[st];
          uint8_t* dst = smem + C::kRing + st * C::kStageBytes + kv * NSTREAM * C::kTile;
          if (it >= kStages && !mbar_wait(emp, ph ^ 1u, p.err, abort_flag)) goto producer_done;
          (kv ? last_v : last_k) = it;
          if (withheld(it, kv)) continue;
          if (!glob || it < n_band) {
            if (lane == 0) load_kv(it, kv);
          } else {
            // gather global-key rows with plain 16-byte loads into the
            // swizzled layout the MMA expects
            const int g0 = (it - n_band) * kTileN;
            const int cnt = min(kTileN, p.n_global - g0);
            const uint16_t* src_base = kv ? p.v_raw : p.k_raw;
            constexpr int kC16 = D / 8;  // 16-byte chunks per row
            for (int s = 0; s < NSTREAM; ++s) {
              for (int idx = lane; idx < kTileN * kC16; idx += 32) {
                const int row = idx / kC16, c16 = idx % kC16;
                uint4 val = make_uint4(0u, 0u, 0u, 0u);
                if (row < cnt) {
                  int gv = __ldg(p.G + g0 + row);
                  gv = gv < 0 ? 0 : (gv >= p.N ? p.N - 1 : gv);
                  const uint16_t* src =
                      src_base + (((size_t)b * p.N + gv) * p.Hkv + kvh[s]) * D + c16 * 8;
                  val = __ldg(reinterpret_cast<const uint4*>(src));
                }
                uint8_t* d8 = dst + s * C::kTile + (c16 / 8) * kChunkBytes + row * 128 +
                              (((c16 % 8) ^ (row % 8)) * 16);
                *reinterpret_cast<uint4*>(d8) = val;
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(ful);
          }
        }
      }
    producer_done:
      if (lane == 0 && *abort_flag) {
        // leave no copy writing shared memory behind
#ifdef SWA_TEST_WITHHOLD_TILE
        const int skip = SWA_TEST_WITHHOLD_TILE;
#else
        const int skip = -1;
#endif
        drain_copies(full_q, 1, 0, 0);
        drain_copies(full_k, kStages, 0, last_k, skip);
        drain_copies(full_v, kStages, 0, last_v);
      }
    } else if (warp <= NSLOT) {
      // =========================== MMA issuers ===========================
      // Warp 1 + s issues the MMAs of slot s (lane 0; the rest of the warp
      // idles at __syncwarp).  Each issuer sits on its own SM sub-partition:
      // a single issuer sharing its sub-partition with two busy softmax
      // warps gets too few issue slots to keep the tensor core fed, two of
      // them together do.  A wait of one issuer leaves the tensor core to
      // the other's MMAs.
      //
      // S of a slot is computed in two 64-key halves.  Tile j's P lives in
      // the TMEM columns of its early half E(j) = j & 1, so the other half's
      // columns are free as soon as the softmax has read them: the early
      // half of tile j+1 (same columns) is issued then, while the softmax
      // is still busy with tile j, and only the late half waits for PV(j).
      const int s = warp - 1;
      if (n_tiles > 0 && slot_ok[s] && lane == 0) {
        const uint32_t idesc_qk = idesc_bf16_f32(kTileM, kTileN / 2, 0, 0);
        const uint32_t idesc_pv = idesc_bf16_f32(kTileM, D, 0, 1);
        // Descriptors are built once; every MMA then only adds a compile-time
        // offset (start address field, 16-byte units) to a base descriptor.
        const uint64_t dq = sdesc_sw128(q_addr, 16, 1024) + (uint64_t)s * (C::kTile >> 4);
        const uint64_t dk0 = sdesc_sw128(ring_addr, 16, 1024) +
                             (NSTREAM == 2 ? (uint64_t)s * (C::kTile >> 4) : 0ull);
        const uint64_t dv0 = sdesc_sw128(ring_addr + NSTREAM * C::kTile, kChunkBytes, 1024) +
                             (NSTREAM == 2 ? (uint64_t)s * (C::kTile >> 4) : 0ull);
        constexpr uint64_t kStageStep = C::kStageBytes >> 4;
        constexpr uint64_t kHalfRows = (64 * 128) >> 4;  // 64 K rows inside a 64-column chunk
        const uint32_t tslot = tmem + 128u * s;
        // S[:, 64 hf : 64 hf + 64] = Q_s K[64 hf : 64 hf + 64]^T of tile it
        auto qk_half = [&](int it, int hf, uint64_t* done) {
          const uint64_t dk = dk0 + (uint64_t)(it % kStages) * kStageStep + (uint64_t)hf * kHalfRows;
          const uint32_t ts = tslot + 64u * hf;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint64_t off = (uint64_t)(((k / 4) * kChunkBytes + (k % 4) * 32) >> 4);
            mma_ss(ts, dq + off, dk + off, idesc_qk, k > 0 ? 1u : 0u);
          }
          tc_commit(done);
        };
        // O_s += P_s V over the keys of one half of tile it.  P (bf16 pairs)
        // sits in the columns of the tile's early half e = it & 1: the early
        // keys' P at [64 e, 64 e + 32), the late keys' at [64 e + 32, 64 e + 64).
        // The early half's share is issued as soon as its P is written, so
        // after the softmax finishes a tile only a quarter-tile of PV stands
        // between it and the late half of the next tile's S.
        auto pv_half = [&](int it, bool early) {
          const uint64_t dv = dv0 + (uint64_t)(it % kStages) * kStageStep;
          const uint32_t to = tmem + C::kOcol + (uint32_t)D * s;
          const int e = it & 1;
          const uint32_t tp = tslot + 64u * (uint32_t)e + (early ? 0u : 32u);
          const int kh = early ? e : (e ^ 1);  // key half
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int k = kh * 4 + kk;
            mma_ts(to, tp + 8u * kk, dv + (uint64_t)((k * 2048) >> 4), idesc_pv,
                   (it > 0 || !early || kk > 0) ? 1u : 0u);
          }
        };
        bool ok = mbar_wait(full_q, 0, p.err, abort_flag) &&
                  mbar_wait(&full_k[0], 0, p.err, abort_flag);
        tc_fence_after();
        if (ok) {
          qk_half(0, 0, &se_full[s]);
          qk_half(0, 1, &sl_full[s]);
          tc_commit(&empty_k[0]);
        }
        for (int it = 0; ok && it < n_tiles; ++it) {
          const int st = it % kStages;
          const bool more = it + 1 < n_tiles;
          const int e_next = (it + 1) & 1;  // early half of tile it + 1
          // the early half's P is in TMEM: its share of PV goes first
          if (!mbar_wait(&pe_full[s], (uint32_t)it & 1u, p.err, abort_flag)) break;
          if (!mbar_wait(&full_v[st], (uint32_t)(it / kStages) & 1u, p.err, abort_flag)) break;
          tc_fence_after();
          pv_half(it, true);
          tc_commit(&oe_done[s]);
          if (more) {
            // the softmax has read the late half of tile it; K of tile it + 1
            if (!mbar_wait(&l_free[s], (uint32_t)it & 1u, p.err, abort_flag)) break;
            if (!mbar_wait(&full_k[(it + 1) % kStages], (uint32_t)((it + 1) / kStages) & 1u,
                           p.err, abort_flag))
              break;
            tc_fence_after();
            qk_half(it + 1, e_next, &se_full[s]);
          }
          // P of tile it is in TMEM; V of tile it
          if (!mbar_wait(&p_full[s], (uint32_t)it & 1u, p.err, abort_flag)) break;
          tc_fence_after();
          pv_half(it, false);
          tc_commit(&o_done[s]);
          tc_commit(&empty_v[st]);
          if (more) {
            qk_half(it + 1, e_next ^ 1, &sl_full[s]);
            tc_commit(&empty_k[(it + 1) % kStages]);
          }
        }
        // o_final completes once every MMA issued above has finished (also on
        // the abort path, so TMEM is quiescent before it is freed).
        tc_commit(&o_final[s]);
      }
      __syncwarp();
    }
  } else {
    if (NSLOT == 2) asm volatile("setmaxnreg.inc.sync.aligned.u32 208;" ::: "memory");
    if (NSLOT == 1 && C::kMinBlocks == 2)
      asm volatile("setmaxnreg.inc.sync.aligned.u32 200;" ::: "memory");
    // ============================ softmax ============================
    const int slot = warp / 4 - 1;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + 128u * slot + lane_off;
    const uint32_t tO = tmem + C::kOcol + (uint32_t)D * slot + lane_off;
    // stacked: lanes 64-127 are the slot's second head, same tokens
    const int h = head[slot] + (stack ? (r >> 6) : 0);
    const int m_row = stack ? (r & 63) : qt * kTileM + r;  // local query row
    const int m_v = q0 + m_row;         // its virtual row among the keys
    bool row_valid;
    int klo, khi, i_phys;
    if (gitem) {
      // global row: every key of the sequence (causal: up to the row)
      row_valid = r < gcnt && slot_ok[slot];
      int gv = r < gcnt ? __ldg(p.G + gq0 + r) : 0;
      gv = gv < 0 ? 0 : (gv >= p.N ? p.N - 1 : gv);
      i_phys = gv;
      klo = 0;
      khi = r < gcnt ? (p.R == 0 ? gv : p.N - 1) : -1;
    } else {
      row_valid = m_row < Mq && slot_ok[slot];
      klo = max(key_lo(g, m_v), lo_b);
      // in place: a window that starts past the history starts in the
      // chunk, beyond the masked rows between the two
      if (inplace && klo >= gap_lo) klo += gap_hi - gap_lo;
      khi = key_hi(g, m_v, Mv);
      i_phys = (int)phys_row(g, c, m_v);
      // a global row is written by its global tile, not by the band
      if (glob && row_valid) {
        int lo = 0, hi = p.n_global - 1;
        while (lo <= hi) {
          const int mid = (lo + hi) >> 1;
          const int gv = __ldg(p.G + mid);
          if (gv == i_phys) {
            row_valid = false;
            break;
          }
          if (gv < i_phys) lo = mid + 1;
          else hi = mid - 1;
        }
      }
    }
    // a warp of a global tile whose 32 rows are all past the tile's last
    // global row only keeps the barriers going
    const bool warp_idle = gitem && quad * 32 >= gcnt;
    const bool causal = p.R == 0;
    // band of the row in physical positions, for the global-key test
    const int glo = p.L < 0 ? -0x40000000
                            : (block_mode ? (i_phys / p.bs - (p.L / p.bs) * p.d) * p.bs
                                          : i_phys - p.L * p.d);
    const int ghi = p.R < 0 ? 0x40000000
                            : (block_mode ? (i_phys / p.bs + (p.R / p.bs) * p.d + 1) * p.bs - 1
                                          : i_phys + p.R * p.d);
    const float sl2 = p.scale_log2;
    float m_used = -INFINITY;  // running max, scaled log2 units
    float l = 0.f;
    bool ok = slot_ok[slot];

    float m_pend = -INFINITY;  // max seen but not yet adopted (adopted next tile)
    int int_lo, int_hi;        // key tiles that need no element mask
    // (stacked: from the tokens' rows, conservatively as if they were the
    // last 128 rows below the last token)
    interior_tiles_rows(g, Mv, stack ? q0 + Mq - kTileM : qm0, &int_lo, &int_hi);
    const int last_row = stack ? Mq - 1 : qt * kTileM + kTileM - 1;  // local
    // mask every tile: global tiles, rows of negative positions, partial
    // query tiles, and in-place windows that start in the chunk
    if (gitem || lo_b > ip_hs || (stack ? Mq < 64 : qt * kTileM + kTileM > Mq) ||
        (inplace && last_row >= p.win - 1))
      int_hi = int_lo - 1;

    // the 64 score columns of key half hf (TMEM -> registers)
    auto read_half = [&](int hf, float (&sv)[64]) {
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        uint32_t v[32];
        tmem_ld32(tS + hf * 64 + jj * 32, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[jj * 32 + e] = __uint_as_float(v[e]);
      }
      tmem_wait_ld();
    };
    // -inf outside the row's key set, on edge and global tiles: a keep-mask
    // of the half's 64 keys (bit j: key j is in the set) applied by one
    // shared select loop
    auto mask_half = [&](int it, int hf, bool edge, float (&sv)[64]) {
      uint64_t keep = ~0ull;
      if (!glob || it < n_band) {
        if (edge) {
          const int n0 = (tr.kv_begin + it) * kTileN + hf * 64;
          const int lo = max(klo - n0, 0);
          const int hi = min(min(khi, Mv - 1) - n0, 63);  // inclusive
          keep = hi < lo ? 0ull : ((~0ull >> (63 - hi)) & (~0ull << lo));
          if (inplace) {
            const int a = max(gap_lo - n0, 0), z = min(gap_hi - n0, 64);  // [a, z)
            if (a < z) keep &= ~((z >= 64 ? ~0ull : ((1ull << z) - 1ull)) & (~0ull << a));
          }
        }
      } else {
        // a global key joins the row unless it is already in the row's band
        // (same residue class and inside [glo, ghi]) or, causal, after it
        const int g0 = (it - n_band) * kTileN + hf * 64;
        keep = 0ull;
#pragma unroll 1
        for (int j = 0; j < 64 && g0 + j < p.n_global; ++j) {
          int gv = __ldg(p.G + g0 + j);
          gv = gv < 0 ? 0 : (gv >= p.N ? p.N - 1 : gv);
          bool same = true;
          if (p.d > 1) same = ((block_mode ? gv / p.bs : gv) % p.d) == c;
          const bool inband = same && gv >= glo && gv <= ghi;
          if (!inband && (!causal || gv <= i_phys)) keep |= 1ull << j;
        }
      }
      if (__any_sync(0xffffffffu, keep != ~0ull)) {
#pragma unroll
        for (int j = 0; j < 64; ++j)
          if (!((keep >> j) & 1ull)) sv[j] = -INFINITY;
      }
    };
    auto half_max = [&](const float (&sv)[64]) -> float {
      float t[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) t[e] = max3f(sv[e], sv[8 + e], sv[16 + e]);
#pragma unroll
      for (int j = 24; j < 64; j += 16)
#pragma unroll
        for (int e = 0; e < 8; ++e) t[e] = max3f(t[e], sv[j + e], sv[j + 8 + e]);
      return max3f(max3f(t[0], t[1], t[2]), max3f(t[3], t[4], t[5]), fmaxf(t[6], t[7]));
    };
    // P = 2^(s * scale * log2 e - m_ref) for one key half, stored as 32
    // columns of bf16 pairs from TMEM column pcol.  At D = 128 seven of
    // every eight column pairs go to the MUFU ex2 unit and one to the FMA
    // pipe (polynomial), which takes some load off MUFU (measured best of 0,
    // 1/8, 1/4 and 1/2 on the FMA pipe with the split PV and the register
    // split); at D = 64 all go to MUFU (1/8 and 1/4 measured 1-4 % slower
    // on the one-head form).
    auto exp_half = [&](int pcol, const float (&sv)[64], float m_ref, float2 (&ls)[4]) {
      const float2 sl2_2 = make_float2(sl2, sl2), negm2 = make_float2(-m_ref, -m_ref);
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 xa =
              fma2(make_float2(sv[jj * 32 + 2 * e], sv[jj * 32 + 2 * e + 1]), sl2_2, negm2);
          float2 pr;
          if (D != 64 && (e & 7) == 7) {
            pr = exp2_poly2(xa);
          } else {
            pr.x = ex2_approx(xa.x);
            pr.y = ex2_approx(xa.y);
          }
          ls[e & 3] = add2(ls[e & 3], pr);
          pk[e] = pack_bf16x2(pr.x, pr.y);
        }
        tmem_st16(tS + pcol + jj * 16, pk);
      }
    };
    // zeros as the P of a key half (32 columns of bf16 pairs from pcol)
    auto zero_p = [&](int pcol) {
      uint32_t z[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) z[i] = 0u;
      tmem_st16(tS + pcol, z);
      tmem_st16(tS + pcol + 16, z);
    };
    // Multiplies O (and l) by 2^(m_from - m_to) and adopts m_to; O holds
    // P_0..P_{it-1} V, whose MMAs are complete once o_done says so.
    auto rescale_o = [&](int it, bool mine, float m_to) -> bool {
      const bool o_ok = mbar_wait(&o_done[slot], (uint32_t)(it - 1) & 1u, p.err, abort_flag);
      if (!__all_sync(0xffffffffu, o_ok)) return false;
      tc_fence_after();
      const float f = mine ? ex2_approx(m_used - m_to) : 1.f;
      l *= f;
#pragma unroll
      for (int j = 0; j < D / 32; ++j) {
        uint32_t v[32];
        tmem_ld32(tO + j * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * f);
        tmem_st32(tO + j * 32, v);
      }
      tmem_wait_st();
      if (mine) m_used = m_to;
      return true;
    };

    // Scores are exponentiated against the running max as it stands (a row
    // without keys so far adopts the max of the half at hand; its O and l
    // are still zero), and the tile max is tracked on the way.  Scores
    // above the running max only enlarge P, by at most 2^64 (safe in fp32
    // and bf16); a larger jump is adopted at once by rescaling O, l, the
    // partial sums and the P already written.
    for (int it = 0; ok && warp_idle && it < n_tiles; ++it) {
      // rows without a query: no scores to read and no P to write (the PV
      // MMA reads whatever these TMEM lanes hold; those O rows are never
      // stored), but the arrivals keep the phases of the barriers in step
      const uint32_t ph = (uint32_t)it & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(&sl_full[slot], ph, p.err, abort_flag))) {
        ok = false;
        break;
      }
      mbar_arrive(&pe_full[slot]);
      mbar_arrive(&l_free[slot]);
      mbar_arrive(&p_full[slot]);
    }
    for (int it = 0; ok && !warp_idle && it < n_tiles; ++it) {
      const int e = it & 1;  // early key half; P of the tile lives in its columns
      const uint32_t ph = (uint32_t)it & 1u;
      const int t_kv = tr.kv_begin + it;
      const bool edge = ((!glob || it < n_band) && !(t_kv >= int_lo && t_kv <= int_hi)) ||
                        (inplace && t_kv * kTileN < gap_hi && t_kv * kTileN + kTileN > gap_lo);

      // adopt a larger max seen on the previous tile (rare after the start)
      const bool pend = m_pend > m_used;
      if (__any_sync(0xffffffffu, pend)) {
        if (!rescale_o(it, pend, m_pend)) { ok = false; break; }
      }

      float2 ls[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                      make_float2(0.f, 0.f)};
      float sv[64];

      // ---- early half
      bool w_ok = mbar_wait(&se_full[slot], ph, p.err, abort_flag);
      if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
      tc_fence_after();
      // key halves of a global-key tile past the last global key hold no
      // key of any row: no scores to read, P = 0 (the same for every row)
      const bool gskip_e = glob && it >= n_band && (it - n_band) * kTileN + 64 * e >= p.n_global;
      float tmax = -INFINITY;
      if (gskip_e) {
        zero_p(64 * e);
      } else {
      read_half(e, sv);
      mask_half(it, e, edge, sv);
      if (!__any_sync(0xffffffffu, m_used == -INFINITY)) {
        // optimistic: exponentiate against the running max while the half's
        // max is found (no dependence between the two); a jump (rare)
        // rescales O and l and redoes the half against the new max
        exp_half(64 * e, sv, m_used, ls);
        tmax = half_max(sv);
        const bool jump = tmax * sl2 > m_used + 64.f;
        if (__any_sync(0xffffffffu, jump)) {
          if (!rescale_o(it, jump, fmaxf(m_used, tmax * sl2))) { ok = false; break; }
#pragma unroll
          for (int j = 0; j < 4; ++j) ls[j] = make_float2(0.f, 0.f);
          tmem_wait_st();
          exp_half(64 * e, sv, m_used, ls);
        }
      } else {
        // some row of the warp meets its first keys: find the max first
        tmax = half_max(sv);
        const bool adopt = m_used == -INFINITY;
        const bool jump = !adopt && tmax * sl2 > m_used + 64.f;
        if (adopt) m_used = tmax * sl2;
        if (__any_sync(0xffffffffu, jump)) {
          if (!rescale_o(it, jump, fmaxf(m_used, tmax * sl2))) { ok = false; break; }
        }
        exp_half(64 * e, sv, m_used == -INFINITY ? 0.f : m_used, ls);
      }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&pe_full[slot]);

      // ---- late half
      w_ok = mbar_wait(&sl_full[slot], ph, p.err, abort_flag);
      if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
      tc_fence_after();
      const bool gskip_l =
          glob && it >= n_band && (it - n_band) * kTileN + 64 * (e ^ 1) >= p.n_global;
      if (gskip_l) {
        tc_fence_before();
        mbar_arrive(&l_free[slot]);
        zero_p(64 * e + 32);
      } else {
      read_half(e ^ 1, sv);
      // these columns now belong to the early half of the next tile
      tc_fence_before();
      mbar_arrive(&l_free[slot]);
      mask_half(it, e ^ 1, edge, sv);
      if (!__any_sync(0xffffffffu, m_used == -INFINITY)) {
        // optimistic as above; on a jump O must also hold the early half's
        // PV (issued once its P was written) before it is scaled
        float2 lh[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
        exp_half(64 * e + 32, sv, m_used, lh);
        const float tmax1 = half_max(sv);
        tmax = fmaxf(tmax, tmax1);
        const bool jump = tmax1 * sl2 > m_used + 64.f;
        if (__any_sync(0xffffffffu, jump)) {
          const float m_old = m_used;
          const bool oe_ok = mbar_wait(&oe_done[slot], (uint32_t)it & 1u, p.err, abort_flag);
          if (!__all_sync(0xffffffffu, oe_ok)) { ok = false; break; }
          if (!rescale_o(it, jump, fmaxf(m_used, tmax1 * sl2))) { ok = false; break; }
          const float f = jump ? ex2_approx(m_old - m_used) : 1.f;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            ls[j] = make_float2(ls[j].x * f, ls[j].y * f);
            lh[j] = make_float2(0.f, 0.f);
          }
          tmem_wait_st();
          exp_half(64 * e + 32, sv, m_used, lh);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) ls[j] = add2(ls[j], lh[j]);
      } else {
        const float tmax1 = half_max(sv);
        tmax = fmaxf(tmax, tmax1);
        const bool adopt = m_used == -INFINITY;
        const bool jump = !adopt && tmax1 * sl2 > m_used + 64.f;
        if (adopt) m_used = tmax1 * sl2;
        if (__any_sync(0xffffffffu, jump)) {
          const float m_old = m_used;
          const bool oe_ok = mbar_wait(&oe_done[slot], (uint32_t)it & 1u, p.err, abort_flag);
          if (!__all_sync(0xffffffffu, oe_ok)) { ok = false; break; }
          if (!rescale_o(it, jump, fmaxf(m_used, tmax1 * sl2))) { ok = false; break; }
          const float f = jump ? ex2_approx(m_old - m_used) : 1.f;
#pragma unroll
          for (int j = 0; j < 4; ++j) ls[j] = make_float2(ls[j].x * f, ls[j].y * f);
        }
        exp_half(64 * e + 32, sv, m_used == -INFINITY ? 0.f : m_used, ls);
      }
      }
      {
        const float2 a2 = add2(add2(ls[0], ls[1]), add2(ls[2], ls[3]));
        l += a2.x + a2.y;
      }
      // a max that grew by more than 2^8 is adopted before the next tile
      if (tmax * sl2 > m_used + kRescaleThreshold) m_pend = tmax * sl2;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[slot]);
    }

    // split key walk: this CTA's part goes to the partials (fp32 O / l and
    // lse); an empty part contributes nothing (lse = -inf)
    const bool split = qwin && p.nsplit > 1 && !pair;
    const size_t prow = (((size_t)sp * p.B + b) * p.H + h) * (size_t)Mq + m_row;
    if (split && ok && n_tiles == 0 && row_valid && !warp_idle) {
      float4* dst = reinterpret_cast<float4*>(p.part_o + prow * D);
      for (int e = 0; e < D / 4; ++e) dst[e] = make_float4(0.f, 0.f, 0.f, 0.f);
      p.part_lse[prow] = -INFINITY;
    }
    bool fin = ok && n_tiles > 0 && !warp_idle;
    if (fin) fin = mbar_wait(&o_final[slot], 0, p.err, abort_flag);
    if (pair) {
      // The two parts of the key walk merge through distributed shared
      // memory.  Once both have finished their MMAs (each tells the other
      // on peer_free), each sends the other the half of its O columns that
      // the other writes, with its (m, l), and merges the half it keeps:
      // with M = max(m_0, m_1) and a_i = 2^(m_i - M), out = (a_0 O_0 + a_1
      // O_1) / (a_0 l_0 + a_1 l_1) (the split softmax's lse identity).
      constexpr int kHalf = D / 2;  // columns a part writes
      constexpr int kV4 = kHalf / 4;
      const uint32_t peer = (uint32_t)(sp ^ 1);
      const int rrow = slot * 128 + r;
      // receive area (the ring, free once this CTA's MMAs are done): row
      // rrow's kV4 float4, XOR-swizzled by the row against bank conflicts,
      // then (m, l) per row
      const uint32_t rx_o = smem_u32(smem + C::kRing) + (uint32_t)(rrow * kV4 * 16);
      const uint32_t rx_ml = smem_u32(smem + C::kRing) + (uint32_t)(C::kRxO + rrow * 8);
      // O in TMEM is complete (an empty part, or one that gave up, sends
      // zeros with m = -inf)
      const bool have = __all_sync(0xffffffffu, fin);
      const float m_me = have ? m_used : -INFINITY, l_me = have ? l : 0.f;
      __syncwarp();
      cluster_wait();  // the other part's barriers exist
      mbar_arrive_cluster(map_shared_rank(smem_u32(peer_free), peer));
      const bool go = __all_sync(0xffffffffu, mbar_wait<true>(peer_free, 0, p.err, abort_flag));
      if (go) {
        const uint32_t dst = map_shared_rank(rx_o, peer);
#pragma unroll
        for (int j = 0; j < kHalf / 32; ++j) {
          uint32_t v[32];
          if (have) {
            tmem_ld32(tO + (uint32_t)(peer * kHalf + 32 * j), v);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0u;
          }
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4)
            st_cluster_f4(dst + (uint32_t)(((j * 8 + e4) ^ (r & 7)) * 16),
                          __uint_as_float(v[4 * e4]), __uint_as_float(v[4 * e4 + 1]),
                          __uint_as_float(v[4 * e4 + 2]), __uint_as_float(v[4 * e4 + 3]));
        }
        st_cluster_f2(map_shared_rank(rx_ml, peer), m_me, l_me);
      }
      mbar_arrive_cluster(map_shared_rank(smem_u32(xfer), peer));
      // both parts' MMAs are done, so every read of this kv head's ring rows
      // is: the chunk enters the ring (keys from part 0, values from part 1)
      if (p.ring_store && go && (have || n_tiles == 0)) {
        const long long p0 = p.pos0[b];
        constexpr int kRv = D / 8;  // 16-byte vectors per row
        const int c_first = Mq > p.win ? Mq - p.win : 0;
        const uint4* src = sp == 0 ? p.kn_raw : p.vn_raw;
        uint4* dst = sp == 0 ? p.k_ring : p.v_ring;
        const int kv = kvh[0];
        if (p0 >= 0) {
          for (int t = (int)threadIdx.x - 128; t < (Mq - c_first) * kRv; t += 128 * NSLOT) {
            const int cc = c_first + t / kRv, i = t % kRv;
            const long long slot_r = (p0 + cc) % p.win;
            dst[(((long long)b * p.win + slot_r) * p.Hkv + kv) * kRv + i] =
                __ldg(src + (((long long)b * Mq + cc) * p.Hkv + kv) * kRv + i);
          }
        }
      }
      const bool got = __all_sync(0xffffffffu, mbar_wait<true>(xfer, 0, p.err, abort_flag));
      if (got) {
        const float2 mlp = ld_shared_f2(rx_ml);
        const float M = fmaxf(m_me, mlp.x);
        const float a_me = m_me == -INFINITY ? 0.f : ex2_approx(m_me - M);
        const float a_pe = mlp.x == -INFINITY ? 0.f : ex2_approx(mlp.x - M);
        const float L_ = a_me * l_me + a_pe * mlp.y;
        const float inv = L_ > 0.f ? 1.f / L_ : 0.f;
        const float c_me = a_me * inv, c_pe = a_pe * inv;
        uint16_t* orow = p.out + (((size_t)b * Mq + m_row) * p.H + h) * D + sp * kHalf;
#pragma unroll
        for (int j = 0; j < kHalf / 32; ++j) {
          uint32_t v[32];
          if (have) {
            tmem_ld32(tO + (uint32_t)(sp * kHalf + 32 * j), v);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0u;
          }
          uint32_t pk[16];
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 o = ld_shared_f4(rx_o + (uint32_t)(((j * 8 + e4) ^ (r & 7)) * 16));
            pk[2 * e4] = pack_bf16x2(__uint_as_float(v[4 * e4]) * c_me + o.x * c_pe,
                                     __uint_as_float(v[4 * e4 + 1]) * c_me + o.y * c_pe);
            pk[2 * e4 + 1] = pack_bf16x2(__uint_as_float(v[4 * e4 + 2]) * c_me + o.z * c_pe,
                                         __uint_as_float(v[4 * e4 + 3]) * c_me + o.w * c_pe);
          }
          if (row_valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * j);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
          }
        }
        if (row_valid && sp == 0 && p.lse)
          p.lse[((size_t)b * p.H + h) * Mq + m_row] = (M + __log2f(L_)) * 0.69314718055994531f;
      }
    } else if (__all_sync(0xffffffffu, fin)) {
      tc_fence_after();
      // (l == 0: a part of a split walk with none of the row's keys; its
      // lse is -inf and the merge skips it)
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const size_t orow_i = qwin ? (size_t)b * Mq + m_row : (size_t)b * p.N + i_phys;
      uint16_t* orow = p.out + (orow_i * p.H + h) * D;
      // rows start on 128-byte multiples from out: 32-byte stores when out
      // itself is 32-byte aligned
      const bool out_v8 = (reinterpret_cast<uintptr_t>(p.out) & 31u) == 0;
      // 64 columns of O per TMEM round trip (two loads, one wait)
#pragma unroll
      for (int j2 = 0; j2 < D / 64; ++j2) {
        uint32_t v[2][32];
        __syncwarp();
        tmem_ld32(tO + j2 * 64, v[0]);
        tmem_ld32(tO + j2 * 64 + 32, v[1]);
        tmem_wait_ld();
        if (split) {
          if (row_valid) {
            float4* dst = reinterpret_cast<float4*>(p.part_o + prow * D + j2 * 64);
#pragma unroll
            for (int e = 0; e < 16; ++e)
              dst[e] = make_float4(__uint_as_float(v[e >> 3][(e & 7) * 4]) * inv,
                                   __uint_as_float(v[e >> 3][(e & 7) * 4 + 1]) * inv,
                                   __uint_as_float(v[e >> 3][(e & 7) * 4 + 2]) * inv,
                                   __uint_as_float(v[e >> 3][(e & 7) * 4 + 3]) * inv);
          }
          continue;
        }
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(v[jj][2 * e]) * inv,
                                __uint_as_float(v[jj][2 * e + 1]) * inv);
          if (row_valid) {
            if (out_v8) {
              // two full 32-byte sectors per lane
              st_global_v8(orow + j2 * 64 + jj * 32, pk);
              st_global_v8(orow + j2 * 64 + jj * 32 + 16, pk + 8);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(orow + j2 * 64 + jj * 32);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
            }
          }
        }
      }
      const float lse_v = (m_used + __log2f(l)) * 0.69314718055994531f;
      if (row_valid && split)
        p.part_lse[prow] = lse_v;
      else if (row_valid && p.lse)
        p.lse[((size_t)b * p.H + h) * (qwin ? Mq : p.N) + (qwin ? m_row : i_phys)] = lse_v;
    }
  }

  // ---- teardown: make sure no MMA is in flight, then free TMEM.
  if (warp >= 1 && warp <= NSLOT && lane == 0 && n_tiles > 0 && slot_ok[warp - 1] &&
      *abort_flag) {
    // abort path: o_final was committed after the last MMA this issuer
    // issued; give it a bounded chance to land before TMEM is released.
    volatile int no_abort = 0;
    mbar_wait(&o_final[warp - 1], 0, nullptr, &no_abort, 100000000ull);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
  // paired parts: neither CTA exits while the other may still write its
  // shared memory (the softmax warps waited on the first cluster barrier
  // in their epilogue, the others do here)
  if (pair) {
    if (warp < 4) cluster_wait();
    cluster_arrive();
    cluster_wait();
  }
}

// Whether the device can place clusters of two CTAs of the query-window
// form (paired parts); asked once per form.
template <int D, int NSLOT, int NSTREAM>
bool pair_clusters_fit() {
  using C = Cfg<D, NSLOT, NSTREAM>;
  static std::atomic<int> known{0};  // 0 not asked, 1 yes, -1 no
  int k = known.load(std::memory_order_acquire);
  if (k == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kAlloc;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    const cudaError_t e = cudaOccupancyMaxActiveClusters(
        &n, reinterpret_cast<const void*>(swa_fwd_sm100_kernel<D, NSLOT, NSTREAM, 1>), &cfg);
    if (e != cudaSuccess) cudaGetLastError();
    k = (e == cudaSuccess && n > 0) ? 1 : -1;
    known.store(k, std::memory_order_release);
  }
  return k > 0;
}

template <int D, int NSLOT, int NSTREAM>
int launch_impl(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H,
                int Hkv, int N, int L, int R, int d, int bs, const int32_t* G, int ng,
                float scale, cudaStream_t stream, const QueryWindow* qw, int qt_lo, int qt_hi) {
  using C = Cfg<D, NSLOT, NSTREAM>;
  static std::atomic<unsigned long long> attr_kind[3] = {{0}, {0}, {0}};
  const int kind = qw ? 1 : (ng > 0 ? 2 : 0);
  const void* kfn[3] = {reinterpret_cast<const void*>(swa_fwd_sm100_kernel<D, NSLOT, NSTREAM, 0>),
                        reinterpret_cast<const void*>(swa_fwd_sm100_kernel<D, NSLOT, NSTREAM, 1>),
                        reinterpret_cast<const void*>(swa_fwd_sm100_kernel<D, NSLOT, NSTREAM, 2>)};
  if (!smem_attr_once(kfn[kind], C::kAlloc, attr_kind[kind])) return SWA_ERR_CUDA;
  if (NSLOT == 2 || C::kMinBlocks == 2) {
    // The register split (warpgroup 0: 56 per thread, each softmax
    // warpgroup: 208 with two slots, 200 with one) must fit in what the
    // block is launched with, or setmaxnreg.inc would never return: checked
    // once per kernel form.
    const long need = NSLOT == 2 ? 128L * 56 + 256L * 208 : 128L * 56 + 128L * 200;
    static std::atomic<int> regs_ok[3] = {{0}, {0}, {0}};
    if (regs_ok[kind].load(std::memory_order_acquire) == 0) {
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, kfn[kind]) != cudaSuccess) return SWA_ERR_CUDA;
      regs_ok[kind].store((long)fa.numRegs * C::kThreads >= need ? 1 : -1,
                          std::memory_order_release);
    }
    if (regs_ok[kind].load(std::memory_order_acquire) < 0) return SWA_ERR_UNSUPPORTED;
  }
  int* err = device_error_word();
  if (!err) return SWA_ERR_CUDA;
  const Geometry geo = make_geometry(N, L, R, d, bs);
  const bool block_mode = geo.bs > 1;
  for (int c0 = 0; c0 < geo.nclass; c0 += kMaxClasses) {
    FwdParams p;
    std::memset(&p, 0, sizeof(p));
    p.nclass = geo.nclass - c0 < kMaxClasses ? geo.nclass - c0 : kMaxClasses;
    p.class0 = c0;
    p.out = static_cast<uint16_t*>(out);
    p.lse = lse;
    p.G = G;
    p.q_raw = static_cast<const uint16_t*>(q);
    p.k_raw = static_cast<const uint16_t*>(k);
    p.v_raw = static_cast<const uint16_t*>(v);
    p.err = err;
    p.n_global = ng;
    p.B = B;
    p.H = H;
    p.Hkv = Hkv;
    p.N = N;
    p.L = L;
    p.R = R;
    p.d = d;
    p.bs = geo.bs;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.qtile_prefix[0] = 0;
    for (int cl = 0; cl < p.nclass; ++cl) {
      p.Mv[cl] = class_valid_rows(geo, c0 + cl);
      const int rows_q = qw ? qw->Mq : p.Mv[cl];
      p.qtile_prefix[cl + 1] = p.qtile_prefix[cl] + (rows_q + kTileM - 1) / kTileM;
    }
    if (qt_hi >= 0) {
      // a row-range launch (one class): only query tiles [qt_lo, qt_hi)
      if (geo.nclass != 1 || qw) return SWA_ERR_UNSUPPORTED;
      const int all = p.qtile_prefix[1];
      const int lo = qt_lo < 0 ? 0 : (qt_lo > all ? all : qt_lo);
      const int hi = qt_hi > all ? all : (qt_hi < lo ? lo : qt_hi);
      p.qt_base = lo;
      p.qtile_prefix[1] = hi - lo;
    }
    const bool inplace = qw && qw->kn;
    if (qw) {
      p.pos0 = qw->pos0;
      p.q0 = qw->q0;
      p.Mq = qw->Mq;
      p.win = qw->win;
      p.inplace = inplace ? 1 : 0;
      p.stack = (NSLOT == 2 && qw->stack) ? 1 : 0;
      p.nsplit = qw->nsplit > 1 ? qw->nsplit : 1;
      p.pair = (p.nsplit == 2 && qw->pair && pair_clusters_fit<D, NSLOT, NSTREAM>()) ? 1 : 0;
      if (p.nsplit > 1 && !p.pair) {
        if (!qw->part) return SWA_ERR_ARG;
        p.part_o = qw->part;
        p.part_lse = qw->part + (size_t)p.nsplit * B * H * qw->Mq * D;
      }
      // the chunk enters the rings inside the launch when each cluster holds
      // every reader of its kv head's ring rows: one query tile and all the
      // kv head's query heads in one item
      const int heads_per_item = p.stack ? 2 * NSLOT : NSLOT;
      if (p.pair && inplace && qw->ring_k && qw->ring_v && p.nclass == 1 &&
          p.qtile_prefix[1] == 1 && heads_per_item == H / Hkv) {
        p.ring_store = 1;
        p.k_ring = static_cast<uint4*>(qw->ring_k);
        p.v_ring = static_cast<uint4*>(qw->ring_v);
        p.kn_raw = static_cast<const uint4*>(qw->kn);
        p.vn_raw = static_cast<const uint4*>(qw->vn);
      }
      if (qw->done) *qw->done = p.pair | (p.ring_store << 1);
    }
    const uint32_t box[4] = {64, 1, (uint32_t)kBlockRows, 1};
    const int nmaps = block_mode ? 1 : p.nclass;
    for (int cl = 0; cl < nmaps; ++cl) {
      const int cc = c0 + cl;
      const uint64_t rows = block_mode ? (uint64_t)N : (uint64_t)class_rows(geo, cc);
      const uint64_t rstep = block_mode ? 1 : (uint64_t)d;
      const size_t qoff = block_mode ? 0 : (size_t)cc * H * D;
      const size_t kvoff = block_mode ? 0 : (size_t)cc * Hkv * D;
      const uint64_t qrows = qw ? (uint64_t)qw->Mq : rows;
      const uint64_t qN = qw ? (uint64_t)qw->Mq : (uint64_t)N;
      const uint64_t dq[4] = {(uint64_t)D, (uint64_t)H, qrows, (uint64_t)B};
      const uint64_t sq[3] = {(uint64_t)D * 2, rstep * H * D * 2, qN * H * D * 2};
      // in place: K / V are the rings, win rows per batch
      const uint64_t krows = inplace ? (uint64_t)qw->win : rows;
      const uint64_t kN = inplace ? (uint64_t)qw->win : (uint64_t)N;
      const uint64_t dk[4] = {(uint64_t)D, (uint64_t)Hkv, krows, (uint64_t)B};
      const uint64_t sk[3] = {(uint64_t)D * 2, rstep * Hkv * D * 2, kN * Hkv * D * 2};
      void* qb = (void*)(static_cast<const uint16_t*>(q) + qoff);
      void* kb = (void*)(static_cast<const uint16_t*>(k) + kvoff);
      void* vb = (void*)(static_cast<const uint16_t*>(v) + kvoff);
      if (encode_tiled(&p.tmQ[cl], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, qb, dq, sq, box,
                       CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
          encode_tiled(&p.tmK[cl], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, kb, dk, sk, box,
                       CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
          encode_tiled(&p.tmV[cl], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, vb, dk, sk, box,
                       CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return SWA_ERR_CUDA;
    }
    if (inplace) {
      // the chunk's keys and values, [B, Mq, Hkv, D]
      const uint64_t dn[4] = {(uint64_t)D, (uint64_t)Hkv, (uint64_t)qw->Mq, (uint64_t)B};
      const uint64_t sn[3] = {(uint64_t)D * 2, (uint64_t)Hkv * D * 2,
                              (uint64_t)qw->Mq * Hkv * D * 2};
      if (encode_tiled(&p.tmKf, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(qw->kn),
                       dn, sn, box, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
          encode_tiled(&p.tmVf, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(qw->vn),
                       dn, sn, box, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return SWA_ERR_CUDA;
    }
    // the global tiles ride with the first launch
    if (c0 == 0 && kind == 2) {
      p.n_gq_tiles = (ng + kTileM - 1) / kTileM;
      p.n_gitems = p.n_gq_tiles * B * ((H + NSLOT - 1) / NSLOT);
      const uint64_t df[4] = {(uint64_t)D, (uint64_t)Hkv, (uint64_t)N, (uint64_t)B};
      const uint64_t sf[3] = {(uint64_t)D * 2, (uint64_t)Hkv * D * 2,
                              (uint64_t)N * Hkv * D * 2};
      if (encode_tiled(&p.tmKf, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(k), df, sf,
                       box, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
          encode_tiled(&p.tmVf, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(v), df, sf,
                       box, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return SWA_ERR_CUDA;
    }
    const long heads_per_item = p.stack ? 2 * NSLOT : NSLOT;
    const long grid = (long)p.n_gitems + (long)p.qtile_prefix[p.nclass] * B *
                                             ((H + heads_per_item - 1) / heads_per_item) *
                                             (qw ? p.nsplit : 1);
    if (grid <= 0) continue;
    if (grid > 0x7fffffffL) return SWA_ERR_UNSUPPORTED;
    if (kind == 1 && p.pair) {
      // clusters of two: the two parts of an item are consecutive CTAs
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)grid);
      cfg.blockDim = dim3(C::kThreads);
      cfg.dynamicSmemBytes = C::kAlloc;
      cfg.stream = stream;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = 2;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      if (cudaLaunchKernelEx(&cfg, swa_fwd_sm100_kernel<D, NSLOT, NSTREAM, 1>, p) != cudaSuccess)
        return SWA_ERR_CUDA;
    } else if (kind == 1)
      swa_fwd_sm100_kernel<D, NSLOT, NSTREAM, 1><<<(unsigned)grid, C::kThreads, C::kAlloc,
                                                   stream>>>(p);
    else if (kind == 2)
      swa_fwd_sm100_kernel<D, NSLOT, NSTREAM, 2><<<(unsigned)grid, C::kThreads, C::kAlloc,
                                                   stream>>>(p);
    else
      swa_fwd_sm100_kernel<D, NSLOT, NSTREAM, 0><<<(unsigned)grid, C::kThreads, C::kAlloc,
                                                   stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return SWA_ERR_CUDA;
  }
  return SWA_OK;
}

}  // namespace

bool fwd_qwin_stacks(int H, int Hkv, int Mq) {
  const int grp = H / Hkv;
  return grp % 4 == 0 && Mq <= 64;  // two slots (even group), four heads per CTA
}

// Two query heads per CTA when they share a kv head (GQA group of even
// size); otherwise one head per CTA, two CTAs per SM at D = 64 (measured on
// the D = 64 MHA workloads against two heads with two K/V streams per CTA:
// Longformer 133 -> 125 us, token dilation 172 -> 155, block 169 -> 156).
int launch_fwd_sm100(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                     int H, int Hkv, int N, int D, int L, int R, int d, int bs, const int32_t* G,
                     int ng, float scale, cudaStream_t stream, const QueryWindow* qw, int qt_lo,
                     int qt_hi) {
  const bool gqa_pair = (H / Hkv) % 2 == 0;
  if (D == 128) {
    if (gqa_pair)
      return launch_impl<128, 2, 1>(q, k, v, out, lse, B, H, Hkv, N, L, R, d, bs, G, ng, scale,
                                    stream, qw, qt_lo, qt_hi);
    return launch_impl<128, 1, 1>(q, k, v, out, lse, B, H, Hkv, N, L, R, d, bs, G, ng, scale,
                                  stream, qw, qt_lo, qt_hi);
  }
  if (D == 64) {
    if (gqa_pair)
      return launch_impl<64, 2, 1>(q, k, v, out, lse, B, H, Hkv, N, L, R, d, bs, G, ng, scale,
                                   stream, qw, qt_lo, qt_hi);
    return launch_impl<64, 1, 1>(q, k, v, out, lse, B, H, Hkv, N, L, R, d, bs, G, ng, scale,
                                 stream, qw, qt_lo, qt_hi);
  }
  return SWA_ERR_UNSUPPORTED;
}

}  // namespace swa
