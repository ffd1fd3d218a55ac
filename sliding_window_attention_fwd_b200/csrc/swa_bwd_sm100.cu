// swa_bwd_sm100.cu -- sliding-window attention backward on the tcgen05
// tensor cores (bf16 operands, fp32 accumulators in TMEM).
//
// The pages train with the method but print no backward pass; this is the
// derivative of the forward definition over the same key sets (band with
// token- or block-level dilation, causal clip), with keys outside the
// window never touched.  With P_ij = exp(s_ij - lse_i) recomputed from the
// forward's lse and Delta_i = dO_i . out_i:
//   dP_ij = dO_i . v_j,   dS_ij = P_ij (dP_ij - Delta_i),
//   dQ_i = scale sum_j dS_ij k_j,   dK_j = scale sum_i dS_ij q_i,
//   dV_j = sum_i P_ij dO_i.
// Every product above is a dense contraction inside a 128 x 128 tile, so it
// runs on the tensor cores; the element-wise steps (exp, dS) run on the
// CUDA cores of four "compute" warps, one thread per TMEM lane.
//
// Two kernels, no atomics:
//  * swa_bwd_dq_kernel, query-stationary: a CTA owns 128 query rows of one
//    head (Q and dO tiles in shared memory) and walks the key tiles of the
//    band (the forward's scheduler):
//        S = Q K^T, dP = dO V^T      tcgen05.mma (smem x smem), TMEM fp32
//        dS (bf16) over S's columns  compute warps
//        dQ += dS K                  tcgen05.mma (TMEM x smem)
//    It also writes Delta_i for the second kernel.
//  * swa_bwd_dkdv_kernel, key-stationary: a CTA owns 128 key rows of one kv
//    head (K and V tiles in shared memory) and walks every (query tile,
//    query head of the GQA group) whose rows see those keys (the transposed
//    scheduler, query_lo / query_hi):
//        S^T = K Q^T, dP^T = V dO^T  tcgen05.mma (smem x smem)
//        P^T, dS^T (bf16) in place   compute warps (one key row per thread)
//        dV += P^T dO, dK += dS^T Q  tcgen05.mma (TMEM x smem)
//    dK and dV stay in TMEM for the CTA's whole walk.
// Warp roles: warp 0 TMA producer, warp 1 MMA issuer (and TMEM owner),
// warps 4.. compute (kGroupsB warpgroups).  Every wait is bounded
// (swa_ptx.cuh).
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

constexpr int kMaxClassesB = 8;                 // residue classes per launch
constexpr int kChunkB = kTileM * 128;           // 128 rows x 64 bf16 columns
constexpr float kLog2e = 1.4426950408889634f;
// Compute warpgroups: each takes 128 / kGroupsB of a step's 128 columns
// (a TMEM lane quadrant belongs to one warp of every group), so several
// warps per SM sub-partition hide each other's latencies.  Measured on the
// Mistral-shaped backward: 1 group 3.12 ms, 2 groups 2.26, 4 groups 2.05.
#ifndef SWA_BWD_GROUPS
#define SWA_BWD_GROUPS 4
#endif
constexpr int kGroupsB = SWA_BWD_GROUPS;
constexpr int kCpg = 4 / kGroupsB;  // 32-column chunks per group
constexpr int kThreadsB = 128 * (1 + kGroupsB);
static_assert(kGroupsB == 1 || kGroupsB == 2 || kGroupsB == 4, "1, 2 or 4 compute groups");

// TMEM column (relative to the operand block) of the bf16 pairs of K-step k
// (16 elements) of a P / dS operand written in place over fp32 scores: chunk
// ch of 32 scores (group g = ch / kCpg, its i-th chunk) is packed into the 16
// columns 32 kCpg g + 16 i, inside the group's own (already read) columns.
// dq kernel: TMEM column of step it's S buffer
__device__ __forceinline__ uint32_t sbuf(int it) { return (it & 1) ? 384u : 0u; }

__device__ __forceinline__ uint32_t pcol(int k) {
  const int ch = k / 2, g = ch / kCpg, i = ch % kCpg;
  return (uint32_t)(32 * kCpg * g + 16 * i + 8 * (k % 2));
}

struct BwdTcParams {
  CUtensorMap tmQ[kMaxClassesB];
  CUtensorMap tmDO[kMaxClassesB];
  CUtensorMap tmK[kMaxClassesB];
  CUtensorMap tmV[kMaxClassesB];
  const uint16_t* out;
  const uint16_t* dout;
  const float* lse;
  float* delta;  // [B, H, N] fp32: written by the dq kernel, read by the dkdv kernel
  uint16_t* dq;
  uint16_t* dk;
  uint16_t* dv;
  int* err;
  int B, H, Hkv, N, grp;
  int L, R, d, bs;
  int class0, nclass;
  int tile_prefix[kMaxClassesB + 1];  // 128-row tiles per class, prefix sums
  int Mv[kMaxClassesB];
  float scale, scale_log2;
};

template <int D>
struct BCfg {
  static constexpr int kTile = D / 64 * kChunkB;  // 128 rows x D bf16
  static constexpr int kStages = D == 128 ? 2 : 3;
  // two fixed tiles at offset 0 (dq: Q, dO; dkdv: K, V), then the stages of
  // two streamed tiles (dq: K, V; dkdv: Q, dO)
  static constexpr int kRing = 2 * kTile;
  static constexpr int kStageBytes = 2 * kTile;
  static constexpr int kVec = kRing + kStages * kStageBytes;  // dkdv: [stage][lse2 | delta][128]
  static constexpr int kBar = kVec + kStages * 2 * kTileM * 4;
  static constexpr int kNumBars = 1 + 2 * kStages + 2 * kStages + 5;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kAlloc = kMisc + 16 + 1024;  // slack for 1024-byte alignment
  static_assert(kAlloc <= 232448, "shared memory budget");
  static_assert(2 * kStages >= kGroupsB, "dq kernel: the Delta parts fit in the vector area");
  // TMEM columns: S (or S^T) [0, 128), dP (or dP^T) [128, 256), then the
  // accumulators: dq kernel dQ [256, 256 + D) and its second S buffer
  // [384, 512); dkdv kernel dV, dK.
  static constexpr uint32_t kTmemCols = 512;
};

__device__ __forceinline__ int box_row_of(const BwdTcParams& p, int c, int vrow) {
  return p.bs > 1 ? (c + p.d * (vrow / kBlockRows)) * kBlockRows + vrow % kBlockRows : vrow;
}

// Loads one 128-row tile (D columns) as 64-row x 64-column boxes into the
// swizzled layout the MMA descriptors expect.
template <int D>
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* m, uint64_t* bar,
                                          const BwdTcParams& p, int c, int head, int vrow0,
                                          int b) {
  for (int cc = 0; cc < D / 64; ++cc)
    for (int hh = 0; hh < 2; ++hh)
      tma_load_4d(dst + cc * kChunkB + hh * (kChunkB / 2), m, bar, cc * 64, head,
                  box_row_of(p, c, vrow0 + hh * 64), b);
}

// K-major operand tile descriptor offset of K-step k (16 columns).
__device__ __forceinline__ uint64_t kmajor_off(int k) {
  return (uint64_t)(((k / 4) * kChunkB + (k % 4) * 32) >> 4);
}

// 2^x for a pair: MUFU for one element, the FMA-pipe polynomial for the
// other when `poly` (one warp per sub-partition: the FMA pipe is idle).
__device__ __forceinline__ float2 exp2_pair(float2 x, bool poly) {
  if (poly) return exp2_poly2(x);
  return make_float2(ex2_approx(x.x), ex2_approx(x.y));
}

// ======================================================== dq kernel
template <int D>
__global__ void __launch_bounds__(kThreadsB, 1)
    swa_bwd_dq_kernel(const __grid_constant__ BwdTcParams p) {
  using C = BCfg<D>;
  constexpr int S_ = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBar);
  uint64_t* full_q = bars;              // Q and dO tiles
  uint64_t* full_k = bars + 1;          // [S_]
  uint64_t* full_v = full_k + S_;       // [S_]
  uint64_t* empty_k = full_v + S_;      // [S_]
  uint64_t* empty_v = empty_k + S_;     // [S_]
  uint64_t* s_full = empty_v + S_;      // [it & 1]: S of step it in its TMEM buffer
  uint64_t* dp_full = s_full + 2;       // dP of the step in TMEM
  uint64_t* ds_full = dp_full + 1;      // dS of the step written (128 arrivals)
  uint64_t* done = ds_full + 1;         // every MMA finished
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMisc + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // ---- work item: (class, query tile, batch, head); heavy (late) tiles first
  int x = blockIdx.x;
  const int h = x % p.H;
  x /= p.H;
  const int b = x % p.B;
  x /= p.B;
  const int jt = p.tile_prefix[p.nclass] - 1 - x;
  int cl = 0;
  while (cl + 1 < p.nclass && p.tile_prefix[cl + 1] <= jt) ++cl;
  const int qt = jt - p.tile_prefix[cl];
  const int c = p.class0 + cl;
  const int g_kv = h / p.grp;
  const Geometry geo = make_geometry(p.N, p.L, p.R, p.d, p.bs);
  const int Mv = p.Mv[cl];
  const TileRange tr = tile_range(geo, Mv, qt);
  const int n_tiles = tr.kv_end - tr.kv_begin;
  const int map_idx = p.bs > 1 ? 0 : cl;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(full_q, 1);
    for (int s = 0; s < S_; ++s) {
      mbar_init(&full_k[s], 1);
      mbar_init(&full_v[s], 1);
      mbar_init(&empty_k[s], 1);
      mbar_init(&empty_v[s], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, 128 * kGroupsB);
    mbar_init(done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t q_addr = smem_u32(smem);
  const uint32_t do_addr = q_addr + C::kTile;
  const uint32_t ring_addr = smem_u32(smem + C::kRing);

  if (warp == 0) {
    // ============================== producer ==============================
    if (lane == 0) {
      prefetch_tensormap(&p.tmQ[map_idx]);
      prefetch_tensormap(&p.tmDO[map_idx]);
      prefetch_tensormap(&p.tmK[map_idx]);
      prefetch_tensormap(&p.tmV[map_idx]);
      mbar_arrive_expect_tx(full_q, 2 * C::kTile);
      load_tile<D>(smem, &p.tmQ[map_idx], full_q, p, c, h, qt * kTileM, b);
      load_tile<D>(smem + C::kTile, &p.tmDO[map_idx], full_q, p, c, h, qt * kTileM, b);
      int last_k = -1, last_v = -1;
      for (int it = 0; it < n_tiles; ++it) {
        const int st = it % S_;
        const uint32_t ph = (uint32_t)(it / S_) & 1u;
        const int t = tr.kv_begin + it;
        uint8_t* kb = smem + C::kRing + st * C::kStageBytes;
        if (it >= S_ && !mbar_wait(&empty_k[st], ph ^ 1u, p.err, abort_flag)) break;
        mbar_arrive_expect_tx(&full_k[st], C::kTile);
        load_tile<D>(kb, &p.tmK[map_idx], &full_k[st], p, c, g_kv, t * kTileN, b);
        last_k = it;
        if (it >= S_ && !mbar_wait(&empty_v[st], ph ^ 1u, p.err, abort_flag)) break;
        mbar_arrive_expect_tx(&full_v[st], C::kTile);
        load_tile<D>(kb + C::kTile, &p.tmV[map_idx], &full_v[st], p, c, g_kv, t * kTileN, b);
        last_v = it;
      }
      if (*abort_flag) {  // leave no copy writing shared memory behind
        drain_copies(full_q, 1, 0, 0);
        drain_copies(full_k, S_, 0, last_k);
        drain_copies(full_v, S_, 0, last_v);
      }
    }
  } else if (warp == 1) {
    // ============================== MMA issuer ==============================
    if (lane == 0 && n_tiles > 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kTileM, kTileN, 0, 0);
      const uint32_t idesc_dq = idesc_bf16_f32(kTileM, D, 0, 1);
      const uint64_t dq_ = sdesc_sw128(q_addr, 16, 1024);
      const uint64_t ddo = sdesc_sw128(do_addr, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(ring_addr, 16, 1024);                // K, K-major
      const uint64_t dkmn0 = sdesc_sw128(ring_addr, kChunkB, 1024);         // K, MN-major
      const uint64_t dv0 = sdesc_sw128(ring_addr + C::kTile, 16, 1024);     // V, K-major
      constexpr uint64_t kStageStep = C::kStageBytes >> 4;
      // S of step it goes to TMEM buffer it & 1 ([0, 128) or [384, 512)), so
      // S(it + 1) is issued before dQ(it) reads dS(it) from the other one;
      // order: S(0), dP(0), then per step S(it + 1), dQ(it), dP(it + 1)
      auto issue_s = [&](int it) -> bool {
        const int st = it % S_;
        if (!mbar_wait(&full_k[st], (uint32_t)(it / S_) & 1u, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint64_t dk = dk0 + (uint64_t)st * kStageStep;
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_ss(tmem + sbuf(it), dq_ + kmajor_off(k), dk + kmajor_off(k), idesc_s,
                 k > 0 ? 1u : 0u);
        tc_commit(&s_full[it & 1]);
        return true;
      };
      auto issue_dp = [&](int it) -> bool {
        const int st = it % S_;
        if (!mbar_wait(&full_v[st], (uint32_t)(it / S_) & 1u, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint64_t dv = dv0 + (uint64_t)st * kStageStep;
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_ss(tmem + 128u, ddo + kmajor_off(k), dv + kmajor_off(k), idesc_s,
                 k > 0 ? 1u : 0u);
        tc_commit(dp_full);
        tc_commit(&empty_v[st]);
        return true;
      };
      bool ok = mbar_wait(full_q, 0, p.err, abort_flag) && issue_s(0) && issue_dp(0);
      for (int it = 0; ok && it < n_tiles; ++it) {
        const int st = it % S_;
        if (it + 1 < n_tiles && !issue_s(it + 1)) break;
        // dQ += dS K, dS (bf16) over S's columns; then dP of the next step
        // (the compute warps have read dP(it))
        if (!mbar_wait(ds_full, (uint32_t)it & 1u, p.err, abort_flag)) break;
        tc_fence_after();
        const uint64_t dkmn = dkmn0 + (uint64_t)st * kStageStep;
#pragma unroll
        for (int k = 0; k < kTileN / 16; ++k)
          mma_ts(tmem + 256u, tmem + sbuf(it) + pcol(k), dkmn + (uint64_t)((k * 2048) >> 4),
                 idesc_dq, (it > 0 || k > 0) ? 1u : 0u);
        tc_commit(&empty_k[st]);
        if (it + 1 < n_tiles && !issue_dp(it + 1)) break;
      }
      tc_commit(done);  // also on the abort path: TMEM quiescent before it is freed
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ============================== compute ==============================
    // group cg takes the keys [32 kCpg cg, 32 kCpg (cg + 1)) of every step
    const int cg = (warp - 4) / 4;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tP = tmem + 128u + lane_off;
    const uint32_t tQ = tmem + 256u + lane_off;
    const int m_v = qt * kTileM + r;
    const bool row_valid = m_v < Mv;
    const int i_phys = (int)phys_row(geo, c, m_v);
    const int klo = key_lo(geo, m_v);
    const int khi = key_hi(geo, m_v, Mv);
    int int_lo, int_hi;
    interior_tiles(geo, Mv, qt, &int_lo, &int_hi);
    const float sl2 = p.scale_log2;
    // Delta_i = dO_i . out_i (each group sums a quarter of the row, the
    // parts meet in shared memory) and lse in log2 units; rows past the
    // class end get P = 0
    float delta = 0.f, lse2 = INFINITY;
    {
      float* part = reinterpret_cast<float*>(smem + C::kVec);  // [group][128]
      float acc0 = 0.f, acc1 = 0.f;
      if (row_valid) {
        const size_t row = ((size_t)b * p.N + i_phys) * p.H + h;
        const uint4* a = reinterpret_cast<const uint4*>(p.dout + row * D);
        const uint4* o = reinterpret_cast<const uint4*>(p.out + row * D);
        constexpr int kU = D / 8 / kGroupsB;  // 16-byte chunks per group
#pragma unroll
        for (int u = cg * kU; u < (cg + 1) * kU; ++u) {
          const uint4 wa = __ldg(a + u), wo = __ldg(o + u);
          const uint32_t xa[4] = {wa.x, wa.y, wa.z, wa.w}, xo[4] = {wo.x, wo.y, wo.z, wo.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc0 = fmaf(__uint_as_float(xa[e] << 16), __uint_as_float(xo[e] << 16), acc0);
            acc1 = fmaf(__uint_as_float(xa[e] & 0xFFFF0000u),
                        __uint_as_float(xo[e] & 0xFFFF0000u), acc1);
          }
        }
      }
      part[cg * kTileM + r] = acc0 + acc1;
      asm volatile("bar.sync 1, %0;" ::"r"(kGroupsB * 128) : "memory");
#pragma unroll
      for (int g2 = 0; g2 < kGroupsB; ++g2) delta += part[g2 * kTileM + r];
      if (row_valid) {
        const size_t li = ((size_t)b * p.H + h) * p.N + i_phys;
        lse2 = __ldg(p.lse + li) * kLog2e;
        if (cg == 0) p.delta[li] = delta;
      }
    }
    bool ok = true;
    for (int it = 0; it < n_tiles; ++it) {
      const uint32_t ph = (uint32_t)it & 1u;
      const int t = tr.kv_begin + it;
      const bool edge = !(t >= int_lo && t <= int_hi);
      // P as soon as S is in TMEM (dP is still being computed)
      const uint32_t tS = tmem + sbuf(it) + lane_off;
      bool w = mbar_wait(&s_full[it & 1], (uint32_t)(it >> 1) & 1u, p.err, abort_flag);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float2 pr[kCpg][16];
#pragma unroll
      for (int i = 0; i < kCpg; ++i) {
        const int ch = cg * kCpg + i;
        uint32_t sv[32];
        tmem_ld32(tS + 32 * ch, sv);
        tmem_wait_ld();
        const int n0 = t * kTileN + 32 * ch;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float2 xs = fma2(make_float2(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])),
                           make_float2(sl2, sl2), make_float2(-lse2, -lse2));
          if (edge) {
            const int j0 = n0 + 2 * e;
            if (!(j0 >= klo && j0 <= khi && j0 < Mv)) xs.x = -INFINITY;
            if (!(j0 + 1 >= klo && j0 + 1 <= khi && j0 + 1 < Mv)) xs.y = -INFINITY;
          }
          pr[i][e] = exp2_pair(xs, (e & 1) != 0 && !edge);
        }
      }
      // then dS = P (dP - Delta)
      w = mbar_wait(dp_full, ph, p.err, abort_flag);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int i = 0; i < kCpg; ++i) {
        const int ch = cg * kCpg + i;
        uint32_t dpv[32];
        tmem_ld32(tP + 32 * ch, dpv);
        tmem_wait_ld();
        const float2 ndl = make_float2(-delta, -delta);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 ds = mul2(pr[i][e], add2(make_float2(__uint_as_float(dpv[2 * e]),
                                                            __uint_as_float(dpv[2 * e + 1])), ndl));
          pk[e] = pack_bf16x2(ds.x, ds.y);
        }
        // dS of these 32 keys over the group's own (already read) S columns
        tmem_st16(tS + 32 * kCpg * cg + 16 * i, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    bool fin = ok && n_tiles > 0 && mbar_wait(done, 0, p.err, abort_flag);
    if (__all_sync(0xffffffffu, fin)) {
      tc_fence_after();
      uint16_t* orow = p.dq + (((size_t)b * p.N + i_phys) * p.H + h) * D;
      // the groups share the row's D / 32 column chunks
#pragma unroll 1
      for (int j = cg; j < D / 32; j += kGroupsB) {
        uint32_t v[32];
        tmem_ld32(tQ + 32 * j, v);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * p.scale,
                              __uint_as_float(v[2 * e + 1]) * p.scale);
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + j * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
    } else if (row_valid && n_tiles == 0 && cg == 0) {
      // no key at all (cannot happen for a valid row: its own key is always
      // in the window), kept for completeness
      uint4* dst = reinterpret_cast<uint4*>(p.dq + (((size_t)b * p.N + i_phys) * p.H + h) * D);
      for (int e = 0; e < D / 8; ++e) dst[e] = make_uint4(0u, 0u, 0u, 0u);
    }
  }

  // ---- teardown: no MMA in flight, then free TMEM
  if (warp == 1 && lane == 0 && n_tiles > 0 && *abort_flag) {
    volatile int no_abort = 0;
    mbar_wait(done, 0, nullptr, &no_abort, 100000000ull);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ======================================================== dk / dv kernel
template <int D>
__global__ void __launch_bounds__(kThreadsB, 1)
    swa_bwd_dkdv_kernel(const __grid_constant__ BwdTcParams p) {
  using C = BCfg<D>;
  constexpr int S_ = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBar);
  uint64_t* full_kv = bars;           // K and V tiles
  uint64_t* full = bars + 1;          // [S_]: Q, dO tiles + lse / Delta vectors
  uint64_t* empty = full + S_;        // [S_]
  uint64_t* st_full = empty + S_;     // S^T of the step in TMEM
  uint64_t* dpt_full = st_full + 1;   // dP^T of the step in TMEM
  uint64_t* pt_full = dpt_full + 1;   // dS^T written (128 arrivals per group)
  uint64_t* done = pt_full + 1;
  uint64_t* p_full = done + 1;        // P^T written (128 arrivals per group)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMisc + 4);
  float* vec = reinterpret_cast<float*>(smem + C::kVec);  // [S_][2][128]

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // ---- work item: (class, key tile, batch, kv head); early (heavy) tiles first
  int x = blockIdx.x;
  const int g_kv = x % p.Hkv;
  x /= p.Hkv;
  const int b = x % p.B;
  x /= p.B;
  const int jt = x;
  int cl = 0;
  while (cl + 1 < p.nclass && p.tile_prefix[cl + 1] <= jt) ++cl;
  const int kt = jt - p.tile_prefix[cl];
  const int c = p.class0 + cl;
  const Geometry geo = make_geometry(p.N, p.L, p.R, p.d, p.bs);
  const int Mv = p.Mv[cl];
  const TileRange qr = qtile_range_keys(geo, Mv, kt * kTileN);
  const int grp = p.grp;
  const int n_steps = (qr.kv_end - qr.kv_begin) * grp;  // (query tile, head of the group)
  const int map_idx = p.bs > 1 ? 0 : cl;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(full_kv, 1);
    for (int s = 0; s < S_; ++s) {
      mbar_init(&full[s], 1 + 32);  // the TMA bytes + every producer lane's vectors
      mbar_init(&empty[s], 1);
    }
    mbar_init(st_full, 1);
    mbar_init(dpt_full, 1);
    mbar_init(pt_full, 128 * kGroupsB);
    mbar_init(done, 1);
    mbar_init(p_full, 128 * kGroupsB);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t k_addr = smem_u32(smem);
  const uint32_t v_addr = k_addr + C::kTile;
  const uint32_t ring_addr = smem_u32(smem + C::kRing);

  if (warp == 0) {
    // ============================== producer ==============================
    if (lane == 0) {
      prefetch_tensormap(&p.tmQ[map_idx]);
      prefetch_tensormap(&p.tmDO[map_idx]);
      prefetch_tensormap(&p.tmK[map_idx]);
      prefetch_tensormap(&p.tmV[map_idx]);
      mbar_arrive_expect_tx(full_kv, 2 * C::kTile);
      load_tile<D>(smem, &p.tmK[map_idx], full_kv, p, c, g_kv, kt * kTileN, b);
      load_tile<D>(smem + C::kTile, &p.tmV[map_idx], full_kv, p, c, g_kv, kt * kTileN, b);
    }
    int last = -1;
    for (int s = 0; s < n_steps; ++s) {
      const int st = s % S_;
      const uint32_t ph = (uint32_t)(s / S_) & 1u;
      const int qt = qr.kv_begin + s / grp;
      const int h = g_kv * grp + s % grp;
      // lse (log2 units) and Delta of the tile's 128 query rows, loaded into
      // registers before the wait for the stage so their latency overlaps it;
      // rows past the class end get lse = +inf (P = 0)
      float l2[kTileM / 32], dl[kTileM / 32];
#pragma unroll
      for (int u = 0; u < kTileM / 32; ++u) {
        const int m = qt * kTileM + lane + 32 * u;
        l2[u] = INFINITY;
        dl[u] = 0.f;
        if (m < Mv) {
          const size_t li = ((size_t)b * p.H + h) * p.N + phys_row(geo, c, m);
          l2[u] = __ldg(p.lse + li) * kLog2e;
          dl[u] = p.delta[li];
        }
      }
      if (s >= S_ && !mbar_wait(&empty[st], ph ^ 1u, p.err, abort_flag)) break;
      if (lane == 0) {
        uint8_t* qb = smem + C::kRing + st * C::kStageBytes;
        mbar_arrive_expect_tx(&full[st], 2 * C::kTile);
        load_tile<D>(qb, &p.tmQ[map_idx], &full[st], p, c, h, qt * kTileM, b);
        load_tile<D>(qb + C::kTile, &p.tmDO[map_idx], &full[st], p, c, h, qt * kTileM, b);
      }
      float* vl = vec + st * 2 * kTileM;
#pragma unroll
      for (int u = 0; u < kTileM / 32; ++u) {
        vl[lane + 32 * u] = l2[u];
        vl[kTileM + lane + 32 * u] = dl[u];
      }
      mbar_arrive(&full[st]);
      last = s;
    }
    if (lane == 0 && *abort_flag) {  // leave no copy writing shared memory behind
      drain_copies(full_kv, 1, 0, 0);
      drain_copies(full, S_, 0, last);
    }
  } else if (warp == 1) {
    // ============================== MMA issuer ==============================
    if (lane == 0 && n_steps > 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kTileN, kTileM, 0, 0);
      const uint32_t idesc_o = idesc_bf16_f32(kTileN, D, 0, 1);
      const uint64_t dk_ = sdesc_sw128(k_addr, 16, 1024);                 // K, K-major (A)
      const uint64_t dv_ = sdesc_sw128(v_addr, 16, 1024);                 // V, K-major (A)
      const uint64_t dq0 = sdesc_sw128(ring_addr, 16, 1024);              // Q, K-major (B)
      const uint64_t ddo0 = sdesc_sw128(ring_addr + C::kTile, 16, 1024);  // dO, K-major (B)
      const uint64_t dqmn0 = sdesc_sw128(ring_addr, kChunkB, 1024);       // Q, MN-major (B)
      const uint64_t ddomn0 = sdesc_sw128(ring_addr + C::kTile, kChunkB, 1024);
      constexpr uint64_t kStageStep = C::kStageBytes >> 4;
      const uint32_t t_dv = tmem + 256u, t_dk = tmem + 256u + (uint32_t)D;
      // order: S^T(0), dP^T(0), then per step dV(s) once P^T(s) is written,
      // S^T(s + 1), dK(s) once dS^T(s) is written, dP^T(s + 1): each of
      // S^T(s + 1) / dP^T(s + 1) right after the MMA that reads the columns
      // it overwrites (P^T(s) / dS^T(s)), so S^T(s + 1) is computed while the
      // compute warps form dS^T(s)
      auto issue_st = [&](int s) -> bool {
        const int st = s % S_;
        if (!mbar_wait(&full[st], (uint32_t)(s / S_) & 1u, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint64_t sq = (uint64_t)st * kStageStep;
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_ss(tmem, dk_ + kmajor_off(k), dq0 + sq + kmajor_off(k), idesc_s, k > 0 ? 1u : 0u);
        tc_commit(st_full);
        return true;
      };
      auto issue_dpt = [&](int s) {  // after issue_st(s): the stage is full
        const uint64_t sq = (uint64_t)(s % S_) * kStageStep;
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_ss(tmem + 128u, dv_ + kmajor_off(k), ddo0 + sq + kmajor_off(k), idesc_s,
                 k > 0 ? 1u : 0u);
        tc_commit(dpt_full);
      };
      bool ok = mbar_wait(full_kv, 0, p.err, abort_flag) && issue_st(0);
      if (ok) issue_dpt(0);
      for (int s = 0; ok && s < n_steps; ++s) {
        const int st = s % S_;
        const uint64_t sq = (uint64_t)st * kStageStep;
        // dV += P^T dO, dK += dS^T Q
        if (!mbar_wait(p_full, (uint32_t)s & 1u, p.err, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < kTileM / 16; ++k)
          mma_ts(t_dv, tmem + pcol(k), ddomn0 + sq + (uint64_t)((k * 2048) >> 4), idesc_o,
                 (s > 0 || k > 0) ? 1u : 0u);
        const bool next = s + 1 < n_steps;
        if (next && !issue_st(s + 1)) break;
        if (!mbar_wait(pt_full, (uint32_t)s & 1u, p.err, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < kTileM / 16; ++k)
          mma_ts(t_dk, tmem + 128u + pcol(k), dqmn0 + sq + (uint64_t)((k * 2048) >> 4), idesc_o,
                 (s > 0 || k > 0) ? 1u : 0u);
        tc_commit(&empty[st]);
        if (next) issue_dpt(s + 1);
      }
      tc_commit(done);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ============================== compute ==============================
    // group cg takes the query columns [32 kCpg cg, 32 kCpg (cg + 1))
    const int cg = (warp - 4) / 4;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off;
    const uint32_t tP = tmem + 128u + lane_off;
    const int j_v = kt * kTileN + r;  // this thread's key row (virtual)
    const bool key_valid = j_v < Mv;
    // query rows that see this key
    int qlo = query_lo(geo, j_v), qhi = query_hi(geo, j_v, Mv);
    qhi = qhi > Mv - 1 ? Mv - 1 : qhi;
    int int_lo, int_hi;
    interior_qtiles_keys(geo, Mv, kt * kTileN, &int_lo, &int_hi);
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int s = 0; s < n_steps; ++s) {
      const int st = s % S_;
      const int qt = qr.kv_begin + s / grp;
      const bool edge = !(qt >= int_lo && qt <= int_hi);
      // P^T as soon as S^T is in TMEM (dP^T is still being computed)
      bool w = mbar_wait(st_full, (uint32_t)s & 1u, p.err, abort_flag);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* vl = vec + st * 2 * kTileM;
      float2 pr[kCpg][16];
#pragma unroll
      for (int i = 0; i < kCpg; ++i) {
        const int ch = cg * kCpg + i;
        uint32_t sv[32];
        tmem_ld32(tS + 32 * ch, sv);
        tmem_wait_ld();
        const int i0 = qt * kTileM + 32 * ch;
        const float4* l4 = reinterpret_cast<const float4*>(vl + 32 * ch);
        uint32_t pp[16];
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) {
          const float4 l = l4[e2];  // lse2 of this pair of pairs
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int e = 2 * e2 + h2;
            const float2 lp = h2 ? make_float2(l.z, l.w) : make_float2(l.x, l.y);
            float2 xs = fma2(make_float2(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])),
                             make_float2(sl2, sl2), make_float2(-lp.x, -lp.y));
            if (edge) {
              if (!(i0 + 2 * e >= qlo && i0 + 2 * e <= qhi)) xs.x = -INFINITY;
              if (!(i0 + 2 * e + 1 >= qlo && i0 + 2 * e + 1 <= qhi)) xs.y = -INFINITY;
            }
            pr[i][e] = exp2_pair(xs, h2 != 0 && !edge);
            pp[e] = pack_bf16x2(pr[i][e].x, pr[i][e].y);
          }
        }
        // P^T of these 32 query columns over the group's own (already read)
        // columns of S^T
        tmem_st16(tS + 32 * kCpg * cg + 16 * i, pp);
      }
      // P^T is complete: dV(s), then S^T(s + 1), may go while dS^T is formed
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
      // then dS^T = P^T (dP^T - Delta)
      w = mbar_wait(dpt_full, (uint32_t)s & 1u, p.err, abort_flag);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int i = 0; i < kCpg; ++i) {
        const int ch = cg * kCpg + i;
        uint32_t dpv[32];
        tmem_ld32(tP + 32 * ch, dpv);
        tmem_wait_ld();
        const float4* d4 = reinterpret_cast<const float4*>(vl + kTileM + 32 * ch);
        uint32_t pd[16];
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) {
          const float4 dl = d4[e2];  // Delta of this pair of pairs
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int e = 2 * e2 + h2;
            const float2 dn = h2 ? make_float2(-dl.z, -dl.w) : make_float2(-dl.x, -dl.y);
            const float2 ds = mul2(pr[i][e], add2(make_float2(__uint_as_float(dpv[2 * e]),
                                                              __uint_as_float(dpv[2 * e + 1])), dn));
            pd[e] = pack_bf16x2(ds.x, ds.y);
          }
        }
        tmem_st16(tP + 32 * kCpg * cg + 16 * i, pd);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(pt_full);
    }
    bool fin = ok && n_steps > 0 && mbar_wait(done, 0, p.err, abort_flag);
    if (__all_sync(0xffffffffu, fin)) {
      tc_fence_after();
      const size_t row = ((size_t)b * p.N + phys_row(geo, c, j_v)) * p.Hkv + g_kv;
      // the groups share the 2 x D / 32 column chunks of dV and dK
#pragma unroll 1
      for (int u = cg; u < 2 * (D / 32); u += kGroupsB) {
        const int which = u / (D / 32), j = u % (D / 32);  // which 0: dV, 1: dK (scaled)
        uint16_t* orow = (which ? p.dk : p.dv) + row * D;
        const float f = which ? p.scale : 1.f;
        {
          uint32_t v[32];
          tmem_ld32(tmem + 256u + (uint32_t)(which * D) + lane_off + 32 * j, v);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * f, __uint_as_float(v[2 * e + 1]) * f);
          if (key_valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + j * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
          }
        }
      }
    } else if (key_valid && n_steps == 0 && cg == 0) {
      const size_t row = ((size_t)b * p.N + phys_row(geo, c, j_v)) * p.Hkv + g_kv;
      uint4* a = reinterpret_cast<uint4*>(p.dk + row * D);
      uint4* v = reinterpret_cast<uint4*>(p.dv + row * D);
      for (int e = 0; e < D / 8; ++e) a[e] = v[e] = make_uint4(0u, 0u, 0u, 0u);
    }
  }

  if (warp == 1 && lane == 0 && n_steps > 0 && *abort_flag) {
    volatile int no_abort = 0;
    mbar_wait(done, 0, nullptr, &no_abort, 100000000ull);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D>
int launch_bwd_tc_impl(const void* q, const void* k, const void* v, const void* out,
                       const void* dout, const float* lse, void* dq, void* dk, void* dv,
                       float* delta, int B, int H, int Hkv, int N, int L, int R, int d, int bs,
                       float scale, cudaStream_t stream) {
  using C = BCfg<D>;
  static std::atomic<unsigned long long> attr_dq{0}, attr_dkdv{0};
  if (!smem_attr_once(reinterpret_cast<const void*>(swa_bwd_dq_kernel<D>), C::kAlloc, attr_dq) ||
      !smem_attr_once(reinterpret_cast<const void*>(swa_bwd_dkdv_kernel<D>), C::kAlloc,
                      attr_dkdv))
    return SWA_ERR_CUDA;
  int* err = device_error_word();
  if (!err) return SWA_ERR_CUDA;
  const Geometry geo = make_geometry(N, L, R, d, bs);
  const bool block_mode = geo.bs > 1;
  // two passes over the class chunks: every Delta is written (dq kernel)
  // before any is read (dkdv kernel)
  for (int pass = 0; pass < 2; ++pass) {
    for (int c0 = 0; c0 < geo.nclass; c0 += kMaxClassesB) {
      BwdTcParams p;
      std::memset(&p, 0, sizeof(p));
      p.nclass = geo.nclass - c0 < kMaxClassesB ? geo.nclass - c0 : kMaxClassesB;
      p.class0 = c0;
      p.out = static_cast<const uint16_t*>(out);
      p.dout = static_cast<const uint16_t*>(dout);
      p.lse = lse;
      p.delta = delta;
      p.dq = static_cast<uint16_t*>(dq);
      p.dk = static_cast<uint16_t*>(dk);
      p.dv = static_cast<uint16_t*>(dv);
      p.err = err;
      p.B = B;
      p.H = H;
      p.Hkv = Hkv;
      p.N = N;
      p.grp = H / Hkv;
      p.L = L;
      p.R = R;
      p.d = d;
      p.bs = geo.bs;
      p.scale = scale;
      p.scale_log2 = scale * kLog2e;
      p.tile_prefix[0] = 0;
      for (int cl = 0; cl < p.nclass; ++cl) {
        p.Mv[cl] = class_valid_rows(geo, c0 + cl);
        p.tile_prefix[cl + 1] = p.tile_prefix[cl] + (p.Mv[cl] + kTileM - 1) / kTileM;
      }
      const uint32_t box[4] = {64, 1, (uint32_t)kBlockRows, 1};
      const int nmaps = block_mode ? 1 : p.nclass;
      for (int cl = 0; cl < nmaps; ++cl) {
        const int cc = c0 + cl;
        const uint64_t rows = block_mode ? (uint64_t)N : (uint64_t)class_rows(geo, cc);
        const uint64_t rstep = block_mode ? 1 : (uint64_t)d;
        const size_t qoff = block_mode ? 0 : (size_t)cc * H * D;
        const size_t kvoff = block_mode ? 0 : (size_t)cc * Hkv * D;
        const uint64_t dq_[4] = {(uint64_t)D, (uint64_t)H, rows, (uint64_t)B};
        const uint64_t sq[3] = {(uint64_t)D * 2, rstep * H * D * 2, (uint64_t)N * H * D * 2};
        const uint64_t dk_[4] = {(uint64_t)D, (uint64_t)Hkv, rows, (uint64_t)B};
        const uint64_t sk[3] = {(uint64_t)D * 2, rstep * Hkv * D * 2,
                                (uint64_t)N * Hkv * D * 2};
        void* qb = (void*)(static_cast<const uint16_t*>(q) + qoff);
        void* db = (void*)(static_cast<const uint16_t*>(dout) + qoff);
        void* kb = (void*)(static_cast<const uint16_t*>(k) + kvoff);
        void* vb = (void*)(static_cast<const uint16_t*>(v) + kvoff);
        if (encode_tiled(&p.tmQ[cl], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, qb, dq_, sq, box,
                         CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
            encode_tiled(&p.tmDO[cl], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, db, dq_, sq, box,
                         CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
            encode_tiled(&p.tmK[cl], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, kb, dk_, sk, box,
                         CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
            encode_tiled(&p.tmV[cl], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, vb, dk_, sk, box,
                         CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
          return SWA_ERR_CUDA;
      }
      const long ntiles = (long)p.tile_prefix[p.nclass];
      if (pass == 0) {
        const long grid = ntiles * B * H;
        if (grid <= 0) continue;
        if (grid > 0x7fffffffL) return SWA_ERR_UNSUPPORTED;
        swa_bwd_dq_kernel<D><<<(unsigned)grid, kThreadsB, C::kAlloc, stream>>>(p);
      } else {
        const long grid = ntiles * B * Hkv;
        if (grid <= 0) continue;
        if (grid > 0x7fffffffL) return SWA_ERR_UNSUPPORTED;
        swa_bwd_dkdv_kernel<D><<<(unsigned)grid, kThreadsB, C::kAlloc, stream>>>(p);
      }
      if (cudaGetLastError() != cudaSuccess) return SWA_ERR_CUDA;
    }
  }
  return SWA_OK;
}

}  // namespace

int launch_backward_tc(const void* q, const void* k, const void* v, const void* out,
                       const void* dout, const float* lse, void* dq, void* dk, void* dv,
                       float* delta, int B, int H, int Hkv, int N, int D, int L, int R, int d,
                       int bs, float scale, cudaStream_t stream) {
  if (D == 128)
    return launch_bwd_tc_impl<128>(q, k, v, out, dout, lse, dq, dk, dv, delta, B, H, Hkv, N, L,
                                   R, d, bs, scale, stream);
  if (D == 64)
    return launch_bwd_tc_impl<64>(q, k, v, out, dout, lse, dq, dk, dv, delta, B, H, Hkv, N, L, R,
                                  d, bs, scale, stream);
  return SWA_ERR_UNSUPPORTED;
}

}  // namespace swa
