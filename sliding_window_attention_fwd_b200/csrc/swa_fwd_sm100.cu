// swa_fwd_sm100.cu -- fused bf16 sliding-window attention forward for B200.
//
// One CTA computes one 128-row query tile of one (batch, head, residue
// class).  Only the key tiles the band-aware scheduler lists are visited
// (page "别再只加Mask了", §1: out-of-window pairs are skipped, not masked;
// "空洞滑窗机制" §四: dilation is handled on dense tiles of whole blocks),
// plus, when global tokens exist, tiles of gathered global keys
// (aiqz.cc page, "全局注意力token").
//
// Warp roles (256 threads):
//   warp 0     producer: TMA loads of Q once and K/V tiles into a
//              3-stage shared-memory ring (128-byte swizzle), or a gather of
//              global-key rows with plain loads for global tiles;
//   warp 1     TMEM owner and MMA issuer (one thread):
//                S_j  = Q K_j^T      tcgen05.mma, both operands in smem,
//                                    fp32 accumulator in TMEM (two buffers);
//                O   += P_j V_j      tcgen05.mma, P read from TMEM (bf16,
//                                    aliasing S_j), V from smem;
//   warps 4-7  softmax: thread t owns query row t of the tile, so the row
//              max / row sum are thread-local (no shuffles).  Scores are
//              masked only on tiles the scheduler marks as edge tiles.
//              The running max is rescaled lazily: O is corrected only when
//              the max grows by more than 2^8, otherwise the stale max is
//              kept (the final O / l is exact either way).
//   warps 2-3  idle after set-up.
// Per row: out = O / l (bf16), lse = ln l + m (fp32).
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
constexpr int kThreads = 256;
constexpr int kChunkBytes = kTileM * 128;  // one 64-column slice of a 128-row tile
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr uint32_t kTmemCols = 512;

struct FwdParams {
  CUtensorMap tmQ[kMaxClasses];
  CUtensorMap tmK[kMaxClasses];
  CUtensorMap tmV[kMaxClasses];
  uint16_t* out;
  float* lse;
  const int32_t* G;
  const uint16_t* k_raw;
  const uint16_t* v_raw;
  int* err;
  int n_global;
  int B, H, Hkv, N;
  int L, R, d, bs;
  int class0, nclass;
  int qtile_prefix[kMaxClasses + 1];
  int Mv[kMaxClasses];
  float scale_log2;
};

template <int D>
struct Smem {
  // K/V ring depth; also sized so that exactly one CTA fits on an SM (each
  // CTA owns all 512 TMEM columns).
  static constexpr int kStages = D == 64 ? 4 : 3;
  static constexpr int kTileBytes = D / 64 * kChunkBytes;  // 128 x D bf16
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kBar = kV + kStages * kTileBytes;
  // barriers: full_q, full_k[S], empty_k[S], full_v[S], empty_v[S],
  //           s_full[2], p_full[2], o_done, o_final
  static constexpr int kNumBars = 1 + 4 * kStages + 2 + 2 + 2;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kTotal = kMisc + 16;
  static constexpr int kAlloc = kTotal + 1024;  // slack for 1024-byte alignment
};

__device__ __forceinline__ bool in_band_phys(int L, int R, int d, int bs, int i, int j) {
  long diff, lo, hi;
  if (bs > 1) {
    diff = (long)(j / bs) - (long)(i / bs);
    lo = -(long)(L / bs) * d;
    hi = (long)(R / bs) * d;
  } else {
    diff = (long)j - (long)i;
    lo = -(long)L * d;
    hi = (long)R * d;
  }
  if (diff % d != 0) return false;
  if (L >= 0 && diff < lo) return false;
  if (R >= 0 && diff > hi) return false;
  return true;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) swa_fwd_sm100_kernel(const __grid_constant__ FwdParams p) {
  using S = Smem<D>;
  constexpr int kStages = S::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint64_t* full_q = bars;
  uint64_t* full_k = bars + 1;
  uint64_t* empty_k = full_k + kStages;
  uint64_t* full_v = empty_k + kStages;
  uint64_t* empty_v = full_v + kStages;
  uint64_t* s_full = empty_v + kStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* o_final = o_done + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + S::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kMisc + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  // ---- work item: (class, q tile, batch, head); heavy (late) tiles first.
  int x = blockIdx.x;
  const int h = x % p.H;
  x /= p.H;
  const int b = x % p.B;
  x /= p.B;
  const int jt = p.qtile_prefix[p.nclass] - 1 - x;
  int cl = 0;
  while (cl + 1 < p.nclass && p.qtile_prefix[cl + 1] <= jt) ++cl;
  const int qt = jt - p.qtile_prefix[cl];
  const int c = p.class0 + cl;
  const int hkv = h / (p.H / p.Hkv);
  const Geometry g = make_geometry(p.N, p.L, p.R, p.d, p.bs);
  const int Mv = p.Mv[cl];
  const TileRange tr = tile_range(g, Mv, qt);
  const int n_band = tr.kv_end - tr.kv_begin;
  const int n_gtiles = (p.n_global + kTileN - 1) / kTileN;
  const int n_tiles = n_band + n_gtiles;
  const bool block_mode = p.bs > 1;
  const int map_idx = block_mode ? 0 : cl;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(full_q, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_k[s], 1);
      mbar_init(&empty_k[s], 1);
      mbar_init(&full_v[s], 1);
      mbar_init(&empty_v[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
    }
    mbar_init(o_done, 1);
    mbar_init(o_final, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // TMEM columns: S/P buffers at [0,128) and [128,256), O at [256, 256+D)
  auto tS = [&](int it) -> uint32_t { return tmem + (uint32_t)(it & 1) * 128u; };
  const uint32_t tO = tmem + 256;

  const uint32_t q_addr = smem_u32(smem + S::kQ);
  const uint32_t k_addr = smem_u32(smem + S::kK);
  const uint32_t v_addr = smem_u32(smem + S::kV);

  // virtual row -> TMA row coordinate of a 64-row box
  auto box_row = [&](int vrow) -> int {
    return block_mode ? (c + p.d * (vrow / kBlockRows)) * kBlockRows : vrow;
  };

  if (warp == 0) {
    // =========================== producer ===========================
    if (lane == 0) {
      prefetch_tensormap(&p.tmQ[map_idx]);
      prefetch_tensormap(&p.tmK[map_idx]);
      prefetch_tensormap(&p.tmV[map_idx]);
      mbar_arrive_expect_tx(full_q, S::kTileBytes);
      for (int cc = 0; cc < D / 64; ++cc)
        for (int hh = 0; hh < 2; ++hh)
          tma_load_4d(smem + S::kQ + cc * kChunkBytes + hh * (kChunkBytes / 2), &p.tmQ[map_idx],
                      full_q, cc * 64, h, box_row(qt * kTileM + hh * 64), b);
    }
    for (int it = 0; it < n_tiles; ++it) {
      const int st = it % kStages;
      const uint32_t ph = (uint32_t)(it / kStages) & 1u;
      for (int kv = 0; kv < 2; ++kv) {  // 0: K, 1: V
        uint64_t* emp = kv ? &empty_v[st] : &empty_k[st];
        uint64_t* ful = kv ? &full_v[st] : &full_k[st];
        uint8_t* dst = smem + (kv ? S::kV : S::kK) + st * S::kTileBytes;
        if (it >= kStages && !mbar_wait(emp, ph ^ 1u, p.err, abort_flag)) goto producer_done;
        if (it < n_band) {
          if (lane == 0) {
            const CUtensorMap* m = kv ? &p.tmV[map_idx] : &p.tmK[map_idx];
            const int t = tr.kv_begin + it;
            mbar_arrive_expect_tx(ful, S::kTileBytes);
            for (int cc = 0; cc < D / 64; ++cc)
              for (int hh = 0; hh < 2; ++hh)
                tma_load_4d(dst + cc * kChunkBytes + hh * (kChunkBytes / 2), m, ful, cc * 64,
                            hkv, box_row(t * kTileN + hh * 64), b);
          }
        } else {
          // gather global-key rows with plain 16-byte loads into the
          // swizzled layout the MMA expects
          const int g0 = (it - n_band) * kTileN;
          const int cnt = min(kTileN, p.n_global - g0);
          const uint16_t* src_base = kv ? p.v_raw : p.k_raw;
          constexpr int kC16 = D / 8;  // 16-byte chunks per row
          for (int idx = lane; idx < kTileN * kC16; idx += 32) {
            const int row = idx / kC16, c16 = idx % kC16;
            uint4 val = make_uint4(0u, 0u, 0u, 0u);
            if (row < cnt) {
              int gv = __ldg(p.G + g0 + row);
              gv = gv < 0 ? 0 : (gv >= p.N ? p.N - 1 : gv);
              const uint16_t* src =
                  src_base + (((size_t)b * p.N + gv) * p.Hkv + hkv) * D + c16 * 8;
              val = __ldg(reinterpret_cast<const uint4*>(src));
            }
            uint8_t* d8 = dst + (c16 / 8) * kChunkBytes + row * 128 + (((c16 % 8) ^ (row % 8)) * 16);
            *reinterpret_cast<uint4*>(d8) = val;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(ful);
        }
      }
    }
  producer_done:;
  } else if (warp == 1) {
    // ============================ MMA issuer ============================
    if (lane == 0 && n_tiles > 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(kTileM, kTileN, 0, 0);
      const uint32_t idesc_pv = idesc_bf16_f32(kTileM, D, 0, 1);
      bool ok = mbar_wait(full_q, 0, p.err, abort_flag);
      tc_fence_after();
      auto issue_qk = [&](int it) -> bool {
        const int st = it % kStages;
        if (!mbar_wait(&full_k[st], (uint32_t)(it / kStages) & 1u, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint32_t kb = k_addr + st * S::kTileBytes;
#pragma unroll
        for (int s = 0; s < D / 16; ++s) {
          const uint32_t off = (s / 4) * kChunkBytes + (s % 4) * 32;
          mma_ss(tS(it), sdesc_sw128(q_addr + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024),
                 idesc_qk, s > 0 ? 1u : 0u);
        }
        tc_commit(&empty_k[st]);
        tc_commit(&s_full[it & 1]);
        return true;
      };
      if (ok) ok = issue_qk(0);
      for (int it = 0; ok && it < n_tiles; ++it) {
        if (it + 1 < n_tiles && !issue_qk(it + 1)) break;
        if (!mbar_wait(&p_full[it & 1], (uint32_t)(it >> 1) & 1u, p.err, abort_flag)) break;
        tc_fence_after();
        const int st = it % kStages;
        if (!mbar_wait(&full_v[st], (uint32_t)(it / kStages) & 1u, p.err, abort_flag)) break;
        tc_fence_after();
        const uint32_t vb = v_addr + st * S::kTileBytes;
#pragma unroll
        for (int s = 0; s < kTileN / 16; ++s) {
          mma_ts(tO, tS(it) + s * 8, sdesc_sw128(vb + s * 2048, kChunkBytes, 1024), idesc_pv,
                 (it > 0 || s > 0) ? 1u : 0u);
        }
        tc_commit(&empty_v[st]);
        tc_commit(o_done);
      }
      // o_final completes once every MMA issued above has finished (also on
      // the abort path, so TMEM is quiescent before it is freed).
      tc_commit(o_final);
    }
  } else if (warp >= 4) {
    // ============================ softmax ============================
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const int m_row = qt * kTileM + r;
    const bool row_valid = m_row < Mv;
    const int klo = key_lo(g, m_row);
    const int khi = key_hi(g, m_row, Mv);
    const int64_t i_phys = phys_row(g, c, m_row);
    const bool causal = p.R == 0;
    const float sl2 = p.scale_log2;
    float m_used = -INFINITY;  // running max, scaled log2 units
    float l = 0.f;
    bool ok = true;

    for (int it = 0; it < n_tiles; ++it) {
      const bool w_ok = mbar_wait(&s_full[it & 1], (uint32_t)(it >> 1) & 1u, p.err, abort_flag);
      if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
      tc_fence_after();
      float s[kTileN];
#pragma unroll
      for (int j = 0; j < kTileN / 32; ++j) {
        uint32_t v[32];
        tmem_ld32(tS(it) + lane_off + j * 32, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) s[j * 32 + e] = __uint_as_float(v[e]);
      }
      tmem_wait_ld();

      if (it < n_band) {
        const int t = tr.kv_begin + it;
        if (!tile_interior(g, Mv, qt, t)) {
          const int n0 = t * kTileN;
#pragma unroll
          for (int j = 0; j < kTileN; ++j) {
            const int n = n0 + j;
            if (n < klo || n > khi || n >= Mv) s[j] = -INFINITY;
          }
        }
      } else {
        const int g0 = (it - n_band) * kTileN;
#pragma unroll
        for (int j = 0; j < kTileN; ++j) {
          bool keep = false;
          if (g0 + j < p.n_global) {
            int gv = __ldg(p.G + g0 + j);
            gv = gv < 0 ? 0 : (gv >= p.N ? p.N - 1 : gv);
            keep = !in_band_phys(p.L, p.R, p.d, p.bs, (int)i_phys, gv) &&
                   (!causal || gv <= i_phys);
          }
          if (!keep) s[j] = -INFINITY;
        }
      }

      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < kTileN; ++j) mx = fmaxf(mx, s[j]);
      const float m_new = fmaxf(m_used, mx * sl2);
      const bool rescale = m_new > m_used + kRescaleThreshold;
      if (it > 0 && __any_sync(0xffffffffu, rescale)) {
        // O holds P_0..P_{it-1} V; wait until the last of those MMAs is done.
        const bool o_ok = mbar_wait(o_done, (uint32_t)(it - 1) & 1u, p.err, abort_flag);
        if (!__all_sync(0xffffffffu, o_ok)) { ok = false; break; }
        tc_fence_after();
        const float f = rescale ? ex2_approx(m_used - m_new) : 1.f;
        l *= f;
#pragma unroll
        for (int j = 0; j < D / 32; ++j) {
          uint32_t v[32];
          tmem_ld32(tO + lane_off + j * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * f);
          tmem_st32(tO + lane_off + j * 32, v);
        }
        tmem_wait_st();
      }
      if (rescale) m_used = m_new;
      const float m_safe = m_used == -INFINITY ? 0.f : m_used;

      float lsum = 0.f;
#pragma unroll
      for (int j = 0; j < kTileN / 32; ++j) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = ex2_approx(fmaf(s[j * 32 + 2 * e], sl2, -m_safe));
          const float p1 = ex2_approx(fmaf(s[j * 32 + 2 * e + 1], sl2, -m_safe));
          lsum += p0 + p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS(it) + lane_off + j * 16, pk);
      }
      l += lsum;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[it & 1]);
    }

    bool fin = ok && n_tiles > 0;
    if (fin) fin = mbar_wait(o_final, 0, p.err, abort_flag);
    if (__all_sync(0xffffffffu, fin)) {
      tc_fence_after();
      const float inv = 1.f / l;
      uint16_t* orow = p.out + (((size_t)b * p.N + i_phys) * p.H + h) * D;
#pragma unroll
      for (int j = 0; j < D / 32; ++j) {
        uint32_t v[32];
        __syncwarp();
        tmem_ld32(tO + lane_off + j * 32, v);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * inv, __uint_as_float(v[2 * e + 1]) * inv);
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + j * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      if (row_valid && p.lse)
        p.lse[((size_t)b * p.H + h) * p.N + i_phys] = (m_used + __log2f(l)) * 0.69314718055994531f;
    }
  }

  // ---- teardown: make sure no MMA is in flight, then free TMEM.
  if (warp == 1 && lane == 0 && n_tiles > 0 && *abort_flag) {
    // abort path: o_final was committed after the last issued MMA; give it
    // a bounded chance to land before TMEM is released.
    volatile int no_abort = 0;
    mbar_wait(o_final, 0, nullptr, &no_abort, 100000000ull);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
int launch_impl(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H,
                int Hkv, int N, int L, int R, int d, int bs, const int32_t* G, int ng,
                float scale, cudaStream_t stream) {
  using S = Smem<D>;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(swa_fwd_sm100_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             S::kAlloc) != cudaSuccess)
      return SWA_ERR_CUDA;
    attr_set = true;
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
      p.qtile_prefix[cl + 1] = p.qtile_prefix[cl] + (p.Mv[cl] + kTileM - 1) / kTileM;
    }
    const uint32_t box[4] = {64, 1, (uint32_t)kBlockRows, 1};
    const int nmaps = block_mode ? 1 : p.nclass;
    for (int cl = 0; cl < nmaps; ++cl) {
      const int cc = c0 + cl;
      const uint64_t rows = block_mode ? (uint64_t)N : (uint64_t)class_rows(geo, cc);
      const uint64_t rstep = block_mode ? 1 : (uint64_t)d;
      const size_t qoff = block_mode ? 0 : (size_t)cc * H * D;
      const size_t kvoff = block_mode ? 0 : (size_t)cc * Hkv * D;
      const uint64_t dq[4] = {(uint64_t)D, (uint64_t)H, rows, (uint64_t)B};
      const uint64_t sq[3] = {(uint64_t)D * 2, rstep * H * D * 2, (uint64_t)N * H * D * 2};
      const uint64_t dk[4] = {(uint64_t)D, (uint64_t)Hkv, rows, (uint64_t)B};
      const uint64_t sk[3] = {(uint64_t)D * 2, rstep * Hkv * D * 2, (uint64_t)N * Hkv * D * 2};
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
    const long grid = (long)p.qtile_prefix[p.nclass] * B * H;
    if (grid <= 0) continue;
    if (grid > 0x7fffffffL) return SWA_ERR_UNSUPPORTED;
    swa_fwd_sm100_kernel<D><<<(unsigned)grid, kThreads, S::kAlloc, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return SWA_ERR_CUDA;
  }
  return SWA_OK;
}

}  // namespace

int launch_fwd_sm100(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                     int H, int Hkv, int N, int D, int L, int R, int d, int bs, const int32_t* G,
                     int ng, float scale, cudaStream_t stream) {
  if (D == 128)
    return launch_impl<128>(q, k, v, out, lse, B, H, Hkv, N, L, R, d, bs, G, ng, scale, stream);
  if (D == 64)
    return launch_impl<64>(q, k, v, out, lse, B, H, Hkv, N, L, R, d, bs, G, ng, scale, stream);
  return SWA_ERR_UNSUPPORTED;
}

}  // namespace swa
