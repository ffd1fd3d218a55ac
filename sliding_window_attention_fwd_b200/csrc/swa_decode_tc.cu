// swa_decode_tc.cu -- single-token decode over a ring-buffer KV cache on the
// tensor cores (page "大模型窗口扩展技术" §3.1: position t lives in slot t %
// W; the new token attends the last W positions).
//
// A decode step is a matrix-vector product per (batch, kv head): the GQA
// group's query vectors against every valid ring slot.  With the keys on the
// MMA's M side it still fits the tensor core:
//   S^T [128 keys x 16]  = K_tile [128 x D] . Q^T [D x 16]     (tcgen05, SS)
//   O^T [D x 16]        += V_tile^T [D x 128] . P^T [128 x 16] (tcgen05, SS)
// where the 16 columns are the group's query vectors (up to 8) padded with
// zero rows of Q.  TMEM lane k of S^T is key k of the tile, so thread k of
// the softmax warpgroup owns that key's scores; lane d of O^T is dimension d.
// The key order does not matter to softmax, so the keys are walked in ring
// slot order (slots >= min(pos + 1, W) are empty and masked).  Over a paged
// cache the keys are the window's positions from a 64-aligned start, each
// 64-row box looked up in the block table.  A CTA takes a part of about
// 1024 keys of one (batch, kv head), streams its K and V tiles through a
// three-slot TMA ring (128-byte swizzle), and writes O / l and the lse of
// its part; a merge kernel combines the parts (lse identity).
//
// Warp roles (192 threads, two CTAs per SM): warp 0 TMA producer, warp 1
// MMA issuer (and TMEM owner), warps 2-5 softmax (their lane quadrants
// warp % 4 cover TMEM lanes 0-127).  Per key tile the softmax warpgroup
// finds each query's tile max (warp shuffles, then the four warps through
// shared memory and a named barrier), keeps a running max that it adopts
// lazily (when it grows by more than 2^8; O^T is then rescaled), and
// writes P^T (bf16) to shared memory as the B operand of the PV MMA.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "swa_internal.h"
#include "swa_ptx.cuh"

namespace swa {
namespace {

constexpr int kTK = 128;        // keys per tile (MMA M)
constexpr int kPart = 1024;     // key indices per CTA, about
constexpr int kNQ = 8;          // query vectors of a GQA group, at most
constexpr int kN = 16;          // MMA N: the group padded with zero rows
constexpr int kRingSlots = 3;   // TMA ring (each slot one K or one V tile)
constexpr int kDecChunk = kTK * 128;  // one 64-column slice of a 128-row tile (bytes)
constexpr float kLazy = 8.0f;   // log2 units

struct DecParams {
  // rings [B, W, Hkv, D] (dims {D, Hkv, W, B}), or the page pools
  // [num_pages * page_size, Hkv, D] (batch dimension 1); 64 x 64 boxes
  CUtensorMap tmK, tmV;
  const uint16_t* q;     // [B, H, D]
  const int64_t* pos;    // [B]
  // paged cache: logical page lp of sequence b is physical page
  // table[b * max_pages + lp] (page_size a multiple of 64)
  const int32_t* table;
  int paged, page_size, max_pages;
  float* part_o;         // [nsplit, B, H, D]: O / l of each part
  float* part_lse;       // [nsplit, B, H]: ln-sum-exp of each part (-inf: empty)
  int* err;
  int B, H, Hkv, W, grp, nsplit;
  int part_keys;  // key indices per CTA (a multiple of 128)
  float scale_log2;
};

// D = 128 (the head size of the ring-decode workload).
struct DecCfg {
  static constexpr int D = 128;
  static constexpr int kTile = kTK * D * 2;       // 32 KB: one K or V tile
  static constexpr int kQ = 0;                    // Q: 16 rows x D, two 2 KB slices
  static constexpr int kQBytes = kN * D * 2;      // 4 KB
  static constexpr int kP = kQ + kQBytes;         // P^T: 16 rows x 128 keys, two 2 KB slices
  static constexpr int kPBytes = kN * kTK * 2;    // 4 KB, two buffers
  static constexpr int kRing = kP + 2 * kPBytes;  // 12 KB (1024-aligned)
  static constexpr int kBar = kRing + kRingSlots * kTile;
  // full[S], empty[S], s_full[2], p_full[2], o_done[2], o_final
  static constexpr int kNumBars = 2 * kRingSlots + 7;
  static constexpr int kRed = kBar + kNumBars * 8;  // per-warp partial max / sum: 4 x kNQ floats
  static constexpr int kMisc = kRed + 4 * kNQ * 4;
  static constexpr int kTotal = kMisc + 16;
  static constexpr int kAlloc = kTotal + 1024;  // slack for 1024-byte alignment
  static constexpr int kThreads = 192;
  static constexpr uint32_t kTmemCols = 64;  // S^T x 2 (16 columns each), O^T (16)
  static_assert(kRing % 1024 == 0, "ring alignment");
  static_assert(2 * (kAlloc + 1024) <= 233472, "two CTAs per SM");
};

// byte offset of element (row, col) in a 128-byte-swizzled K-major operand
// of 16 rows, 64 columns per 2 KB slice
__device__ __forceinline__ uint32_t sw128_off16(int row, int col) {
  const int slice = col >> 6, c = col & 63;
  return (uint32_t)(slice * 2048 + row * 128 + ((((c >> 3) ^ (row & 7)) & 7) << 4) + ((c & 7) << 1));
}

__global__ void __launch_bounds__(DecCfg::kThreads, 2)
    swa_decode_tc_kernel(const __grid_constant__ DecParams p) {
  using C = DecCfg;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBar);
  uint64_t* full = bars;                  // [slot]
  uint64_t* empty = full + kRingSlots;    // [slot]
  uint64_t* s_full = empty + kRingSlots;  // [t & 1]: S^T of tile t ready
  uint64_t* p_full = s_full + 2;          // [t & 1]: P^T of tile t written
  uint64_t* o_done = p_full + 2;          // [t & 1]: PV of tile t done
  uint64_t* o_final = o_done + 2;         // every MMA done
  float* red = reinterpret_cast<float*>(smem + C::kRed);  // [warp][query]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMisc + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  // work item: (part, kv head, batch), parts fastest
  int x = blockIdx.x;
  const int part = x % p.nsplit;
  x /= p.nsplit;
  const int g = x % p.Hkv;
  const int b = x / p.Hkv;
  const long long pb = p.pos[b];
  // key index space of the CTA's part: ring slots [0, min(pos + 1, W)), or,
  // paged, positions a64 + idx for idx in [0, pos - a64] from the window's
  // first position a rounded down to 64 (so no 64-row box crosses a page),
  // the positions below a masked
  long long a64 = 0;
  int lo_idx = 0, n_idx;
  if (p.paged) {
    const long long a = pb - p.W + 1 > 0 ? pb - p.W + 1 : 0;
    a64 = a & ~63LL;
    lo_idx = (int)(a - a64);
    n_idx = (int)(pb - a64 + 1);
  } else {
    n_idx = pb + 1 < (long long)p.W ? (int)(pb + 1) : p.W;  // filled slots
  }
  const int s0 = part * p.part_keys;
  const int s1 = min(s0 + p.part_keys, n_idx);
  const int ntiles = s1 > s0 ? (s1 - s0 + kTK - 1) / kTK : 0;
  const int nq = p.grp;

  // load j of the walk: K of tile j / 2 (j even) or its V (j odd), into
  // ring slot j % 3 (one thread)
  auto load_j = [&](int j) {
    const int st = j % kRingSlots;
    const int kv = j & 1, t = j >> 1;
#ifdef SWA_TEST_WITHHOLD_TILE
    // failure-detection test build only: this K tile is never loaded, so
    // the issuer's bounded wait for it runs out
    if (kv == 0 && t == SWA_TEST_WITHHOLD_TILE) return;
#endif
    const CUtensorMap* m = kv ? &p.tmV : &p.tmK;
    uint8_t* dst = smem + C::kRing + st * C::kTile;
    mbar_arrive_expect_tx(&full[st], C::kTile);
    for (int hh = 0; hh < 2; ++hh) {
      // source row of the 64 keys from index idx0: a ring slot, or a row of
      // the page pool (a page id past the table reads as zeros, masked
      // below)
      const int idx0 = s0 + t * kTK + hh * 64;
      int row = idx0, bc = b;
      if (p.paged) {
        const long long t0 = a64 + idx0;
        const long long lp = t0 / p.page_size;
        const long long page = lp < p.max_pages ? p.table[(long)b * p.max_pages + lp] : -1;
        row = page < 0 ? -64 : (int)(page * p.page_size + t0 % p.page_size);
        bc = 0;
      }
      for (int cc = 0; cc < D / 64; ++cc)
        tma_load_4d(dst + cc * kDecChunk + hh * (kDecChunk / 2), m, &full[st], cc * 64, g, row,
                    bc);
    }
  };
  // the first ring pass is issued by thread 0 as soon as the barriers
  // exist, so its latency overlaps TMEM allocation and the Q gather
  const int n_early = min(kRingSlots, 2 * ntiles);

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kRingSlots; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(o_final, 1);
    fence_mbar_init();
    if (ntiles > 0) {
      prefetch_tensormap(&p.tmK);
      prefetch_tensormap(&p.tmV);
      for (int j = 0; j < n_early; ++j) load_j(j);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp >= 2) {
    // Q of the group as 16 K-major rows (zeros past the group), and both
    // P^T buffers zeroed (their rows past the group stay zero)
    const int t = threadIdx.x - 64;  // 0..127
    for (int i = t; i < kN * D / 8; i += 128) {
      const int row = i / (D / 8), c8 = i % (D / 8);
      uint4 val = make_uint4(0u, 0u, 0u, 0u);
      if (row < nq)
        val = __ldg(reinterpret_cast<const uint4*>(
            p.q + ((size_t)b * p.H + (size_t)g * p.grp + row) * D + c8 * 8));
      *reinterpret_cast<uint4*>(smem + C::kQ + sw128_off16(row, c8 * 8)) = val;
    }
    for (int i = t; i < 2 * C::kPBytes / 16; i += 128)
      *reinterpret_cast<uint4*>(smem + C::kP + i * 16) = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t ring_addr = smem_u32(smem + C::kRing);

  if (warp == 0) {
    // =========================== producer ===========================
    // the rest of the walk (the first ring pass is already issued)
    int last = n_early - 1;
    if (lane == 0 && ntiles > 0) {
      for (int j = n_early; j < 2 * ntiles; ++j) {
        const int st = j % kRingSlots;
        if (j >= kRingSlots &&
            !mbar_wait(&empty[st], (uint32_t)((j / kRingSlots) - 1) & 1u, p.err, abort_flag))
          break;
        last = j;
        load_j(j);
      }
#ifdef SWA_TEST_WITHHOLD_TILE
      const int skip = 2 * SWA_TEST_WITHHOLD_TILE;
#else
      const int skip = -1;
#endif
      if (*abort_flag) drain_copies(full, kRingSlots, 0, last, skip);
    }
  } else if (warp == 1) {
    // =========================== MMA issuer ===========================
    // order: S(0), then per tile t: S(t + 1), PV(t).  S(t + 1) reuses the S^T
    // buffer of tile t - 1, whose P^T the issuer has already waited for.
    if (lane == 0 && ntiles > 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kTK, kN, 0, 0);  // K-major A (K), K-major B (Q)
      const uint32_t idesc_o = idesc_bf16_f32(D, kN, 1, 0);    // MN-major A (V^T), K-major B (P^T)
      const uint64_t dq = sdesc_sw128(smem_u32(smem + C::kQ), 16, 1024);
      const uint64_t dp0 = sdesc_sw128(smem_u32(smem + C::kP), 16, 1024);
      const uint64_t dring_k = sdesc_sw128(ring_addr, 16, 1024);
      const uint64_t dring_v = sdesc_sw128(ring_addr, kDecChunk, 1024);
      constexpr uint64_t kSlotStep = C::kTile >> 4;
      bool ok = true;
      auto issue_s = [&](int t) -> bool {
        const int j = 2 * t, st = j % kRingSlots;
        if (!mbar_wait(&full[st], (uint32_t)(j / kRingSlots) & 1u, p.err, abort_flag)) return false;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t ka = (uint64_t)(((k / 4) * kDecChunk + (k % 4) * 32) >> 4);
          const uint64_t kb = (uint64_t)(((k / 4) * 2048 + (k % 4) * 32) >> 4);
          mma_ss(tmem + 16u * (t & 1), dring_k + st * kSlotStep + ka, dq + kb, idesc_s,
                 k > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[t & 1]);
        tc_commit(&empty[st]);
        return true;
      };
      ok = issue_s(0);
      for (int t = 0; ok && t < ntiles; ++t) {
        if (t + 1 < ntiles && !issue_s(t + 1)) break;
        const int j = 2 * t + 1, st = j % kRingSlots;
        if (!mbar_wait(&p_full[t & 1], (uint32_t)(t >> 1) & 1u, p.err, abort_flag) ||
            !mbar_wait(&full[st], (uint32_t)(j / kRingSlots) & 1u, p.err, abort_flag))
          break;
        tc_fence_after();
        const uint64_t dp = dp0 + (uint64_t)((t & 1) * C::kPBytes >> 4);
#pragma unroll
        for (int k = 0; k < kTK / 16; ++k) {
          const uint64_t ka = (uint64_t)((k * 2048) >> 4);  // 16 keys of the V tile
          const uint64_t kb = (uint64_t)(((k / 4) * 2048 + (k % 4) * 32) >> 4);
          mma_ss(tmem + 32u, dring_v + st * kSlotStep + ka, dp + kb, idesc_o,
                 (t > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(&o_done[t & 1]);
        tc_commit(&empty[st]);
      }
      tc_commit(o_final);
    }
    __syncwarp();
  } else {
    // ============================ softmax ============================
    const int quad = warp & 3;          // TMEM lane quadrant
    const int r = quad * 32 + lane;     // key of the tile (S^T) / dimension (O^T)
    const int wi = warp - 2;            // index among the four softmax warps
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const float sl2 = p.scale_log2;
    float m_run[kNQ], lsum[kNQ];
#pragma unroll
    for (int n = 0; n < kNQ; ++n) {
      m_run[n] = -INFINITY;
      lsum[n] = 0.f;
    }
    bool ok = true;
    for (int t = 0; t < ntiles; ++t) {
      bool w_ok = mbar_wait(&s_full[t & 1], (uint32_t)(t >> 1) & 1u, p.err, abort_flag);
      tc_fence_after();
      uint32_t sv[16];
      tmem_ld16(tmem + 16u * (t & 1) + lane_off, sv);
      tmem_wait_ld();
      const int idx = s0 + t * kTK + r;
      const bool valid = idx < s1 && idx >= lo_idx;
      float xs[kNQ];
#pragma unroll
      for (int n = 0; n < kNQ; ++n) xs[n] = valid ? __uint_as_float(sv[n]) * sl2 : -INFINITY;
      // tile max per query: the warp, then the four warps
#pragma unroll
      for (int n = 0; n < kNQ; ++n) {
        float v = xs[n];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) red[wi * kNQ + n] = v;
      }
      // every softmax thread passes this barrier on every tile (a failed
      // wait above only leaves garbage scores); the barrier also ANDs the
      // threads' verdicts, so all four warps leave the loop on the same tile
      // and meet at the same named barriers after it
      ok = bar_red_and(1, 128, ok && w_ok && !*abort_flag);
      float m_tile[kNQ];
#pragma unroll
      for (int n = 0; n < kNQ; ++n)
        m_tile[n] = fmaxf(fmaxf(red[n], red[kNQ + n]), fmaxf(red[2 * kNQ + n], red[3 * kNQ + n]));
      asm volatile("bar.sync 1, 128;" ::: "memory");  // red is rewritten next tile
      if (!ok) break;
      // adopt a tile max that exceeds the running max by more than 2^8 (or
      // a first one): P stays <= 2^8 otherwise
      bool grow = false;
      float f[kNQ];
#pragma unroll
      for (int n = 0; n < kNQ; ++n) {
        f[n] = 1.f;
        if (m_tile[n] > m_run[n] + kLazy) {
          f[n] = m_run[n] == -INFINITY ? 0.f : ex2_approx(m_run[n] - m_tile[n]);
          m_run[n] = m_tile[n];
          lsum[n] *= f[n];
          grow = true;
        }
      }
      if (grow && t > 0) {
        // O^T holds P V of tiles < t: rescale its columns once PV(t - 1) is done
        if (!mbar_wait(&o_done[(t - 1) & 1], (uint32_t)((t - 1) >> 1) & 1u, p.err, abort_flag))
          ok = false;
        tc_fence_after();
        uint32_t ov[16];
        tmem_ld16(tmem + 32u + lane_off, ov);
        tmem_wait_ld();
#pragma unroll
        for (int n = 0; n < kNQ; ++n) ov[n] = __float_as_uint(__uint_as_float(ov[n]) * f[n]);
        tmem_st16(tmem + 32u + lane_off, ov);
        tmem_wait_st();
      }
      float pr[kNQ];
#pragma unroll
      for (int n = 0; n < kNQ; ++n) {
        pr[n] = ex2_approx(xs[n] - (m_run[n] == -INFINITY ? 0.f : m_run[n]));
        lsum[n] += pr[n];
      }
      // P^T buffer t & 1 was last read by PV(t - 2)
      if (t >= 2 &&
          !mbar_wait(&o_done[t & 1], (uint32_t)((t - 2) >> 1) & 1u, p.err, abort_flag))
        ok = false;
      uint8_t* pbuf = smem + C::kP + (t & 1) * C::kPBytes;
#pragma unroll
      for (int n = 0; n < kNQ; ++n) {
        const __nv_bfloat16 hv = __float2bfloat16_rn(pr[n]);
        *reinterpret_cast<__nv_bfloat16*>(pbuf + sw128_off16(n, r)) = hv;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[t & 1]);
    }
    // ---- the part's result: l per query over the 128 threads, then O / l
    float l_tot[kNQ];
#pragma unroll
    for (int n = 0; n < kNQ; ++n) {
      float v = lsum[n];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) red[wi * kNQ + n] = v;
    }
    ok = bar_red_and(1, 128, ok);
#pragma unroll
    for (int n = 0; n < kNQ; ++n)
      l_tot[n] = red[n] + red[kNQ + n] + red[2 * kNQ + n] + red[3 * kNQ + n];
    const size_t rowbase = ((size_t)part * p.B + b) * p.H + (size_t)g * p.grp;  // query 0
    if (ntiles == 0) {
      // an empty part (slots past the filled ones): contributes nothing
      if (r < nq) p.part_lse[rowbase + r] = -INFINITY;
    } else if (__all_sync(0xffffffffu, ok && mbar_wait(o_final, 0, p.err, abort_flag))) {
      tc_fence_after();
      uint32_t ov[16];
      tmem_ld16(tmem + 32u + lane_off, ov);
      tmem_wait_ld();
      for (int n = 0; n < nq; ++n) {
        p.part_o[(rowbase + n) * D + r] = __uint_as_float(ov[n]) / l_tot[n];
        if (r == 0) p.part_lse[rowbase + n] = (m_run[n] + __log2f(l_tot[n])) * 0.69314718055994531f;
      }
    }
  }

  // ---- teardown: no MMA in flight, then free TMEM
  if (warp == 1 && lane == 0 && ntiles > 0 && *abort_flag) {
    volatile int no_abort = 0;
    mbar_wait(o_final, 0, nullptr, &no_abort, 100000000ull);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace

namespace {
int launch_tc(DecParams& p, const void* q, void* out, float* lse, const int64_t* pos, int B,
              int H, int Hkv, int D, int W, int span, float scale, cudaStream_t stream) {
  static std::atomic<unsigned long long> attr{0};
  if (!smem_attr_once(reinterpret_cast<const void*>(swa_decode_tc_kernel), DecCfg::kAlloc, attr))
    return SWA_ERR_CUDA;
  // about kPart keys per CTA: as many parts as W needs, the span (W, or
  // W + 63 from a 64-aligned start) shared evenly in whole 128-key tiles
  p.nsplit = (W + kPart - 1) / kPart;
  p.part_keys = ((span + p.nsplit - 1) / p.nsplit + kTK - 1) / kTK * kTK;
  const size_t rows = (size_t)B * H;
  float* part = nullptr;
  if (!split_workspace(1, (size_t)p.nsplit * rows * (D + 1) * sizeof(float), stream, &part))
    return SWA_ERR_NOMEM;
  p.q = static_cast<const uint16_t*>(q);
  p.pos = pos;
  p.part_o = part;
  p.part_lse = part + (size_t)p.nsplit * rows * D;
  p.err = device_error_word();
  if (!p.err) return SWA_ERR_CUDA;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.W = W;
  p.grp = H / Hkv;
  p.scale_log2 = scale * 1.4426950408889634f;
  const long long grid = (long long)B * Hkv * p.nsplit;
  if (grid > 0x7fffffffLL) return SWA_ERR_UNSUPPORTED;
  swa_decode_tc_kernel<<<(unsigned)grid, DecCfg::kThreads, DecCfg::kAlloc, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return SWA_ERR_CUDA;
  return split_merge(part, out, lse, p.nsplit, B, 1, H, D, stream);
}
}  // namespace

int launch_decode_tc(const void* q, const void* k_ring, const void* v_ring, void* out, float* lse,
                     const int64_t* pos, int B, int H, int Hkv, int D, int W, float scale,
                     cudaStream_t stream) {
  const int grp = H / Hkv;
  if (D != 128 || grp > kNQ || grp < 1) return SWA_ERR_UNSUPPORTED;
  DecParams p;
  std::memset(&p, 0, sizeof(p));
  if (encode_kv_map(&p.tmK, k_ring, D, Hkv, W, B) != SWA_OK ||
      encode_kv_map(&p.tmV, v_ring, D, Hkv, W, B) != SWA_OK)
    return SWA_ERR_CUDA;
  return launch_tc(p, q, out, lse, pos, B, H, Hkv, D, W, W, scale, stream);
}

int launch_decode_paged_tc(const void* q, const void* k_pages, const void* v_pages, void* out,
                           float* lse, const int32_t* table, const int64_t* pos, int B, int H,
                           int Hkv, int D, int page_size, int num_pages, int max_pages, int W,
                           float scale, cudaStream_t stream) {
  const int grp = H / Hkv;
  if (D != 128 || grp > kNQ || grp < 1 || page_size % 64 != 0) return SWA_ERR_UNSUPPORTED;
  const long long pool_rows = (long long)num_pages * page_size;
  if (pool_rows > 0x7fffffffLL || (long long)W + 64 > 0x7fffffffLL) return SWA_ERR_UNSUPPORTED;
  DecParams p;
  std::memset(&p, 0, sizeof(p));
  if (encode_kv_map(&p.tmK, k_pages, D, Hkv, (int)pool_rows, 1) != SWA_OK ||
      encode_kv_map(&p.tmV, v_pages, D, Hkv, (int)pool_rows, 1) != SWA_OK)
    return SWA_ERR_CUDA;
  p.paged = 1;
  p.table = table;
  p.page_size = page_size;
  p.max_pages = max_pages;
  // the window's positions from a 64-aligned start: at most W + 63 indices
  return launch_tc(p, q, out, lse, pos, B, H, Hkv, D, W, W + 63, scale, stream);
}

}  // namespace swa
