// swa_rowattn.cu -- split-KV attention of a few query vectors against a long
// contiguous run of key rows, on CUDA cores.  Three users:
//
//  * ring-buffer decode: one new token per sequence attends the valid slots
//    of its W-slot cache (page "大模型窗口扩展技术" §3.1: token t lives in
//    slot t % W; aiqz.cc page, "推理优化策略": the cache rolls like a
//    conveyor belt, old entries are overwritten);
//  * paged decode: the cache lives in fixed-size pages found through a block
//    table, so pages that leave the window can be released ("空洞滑窗机制"
//    page, §四, KV cache management with PagedAttention);
//  * chunked append: C new tokens attend the ring history and the chunk
//    itself, each over its own window (aiqz.cc page, "推理优化策略":
//    streaming inference).
//
// The work is HBM-bound (each key/value byte is used for a handful of
// flops), so the kernel is built for bandwidth: one CTA streams a chunk of
// key rows of one (batch, kv head) through a 2-stage TMA ring (64 rows per
// stage, 128-byte swizzle so the reads below are bank-conflict free) and
// serves all NQ query vectors that read those rows (the GQA group of the kv
// head, and for an append several tokens) from that single read.
// Math is fp32 on the FMA pipe.  Chunks of one query set are merged with
// the log-sum-exp identity by whichever CTA of the set finishes last.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "swa_internal.h"
#include "swa_ptx.cuh"

namespace swa {
namespace {

constexpr int kRows = 64;           // key rows per stage
constexpr int kDecodeChunk = 1024;  // ring-decode keys per CTA: amortises set-up and merge
constexpr int kStagesR = 2;
constexpr int kComputeWarps = 4;
constexpr int kThreadsR = (kComputeWarps + 1) * 32;

struct RowParams {
  CUtensorMap tmK;   // decode: ring; paged: page pool; append: ring
  CUtensorMap tmV;
  CUtensorMap tmKn;  // chunked append: the chunk's new keys / values
  CUtensorMap tmVn;
  const int32_t* table;  // paged: block table [B, max_pages]
  int page_size, max_pages;
  const uint16_t* q;
  uint16_t* out;
  float* lse;
  const int64_t* pos;
  float* ws_o;
  float* ws_ml;
  int* cnt;
  int* err;
  int mode;  // 0: decode, 2: paged decode, 3: chunked append
  int B, H, Hkv, N, W, grp;
  int rows_per_cta, nrowchunks;
  int chunk, nsplit;
  float scale_log2;
};

template <int D, int NQ>
struct RSmem {
  static constexpr int kTile = kRows * D * 2;
  static constexpr int kStage = 2 * kTile;
  static constexpr int kSc = kStagesR * kStage;       // scores [row][slot]
  static constexpr int kPc = kSc + kRows * NQ * 4;    // probabilities [row][slot]
  static constexpr int kCorr = kPc + kRows * NQ * 4;  // per-slot rescale factor
  static constexpr int kBar = kCorr + 64;
  static constexpr int kMisc = kBar + 2 * kStagesR * 8;
  static constexpr int kTotal = kMisc + 16;
  static constexpr int kAlloc = kTotal + 1024;
  // epilogue reduction buffer [warp][slot][D] floats, reusing the ring
  static_assert(kComputeWarps * NQ * D * 4 <= kSc, "reduction buffer must fit in the ring");
  static_assert((kRows / 4) % kComputeWarps == 0, "row groups split evenly over the warps");
};

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float2 bf2(uint32_t w) { return make_float2(bf_lo(w), bf_hi(w)); }

// Sum of v[0..NQ) over the 8 lanes of a row group, transposed: at each of
// the three exchange levels a lane sends the half of its values it does not
// keep, so NQ values need NQ-1 shuffles (butterfly: 3 NQ).  Lane t ends up
// with the full sum of slot (t >> (3 - log2 NQ)) & (NQ - 1) (for NQ < 8 two
// or more neighbouring lanes hold the same slot).
template <int NQ>
__device__ __forceinline__ float reduce8_transposed(float (&v)[NQ], int t, int* slot_out) {
  float w[NQ];
#pragma unroll
  for (int i = 0; i < NQ; ++i) w[i] = v[i];
  int n = NQ, base = 0;
#pragma unroll
  for (int lvl = 4; lvl >= 1; lvl >>= 1) {
    if (n > 1) {
      const bool upper = (t & lvl) != 0;  // keep the upper half of the values
      const int h = n / 2;
#pragma unroll
      for (int i = 0; i < NQ / 2; ++i) {
        if (i < h) {
          const float send = upper ? w[i] : w[i + h];
          const float keep = upper ? w[i + h] : w[i];
          w[i] = keep + __shfl_xor_sync(0xffffffffu, send, lvl);
        }
      }
      base += upper ? h : 0;
      n = h;
    } else {
      w[0] += __shfl_xor_sync(0xffffffffu, w[0], lvl);
    }
  }
  *slot_out = base;
  return w[0];
}

// MODE: 0 ring decode, 2 paged decode, 3 chunked append
// (compile-time, so each user's kernel carries only its own addressing).
template <int D, int NQ, int MODE>
__global__ void __launch_bounds__(kThreadsR, (NQ <= 4 ? 3 : 1))
    swa_rowattn_kernel(const __grid_constant__ RowParams p) {
  using S = RSmem<D, NQ>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  float* sc = reinterpret_cast<float*>(smem + S::kSc);
  float* pc = reinterpret_cast<float*>(smem + S::kPc);
  float* corr_s = reinterpret_cast<float*>(smem + S::kCorr);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint64_t* empty = full + kStagesR;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kMisc);
  int* last_flag = reinterpret_cast<int*>(smem + S::kMisc + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int split = blockIdx.x;
  const int gi = blockIdx.y;  // query set

  // ---- the query set: kv head, batch, query vectors and their key sets.
  // Keys are walked by an index idx in [0, max_limit).  Key positions are
  // kept relative to tA (32-bit): rel(idx) = idx below seg_n, idx + off_b
  // from seg_n on (the chunk of an append); slot s sees the keys with
  // lo_r[s] <= rel <= hi_r[s] (and, below seg_n, rel < a_end_r).
  int b, g, rowchunk = 0;
  if (MODE == 0 || MODE == 2) {
    g = gi % p.Hkv;
    b = gi / p.Hkv;
  } else {
    rowchunk = gi % p.nrowchunks;
    g = (gi / p.nrowchunks) % p.Hkv;
    b = gi / (p.nrowchunks * p.Hkv);
  }
  long long tA = 0;
  int seg_n = 0x7fffffff, off_b = 0, a_end_r = 0x7fffffff;
  long qoff[NQ];
  int lo_r[NQ], hi_r[NQ];
  int max_limit = 0;
  if (MODE == 2) {
    const long long ps = p.pos[b];
    const long long start = ps - p.W + 1 < 0 ? 0 : ps - p.W + 1;
    tA = start & ~(long long)(kRows - 1);
    const long long lim = ps + 1 - tA;
    max_limit = lim < 0 ? 0 : (int)lim;
  } else if (MODE == 3) {
    const long long pos0 = p.pos[b];
    const long long r0 = (long long)rowchunk * p.rows_per_cta;
    const long long start = pos0 + r0 - p.W + 1 < 0 ? 0 : pos0 + r0 - p.W + 1;
    tA = start & ~(long long)(kRows - 1);
    const long long na = pos0 > tA ? ((pos0 - tA + kRows - 1) / kRows) * kRows : 0;
    seg_n = (int)na;
    a_end_r = (int)(pos0 - tA);
    off_b = (int)(pos0 - na - tA);
    const long long last = r0 + p.rows_per_cta < p.N ? r0 + p.rows_per_cta : p.N;
    max_limit = (int)(na + last);
  }
#pragma unroll
  for (int s = 0; s < NQ; ++s) {
    const int hsub = s % p.grp, rsub = s / p.grp;
    const int h = g * p.grp + hsub;
    qoff[s] = -1;
    lo_r[s] = 0;
    hi_r[s] = -1;
    if (rsub < p.rows_per_cta) {
      if (MODE == 0) {
        long long ps = p.pos[b];
        const int limit = ps + 1 < (long long)p.W ? (int)(ps + 1) : p.W;
        hi_r[s] = limit - 1;
        qoff[s] = ((long)b * p.H + h) * D;
        max_limit = limit > max_limit ? limit : max_limit;
      } else if (MODE == 2) {
        const long long ps = p.pos[b];
        lo_r[s] = (int)((ps - p.W + 1 < 0 ? 0 : ps - p.W + 1) - tA);
        hi_r[s] = (int)(ps - tA);
        qoff[s] = ((long)b * p.H + h) * D;
      } else {
        const int c = rowchunk * p.rows_per_cta + rsub;
        if (c < p.N) {
          const long long pc = p.pos[b] + c;
          lo_r[s] = (int)((pc - p.W + 1 < 0 ? 0 : pc - p.W + 1) - tA);
          hi_r[s] = (int)(pc - tA);
          qoff[s] = (((long)b * p.N + c) * p.H + h) * D;
        }
      }
    }
  }
  const int key0 = split * p.chunk;
  int nk = max_limit - key0;
  nk = nk < 0 ? 0 : (nk > p.chunk ? p.chunk : nk);
  const int n_stages = (nk + kRows - 1) / kRows;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kStagesR; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kComputeWarps * 32);
    }
    fence_mbar_init();
  }
  __syncthreads();

  // PV mapping: every warp handles whole value rows; lane owns EPL columns.
  constexpr int EPL = D / 32;
  // running stats of the slots this warp owns: warp + 4 u
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  float2 acc[NQ][EPL / 2];
#pragma unroll
  for (int s = 0; s < NQ; ++s)
#pragma unroll
    for (int e = 0; e < EPL / 2; ++e) acc[s][e] = make_float2(0.f, 0.f);

  if (warp == kComputeWarps) {
    // ============================ producer ============================
    if (lane == 0) {
      prefetch_tensormap(&p.tmK);
      prefetch_tensormap(&p.tmV);
      if (MODE == 3) {
        prefetch_tensormap(&p.tmKn);
        prefetch_tensormap(&p.tmVn);
      }
      int last = -1;  // last stage whose loads were issued
#ifdef SWA_TEST_WITHHOLD_TILE
      const int skip = SWA_TEST_WITHHOLD_TILE;
#else
      const int skip = -1;
#endif
      for (int k = 0; k < n_stages; ++k) {
        const int st = k % kStagesR;
        if (k >= kStagesR &&
            !mbar_wait(&empty[st], ((uint32_t)(k / kStagesR) & 1u) ^ 1u, p.err, abort_flag))
          break;
        last = k;
        // failure-detection test build only: these 64 rows are never loaded,
        // so the compute warps' bounded wait for them runs out
        if (k == skip) continue;
        uint8_t* kb = smem + st * S::kStage;
        uint8_t* vb = kb + S::kTile;
        // source of the 64 key rows [idx0, idx0 + 64): a row of the ring /
        // sequence, a page of the pool, or rows of the chunk.  Rows past a
        // tensor's end (or a page id past the pool) read as zeros and are
        // masked below.
        const int idx0 = key0 + k * kRows;
        const CUtensorMap* mk = &p.tmK;
        const CUtensorMap* mv = &p.tmV;
        int row = idx0, bc = b;
        if (MODE == 2) {
          const long long t0 = tA + idx0;
          const long long lp = t0 / p.page_size;
          const long long page = lp < p.max_pages ? p.table[(long)b * p.max_pages + lp] : -1;
          row = page < 0 ? -kRows : (int)(page * p.page_size + t0 % p.page_size);
          bc = 0;
        } else if (MODE == 3) {
          if (idx0 < seg_n) {
            row = (int)((tA + idx0) % p.W);
          } else {
            row = idx0 - seg_n;
            mk = &p.tmKn;
            mv = &p.tmVn;
          }
        }
        mbar_arrive_expect_tx(&full[st], S::kStage);
        for (int cc = 0; cc < D / 64; ++cc) {
          tma_load_4d(kb + cc * (kRows * 128), mk, &full[st], cc * 64, g, row, bc);
          tma_load_4d(vb + cc * (kRows * 128), mv, &full[st], cc * 64, g, row, bc);
        }
      }
      // leave no copy writing shared memory behind
      if (*abort_flag) drain_copies(full, kStagesR, 0, last, skip);
    }
  } else {
    // ============================ compute ============================
    // QK mapping: 8 lanes per key row, lane t reads 16-byte chunk t of each
    // 128-byte half of the row (conflict free under the swizzle); a warp
    // covers 4 rows per step, the 8 warps a 64-row stage in two steps.
    constexpr int kCPL = D / 64;
    const int t8 = lane & 7, rsub = lane >> 3;
    float2 qv[NQ][kCPL * 4];
#pragma unroll
    for (int s = 0; s < NQ; ++s) {
#pragma unroll
      for (int hh = 0; hh < kCPL; ++hh) {
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (qoff[s] >= 0) w = __ldg(reinterpret_cast<const uint4*>(p.q + qoff[s] + hh * 64 + t8 * 8));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = bf2(ws[e]);
          qv[s][hh * 4 + e] = make_float2(f.x * p.scale_log2, f.y * p.scale_log2);
        }
      }
    }

    for (int k = 0; k < n_stages; ++k) {
      const int st = k % kStagesR;
      // A wait that gives up (error recorded, abort set) does not leave the
      // loop: every compute warp keeps taking the same named barriers, so the
      // CTA always finishes; its output is then garbage and the host sees
      // SWA_ERR_TIMEOUT.
      mbar_wait(&full[st], (uint32_t)(k / kStagesR) & 1u, p.err, abort_flag);
      const uint8_t* kb = smem + st * S::kStage;
      const uint8_t* vb = kb + S::kTile;
      // ---- scores of the stage's 64 key rows, for every slot
#pragma unroll
      for (int j = 0; j < kRows / 4 / kComputeWarps; ++j) {
        const int r = (warp + j * kComputeWarps) * 4 + rsub;
        float2 d2[NQ];
#pragma unroll
        for (int s = 0; s < NQ; ++s) d2[s] = make_float2(0.f, 0.f);
#pragma unroll
        for (int hh = 0; hh < kCPL; ++hh) {
          const uint4 w = *reinterpret_cast<const uint4*>(kb + hh * (kRows * 128) + r * 128 +
                                                          ((t8 ^ (r & 7)) * 16));
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 kk = bf2(ws[e]);
#pragma unroll
            for (int s = 0; s < NQ; ++s) d2[s] = fma2(qv[s][hh * 4 + e], kk, d2[s]);
          }
        }
        float dot[NQ];
#pragma unroll
        for (int s = 0; s < NQ; ++s) dot[s] = d2[s].x + d2[s].y;
        int myslot;
        const float tot = reduce8_transposed<NQ>(dot, t8, &myslot);
        // after the reduction lanes t with t % (8 / NQ) == 0 hold distinct
        // slots; each writes its (row, slot) score
        if ((t8 & (8 / NQ - 1)) == 0) {
          const int idx = key0 + k * kRows + r;
          const int rel = idx < seg_n ? idx : idx + off_b;
          int lo = lo_r[0], hi = hi_r[0];  // decode, paged: one sequence per set
          if (MODE == 3) {
#pragma unroll
            for (int s = 1; s < NQ; ++s)
              if (s == myslot) {
                lo = lo_r[s];
                hi = hi_r[s];
              }
          }
          const bool ok = MODE == 0
                              ? idx <= hi
                              : (rel >= lo && rel <= hi && (idx >= seg_n || rel < a_end_r));
          sc[r * NQ + myslot] = ok ? tot : -INFINITY;
        }
      }
      named_sync(1, kComputeWarps * 32);
      // ---- online softmax statistics: warp w owns slots w, w + 4
      for (int s = warp; s < NQ; s += kComputeWarps) {
        const int u = s / kComputeWarps;
        const float a0 = sc[lane * NQ + s], a1 = sc[(lane + 32) * NQ + s];
        float mx = fmaxf(a0, a1);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float m_new = fmaxf(m_run[u], mx);
        const float m_safe = m_new == -INFINITY ? 0.f : m_new;
        const float cf = ex2_approx(m_run[u] - m_safe);
        const float p0 = ex2_approx(a0 - m_safe), p1 = ex2_approx(a1 - m_safe);
        pc[lane * NQ + s] = p0;
        pc[(lane + 32) * NQ + s] = p1;
        float sum = p0 + p1;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        l_run[u] = l_run[u] * cf + sum;
        m_run[u] = m_new;
        if (lane == 0) corr_s[s] = cf;
      }
      named_sync(1, kComputeWarps * 32);
      // ---- O += P V: warp w takes rows w, w + 4, ...; lane owns EPL columns
#pragma unroll
      for (int s = 0; s < NQ; ++s) {
        const float cf = corr_s[s];
#pragma unroll
        for (int e = 0; e < EPL / 2; ++e) acc[s][e] = make_float2(acc[s][e].x * cf, acc[s][e].y * cf);
      }
      // lane's EPL columns: byte offset lane * 2 * EPL of the row, in the
      // 128-byte half (lane * 2 * EPL) / 128
      const int byte0 = lane * 2 * EPL;
      const int hh = byte0 / 128, c16 = (byte0 % 128) / 16, in16 = byte0 % 16;
#pragma unroll 4
      for (int r = warp; r < kRows; r += kComputeWarps) {
        const uint8_t* src = vb + hh * (kRows * 128) + r * 128 + ((c16 ^ (r & 7)) * 16) + in16;
        uint32_t vw[EPL / 2];
        if (EPL == 4) {
          const uint2 w = *reinterpret_cast<const uint2*>(src);
          vw[0] = w.x;
          vw[EPL / 2 - 1] = w.y;
        } else {
          vw[0] = *reinterpret_cast<const uint32_t*>(src);
        }
        float pr[NQ];
        if (NQ >= 4) {
#pragma unroll
          for (int s4 = 0; s4 < NQ; s4 += 4) {
            const float4 p4 = *reinterpret_cast<const float4*>(pc + r * NQ + s4);
            pr[s4] = p4.x;
            pr[s4 + 1] = p4.y;
            pr[s4 + 2] = p4.z;
            pr[s4 + 3] = p4.w;
          }
        } else {
#pragma unroll
          for (int s = 0; s < NQ; ++s) pr[s] = pc[r * NQ + s];
        }
#pragma unroll
        for (int e = 0; e < EPL / 2; ++e) {
          const float2 vv = bf2(vw[e]);
#pragma unroll
          for (int s = 0; s < NQ; ++s) acc[s][e] = fma2(make_float2(pr[s], pr[s]), vv, acc[s][e]);
        }
      }
      mbar_arrive(&empty[st]);
    }
  }
  __syncthreads();  // every stage consumed: the ring can be reused below

  // ---- reduce the warps' partial sums: red[warp][slot][D]
  float* red = reinterpret_cast<float*>(smem);
  if (warp < kComputeWarps) {
#pragma unroll
    for (int s = 0; s < NQ; ++s) {
      float* dst = red + (warp * NQ + s) * D + lane * EPL;
      if (EPL == 4) {
        *reinterpret_cast<float4*>(dst) = make_float4(acc[s][0].x, acc[s][0].y, acc[s][EPL / 2 - 1].x,
                                                      acc[s][EPL / 2 - 1].y);
      } else {
        *reinterpret_cast<float2*>(dst) = acc[s][0];
      }
    }
    if (lane == 0) {
      for (int s = warp; s < NQ; s += kComputeWarps) {
        sc[s] = m_run[s / kComputeWarps];
        sc[NQ + s] = l_run[s / kComputeWarps];
      }
    }
  }
  __syncthreads();

  const size_t part = (size_t)gi * p.nsplit + split;
  if (p.nsplit == 1) {
    // single chunk: finish in place
    for (int idx = threadIdx.x; idx < NQ * D; idx += blockDim.x) {
      const int s = idx / D, dd = idx % D;
      if (qoff[s] < 0) continue;
      float o = 0.f;
      for (int w = 0; w < kComputeWarps; ++w) o += red[(w * NQ + s) * D + dd];
      const float l = sc[NQ + s];
      p.out[qoff[s] + dd] = __bfloat16_as_ushort(__float2bfloat16_rn(o / l));
    }
    if (p.lse && threadIdx.x < NQ && qoff[threadIdx.x] >= 0) {
      const int s = threadIdx.x;
      const float lv = (sc[s] + __log2f(sc[NQ + s])) * 0.69314718055994531f;
      const long row = qoff[s] / D;  // decode: b*H + h; append: (b*C + c)*H + h
      long li;
      if (MODE == 0 || MODE == 2) li = row;
      else {
        const int h = (int)(row % p.H);
        const long bi = row / p.H;
        li = ((bi / p.N) * p.H + h) * p.N + (bi % p.N);
      }
      p.lse[li] = lv;
    }
    return;
  }
  for (int idx = threadIdx.x; idx < NQ * D; idx += blockDim.x) {
    const int s = idx / D, dd = idx % D;
    float o = 0.f;
    for (int w = 0; w < kComputeWarps; ++w) o += red[(w * NQ + s) * D + dd];
    p.ws_o[part * NQ * D + idx] = o;
  }
  if (threadIdx.x < NQ) {
    p.ws_ml[(part * NQ + threadIdx.x) * 2] = sc[threadIdx.x];
    p.ws_ml[(part * NQ + threadIdx.x) * 2 + 1] = sc[NQ + threadIdx.x];
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int ticket = atomicAdd(&p.cnt[gi], 1);
    *last_flag = ticket == p.nsplit - 1;
  }
  __syncthreads();
  if (!*last_flag) return;
  __threadfence();
  // ---- last chunk of this query set: merge all chunks
  const size_t base = (size_t)gi * p.nsplit;
  float* Ms = sc;          // [NQ] global max
  float* Ls = sc + NQ;     // [NQ] merged denominator
  if (threadIdx.x < NQ) {
    const int s = threadIdx.x;
    float M = -INFINITY;
    for (int sp = 0; sp < p.nsplit; ++sp) M = fmaxf(M, __ldcg(&p.ws_ml[((base + sp) * NQ + s) * 2]));
    const float Msafe = M == -INFINITY ? 0.f : M;
    float L = 0.f;
    for (int sp = 0; sp < p.nsplit; ++sp) {
      const float m = __ldcg(&p.ws_ml[((base + sp) * NQ + s) * 2]);
      L += __ldcg(&p.ws_ml[((base + sp) * NQ + s) * 2 + 1]) * ex2_approx(m - Msafe);
    }
    Ms[s] = Msafe;
    Ls[s] = L;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < NQ * D; idx += blockDim.x) {
    const int s = idx / D, dd = idx % D;
    if (qoff[s] < 0) continue;
    float o = 0.f;
    for (int sp = 0; sp < p.nsplit; ++sp) {
      const float m = __ldcg(&p.ws_ml[((base + sp) * NQ + s) * 2]);
      o += __ldcg(&p.ws_o[(base + sp) * NQ * D + idx]) * ex2_approx(m - Ms[s]);
    }
    p.out[qoff[s] + dd] = __bfloat16_as_ushort(__float2bfloat16_rn(o / Ls[s]));
  }
  if (p.lse && threadIdx.x < NQ && qoff[threadIdx.x] >= 0) {
    const int s = threadIdx.x;
    const float lv = (Ms[s] + __log2f(Ls[s])) * 0.69314718055994531f;
    const long row = qoff[s] / D;
    long li;
    if (MODE == 0 || MODE == 2) li = row;
    else {
      const int h = (int)(row % p.H);
      const long bi = row / p.H;
      li = ((bi / p.N) * p.H + h) * p.N + (bi % p.N);
    }
    p.lse[li] = lv;
  }
  if (threadIdx.x == 0) p.cnt[gi] = 0;  // ready for the next call
}

// ------------------------------------------------------------ workspaces
// Per device and per user (0: decode, 1: unused, 2: paged decode,
// 3: chunked append, 4: the split partials of a tensor-core append):
// split counters and
// split partials in separate buffers.  Every merge resets its counter to
// zero, so between complete calls all counters are zero; the counter buffer
// is zeroed whenever it is (re)allocated and is never overlapped by the
// partials, whatever the number of query sets of later calls.
struct Workspace {
  void* cnt = nullptr;
  size_t cnt_bytes = 0;
  void* part = nullptr;
  size_t part_bytes = 0;
};
constexpr int kMaxDev = 64;
Workspace g_ws[kMaxDev][5];  // users: decode, (unused), paged, append, tensor-core append
std::mutex g_ws_mu;

bool get_workspace(int which, size_t cnt_bytes, size_t part_bytes, cudaStream_t stream,
                   int** cnt, void** part) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return false;
  std::lock_guard<std::mutex> lk(g_ws_mu);
  Workspace& w = g_ws[dev][which];
  if (w.cnt_bytes < cnt_bytes) {
    if (w.cnt) {
      cudaStreamSynchronize(stream);
      ws_free(w.cnt);
      w.cnt = nullptr;
      w.cnt_bytes = 0;
    }
    void* p = ws_alloc(cnt_bytes);
    if (!p) return false;
    if (cudaMemsetAsync(p, 0, cnt_bytes, stream) != cudaSuccess) {
      ws_free(p);
      return false;
    }
    w.cnt = p;
    w.cnt_bytes = cnt_bytes;
  }
  if (w.part_bytes < part_bytes) {
    if (w.part) {
      cudaStreamSynchronize(stream);
      ws_free(w.part);
      w.part = nullptr;
      w.part_bytes = 0;
    }
    void* p = ws_alloc(part_bytes);
    if (!p) return false;
    w.part = p;
    w.part_bytes = part_bytes;
  }
  *cnt = static_cast<int*>(w.cnt);
  *part = w.part;
  return true;
}

template <int D, int NQ, int MODE>
int launch_rows(RowParams& p, int nsets, cudaStream_t stream) {
  using S = RSmem<D, NQ>;
  static std::atomic<unsigned long long> attr{0};
  if (!smem_attr_once(reinterpret_cast<const void*>(swa_rowattn_kernel<D, NQ, MODE>), S::kAlloc,
                      attr))
    return SWA_ERR_CUDA;
  dim3 grid(p.nsplit, nsets);
  swa_rowattn_kernel<D, NQ, MODE><<<grid, kThreadsR, S::kAlloc, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

// decode and paged decode serve a GQA group (1, 2, 4 or 8 query vectors);
// a chunked append fills 4 or 8 slots with whole groups
template <int D>
int dispatch_nq(RowParams& p, int nq, int nsets, cudaStream_t stream) {
  if (p.mode == 3)
    return nq == 8 ? launch_rows<D, 8, 3>(p, nsets, stream)
                   : (nq == 4 ? launch_rows<D, 4, 3>(p, nsets, stream) : SWA_ERR_UNSUPPORTED);
  if (p.mode == 0) {
    switch (nq) {
      case 1: return launch_rows<D, 1, 0>(p, nsets, stream);
      case 2: return launch_rows<D, 2, 0>(p, nsets, stream);
      case 4: return launch_rows<D, 4, 0>(p, nsets, stream);
      case 8: return launch_rows<D, 8, 0>(p, nsets, stream);
      default: return SWA_ERR_UNSUPPORTED;
    }
  }
  switch (nq) {
    case 1: return launch_rows<D, 1, 2>(p, nsets, stream);
    case 2: return launch_rows<D, 2, 2>(p, nsets, stream);
    case 4: return launch_rows<D, 4, 2>(p, nsets, stream);
    case 8: return launch_rows<D, 8, 2>(p, nsets, stream);
    default: return SWA_ERR_UNSUPPORTED;
  }
}

int pow2_at_least(int x) {
  int r = 1;
  while (r < x) r <<= 1;
  return r;
}

int encode_kv(CUtensorMap* m, const void* base, int D, int Hkv, int rows, int B) {
  const uint64_t dims[4] = {(uint64_t)D, (uint64_t)Hkv, (uint64_t)rows, (uint64_t)B};
  const uint64_t strides[3] = {(uint64_t)D * 2, (uint64_t)Hkv * D * 2, (uint64_t)rows * Hkv * D * 2};
  const uint32_t box[4] = {64, 1, (uint32_t)kRows, 1};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                      strides, box, CU_TENSOR_MAP_SWIZZLE_128B) == CUDA_SUCCESS
             ? SWA_OK
             : SWA_ERR_CUDA;
}

int run(RowParams& p, int D, int nq, int nsets, int which, cudaStream_t stream) {
  if (p.nsplit > 1) {
    const size_t cnt_bytes = ((size_t)nsets * 4 + 255) & ~size_t(255);
    const size_t o_bytes = (size_t)nsets * p.nsplit * nq * D * 4;
    const size_t ml_bytes = (size_t)nsets * p.nsplit * nq * 2 * 4;
    int* cnt = nullptr;
    void* part = nullptr;
    if (!get_workspace(which, cnt_bytes, o_bytes + ml_bytes, stream, &cnt, &part))
      return SWA_ERR_NOMEM;
    p.cnt = cnt;
    p.ws_o = static_cast<float*>(part);
    p.ws_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(part) + o_bytes);
  }
  if (D == 128) return dispatch_nq<128>(p, nq, nsets, stream);
  if (D == 64) return dispatch_nq<64>(p, nq, nsets, stream);
  return SWA_ERR_UNSUPPORTED;
}

// Writes the chunk's keys and values into their ring slots (pos0 + c) % W,
// 16 bytes per thread.  grid (ceil(row_vecs / 256), C - c_first, B).
__global__ void ring_store_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                                  uint4* __restrict__ k_ring, uint4* __restrict__ v_ring,
                                  const int64_t* __restrict__ pos0, int C, int W, int row_vecs,
                                  int c_first) {
  const int b = blockIdx.z, c = c_first + (int)blockIdx.y;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const long long p0 = pos0[b];
  if (i >= row_vecs || p0 < 0) return;
  const long long slot = (p0 + c) % W;
  const long src = ((long)b * C + c) * row_vecs + i;
  const long dst = ((long)b * W + slot) * row_vecs + i;
  k_ring[dst] = k_new[src];
  v_ring[dst] = v_new[src];
}

// The chunk of an append entering its ring slots (pos0 + c) % W: the rows
// c >= c_first of k_new / v_new, row_vecs 16-byte vectors each.
struct RingStore {
  const uint4* k_new = nullptr;
  const uint4* v_new = nullptr;
  uint4* k_ring = nullptr;
  uint4* v_ring = nullptr;
  const int64_t* pos0 = nullptr;
  int B = 0, C = 0, W = 0, row_vecs = 0, c_first = 0;
};

// Combines split key walks (the parts of a tensor-core append or decode):
// row (b, c, h) has nsplit partial results O_i / l_i (fp32) with lse_i
// (any number of parts, taken eight at a time); with m = max lse_i
// and w_i = exp(lse_i - m), out = sum w_i O_i / sum w_i (bf16) and lse = m +
// ln sum w_i (the lse identity of split softmax).  One warp per row, D / 32
// columns per lane.  An append also hands its ring store to this launch
// (every key walk has read the ring by then): the grid's threads copy the
// chunk's vectors into their slots before merging.
template <int D>
__global__ void __launch_bounds__(256) split_merge_kernel(const float* __restrict__ part_o,
                                                           const float* __restrict__ part_lse,
                                                           uint16_t* __restrict__ out,
                                                           float* __restrict__ lse, int nsplit,
                                                           int B, int C, int H, RingStore rs) {
  constexpr int kPer = D / 32;  // 4 (D = 128) or 2 (D = 64) columns per lane
  constexpr int kBatch = 8;     // parts whose loads are in flight together
  using Vec = typename std::conditional<kPer == 4, float4, float2>::type;
  if (rs.k_new) {
    const long long per_b = (long long)(rs.C - rs.c_first) * rs.row_vecs;
    const long long total = per_b * rs.B;
    const long long nthr = (long long)gridDim.x * blockDim.x;
    for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += nthr) {
      const int b = (int)(t / per_b);
      const long long rem = t - (long long)b * per_b;
      const int c = rs.c_first + (int)(rem / rs.row_vecs);
      const int i = (int)(rem % rs.row_vecs);
      const long long p0 = rs.pos0[b];
      if (p0 < 0) continue;
      const long long slot = (p0 + c) % rs.W;
      const long long src = ((long long)b * rs.C + c) * rs.row_vecs + i;
      const long long dst = ((long long)b * rs.W + slot) * rs.row_vecs + i;
      rs.k_ring[dst] = __ldg(rs.k_new + src);
      rs.v_ring[dst] = __ldg(rs.v_new + src);
    }
  }
  // launched as a programmatic dependent of the kernel that wrote the
  // partials: wait here until that grid has completed (a no-op otherwise)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const long long row = (long long)blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const long long rows = (long long)B * H * C;
  if (row >= rows) return;
  // part index ((sp * B + b) * H + h) * C + c = sp * rows + row
  const int c = (int)(row % C);
  const long long bh = row / C;  // b * H + h
  const int h = (int)(bh % H);
  const int b = (int)(bh / H);
  // m = max lse_i: with at most kBatch parts it comes from the batch loaded
  // below (one pass, every load in flight at once); otherwise a first pass
  float m = -INFINITY;
  if (nsplit > kBatch) {
    for (int sp = lane; sp < nsplit; sp += 32)
      m = fmaxf(m, __ldg(part_lse + (long long)sp * rows + row));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  }
  float acc[kPer] = {};
  float wsum = 0.f;
  for (int sp0 = 0; sp0 < nsplit; sp0 += kBatch) {
    // a batch of parts: every load issued before any is used
    float li[kBatch];
    Vec o[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      if (sp0 + i < nsplit) {
        const long long pr = (long long)(sp0 + i) * rows + row;
        li[i] = __ldg(part_lse + pr);
        o[i] = __ldg(reinterpret_cast<const Vec*>(part_o + pr * D) + lane);
      }
    }
    if (nsplit <= kBatch) {
#pragma unroll
      for (int i = 0; i < kBatch; ++i)
        if (i < nsplit) m = fmaxf(m, li[i]);
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      // a part holding none of the row's keys has lse = -inf: skipped
      if (sp0 + i >= nsplit || li[i] == -INFINITY) continue;
      const float w = __expf(li[i] - m);
      wsum += w;
      const float* f = reinterpret_cast<const float*>(&o[i]);
#pragma unroll
      for (int e = 0; e < kPer; ++e) acc[e] += w * f[e];
    }
  }
  const float inv = 1.f / wsum;
  uint16_t* dst = out + (((long long)b * C + c) * H + h) * D + lane * kPer;
  uint32_t pk[kPer / 2];
#pragma unroll
  for (int e = 0; e < kPer; e += 2) pk[e / 2] = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
  if (kPer == 4)
    *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[kPer / 2 - 1]);
  else
    *reinterpret_cast<uint32_t*>(dst) = pk[0];
  if (lse && lane == 0) lse[bh * C + c] = m + __logf(wsum);
}

}  // namespace

bool split_workspace(int which, size_t bytes, cudaStream_t stream, float** part) {
  int* cnt = nullptr;
  void* p = nullptr;
  if (!get_workspace(which, 256, bytes, stream, &cnt, &p)) return false;
  *part = static_cast<float*>(p);
  return true;
}

int encode_kv_map(CUtensorMap* m, const void* base, int D, int Hkv, int rows, int B) {
  return encode_kv(m, base, D, Hkv, rows, B);
}

int launch_decode(const void* q, const void* k_ring, const void* v_ring, void* out, float* lse,
                  const int64_t* pos, int B, int H, int Hkv, int D, int W, float scale,
                  cudaStream_t stream) {
  // D = 128: the tensor-core decode (swa_decode_tc.cu); other sizes the
  // split-KV row kernel below
  if (D == 128) {
    const int st = launch_decode_tc(q, k_ring, v_ring, out, lse, pos, B, H, Hkv, D, W, scale,
                                    stream);
    if (st != SWA_ERR_UNSUPPORTED) return st;
  }
  RowParams p;
  std::memset(&p, 0, sizeof(p));
  if (encode_kv(&p.tmK, k_ring, D, Hkv, W, B) != SWA_OK ||
      encode_kv(&p.tmV, v_ring, D, Hkv, W, B) != SWA_OK)
    return SWA_ERR_CUDA;
  p.q = static_cast<const uint16_t*>(q);
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.pos = pos;
  p.err = device_error_word();
  if (!p.err) return SWA_ERR_CUDA;
  p.mode = 0;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.W = W;
  p.grp = H / Hkv;
  p.rows_per_cta = 1;
  p.nrowchunks = 1;
  p.chunk = kDecodeChunk;
  p.nsplit = (W + p.chunk - 1) / p.chunk;
  p.scale_log2 = scale * 1.4426950408889634f;
  const int nq = pow2_at_least(p.grp);
  return run(p, D, nq, B * Hkv, 0, stream);
}

int launch_decode_paged(const void* q, const void* k_pages, const void* v_pages, void* out,
                        float* lse, const int32_t* table, const int64_t* pos, int B, int H,
                        int Hkv, int D, int page_size, int num_pages, int max_pages, int W,
                        float scale, cudaStream_t stream) {
  if (D == 128) {
    const int st = launch_decode_paged_tc(q, k_pages, v_pages, out, lse, table, pos, B, H, Hkv,
                                          D, page_size, num_pages, max_pages, W, scale, stream);
    if (st != SWA_ERR_UNSUPPORTED) return st;
  }
  RowParams p;
  std::memset(&p, 0, sizeof(p));
  const long long rows = (long long)num_pages * page_size;
  if (rows > 0x7fffffffLL) return SWA_ERR_UNSUPPORTED;
  if (encode_kv(&p.tmK, k_pages, D, Hkv, (int)rows, 1) != SWA_OK ||
      encode_kv(&p.tmV, v_pages, D, Hkv, (int)rows, 1) != SWA_OK)
    return SWA_ERR_CUDA;
  p.q = static_cast<const uint16_t*>(q);
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.pos = pos;
  p.table = table;
  p.page_size = page_size;
  p.max_pages = max_pages;
  p.err = device_error_word();
  if (!p.err) return SWA_ERR_CUDA;
  p.mode = 2;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.W = W;
  p.grp = H / Hkv;
  p.rows_per_cta = 1;
  p.nrowchunks = 1;
  // the window's keys, from a 64-aligned start: at most W + 63 indices,
  // split into near-equal multiples of 64 of about 1024 keys
  const int span = W + kRows;
  p.nsplit = (span + 1023) / 1024;
  p.chunk = (((span + p.nsplit - 1) / p.nsplit) + kRows - 1) / kRows * kRows;
  p.scale_log2 = scale * 1.4426950408889634f;
  const int nq = pow2_at_least(p.grp);
  return run(p, D, nq, B * Hkv, 2, stream);
}

namespace {
// The new tokens enter the ring (launched after every query has read the
// slots they overwrite); of a chunk longer than W only the last W stay.
int ring_store(const void* k_new, const void* v_new, void* k_ring, void* v_ring,
               const int64_t* pos0, int B, int C, int Hkv, int D, int W, cudaStream_t stream) {
  const int c_first = C > W ? C - W : 0;
  const int row_vecs = Hkv * D / 8;
  dim3 grid((row_vecs + 255) / 256, C - c_first, B);
  ring_store_kernel<<<grid, 256, 0, stream>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new),
      static_cast<uint4*>(k_ring), static_cast<uint4*>(v_ring), pos0, C, W, row_vecs, c_first);
  return cudaGetLastError() == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}
}  // namespace

namespace {
int merge_parts(const float* part, void* out, float* lse, int nsplit, int B, int C, int H, int D,
                 cudaStream_t stream, const RingStore& rs = RingStore()) {
  const long long rows = (long long)B * H * C;
  const float* part_lse = part + (size_t)nsplit * rows * D;
  const long long blocks = (rows + 7) / 8;
  if (blocks > 0x7fffffffLL) return SWA_ERR_UNSUPPORTED;
  // a programmatic dependent launch: its launch overlaps the tail of the
  // kernel before it, and griddepcontrol.wait orders the reads
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (D == 128)
    e = cudaLaunchKernelEx(&cfg, split_merge_kernel<128>, (const float*)part, part_lse,
                           static_cast<uint16_t*>(out), lse, nsplit, B, C, H, rs);
  else
    e = cudaLaunchKernelEx(&cfg, split_merge_kernel<64>, (const float*)part, part_lse,
                           static_cast<uint16_t*>(out), lse, nsplit, B, C, H, rs);
  if (e != cudaSuccess) return SWA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

// Chunks of 32 tokens and more: the tcgen05 forward with a causal window of
// W keys over the ring history below pos0 followed by the chunk (both read
// in place), its queries being the chunk's C rows.  Shorter chunks would
// leave most of a 128-row query tile idle and take the row kernel below.
int append_attention_tc(const void* q, const void* k_new, const void* v_new, void* k_ring,
                        void* v_ring, void* out, float* lse, const int64_t* pos0, int B, int C,
                        int H, int Hkv, int D, int W, float scale, cudaStream_t stream) {
  // Work items: query tiles x head groups (four heads per CTA when two are
  // stacked per tile, else two or one); when they do not fill the SMs the
  // key walks are split (the partials merged after), at least two key
  // tiles per part.
  int nsm = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm <= 0)
    return SWA_ERR_CUDA;
  const int grp = H / Hkv;
  const bool stack = fwd_qwin_stacks(H, Hkv, C);
  const int per_cta = stack ? 4 : (grp % 2 == 0 ? 2 : 1);
  const long long items = (long long)B * ((H + per_cta - 1) / per_cta) * ((C + 127) / 128);
  const int per_sm = (D == 64 && per_cta == 1) ? 2 : 1;
  const int walk = (W + C + 127) / 128 + 1;  // key tiles of a query tile, at most
  int nsplit = (int)((long long)nsm * per_sm / (items > 0 ? items : 1));
  nsplit = nsplit < 1 ? 1 : (nsplit > 8 ? 8 : nsplit);
  while (nsplit > 1 && walk / nsplit < 2) --nsplit;
  QueryWindow qw{pos0, W - 1, C, W};
  qw.stack = stack ? 1 : 0;
  qw.nsplit = nsplit;
  const size_t part_bytes =
      nsplit > 1 ? (size_t)nsplit * B * H * C * (D + 1) * sizeof(float) : 0;
  // the ring and the chunk are read in place: with W a multiple of 64
  // (swa_append requires it) every 64-row key box lies inside one of them
  // (the kernel's per-batch layout), so no staged copy is needed
  if (W % 64 != 0 || (long long)W + 64 + C > 0x7fffffffLL) return SWA_ERR_UNSUPPORTED;
  if (part_bytes) {
    int* cnt = nullptr;
    void* part = nullptr;
    if (!get_workspace(4, 256, part_bytes, stream, &cnt, &part)) return SWA_ERR_NOMEM;
    qw.part = static_cast<float*>(part);
  }
  qw.kn = k_new;
  qw.vn = v_new;
  // two parts merge each other inside the launch (clusters of two CTAs),
  // which can also store the chunk into the ring
  qw.pair = nsplit == 2 ? 1 : 0;
  qw.ring_k = k_ring;
  qw.ring_v = v_ring;
  int done = 0;
  qw.done = &done;
  const int st = launch_fwd_sm100(q, k_ring, v_ring, out, lse, B, H, Hkv, W + 64 + C, D, W - 1,
                                  0, 1, 0, nullptr, 0, scale, stream, &qw);
  if (st != SWA_OK) return st;
  if (done & 2) return SWA_OK;
  if (nsplit == 1 || (done & 1))
    return ring_store(k_new, v_new, k_ring, v_ring, pos0, B, C, Hkv, D, W, stream);
  // the merge launch also stores the chunk into the ring
  RingStore rs;
  rs.k_new = static_cast<const uint4*>(k_new);
  rs.v_new = static_cast<const uint4*>(v_new);
  rs.k_ring = static_cast<uint4*>(k_ring);
  rs.v_ring = static_cast<uint4*>(v_ring);
  rs.pos0 = pos0;
  rs.B = B;
  rs.C = C;
  rs.W = W;
  rs.row_vecs = Hkv * D / 8;
  rs.c_first = C > W ? C - W : 0;
  return merge_parts(qw.part, out, lse, nsplit, B, C, H, D, stream, rs);
}
}  // namespace

int split_merge(const float* part, void* out, float* lse, int nsplit, int B, int C, int H, int D,
                cudaStream_t stream) {
  return merge_parts(part, out, lse, nsplit, B, C, H, D, stream);
}

int launch_append(const void* q, const void* k_new, const void* v_new, void* k_ring, void* v_ring,
                  void* out, float* lse, const int64_t* pos0, int B, int C, int H, int Hkv, int D,
                  int W, float scale, cudaStream_t stream) {
  if (C >= 32)
    return append_attention_tc(q, k_new, v_new, k_ring, v_ring, out, lse, pos0, B, C, H, Hkv, D,
                               W, scale, stream);
  RowParams p;
  std::memset(&p, 0, sizeof(p));
  if (encode_kv(&p.tmK, k_ring, D, Hkv, W, B) != SWA_OK ||
      encode_kv(&p.tmV, v_ring, D, Hkv, W, B) != SWA_OK ||
      encode_kv(&p.tmKn, k_new, D, Hkv, C, B) != SWA_OK ||
      encode_kv(&p.tmVn, v_new, D, Hkv, C, B) != SWA_OK)
    return SWA_ERR_CUDA;
  p.q = static_cast<const uint16_t*>(q);
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.pos = pos0;
  p.err = device_error_word();
  if (!p.err) return SWA_ERR_CUDA;
  p.mode = 3;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.N = C;
  p.W = W;
  p.grp = H / Hkv;
  const int nq = p.grp <= 4 ? 4 : 8;
  p.rows_per_cta = nq / p.grp;  // query tokens per CTA
  p.nrowchunks = (C + p.rows_per_cta - 1) / p.rows_per_cta;
  // history (at most W + 64 indices from a 64-aligned start) then the chunk
  const int span = W + kRows + C;
  p.nsplit = (span + 1023) / 1024;
  p.chunk = (((span + p.nsplit - 1) / p.nsplit) + kRows - 1) / kRows * kRows;
  p.scale_log2 = scale * 1.4426950408889634f;
  const int st = run(p, D, nq, B * Hkv * p.nrowchunks, 3, stream);
  if (st != SWA_OK) return st;
  return ring_store(k_new, v_new, k_ring, v_ring, pos0, B, C, Hkv, D, W, stream);
}

void release_workspaces() {
  std::lock_guard<std::mutex> lk(g_ws_mu);
  for (int d = 0; d < kMaxDev; ++d)
    for (int w = 0; w < 5; ++w) {
      Workspace& ws = g_ws[d][w];
      if (!ws.cnt && !ws.part) continue;
      int cur = 0;
      cudaGetDevice(&cur);
      cudaSetDevice(d);
      cudaDeviceSynchronize();
      if (ws.cnt) ws_free(ws.cnt);
      if (ws.part) ws_free(ws.part);
      cudaSetDevice(cur);
      ws = Workspace();
    }
}


// ------------------------------------------------------------------------
// Decode without any device allocation by the library.
//
// The ordinary swa_decode path keeps its split partials in a workspace that
// the library cudaMalloc's on first use.  Some callers cannot allow that:
// serving engines that hand every byte of device memory to their own
// pre-sized pool or arena (a stray cudaMalloc breaks their budget and
// fragments the pool), and latency-critical loops that cannot afford the
// implicit device-wide synchronisation cudaMalloc may cause.  For them the
// partials live in this fixed file-scope array instead.  Every GPU that
// loads the library holds it (kNoAllocScratchBytes) until the process
// exits, and all calls share it.
constexpr size_t kNoAllocScratchBytes = 16u << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
void* g_noalloc_ptr[kMaxDev] = {};
std::mutex g_noalloc_mu;

// Device address of g_noalloc_scratch on the current device.  In host code
// the symbol is only a stand-in, so the address is looked up once per
// device with that device current (first call on the device).
void* noalloc_scratch(int* status) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    *status = SWA_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) {
      *status = SWA_ERR_CUDA;
      return nullptr;
    }
    g_noalloc_ptr[dev] = ptr;
  }
  return g_noalloc_ptr[dev];
}
}  // namespace

int launch_decode_noalloc(const void* q, const void* k_ring, const void* v_ring, void* out,
                          const int64_t* pos, int B, int H, int Hkv, int D, int W,
                          float scale, cudaStream_t stream) {
  RowParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = static_cast<const uint16_t*>(q);
  p.out = static_cast<uint16_t*>(out);
  p.lse = nullptr;
  p.pos = pos;
  p.mode = 0;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.W = W;
  p.grp = H / Hkv;
  p.rows_per_cta = 1;
  p.nrowchunks = 1;
  p.chunk = kDecodeChunk;  // the same split as swa_decode
  p.nsplit = (W + p.chunk - 1) / p.chunk;
  p.scale_log2 = scale * 1.4426950408889634f;
  const int nq = pow2_at_least(p.grp);
  const int nsets = B * Hkv;
  const size_t cnt_bytes = ((size_t)nsets * 4 + 255) & ~size_t(255);
  const size_t o_bytes = (size_t)nsets * p.nsplit * nq * D * 4;
  const size_t ml_bytes = (size_t)nsets * p.nsplit * nq * 2 * 4;
  if (p.nsplit > 1 && cnt_bytes + o_bytes + ml_bytes > kNoAllocScratchBytes)
    return SWA_ERR_UNSUPPORTED;  // problem needs more scratch than the array holds
  int status = SWA_OK;
  uint8_t* ws = static_cast<uint8_t*>(noalloc_scratch(&status));
  if (!ws) return status;
  p.err = device_error_word();
  if (!p.err) return SWA_ERR_CUDA;
  if (encode_kv(&p.tmK, k_ring, D, Hkv, W, B) != SWA_OK ||
      encode_kv(&p.tmV, v_ring, D, Hkv, W, B) != SWA_OK)
    return SWA_ERR_CUDA;
  if (p.nsplit > 1) {
    // The array keeps whatever the last call left; the split counters must
    // start at zero, so clear them on the caller's stream.
    if (cudaMemsetAsync(ws, 0, cnt_bytes, stream) != cudaSuccess) return SWA_ERR_CUDA;
    p.cnt = reinterpret_cast<int*>(ws);
    p.ws_o = reinterpret_cast<float*>(ws + cnt_bytes);
    p.ws_ml = reinterpret_cast<float*>(ws + cnt_bytes + o_bytes);
  }
  if (D == 128) return dispatch_nq<128>(p, nq, nsets, stream);
  if (D == 64) return dispatch_nq<64>(p, nq, nsets, stream);
  return SWA_ERR_UNSUPPORTED;
}

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

}  // namespace swa
