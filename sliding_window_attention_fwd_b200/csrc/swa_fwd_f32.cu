// swa_fwd_f32.cu -- fp32 sliding-window attention forward on CUDA cores.
//
// One warp per query row (b, h, i).  The row's keys are walked in index
// order straight from the window arithmetic -- band (token- or
// block-level dilation), then global keys outside the band -- so keys
// outside the window are never touched (page "别再只加Mask了", §1: skip
// the out-of-window pairs instead of masking them).  The softmax is the
// online (running max / running sum) form, in fp32 FFMA: tcgen05
// kind::tf32 would round operands to 10 mantissa bits, too coarse for a
// 1e-4 bound, so this path stays on the FMA pipe.
#include <cuda_runtime.h>

#include <cstdint>

#include "swa_internal.h"

namespace swa {

namespace {

struct F32Params {
  const float* q;
  const float* k;
  const float* v;
  float* out;
  float* lse;
  const int32_t* G;
  int n_global;
  int B, H, Hkv, N, D;
  int L, R, d, bs;
  float scale;
};

__device__ __forceinline__ bool is_global(const int32_t* G, int ng, int i) {
  int lo = 0, hi = ng - 1;
  while (lo <= hi) {
    int mid = (lo + hi) >> 1;
    int x = G[mid];
    if (x == i) return true;
    if (x < i) lo = mid + 1; else hi = mid - 1;
  }
  return false;
}

// Whether key j is in the (uncut) band of query i.
__device__ __forceinline__ bool in_band(const F32Params& p, int i, int j) {
  long diff;
  long lo, hi;
  if (p.bs > 1) {
    diff = (long)(j / p.bs) - (long)(i / p.bs);
    lo = -(long)(p.L / p.bs) * p.d;
    hi = (long)(p.R / p.bs) * p.d;
  } else {
    diff = (long)j - (long)i;
    lo = -(long)p.L * p.d;
    hi = (long)p.R * p.d;
  }
  if (diff % p.d != 0) return false;
  if (p.L >= 0 && diff < lo) return false;
  if (p.R >= 0 && diff > hi) return false;
  return true;
}

template <int NV>  // NV = D / 32 values per lane
__global__ void __launch_bounds__(128) swa_fwd_f32_kernel(F32Params p) {
  const int warp = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  const long rows = (long)p.B * p.H * p.N;
  if (warp >= rows) return;
  const int i = warp % p.N;
  const int h = (warp / p.N) % p.H;
  const int b = warp / (p.N * p.H);
  const int g = h / (p.H / p.Hkv);
  const bool causal = p.R == 0;

  float qv[NV];
  const float* qrow = p.q + (((long)b * p.N + i) * p.H + h) * p.D;
#pragma unroll
  for (int t = 0; t < NV; ++t) qv[t] = qrow[lane + 32 * t];
  const long kv_stride = (long)p.Hkv * p.D;
  const float* kb = p.k + ((long)b * p.N * p.Hkv + g) * p.D;
  const float* vb = p.v + ((long)b * p.N * p.Hkv + g) * p.D;

  float m = -INFINITY, l = 0.f;
  float acc[NV];
#pragma unroll
  for (int t = 0; t < NV; ++t) acc[t] = 0.f;

  auto visit = [&](int j) {
    const float* kr = kb + (long)j * kv_stride;
    float s = 0.f;
#pragma unroll
    for (int t = 0; t < NV; ++t) s = fmaf(qv[t], kr[lane + 32 * t], s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    s *= p.scale;
    float mn = fmaxf(m, s);
    float corr = expf(m - mn);  // 0 when m = -inf
    float e = expf(s - mn);
    l = l * corr + e;
    const float* vr = vb + (long)j * kv_stride;
#pragma unroll
    for (int t = 0; t < NV; ++t) acc[t] = fmaf(e, vr[lane + 32 * t], acc[t] * corr);
    m = mn;
  };

  const int jmax = causal ? i : p.N - 1;
  if (p.n_global > 0 && is_global(p.G, p.n_global, i)) {
    for (int j = 0; j <= jmax; ++j) visit(j);
  } else {
    if (p.bs > 1) {
      const int nb = (p.N + p.bs - 1) / p.bs;
      const int bi = i / p.bs;
      const long mlo = p.L < 0 ? -(long)(bi / p.d) : -(long)(p.L / p.bs);
      const long mhi = p.R < 0 ? (long)((nb - 1 - bi) / p.d) : (long)(p.R / p.bs);
      for (long mm = mlo; mm <= mhi; ++mm) {
        long blk = bi + mm * p.d;
        if (blk < 0 || blk >= nb) continue;
        long j1 = (blk + 1) * p.bs - 1;
        if (j1 > jmax) j1 = jmax;
        for (long j = blk * p.bs; j <= j1; ++j) visit((int)j);
      }
    } else {
      const long klo = p.L < 0 ? -(long)(i / p.d) : -(long)p.L;
      const long khi = p.R < 0 ? (long)((p.N - 1 - i) / p.d) : (long)p.R;
      for (long kk = klo; kk <= khi; ++kk) {
        long j = i + kk * p.d;
        if (j < 0 || j > jmax) continue;
        visit((int)j);
      }
    }
    for (int t = 0; t < p.n_global; ++t) {
      int j = p.G[t];
      j = j < 0 ? 0 : (j >= p.N ? p.N - 1 : j);
      if (j > jmax || in_band(p, i, j)) continue;
      visit(j);
    }
  }

  const float inv = 1.f / l;
  float* orow = p.out + (((long)b * p.N + i) * p.H + h) * p.D;
#pragma unroll
  for (int t = 0; t < NV; ++t) orow[lane + 32 * t] = acc[t] * inv;
  if (p.lse && lane == 0) p.lse[((long)b * p.H + h) * p.N + i] = m + logf(l);
}

}  // namespace

int launch_fwd_f32(const float* q, const float* k, const float* v, float* out, float* lse,
                   int B, int H, int Hkv, int N, int D, int L, int R, int d, int bs,
                   const int32_t* G, int ng, float scale, cudaStream_t stream) {
  F32Params p{q, k, v, out, lse, G, ng, B, H, Hkv, N, D, L, R, d, bs, scale};
  const long rows = (long)B * H * N;
  const int threads = 128;
  const long blocks = (rows + 3) / 4;
  if (blocks > 0x7fffffffL) return SWA_ERR_UNSUPPORTED;
  switch (D) {
    case 32: swa_fwd_f32_kernel<1><<<(unsigned)blocks, threads, 0, stream>>>(p); break;
    case 64: swa_fwd_f32_kernel<2><<<(unsigned)blocks, threads, 0, stream>>>(p); break;
    case 96: swa_fwd_f32_kernel<3><<<(unsigned)blocks, threads, 0, stream>>>(p); break;
    case 128: swa_fwd_f32_kernel<4><<<(unsigned)blocks, threads, 0, stream>>>(p); break;
    default: return SWA_ERR_UNSUPPORTED;
  }
  return cudaGetLastError() == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

}  // namespace swa
