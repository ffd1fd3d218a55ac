// swa_bwd.cu -- sliding-window attention backward (dq, dk, dv): the entry
// point, and the CUDA-core kernel that serves problems with global tokens
// (band problems run on the tensor cores, swa_bwd_sm100.cu).
//
// The pages use the method for training but describe no backward pass; this
// is the derivative of the forward definition, over the same key sets (band
// with token- or block-level dilation, global tokens, causal clip), with
// keys outside the window never touched.  With P_ij = exp(s_ij - lse_i)
// recomputed from the forward's lse:
//   dP_ij = dO_i . v_j,  D_i = dO_i . out_i,  dS_ij = P_ij (dP_ij - D_i),
//   dQ_i = scale sum_j dS_ij k_j,  dK_j += scale dS_ij q_i,  dV_j += P_ij dO_i.
// One warp per (batch, query row, kv head) serves the whole GQA group (their
// key sets are the same), keeps dQ in registers and adds its dK / dV
// contributions into fp32 accumulators with atomics; a second kernel rounds
// those to bf16.  fp32 math on bf16 data.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <type_traits>

#include "swa_internal.h"

namespace swa {

namespace {

struct BwdParams {
  const uint16_t *q, *k, *v, *out, *dout;
  const float* lse;
  uint16_t* dq;
  float *dk_acc, *dv_acc;
  const int32_t* G;
  int n_global;
  int B, H, Hkv, N, D, grp;
  int L, R, d, bs;
  float scale;
};

// NV contiguous bf16 values (NV = 2 or 4) -> fp32
template <int NV>
__device__ __forceinline__ void load_bf(const uint16_t* src, float (&x)[NV]) {
  if (NV == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(src);
    x[0] = __uint_as_float(w.x << 16);
    x[NV > 1 ? 1 : 0] = __uint_as_float(w.x & 0xFFFF0000u);
    x[NV > 2 ? 2 : 0] = __uint_as_float(w.y << 16);
    x[NV > 3 ? 3 : 0] = __uint_as_float(w.y & 0xFFFF0000u);
  } else {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(src);
    x[0] = __uint_as_float(w << 16);
    x[NV > 1 ? 1 : 0] = __uint_as_float(w & 0xFFFF0000u);
  }
}

// adds NV contiguous floats with one vector reduction (no return value)
template <int NV>
__device__ __forceinline__ void red_add(float* dst, const float (&x)[NV]) {
  if (NV == 4) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(x[0]),
                 "f"(x[NV > 1 ? 1 : 0]), "f"(x[NV > 2 ? 2 : 0]), "f"(x[NV > 3 ? 3 : 0])
                 : "memory");
  } else {
    asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(dst), "f"(x[0]),
                 "f"(x[NV > 1 ? 1 : 0])
                 : "memory");
  }
}

__device__ __forceinline__ bool is_global(const int32_t* G, int ng, int i) {
  int lo = 0, hi = ng - 1;
  while (lo <= hi) {
    const int mid = (lo + hi) >> 1;
    const int x = G[mid];
    if (x == i) return true;
    if (x < i) lo = mid + 1; else hi = mid - 1;
  }
  return false;
}

// whether key j is in the (uncut) band of query i
__device__ __forceinline__ bool in_band(const BwdParams& p, int i, int j) {
  long diff, lo, hi;
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

// Sums each of the K values (K a power of two, 2..16) over the 32 lanes of
// the warp and returns all K sums to every lane, with K - 1 + (5 - log2 K)
// exchanges for the reduction and K for the broadcast (a plain butterfly
// per value takes 5 K).  Reduction: at each of the first log2 K levels a
// lane keeps the half of its values selected by its lane bit and sends the
// other half to its partner; after them lane l holds a partial sum of one
// value, which the remaining levels complete.  Broadcast: every sum is read
// from a lane that holds it.
template <int K>
__device__ __forceinline__ void warp_allreduce(float (&v)[K], int lane) {
  constexpr int kLog = K == 2 ? 1 : (K == 4 ? 2 : (K == 8 ? 3 : 4));
  static_assert((1 << kLog) == K, "K must be 2, 4, 8 or 16");
  float w[K];
#pragma unroll
  for (int i = 0; i < K; ++i) w[i] = v[i];
#pragma unroll
  for (int lvl = 0; lvl < kLog; ++lvl) {
    const int o = 16 >> lvl;
    const int h = K >> (lvl + 1);
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < K / 2; ++i) {
      if (i < h) {
        const float send = upper ? w[i] : w[i + h];
        const float keep = upper ? w[i + h] : w[i];
        w[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
  }
#pragma unroll
  for (int o = 16 >> kLog; o > 0; o >>= 1) w[0] += __shfl_xor_sync(0xffffffffu, w[0], o);
  // the sum of value t sits in the lanes whose bits (4 - l) spell t's bits
  // (kLog - 1 - l), l = 0 .. kLog - 1
#pragma unroll
  for (int t = 0; t < K; ++t) {
    int owner = 0;
#pragma unroll
    for (int l = 0; l < kLog; ++l) owner |= ((t >> (kLog - 1 - l)) & 1) << (4 - l);
    v[t] = __shfl_sync(0xffffffffu, w[0], owner);
  }
}

template <int NV, int NQ>  // NV = D / 32 values per lane; NQ = query heads per warp
__global__ void __launch_bounds__(128) swa_bwd_rows_kernel(BwdParams p) {
  const long warp = (long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (warp >= (long)p.B * p.N * p.Hkv) return;
  const int g = (int)(warp % p.Hkv);
  const int i = (int)((warp / p.Hkv) % p.N);
  const int b = (int)(warp / ((long)p.Hkv * p.N));
  const bool causal = p.R == 0;
  const float kLog2e = 1.4426950408889634f;
  const float c2 = p.scale * kLog2e;

  // lane owns the NV contiguous columns [NV * lane, NV * lane + NV)
  const int c0 = NV * lane;
  float qv[NQ][NV], dov[NQ][NV], dq[NQ][NV], lse2[NQ], Dsum[NQ];
#pragma unroll
  for (int s = 0; s < NQ; ++s) {
    const bool ok = s < p.grp;
    const int h = g * p.grp + (ok ? s : 0);
    const long row = (((long)b * p.N + i) * p.H + h) * p.D;
    float ov[NV];
    load_bf<NV>(p.q + row + c0, qv[s]);
    load_bf<NV>(p.dout + row + c0, dov[s]);
    load_bf<NV>(p.out + row + c0, ov);
    float dsum = 0.f;
#pragma unroll
    for (int t = 0; t < NV; ++t) {
      if (!ok) qv[s][t] = dov[s][t] = 0.f;
      dsum = fmaf(dov[s][t], ov[t], dsum);
      dq[s][t] = 0.f;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
    Dsum[s] = dsum;
    lse2[s] = ok ? p.lse[((long)b * p.H + h) * p.N + i] * kLog2e : INFINITY;
  }
  const long kv_stride = (long)p.Hkv * p.D;
  const uint16_t* kb = p.k + ((long)b * p.N * p.Hkv + g) * p.D + c0;
  const uint16_t* vb = p.v + ((long)b * p.N * p.Hkv + g) * p.D + c0;
  float* dkb = p.dk_acc + ((long)b * p.N * p.Hkv + g) * p.D + c0;
  float* dvb = p.dv_acc + ((long)b * p.N * p.Hkv + g) * p.D + c0;

  // gradient contributions of NK key rows js[0..NK) (NK = 1 or 2; two rows
  // give two independent dependency chains and one shared reduction)
  auto visit_n = [&](auto nk_tag, const int (&js)[2]) {
    constexpr int NK = decltype(nk_tag)::value;
    float kv[NK][NV], vv[NK][NV];
#pragma unroll
    for (int u = 0; u < NK; ++u) {
      load_bf<NV>(kb + (long)js[u] * kv_stride, kv[u]);
      load_bf<NV>(vb + (long)js[u] * kv_stride, vv[u]);
    }
    float red[2 * NQ * NK];  // per key: scores, then dO . v, of every head
#pragma unroll
    for (int u = 0; u < NK; ++u)
#pragma unroll
      for (int s = 0; s < NQ; ++s) {
        float a = 0.f, e = 0.f;
#pragma unroll
        for (int t = 0; t < NV; ++t) {
          a = fmaf(qv[s][t], kv[u][t], a);
          e = fmaf(dov[s][t], vv[u][t], e);
        }
        red[2 * NQ * u + s] = a;
        red[2 * NQ * u + NQ + s] = e;
      }
    warp_allreduce<2 * NQ * NK>(red, lane);
#pragma unroll
    for (int u = 0; u < NK; ++u) {
      float dk[NV], dv[NV];
#pragma unroll
      for (int t = 0; t < NV; ++t) dk[t] = dv[t] = 0.f;
#pragma unroll
      for (int s = 0; s < NQ; ++s) {
        const float P = exp2f(red[2 * NQ * u + s] * c2 - lse2[s]);  // 0 for unused slots
        const float ds = P * (red[2 * NQ * u + NQ + s] - Dsum[s]);
#pragma unroll
        for (int t = 0; t < NV; ++t) {
          dq[s][t] = fmaf(ds, kv[u][t], dq[s][t]);
          dk[t] = fmaf(ds, qv[s][t], dk[t]);
          dv[t] = fmaf(P, dov[s][t], dv[t]);
        }
      }
#pragma unroll
      for (int t = 0; t < NV; ++t) dk[t] *= p.scale;
      red_add<NV>(dkb + (long)js[u] * kv_stride, dk);
      red_add<NV>(dvb + (long)js[u] * kv_stride, dv);
    }
  };
  auto visit = [&](int j) {
    const int js[2] = {j, j};
    visit_n(std::integral_constant<int, 1>(), js);
  };
  // pairs of keys where the reduction stays within 16 values
  constexpr bool kPairs = NQ <= 4;
  int pend = -1;
  auto visit_paired = [&](int j) {
    if constexpr (!kPairs) {
      visit(j);
    } else {
      if (pend < 0) {
        pend = j;
      } else {
        const int js[2] = {pend, j};
        visit_n(std::integral_constant<int, 2>(), js);
        pend = -1;
      }
    }
  };

  // the key set of row i, walked as the forward walks it
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
        const long blk = bi + mm * p.d;
        if (blk < 0 || blk >= nb) continue;
        long j1 = (blk + 1) * p.bs - 1;
        if (j1 > jmax) j1 = jmax;
        for (long j = blk * p.bs; j <= j1; ++j) visit((int)j);
      }
    } else {
      const long klo = p.L < 0 ? -(long)(i / p.d) : -(long)p.L;
      const long khi = p.R < 0 ? (long)((p.N - 1 - i) / p.d) : (long)p.R;
      for (long kk = klo; kk <= khi; ++kk) {
        const long j = i + kk * p.d;
        if (j < 0 || j > jmax) continue;
        visit_paired((int)j);
      }
      if (pend >= 0) visit(pend);
      pend = -1;
    }
    for (int t = 0; t < p.n_global; ++t) {
      int j = p.G[t];
      j = j < 0 ? 0 : (j >= p.N ? p.N - 1 : j);
      if (j > jmax || in_band(p, i, j)) continue;
      visit(j);
    }
  }

#pragma unroll
  for (int s = 0; s < NQ; ++s) {
    if (s >= p.grp) continue;
    const int h = g * p.grp + s;
    uint16_t* drow = p.dq + (((long)b * p.N + i) * p.H + h) * p.D + c0;
#pragma unroll
    for (int t = 0; t < NV; ++t)
      drow[t] = __bfloat16_as_ushort(__float2bfloat16_rn(dq[s][t] * p.scale));
  }
}

// fp32 accumulators -> bf16 gradients, 4 values per thread
__global__ void bwd_cast_kernel(const float4* __restrict__ a, uint2* __restrict__ o, long n4) {
  const long t = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n4) return;
  const float4 x = a[t];
  const uint32_t lo = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(x.x)) |
                      ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(x.y)) << 16);
  const uint32_t hi = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(x.z)) |
                      ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(x.w)) << 16);
  o[t] = make_uint2(lo, hi);
}

// library-owned fp32 accumulators for dk and dv, per device, grown on demand
constexpr int kMaxDevB = 64;
void* g_bwd_ws[kMaxDevB] = {};
size_t g_bwd_bytes[kMaxDevB] = {};
std::mutex g_bwd_mu;

float* bwd_workspace(size_t bytes, cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevB) return nullptr;
  std::lock_guard<std::mutex> lk(g_bwd_mu);
  if (g_bwd_bytes[dev] < bytes) {
    if (g_bwd_ws[dev]) {
      cudaStreamSynchronize(stream);
      ws_free(g_bwd_ws[dev]);
      g_bwd_ws[dev] = nullptr;
      g_bwd_bytes[dev] = 0;
    }
    void* ptr = ws_alloc(bytes);
    if (!ptr) return nullptr;
    g_bwd_ws[dev] = ptr;
    g_bwd_bytes[dev] = bytes;
  }
  return static_cast<float*>(g_bwd_ws[dev]);
}

template <int NV>
int launch_rows(const BwdParams& p, int nq, long blocks, cudaStream_t stream) {
  switch (nq) {
    case 1: swa_bwd_rows_kernel<NV, 1><<<(unsigned)blocks, 128, 0, stream>>>(p); break;
    case 2: swa_bwd_rows_kernel<NV, 2><<<(unsigned)blocks, 128, 0, stream>>>(p); break;
    case 4: swa_bwd_rows_kernel<NV, 4><<<(unsigned)blocks, 128, 0, stream>>>(p); break;
    case 8: swa_bwd_rows_kernel<NV, 8><<<(unsigned)blocks, 128, 0, stream>>>(p); break;
    default: return SWA_ERR_UNSUPPORTED;
  }
  return SWA_OK;
}

}  // namespace

int launch_backward(const void* q, const void* k, const void* v, const void* out,
                    const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                    int H, int Hkv, int N, int D, int L, int R, int d, int bs, const int32_t* G,
                    int ng, float scale, cudaStream_t stream) {
  if (ng == 0) {
    // band problems: the tensor-core kernels (swa_bwd_sm100.cu), with a
    // [B, H, N] fp32 workspace for Delta_i = dO_i . out_i
    float* delta = bwd_workspace((size_t)B * H * N * sizeof(float), stream);
    if (!delta) return SWA_ERR_NOMEM;
    return launch_backward_tc(q, k, v, out, dout, lse, dq, dk, dv, delta, B, H, Hkv, N, D, L, R,
                              d, bs, scale, stream);
  }
  // with global tokens (whole-sequence rows and columns of the key sets):
  // one warp per (batch, row, kv head) on CUDA cores, below
  const size_t n_kv = (size_t)B * N * Hkv * D;
  float* acc = bwd_workspace(2 * n_kv * sizeof(float), stream);
  if (!acc) return SWA_ERR_NOMEM;
  if (cudaMemsetAsync(acc, 0, 2 * n_kv * sizeof(float), stream) != cudaSuccess)
    return SWA_ERR_CUDA;
  BwdParams p;
  p.q = static_cast<const uint16_t*>(q);
  p.k = static_cast<const uint16_t*>(k);
  p.v = static_cast<const uint16_t*>(v);
  p.out = static_cast<const uint16_t*>(out);
  p.dout = static_cast<const uint16_t*>(dout);
  p.lse = lse;
  p.dq = static_cast<uint16_t*>(dq);
  p.dk_acc = acc;
  p.dv_acc = acc + n_kv;
  p.G = G;
  p.n_global = ng;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.N = N;
  p.D = D;
  p.grp = H / Hkv;
  p.L = L;
  p.R = R;
  p.d = d;
  p.bs = bs > 1 ? bs : 0;
  p.scale = scale;
  int nq = 1;
  while (nq < p.grp) nq <<= 1;
  const long warps = (long)B * N * Hkv;
  const long blocks = (warps + 3) / 4;
  if (blocks > 0x7fffffffL) return SWA_ERR_UNSUPPORTED;
  int st = D == 128 ? launch_rows<4>(p, nq, blocks, stream)
                    : (D == 64 ? launch_rows<2>(p, nq, blocks, stream) : SWA_ERR_UNSUPPORTED);
  if (st != SWA_OK) return st;
  if (cudaGetLastError() != cudaSuccess) return SWA_ERR_CUDA;
  const long n4 = (long)(n_kv / 4);
  const unsigned cb = (unsigned)((n4 + 255) / 256);
  bwd_cast_kernel<<<cb, 256, 0, stream>>>(reinterpret_cast<const float4*>(acc),
                                          static_cast<uint2*>(dk), n4);
  bwd_cast_kernel<<<cb, 256, 0, stream>>>(reinterpret_cast<const float4*>(acc + n_kv),
                                          static_cast<uint2*>(dv), n4);
  return cudaGetLastError() == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

void release_backward_workspace() {
  std::lock_guard<std::mutex> lk(g_bwd_mu);
  for (int dv = 0; dv < kMaxDevB; ++dv) {
    if (!g_bwd_ws[dv]) continue;
    int cur = 0;
    cudaGetDevice(&cur);
    cudaSetDevice(dv);
    cudaDeviceSynchronize();
    ws_free(g_bwd_ws[dv]);
    cudaSetDevice(cur);
    g_bwd_ws[dv] = nullptr;
    g_bwd_bytes[dv] = 0;
  }
}

}  // namespace swa
