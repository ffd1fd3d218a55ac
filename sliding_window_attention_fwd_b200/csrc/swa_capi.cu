// swa_capi.cu -- the extern "C" boundary of libswa.so: argument checks,
// dispatch to the kernels, device error word, host-side scheduler query.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "swa.h"
#include "swa_internal.h"
#include "swa_ptx.cuh"
#include "swa_sched.cuh"

namespace swa {

__device__ int g_device_error = 0;

namespace {

constexpr int kMaxDevices = 64;
int* g_err_ptr[kMaxDevices] = {};
std::mutex g_mu;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

__global__ void timeout_selftest_kernel(int* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nobody arrives on `bar`: the bounded wait must give up and report.
    mbar_wait(&bar, 0, err, &abort_flag, limit_ns);
  }
  __syncthreads();
}

}  // namespace

int* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<int*>(p);
  }
  return g_err_ptr[dev];
}

CUresult encode_tiled(CUtensorMap* map, CUtensorMapDataType dtype, int rank, void* base,
                      const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                      CUtensorMapSwizzle swizzle) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return CUDA_ERROR_NOT_FOUND;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
  }
  cuuint64_t d[5], s[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1;
    if (i < rank - 1) s[i] = strides_bytes[i];
  }
  return g_encode(map, dtype, (cuuint32_t)rank, base, d, s, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

namespace {
std::mutex g_alloc_mu;
swa_alloc_fn g_alloc = nullptr;
swa_free_fn g_free = nullptr;
void* g_alloc_user = nullptr;
}  // namespace

void* ws_alloc(size_t bytes) {
  std::lock_guard<std::mutex> lk(g_alloc_mu);
  if (g_alloc) return g_alloc(bytes, g_alloc_user);
  void* p = nullptr;
  return cudaMalloc(&p, bytes) == cudaSuccess ? p : nullptr;
}

void ws_free(void* ptr) {
  if (!ptr) return;
  std::lock_guard<std::mutex> lk(g_alloc_mu);
  if (g_free) g_free(ptr, g_alloc_user);
  else cudaFree(ptr);
}

int set_workspace_allocator(swa_alloc_fn alloc, swa_free_fn free_fn, void* user) {
  if ((alloc == nullptr) != (free_fn == nullptr)) return SWA_ERR_ARG;
  // blocks of the old allocator go back to it before the switch
  release_workspaces();
  release_backward_workspace();
  std::lock_guard<std::mutex> lk(g_alloc_mu);
  g_alloc = alloc;
  g_free = free_fn;
  g_alloc_user = user;
  return SWA_OK;
}

int launch_timeout_selftest(int limit_us, cudaStream_t stream) {
  int* err = device_error_word();
  if (!err) return SWA_ERR_CUDA;
  timeout_selftest_kernel<<<1, 32, 0, stream>>>(err, (uint64_t)limit_us * 1000ull);
  return cudaGetLastError() == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

}  // namespace swa

using namespace swa;

namespace {

int check_forward_args(const void* q, const void* k, const void* v, const void* out,
                       const float* lse, int B, int H, int Hkv, int N, int D, int dilation,
                       int dilation_block, const int32_t* global_idx, int n_global) {
  if (B < 0 || N < 0 || H <= 0 || Hkv <= 0 || D <= 0) return SWA_ERR_ARG;
  if (H % Hkv != 0) return SWA_ERR_ARG;
  if (dilation < 1 || dilation_block < 0) return SWA_ERR_ARG;
  if (n_global < 0 || n_global > N || (n_global > 0 && !global_idx)) return SWA_ERR_ARG;
  if (!q || !k || !v || !out) return SWA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SWA_ERR_ALIGN;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return SWA_ERR_ALIGN;
  if (global_idx && (reinterpret_cast<uintptr_t>(global_idx) & 3u)) return SWA_ERR_ALIGN;
  return SWA_OK;
}

float resolve_scale(float scale, int D) {
  return scale > 0.f ? scale : 1.0f / std::sqrt((float)D);
}

}  // namespace

extern "C" {

namespace {
int check_forward_bf16(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                       int H, int Hkv, int N, int D, int dilation, int dilation_block,
                       const int32_t* global_idx, int n_global) {
  int st = check_forward_args(q, k, v, out, lse, B, H, Hkv, N, D, dilation, dilation_block,
                              global_idx, n_global);
  if (st != SWA_OK) return st;
  if (D != 64 && D != 128) return SWA_ERR_UNSUPPORTED;
  if (dilation_block > 1 && dilation_block != kBlockRows) return SWA_ERR_UNSUPPORTED;
  return SWA_OK;
}
}  // namespace

namespace {
// The bf16 forward of one parameter block, validated by the caller.
int forward_bf16(const swa_params& p, cudaStream_t s) {
  if (p.B == 0 || p.N == 0) return SWA_OK;
  // one launch: band tiles, global-key tiles and the global query rows
  return launch_fwd_sm100(p.q, p.k, p.v, p.out, p.lse, p.B, p.H, p.Hkv, p.N, p.D, p.win_left,
                          p.win_right, p.dilation, p.dilation_block, p.global_idx, p.n_global,
                          resolve_scale(p.scale, p.D), s);
}

int forward_f32(const swa_params& p, cudaStream_t s) {
  int st = check_forward_args(p.q, p.k, p.v, p.out, p.lse, p.B, p.H, p.Hkv, p.N, p.D,
                              p.dilation, p.dilation_block, p.global_idx, p.n_global);
  if (st != SWA_OK) return st;
  if (p.D != 32 && p.D != 64 && p.D != 96 && p.D != 128) return SWA_ERR_UNSUPPORTED;
  if (p.B == 0 || p.N == 0) return SWA_OK;
  return launch_fwd_f32(static_cast<const float*>(p.q), static_cast<const float*>(p.k),
                        static_cast<const float*>(p.v), static_cast<float*>(p.out), p.lse, p.B,
                        p.H, p.Hkv, p.N, p.D, p.win_left, p.win_right, p.dilation,
                        p.dilation_block, p.global_idx, p.n_global,
                        resolve_scale(p.scale, p.D), s);
}

swa_params make_params(const void* q, const void* k, const void* v, void* out, float* lse,
                       int B, int H, int Hkv, int N, int D, int win_left, int win_right,
                       int dilation, int dilation_block, const int32_t* global_idx,
                       int n_global, float scale, int dtype) {
  swa_params p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.out = out;
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.N = N;
  p.D = D;
  p.win_left = win_left;
  p.win_right = win_right;
  p.dilation = dilation;
  p.dilation_block = dilation_block;
  p.global_idx = global_idx;
  p.n_global = n_global;
  p.scale = scale;
  p.dtype = dtype;
  return p;
}
}  // namespace

SWA_API int swa_forward_ex(const swa_params* p, void* stream) {
  if (!p) return SWA_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (p->dtype == SWA_DTYPE_F32) return forward_f32(*p, s);
  if (p->dtype != SWA_DTYPE_BF16) return SWA_ERR_ARG;
  const int st = check_forward_bf16(p->q, p->k, p->v, p->out, p->lse, p->B, p->H, p->Hkv, p->N,
                                    p->D, p->dilation, p->dilation_block, p->global_idx,
                                    p->n_global);
  if (st != SWA_OK) return st;
  return forward_bf16(*p, s);
}

SWA_API int swa_forward(const void* q, const void* k, const void* v, void* out, float* lse,
                        int B, int H, int Hkv, int N, int D, int win_left, int win_right,
                        int dilation, const int32_t* global_idx, int n_global, float scale,
                        void* stream) {
  const swa_params p = make_params(q, k, v, out, lse, B, H, Hkv, N, D, win_left, win_right,
                                   dilation, 0, global_idx, n_global, scale, SWA_DTYPE_BF16);
  return swa_forward_ex(&p, stream);
}

SWA_API int swa_forward_host(const void* q_host, const void* k_host, const void* v_host,
                             void* out_host, float* lse_host, void* q_dev, void* k_dev,
                             void* v_dev, void* out_dev, float* lse_dev, int B, int H, int Hkv,
                             int N, int D, int win_left, int win_right, int dilation,
                             int dilation_block, const int32_t* global_idx, int n_global,
                             float scale, void* stream) {
  int st = check_forward_bf16(q_dev, k_dev, v_dev, out_dev, lse_dev, B, H, Hkv, N, D, dilation,
                              dilation_block, global_idx, n_global);
  if (st != SWA_OK) return st;
  if (!q_host || !k_host || !v_host || !out_host) return SWA_ERR_ARG;
  if ((lse_host == nullptr) != (lse_dev == nullptr)) return SWA_ERR_ARG;
  if (B == 0 || N == 0) return SWA_OK;
  return forward_host(q_host, k_host, v_host, out_host, lse_host, const_cast<void*>(q_dev),
                      const_cast<void*>(k_dev), const_cast<void*>(v_dev), out_dev, lse_dev, B, H,
                      Hkv, N, D, win_left, win_right, dilation, dilation_block, global_idx,
                      n_global, resolve_scale(scale, D), static_cast<cudaStream_t>(stream));
}

SWA_API int swa_forward_layers(const swa_layer* layers, int n_layers, int B, int H, int Hkv,
                               int N, int D, int* bad_layer, void* stream) {
  if (bad_layer) *bad_layer = -1;
  if (n_layers < 0 || (n_layers > 0 && !layers)) return SWA_ERR_ARG;
  for (int i = 0; i < n_layers; ++i) {
    const swa_layer& L = layers[i];
    const int st = check_forward_bf16(L.q, L.k, L.v, L.out, L.lse, B, H, Hkv, N, D, L.dilation,
                                      L.dilation_block, L.global_idx, L.n_global);
    if (st != SWA_OK) {
      if (bad_layer) *bad_layer = i;
      return st;
    }
  }
  for (int i = 0; i < n_layers; ++i) {
    const swa_layer& L = layers[i];
    const swa_params p = make_params(L.q, L.k, L.v, L.out, L.lse, B, H, Hkv, N, D, L.win_left,
                                     L.win_right, L.dilation, L.dilation_block, L.global_idx,
                                     L.n_global, L.scale, SWA_DTYPE_BF16);
    const int st = forward_bf16(p, static_cast<cudaStream_t>(stream));
    if (st != SWA_OK) {
      if (bad_layer) *bad_layer = i;
      return st;
    }
  }
  return SWA_OK;
}

SWA_API int swa_backward(const void* q, const void* k, const void* v, const void* out,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                         int H, int Hkv, int N, int D, int win_left, int win_right, int dilation,
                         int dilation_block, const int32_t* global_idx, int n_global,
                         float scale, void* stream) {
  int st = check_forward_bf16(q, k, v, const_cast<void*>(out), nullptr, B, H, Hkv, N, D, dilation,
                              dilation_block, global_idx, n_global);
  if (st != SWA_OK) return st;
  if (!dout || !lse || !dq || !dk || !dv) return SWA_ERR_ARG;
  if (!aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return SWA_ERR_ALIGN;
  if (H / Hkv > 8) return SWA_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return SWA_OK;
  return launch_backward(q, k, v, out, dout, lse, dq, dk, dv, B, H, Hkv, N, D, win_left,
                         win_right, dilation, dilation_block, global_idx, n_global,
                         resolve_scale(scale, D), static_cast<cudaStream_t>(stream));
}

SWA_API int swa_forward_f32(const float* q, const float* k, const float* v, float* out,
                            float* lse, int B, int H, int Hkv, int N, int D, int win_left,
                            int win_right, int dilation, int dilation_block,
                            const int32_t* global_idx, int n_global, float scale,
                            void* stream) {
  const swa_params p = make_params(q, k, v, out, lse, B, H, Hkv, N, D, win_left, win_right,
                                   dilation, dilation_block, global_idx, n_global, scale,
                                   SWA_DTYPE_F32);
  return swa_forward_ex(&p, stream);
}

SWA_API int swa_decode_ex(const void* q, const void* k_ring, const void* v_ring, void* out,
                          float* lse, const int64_t* pos, int B, int H, int Hkv, int D, int W,
                          float scale, void* stream) {
  if (B < 0 || H <= 0 || Hkv <= 0 || D <= 0 || W <= 0) return SWA_ERR_ARG;
  if (H % Hkv != 0) return SWA_ERR_ARG;
  if (!q || !k_ring || !v_ring || !out || !pos) return SWA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k_ring) || !aligned16(v_ring) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(pos) & 7u))
    return SWA_ERR_ALIGN;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return SWA_ERR_ALIGN;
  if (D != 64 && D != 128) return SWA_ERR_UNSUPPORTED;
  if (H / Hkv > 8) return SWA_ERR_UNSUPPORTED;
  if (B == 0) return SWA_OK;
  return launch_decode(q, k_ring, v_ring, out, lse, pos, B, H, Hkv, D, W,
                       resolve_scale(scale, D), static_cast<cudaStream_t>(stream));
}

SWA_API int swa_decode(const void* q, const void* k_ring, const void* v_ring, void* out,
                       const int64_t* pos, int B, int H, int Hkv, int D, int W, void* stream) {
  return swa_decode_ex(q, k_ring, v_ring, out, nullptr, pos, B, H, Hkv, D, W, 0.f, stream);
}

SWA_API int swa_decode_noalloc(const void* q, const void* k_ring, const void* v_ring, void* out,
                               const int64_t* pos, int B, int H, int Hkv, int D, int W,
                               void* stream) {
  if (B < 0 || H <= 0 || Hkv <= 0 || D <= 0 || W <= 0) return SWA_ERR_ARG;
  if (H % Hkv != 0) return SWA_ERR_ARG;
  if (!q || !k_ring || !v_ring || !out || !pos) return SWA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k_ring) || !aligned16(v_ring) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(pos) & 7u))
    return SWA_ERR_ALIGN;
  if (D != 64 && D != 128) return SWA_ERR_UNSUPPORTED;
  if (H / Hkv > 8) return SWA_ERR_UNSUPPORTED;
  if (B == 0) return SWA_OK;
  return launch_decode_noalloc(q, k_ring, v_ring, out, pos, B, H, Hkv, D, W,
                               resolve_scale(0.f, D), static_cast<cudaStream_t>(stream));
}

SWA_API size_t swa_decode_noalloc_scratch_bytes(void) { return noalloc_scratch_bytes(); }

SWA_API int swa_decode_paged(const void* q, const void* k_pages, const void* v_pages, void* out,
                             float* lse, const int32_t* block_table, const int64_t* pos, int B,
                             int H, int Hkv, int D, int page_size, int num_pages, int max_pages,
                             int W, float scale, void* stream) {
  if (B < 0 || H <= 0 || Hkv <= 0 || D <= 0 || W <= 0 || page_size <= 0 || num_pages <= 0 ||
      max_pages <= 0)
    return SWA_ERR_ARG;
  if (H % Hkv != 0) return SWA_ERR_ARG;
  if (!q || !k_pages || !v_pages || !out || !block_table || !pos) return SWA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(pos) & 7u) || (reinterpret_cast<uintptr_t>(block_table) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return SWA_ERR_ALIGN;
  if (D != 64 && D != 128) return SWA_ERR_UNSUPPORTED;
  if (H / Hkv > 8 || page_size % 64 != 0) return SWA_ERR_UNSUPPORTED;
  if (B == 0) return SWA_OK;
  return launch_decode_paged(q, k_pages, v_pages, out, lse, block_table, pos, B, H, Hkv, D,
                             page_size, num_pages, max_pages, W, resolve_scale(scale, D),
                             static_cast<cudaStream_t>(stream));
}

SWA_API int swa_paged_window(int64_t pos, int W, int page_size, int64_t* first_page,
                             int64_t* last_page) {
  if (pos < 0 || W < 1 || page_size < 1 || !first_page || !last_page) return SWA_ERR_ARG;
  const int64_t first = pos - W + 1 < 0 ? 0 : pos - W + 1;
  *first_page = first / page_size;
  *last_page = pos / page_size;
  return SWA_OK;
}

SWA_API int swa_append(const void* q, const void* k_new, const void* v_new, void* k_ring,
                       void* v_ring, void* out, float* lse, const int64_t* pos0, int B, int C,
                       int H, int Hkv, int D, int W, float scale, void* stream) {
  if (B < 0 || C < 0 || H <= 0 || Hkv <= 0 || D <= 0 || W <= 0) return SWA_ERR_ARG;
  if (H % Hkv != 0) return SWA_ERR_ARG;
  if (!q || !k_new || !v_new || !k_ring || !v_ring || !out || !pos0) return SWA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_ring) ||
      !aligned16(v_ring) || !aligned16(out) || (reinterpret_cast<uintptr_t>(pos0) & 7u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return SWA_ERR_ALIGN;
  if (D != 64 && D != 128) return SWA_ERR_UNSUPPORTED;
  if (H / Hkv > 8 || W % 64 != 0 || C > 65535) return SWA_ERR_UNSUPPORTED;
  if (B == 0 || C == 0) return SWA_OK;
  return launch_append(q, k_new, v_new, k_ring, v_ring, out, lse, pos0, B, C, H, Hkv, D, W,
                       resolve_scale(scale, D), static_cast<cudaStream_t>(stream));
}

SWA_API int swa_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SWA_ERR_CUDA;
  int* err = device_error_word();
  if (!err) return SWA_ERR_CUDA;
  int h = 0;
  if (cudaMemcpy(&h, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return SWA_ERR_CUDA;
  if (h != 0) {
    int zero = 0;
    if (cudaMemcpy(err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return SWA_ERR_CUDA;
    // An aborted kernel may have left split counters mid-count.
    release_workspaces();
    return SWA_ERR_TIMEOUT;
  }
  return SWA_OK;
}

SWA_API int swa_selftest_timeout(int limit_us, void* stream) {
  if (limit_us <= 0) return SWA_ERR_ARG;
  return launch_timeout_selftest(limit_us, static_cast<cudaStream_t>(stream));
}

SWA_API int swa_schedule(int N, int win_left, int win_right, int dilation, int dilation_block,
                         int32_t* tile_out, int cap) {
  if (N < 0 || dilation < 1 || dilation_block < 0 || cap < 0) return SWA_ERR_ARG;
  if (dilation_block > 1 && dilation_block != kBlockRows) return SWA_ERR_UNSUPPORTED;
  Geometry g = make_geometry(N, win_left, win_right, dilation, dilation_block);
  int n = 0;
  for (int c = 0; c < g.nclass; ++c) {
    const int Mv = class_valid_rows(g, c);
    const int nqt = (Mv + kTileM - 1) / kTileM;
    for (int qt = 0; qt < nqt; ++qt) {
      if (tile_out && n < cap) {
        TileRange r = tile_range(g, Mv, qt);
        int ilo, ihi;
        interior_tiles(g, Mv, qt, &ilo, &ihi);
        if (ilo < r.kv_begin) ilo = r.kv_begin;
        if (ihi > r.kv_end - 1) ihi = r.kv_end - 1;
        const int edges = (r.kv_end - r.kv_begin) - (ihi >= ilo ? ihi - ilo + 1 : 0);
        int32_t* o = tile_out + 6 * n;
        o[0] = c;
        o[1] = qt;
        o[2] = qt * kTileM;
        o[3] = r.kv_begin;
        o[4] = r.kv_end;
        o[5] = edges;
      }
      ++n;
    }
  }
  return n;
}

SWA_API int swa_set_workspace_allocator(swa_alloc_fn alloc, swa_free_fn free_fn, void* user) {
  return set_workspace_allocator(alloc, free_fn, user);
}

SWA_API int swa_release(void) {
  release_workspaces();
  release_backward_workspace();
  release_host_pipes();
  return SWA_OK;
}

SWA_API const char* swa_status_string(int status) {
  switch (status) {
    case SWA_OK: return "ok";
    case SWA_ERR_ARG: return "invalid argument";
    case SWA_ERR_ALIGN: return "tensor pointer not 16-byte aligned";
    case SWA_ERR_UNSUPPORTED: return "unsupported configuration";
    case SWA_ERR_CUDA: return "CUDA error";
    case SWA_ERR_TIMEOUT: return "device-side wait timed out";
    case SWA_ERR_NOMEM: return "workspace allocation failed";
    default: return "unknown status";
  }
}

SWA_API int swa_version(void) { return 100; }

}  // extern "C"
