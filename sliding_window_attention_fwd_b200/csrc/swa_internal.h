// swa_internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "swa.h"

namespace swa {

// Raises a kernel's dynamic shared memory limit to `bytes` on the current
// device.  The attribute belongs to the kernel's instance on each device,
// so it is set once per device (devices 0-63 are remembered in `done`;
// higher ordinals set it on every call).  False on a CUDA error.
inline bool smem_attr_once(const void* kernel, int bytes, std::atomic<unsigned long long>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const unsigned long long bit = dev >= 0 && dev < 64 ? 1ull << dev : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  if (bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return true;
}

// Device error word of the current device (bounded waits write into it).
int* device_error_word();

// Device memory of the library-owned workspaces, on the current device:
// through the caller's allocator when one is set (swa_set_workspace_allocator),
// else cudaMalloc / cudaFree.  ws_alloc returns nullptr on failure.
void* ws_alloc(size_t bytes);
void ws_free(void* ptr);

// Encodes a tiled tensor map through the driver entry point (no -lcuda).
CUresult encode_tiled(CUtensorMap* map, CUtensorMapDataType dtype, int rank, void* base,
                      const uint64_t* dims, const uint64_t* strides_bytes,
                      const uint32_t* box, CUtensorMapSwizzle swizzle);

int launch_fwd_f32(const float* q, const float* k, const float* v, float* out, float* lse,
                   int B, int H, int Hkv, int N, int D, int L, int R, int d, int bs,
                   const int32_t* G, int ng, float scale, cudaStream_t stream);

// Query window of the forward (chunked append): the Mq query rows are the
// local rows of q / out / lse and sit at virtual rows q0.. of the key
// sequence, whose row v holds position pos0[b] - (win - 1) + v (device
// array; rows of negative positions are masked).
struct QueryWindow {
  const int64_t* pos0;
  int q0, Mq, win;
  // In place (chunked append with win % 64 == 0): k / v passed to the
  // launch are the rings [B, win, Hkv, D] and kn / vn the chunk [B, Mq, Hkv,
  // D]; the kernel lays the keys out per batch (see swa_fwd_sm100.cu) and
  // q0 is not used.  Otherwise k / v hold the key sequence contiguously
  // (row v: position pos0 - (win - 1) + v) and the queries sit at rows q0..
  const void* kn = nullptr;
  const void* vn = nullptr;
  // stack: two heads per 128-row tile (Mq <= 64, two slots, GQA group a
  // multiple of 4); nsplit > 1: split key walks whose partials go to part
  // (nsplit * B * H * Mq * (D + 1) floats: O / l, then lse) for a merge.
  int stack = 0;
  int nsplit = 1;
  float* part = nullptr;
  // pair: with nsplit == 2, let the two parts merge each other through a
  // cluster of two CTAs (no partials written) when the device can place the
  // clusters; ring_k / ring_v (in place): the rings the chunk kn / vn then
  // enters from inside the launch, when one cluster holds every reader of a
  // kv head's ring rows.  *done (if given) reports what the launch did:
  // bit 0 merged in pairs, bit 1 stored the chunk into the rings.
  int pair = 0;
  void* ring_k = nullptr;
  void* ring_v = nullptr;
  int* done = nullptr;
};
// Whether the forward for a query window of Mq rows would stack two heads
// per tile (the launch's slot count follows the GQA group as in
// launch_fwd_sm100).
bool fwd_qwin_stacks(int H, int Hkv, int Mq);
// qt_lo / qt_hi (token-level, d == 1, no query window): launch only the
// query tiles [qt_lo, qt_hi) of the sequence (qt_hi < 0: all).
int launch_fwd_sm100(const void* q, const void* k, const void* v, void* out, float* lse,
                     int B, int H, int Hkv, int N, int D, int L, int R, int d, int bs,
                     const int32_t* G, int ng, float scale, cudaStream_t stream,
                     const QueryWindow* qw = nullptr, int qt_lo = 0, int qt_hi = -1);

int launch_decode(const void* q, const void* k_ring, const void* v_ring, void* out,
                  float* lse, const int64_t* pos, int B, int H, int Hkv, int D, int W,
                  float scale, cudaStream_t stream);
// The tensor-core decode (D = 128, GQA group <= 8; SWA_ERR_UNSUPPORTED
// otherwise, launching nothing).
int launch_decode_tc(const void* q, const void* k_ring, const void* v_ring, void* out,
                     float* lse, const int64_t* pos, int B, int H, int Hkv, int D, int W,
                     float scale, cudaStream_t stream);
// The same over a paged cache (page_size a multiple of 64).
int launch_decode_paged_tc(const void* q, const void* k_pages, const void* v_pages, void* out,
                           float* lse, const int32_t* table, const int64_t* pos, int B, int H,
                           int Hkv, int D, int page_size, int num_pages, int max_pages, int W,
                           float scale, cudaStream_t stream);
// Library workspace `which` (one per device and use) of at least `bytes`.
bool split_workspace(int which, size_t bytes, cudaStream_t stream, float** part);
// Tensor map of a [B, rows, Hkv, D] bf16 tensor: 64-column x 64-row boxes,
// 128-byte swizzle.
int encode_kv_map(CUtensorMap* m, const void* base, int D, int Hkv, int rows, int B);
// Merges nsplit partial results: part = O / l [nsplit, B*H*C, D] fp32, then
// lse [nsplit, B*H*C]; out [B, C, H, D] bf16, lse [B, H, C] (may be NULL).
int split_merge(const float* part, void* out, float* lse, int nsplit, int B, int C, int H, int D,
                cudaStream_t stream);

// Decode with its split partials in a fixed file-scope device array (no
// allocation by the library).
int launch_decode_noalloc(const void* q, const void* k_ring, const void* v_ring, void* out,
                          const int64_t* pos, int B, int H, int Hkv, int D, int W,
                          float scale, cudaStream_t stream);
size_t noalloc_scratch_bytes();

int launch_timeout_selftest(int limit_us, cudaStream_t stream);

int launch_decode_paged(const void* q, const void* k_pages, const void* v_pages, void* out,
                        float* lse, const int32_t* table, const int64_t* pos, int B, int H,
                        int Hkv, int D, int page_size, int num_pages, int max_pages, int W,
                        float scale, cudaStream_t stream);
int launch_append(const void* q, const void* k_new, const void* v_new, void* k_ring, void* v_ring,
                  void* out, float* lse, const int64_t* pos0, int B, int C, int H, int Hkv, int D,
                  int W, float scale, cudaStream_t stream);
void release_workspaces();
// The forward over host-resident inputs and outputs (swa_host.cu).
int forward_host(const void* qh, const void* kh, const void* vh, void* oh, float* lh, void* qd,
                 void* kd, void* vd, void* od, float* ld, int B, int H, int Hkv, int N, int D,
                 int L, int R, int d, int bs, const int32_t* G, int ng, float scale,
                 cudaStream_t stream);
void release_host_pipes();
int launch_backward(const void* q, const void* k, const void* v, const void* out,
                    const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                    int H, int Hkv, int N, int D, int L, int R, int d, int bs, const int32_t* G,
                    int ng, float scale, cudaStream_t stream);
void release_backward_workspace();
// Tensor-core backward of band problems (no global tokens): dq kernel then
// dk / dv kernel; delta is a [B, H, N] fp32 workspace.
int launch_backward_tc(const void* q, const void* k, const void* v, const void* out,
                       const void* dout, const float* lse, void* dq, void* dk, void* dv,
                       float* delta, int B, int H, int Hkv, int N, int D, int L, int R, int d,
                       int bs, float scale, cudaStream_t stream);

}  // namespace swa
