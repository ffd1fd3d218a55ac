// swa_host.cu -- the forward for inputs and outputs that live in host
// memory: host -> device copies, the fused kernel and device -> host copies
// of one call, overlapped chunk by chunk.
//
// The query rows are cut into chunks (whole 128-row query tiles): short
// first and last chunks, long ones between.  Chunk c needs its own q rows and the k / v rows of its windows;
// with a window bounded on the right (causal, or win_right >= 0) those are
// rows below the chunk's end + win_right, most of them already copied for
// the chunks before.  Three streams: copies in (library-owned), the kernel
// (the caller's stream) and copies out (library-owned), ordered by events:
//   in:      q[c], new k / v rows  -> ev_in[c]
//   kernel:  wait ev_in[c]; forward over query tiles of chunk c -> ev_fw[c]
//   out:     wait ev_fw[c]; out[c], lse[c]
// so the host -> device copy of chunk c + 1, the kernel of chunk c and the
// device -> host copy of chunk c - 1 run at once (PCIe is full duplex).
// Windows unbounded on the right, dilation, block dilation and global tokens
// take one chunk (all of k / v is needed by the first rows).
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "swa_internal.h"
#include "swa_sched.cuh"

namespace swa {
namespace {

constexpr int kEdgeRows = 512;   // first and last chunk
constexpr int kMidRows = 2048;   // the chunks between (longer for long inputs)
constexpr int kMaxChunks = 64;   // events per device
constexpr int kMaxDevH = 64;

struct HostPipe {
  bool ready = false;
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t ev_in[kMaxChunks] = {}, ev_fw[kMaxChunks] = {};
};
HostPipe g_pipe[kMaxDevH];
std::mutex g_pipe_mu;

// The copy streams and events of the current device, created on first use.
HostPipe* host_pipe() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevH) return nullptr;
  std::lock_guard<std::mutex> lk(g_pipe_mu);
  HostPipe& hp = g_pipe[dev];
  if (!hp.ready) {
    const unsigned fl = cudaEventDisableTiming;
    if (cudaStreamCreateWithFlags(&hp.s_in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&hp.s_out, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&hp.start, fl) != cudaSuccess ||
        cudaEventCreateWithFlags(&hp.done, fl) != cudaSuccess)
      return nullptr;
    for (int i = 0; i < kMaxChunks; ++i)
      if (cudaEventCreateWithFlags(&hp.ev_in[i], fl) != cudaSuccess ||
          cudaEventCreateWithFlags(&hp.ev_fw[i], fl) != cudaSuccess)
        return nullptr;
    hp.ready = true;
  }
  return &hp;
}

// Rows [r0, r1) of every batch of a [B, N, heads, D] tensor: B runs of
// (r1 - r0) * row bytes, N * row bytes apart.
cudaError_t copy_rows(void* dst, const void* src, int B, int N, size_t row_bytes, int r0, int r1,
                      cudaMemcpyKind kind, cudaStream_t s) {
  if (r1 <= r0) return cudaSuccess;
  const size_t pitch = (size_t)N * row_bytes, off = (size_t)r0 * row_bytes;
  return cudaMemcpy2DAsync(static_cast<char*>(dst) + off, pitch,
                           static_cast<const char*>(src) + off, pitch,
                           (size_t)(r1 - r0) * row_bytes, (size_t)B, kind, s);
}

}  // namespace

int forward_host(const void* qh, const void* kh, const void* vh, void* oh, float* lh, void* qd,
                 void* kd, void* vd, void* od, float* ld, int B, int H, int Hkv, int N, int D,
                 int L, int R, int d, int bs, const int32_t* G, int ng, float scale,
                 cudaStream_t stream) {
  HostPipe* hp = host_pipe();
  if (!hp) return SWA_ERR_CUDA;
  const size_t qrow = (size_t)H * D * 2, kvrow = (size_t)Hkv * D * 2;
  const bool chunked = d == 1 && bs <= 1 && ng == 0 && R >= 0;
  // chunk boundaries (multiples of 128 rows): a short first chunk (its copy
  // in is the one nothing overlaps), long middle chunks (fewer copies), a
  // short last chunk (its kernel and copy out are the ones nothing
  // overlaps)
  int bounds[kMaxChunks + 1];
  int nchunks = 0;
  bounds[0] = 0;
  const int last0 = (N - kEdgeRows) / kTileM * kTileM;  // start of the last chunk
  if (!chunked || last0 <= kEdgeRows) {
    bounds[++nchunks] = N;
  } else {
    int mid = kMidRows;
    while ((last0 - kEdgeRows + mid - 1) / mid > kMaxChunks - 2) mid *= 2;
    int r = kEdgeRows;
    bounds[++nchunks] = r;
    while (r < last0) {
      r = r + mid < last0 ? r + mid : last0;
      bounds[++nchunks] = r;
    }
    bounds[++nchunks] = N;
  }

  // everything below runs after the work already queued on `stream`
  if (cudaEventRecord(hp->start, stream) != cudaSuccess ||
      cudaStreamWaitEvent(hp->s_in, hp->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(hp->s_out, hp->start, 0) != cudaSuccess)
    return SWA_ERR_CUDA;
  int kv_done = 0;
  for (int c = 0; c < nchunks; ++c) {
    const int n0 = bounds[c], n1 = bounds[c + 1];
    // k / v rows the chunk's windows reach (all of them when not chunked)
    const int kv_end = !chunked ? N : (n1 + R < N ? n1 + R : N);
    if (copy_rows(qd, qh, B, N, qrow, n0, n1, cudaMemcpyHostToDevice, hp->s_in) != cudaSuccess ||
        copy_rows(kd, kh, B, N, kvrow, kv_done, kv_end, cudaMemcpyHostToDevice, hp->s_in) !=
            cudaSuccess ||
        copy_rows(vd, vh, B, N, kvrow, kv_done, kv_end, cudaMemcpyHostToDevice, hp->s_in) !=
            cudaSuccess ||
        cudaEventRecord(hp->ev_in[c], hp->s_in) != cudaSuccess ||
        cudaStreamWaitEvent(stream, hp->ev_in[c], 0) != cudaSuccess)
      return SWA_ERR_CUDA;
    kv_done = kv_end > kv_done ? kv_end : kv_done;
    const int st = chunked ? launch_fwd_sm100(qd, kd, vd, od, ld, B, H, Hkv, N, D, L, R, d, 0,
                                              G, ng, scale, stream, nullptr, n0 / kTileM,
                                              (n1 + kTileM - 1) / kTileM)
                           : launch_fwd_sm100(qd, kd, vd, od, ld, B, H, Hkv, N, D, L, R, d, bs,
                                              G, ng, scale, stream);
    if (st != SWA_OK) return st;
    if (cudaEventRecord(hp->ev_fw[c], stream) != cudaSuccess ||
        cudaStreamWaitEvent(hp->s_out, hp->ev_fw[c], 0) != cudaSuccess ||
        copy_rows(oh, od, B, N, qrow, n0, n1, cudaMemcpyDeviceToHost, hp->s_out) != cudaSuccess)
      return SWA_ERR_CUDA;
    // lse [B, H, N]: B * H runs of the chunk's rows
    if (lh && copy_rows(lh, ld, B * H, N, sizeof(float), n0, n1, cudaMemcpyDeviceToHost,
                        hp->s_out) != cudaSuccess)
      return SWA_ERR_CUDA;
  }
  // later work on `stream` sees every copy done
  if (cudaEventRecord(hp->done, hp->s_out) != cudaSuccess ||
      cudaStreamWaitEvent(stream, hp->done, 0) != cudaSuccess)
    return SWA_ERR_CUDA;
  return SWA_OK;
}

void release_host_pipes() {
  std::lock_guard<std::mutex> lk(g_pipe_mu);
  for (int dv = 0; dv < kMaxDevH; ++dv) {
    HostPipe& hp = g_pipe[dv];
    if (!hp.ready) continue;
    int cur = 0;
    cudaGetDevice(&cur);
    cudaSetDevice(dv);
    cudaDeviceSynchronize();
    cudaStreamDestroy(hp.s_in);
    cudaStreamDestroy(hp.s_out);
    cudaEventDestroy(hp.start);
    cudaEventDestroy(hp.done);
    for (int i = 0; i < kMaxChunks; ++i) {
      cudaEventDestroy(hp.ev_in[i]);
      cudaEventDestroy(hp.ev_fw[i]);
    }
    cudaSetDevice(cur);
    hp = HostPipe();
  }
}

}  // namespace swa
