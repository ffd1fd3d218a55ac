/*
 * swa.h -- C ABI of libswa.so: sliding-window attention (SWA) on NVIDIA
 * B200 (sm_100a): forward (also over a per-layer schedule), backward,
 * ring-buffer and paged-cache decode, and chunked append into a ring.
 *
 * Every call is asynchronous on the CUDA stream passed as `stream` (a
 * cudaStream_t as void*; NULL = the legacy default stream).  All pointers
 * to tensors are DEVICE pointers owned by the caller; the library reads the
 * inputs and writes the outputs and keeps no reference after the call
 * returns.  Arguments are validated on the host before anything is
 * launched: on failure the call returns a negative swa_status and launches
 * nothing.  No call synchronises the stream; swa_device_error() does.
 * Library-owned device workspaces (split partials of the decode / global
 * row / paged / append kernels, the backward's accumulators) are one per device and per use: two calls that
 * use the same one must not run on the device at the same time, whichever
 * streams they are on.  Workspaces grow on demand (the growing call
 * synchronises its stream first) and are freed by swa_release().
 * Every call runs on the calling thread's current CUDA device, and the
 * stream must belong to that device.  What the library keeps (workspaces,
 * the device error word, kernel shared-memory limits) is kept per device
 * (ordinals 0-63), so one process may drive several GPUs, one current
 * device at a time.
 *
 * Definitions (page title, section):
 *  - Window and output: "滑动窗口注意力" (bmjup.com/post/11897), section
 *    "滑动窗口注意力的核心原理" 1: query i attends only the keys of its
 *    window, y_i = sum_j softmax(q_i . k_j * scale) v_j; keys outside the
 *    window are not computed at all ("别再只加Mask了", §1: real SWA skips
 *    them physically instead of masking an n x n matrix).
 *  - Causal window: "滑动窗口注意力：Mistral 的长文本“接力跑”智慧"
 *    (aiqz.cc), "Python 演示": the last window_size keys including the
 *    current token.
 *  - Dilation: "空洞滑窗机制" (mhpn.cn/news/940557), §二.1: j = i + k*d,
 *    k in [-w, w]; §四: dilation at the level of 64-token blocks, dense
 *    inside each block.
 *  - Global tokens: aiqz.cc page, "全局注意力token": a global token attends
 *    to all keys and all queries attend to it.
 *  - Ring cache: "大模型窗口扩展技术" (intelliparadigm.com), §3.1: the
 *    stream item with index t is stored in slot t % window_size.
 *
 * Key set of query i (token-level; win_left = L, win_right = R, dilation d):
 *     K(i) = { i + k*d : -L <= k <= R, 0 <= i + k*d < N }
 *            U { global keys }  U { 0 .. N-1 if i is global }
 *     and, when R == 0 (causal), only keys j <= i are kept.
 *  L < 0 (R < 0) means unbounded on the left (right).  A key is counted once
 *  even when it is both in the band and global.
 *  Block-level dilation (dilation_block = Bs > 1): with b_i = i / Bs,
 *     K(i) = union over m in [-(L / Bs), R / Bs] of the block
 *            [(b_i + m*d)*Bs, (b_i + m*d + 1)*Bs) cut to [0, N),
 *     then globals and the causal clip as above.
 *
 * Layouts (row-major, contiguous, "[batch_size, seq_len, num_heads,
 * head_dim]" as on page "别再只加Mask了", §3):
 *     q, out            [B, N, H, D]
 *     k, v              [B, N, Hkv, D]       query head h reads kv head
 *                                            h / (H / Hkv)  (GQA)
 *     lse               [B, H, N]  fp32, natural log of the softmax
 *                                  denominator: ln sum_j exp(s_ij)
 *     global_idx        [n_global] int32, sorted ascending, unique, in
 *                                  [0, N); shared by all batches and heads
 *     decode q, out     [B, H, D]
 *     k_ring, v_ring    [B, W, Hkv, D]
 *     pos               [B] int64 (device)
 */
#ifndef SWA_H_
#define SWA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SWA_API __attribute__((visibility("default")))
#else
#define SWA_API
#endif

typedef enum {
  SWA_OK = 0,
  SWA_ERR_ARG = -1,         /* null pointer, bad size, H % Hkv != 0, d < 1 ... */
  SWA_ERR_ALIGN = -2,       /* a tensor pointer is not 16-byte aligned         */
  SWA_ERR_UNSUPPORTED = -3, /* valid but not implemented (e.g. D not 64/128)   */
  SWA_ERR_CUDA = -4,        /* a CUDA runtime/driver call failed               */
  SWA_ERR_TIMEOUT = -5,     /* a device-side wait gave up (see swa_device_error) */
  SWA_ERR_NOMEM = -6        /* library workspace could not be allocated        */
} swa_status;

/*
 * swa_forward -- bf16 SWA prefill (the fused tcgen05 kernel).
 *
 * q, k, v: bf16 device tensors (layouts above).  out: bf16 [B,N,H,D].
 * lse: fp32 [B,H,N] or NULL.  D must be 64 or 128.  win_left, win_right:
 * window half-widths in dilation steps (negative = unbounded; win_right ==
 * 0 = causal).  dilation >= 1.  global_idx: device int32 array of n_global
 * entries (NULL iff n_global == 0).  scale <= 0 selects 1/sqrt(D) (the
 * "softmax_scale None" default on page "别再只加Mask了", §3).
 * With global tokens the GQA group H / Hkv must be <= 8 (else
 * SWA_ERR_UNSUPPORTED).
 * B == 0 or N == 0 is a no-op returning SWA_OK.  Without global tokens the
 * call allocates no device memory; with them, the global query rows use the
 * library-owned split workspace of the row kernel (allocated on the first
 * such call on a device, kept until swa_release).  Entries of global_idx
 * outside [0, N) are clamped when read (no out-of-bounds access) but then
 * the result is unspecified.
 */
SWA_API int swa_forward(const void* q, const void* k, const void* v, void* out,
                        float* lse, int B, int H, int Hkv, int N, int D,
                        int win_left, int win_right, int dilation,
                        const int32_t* global_idx, int n_global, float scale,
                        void* stream);

/* Element type of q, k, v and out in swa_params.dtype. */
typedef enum {
  SWA_DTYPE_BF16 = 0, /* bf16 tensors: the fused tcgen05 kernel (D 64 or 128) */
  SWA_DTYPE_F32 = 1   /* fp32 tensors: the FFMA path of swa_forward_f32     */
} swa_dtype;

/*
 * Every argument of one forward call.  Each field means what the argument
 * of the same name means for swa_forward; two more:
 *   dilation_block  <= 1: token-level dilation (as swa_forward); Bs > 1:
 *                   the dilation applies to whole Bs-token blocks
 *                   ("空洞滑窗机制" §四), dense inside each block.  The bf16
 *                   kernel supports Bs = 64 (its tile is two 64-row blocks;
 *                   other Bs > 1 return SWA_ERR_UNSUPPORTED); the fp32 path
 *                   any Bs.
 *   dtype           a swa_dtype value: the element type of q, k, v, out.
 * The struct is read during the call only.
 */
typedef struct swa_params {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* lse;
  int B, H, Hkv, N, D;
  int win_left;
  int win_right;
  int dilation;
  int dilation_block;
  const int32_t* global_idx;
  int n_global;
  float scale;
  int dtype;
} swa_params;

/*
 * swa_forward_ex -- the forward over a parameter block: swa_forward plus
 * block-level dilation and a dtype selector (swa_forward is this call with
 * dilation_block = 0 and dtype = SWA_DTYPE_BF16; swa_forward_f32 with
 * dtype = SWA_DTYPE_F32).  p == NULL or an unknown dtype is SWA_ERR_ARG.
 * Everything else (validation, errors, allocation) as for swa_forward or
 * swa_forward_f32.
 */
SWA_API int swa_forward_ex(const swa_params* p, void* stream);

/*
 * swa_forward_host -- swa_forward_ex (bf16) for inputs and outputs in host
 * memory: copies q, k, v from the host into the caller's device buffers,
 * runs the forward and copies out (and lse) back, overlapping the three.
 *   q_host, k_host, v_host, out_host [layouts as above] and lse_host
 *   [B, H, N] (or NULL): host memory, page-locked (cudaHostAlloc /
 *   cudaHostRegister) for the copies to overlap; q_dev ... lse_dev: device
 *   buffers of the same shapes (lse_dev NULL iff lse_host is NULL).
 * The query rows are copied, computed and copied back in chunks of 1024
 * rows (whole query tiles), each chunk's k / v rows just before its
 * kernel, on two library-owned copy streams and `stream` (the kernels),
 * ordered by events: the copy in of chunk c + 1, the kernel of chunk c and
 * the copy out of chunk c - 1 overlap.  Windows unbounded on the right,
 * dilation > 1, block dilation and global tokens are one chunk.  The call
 * is asynchronous on `stream` like the others: work queued on `stream`
 * before it comes first, work queued after it sees out_host / lse_host
 * complete; the host buffers must stay valid until then.  Other arguments,
 * validation and errors as for swa_forward_ex.  The first call on a device
 * creates the copy streams and their events (kept until swa_release); calls
 * on one device share them.
 */
SWA_API int swa_forward_host(const void* q_host, const void* k_host, const void* v_host,
                             void* out_host, float* lse_host, void* q_dev, void* k_dev,
                             void* v_dev, void* out_dev, float* lse_dev, int B, int H, int Hkv,
                             int N, int D, int win_left, int win_right, int dilation,
                             int dilation_block, const int32_t* global_idx, int n_global,
                             float scale, void* stream);

/*
 * One layer of a per-layer window schedule (see swa_forward_layers).  Every
 * field means what the field of the same name means in swa_params (bf16).
 */
typedef struct swa_layer {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* lse;
  int win_left;
  int win_right;
  int dilation;
  int dilation_block;
  const int32_t* global_idx;
  int n_global;
  float scale;
} swa_layer;

/*
 * swa_forward_layers -- swa_forward_ex for each of n_layers layers, in
 * order, on `stream` ("空洞滑窗机制" page, §三: models mix plain windows in
 * the lower layers, growing dilation in the middle ones and a global layer
 * every few layers or a few always-visible "attention sink" tokens).  All
 * layers share B, H, Hkv, N, D; each brings its own tensors, window,
 * dilation, global tokens and scale.  Every layer is validated before the
 * first launch: on an invalid layer nothing is launched, its index is
 * stored in *bad_layer (if not NULL) and its status is returned.
 */
SWA_API int swa_forward_layers(const swa_layer* layers, int n_layers, int B, int H, int Hkv,
                               int N, int D, int* bad_layer, void* stream);

/*
 * swa_backward -- gradients of swa_forward_ex with respect to q, k and v.
 * The pages train with the method but print no backward pass; this is the
 * derivative of the forward definition over the same key sets, with
 * P = exp(s - lse) recomputed from the forward's lse:
 *   dV_j = sum_i P_ij dO_i,  dS_ij = P_ij (dO_i . v_j - dO_i . out_i),
 *   dQ_i = scale sum_j dS_ij k_j,  dK_j = scale sum_i dS_ij q_i.
 *   q, dout, out, dq [B, N, H, D] bf16; k, v, dk, dv [B, N, Hkv, D] bf16;
 *   lse [B, H, N] fp32 (natural log) and out as written by swa_forward_ex
 *   for the same arguments; all device memory, 16-byte aligned.
 * Window arguments as for swa_forward_ex.  Runs on CUDA cores (fp32 math):
 * one warp per (batch, row, kv head) with dk / dv summed in a library-owned
 * fp32 workspace (2 * B * N * Hkv * D floats, kept until swa_release), then
 * rounded to bf16.  D in {64, 128}; H / Hkv <= 8.
 */
SWA_API int swa_backward(const void* q, const void* k, const void* v, const void* out,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                         int H, int Hkv, int N, int D, int win_left, int win_right, int dilation,
                         int dilation_block, const int32_t* global_idx, int n_global,
                         float scale, void* stream);

/*
 * swa_forward_f32 -- the same operation in fp32 (q, k, v, out are float*),
 * computed with fp32 FFMA on CUDA cores (no TF32), for callers that need
 * fp32 accuracy.  D in {32, 64, 96, 128}; any dilation_block >= 0.
 */
SWA_API int swa_forward_f32(const float* q, const float* k, const float* v,
                            float* out, float* lse, int B, int H, int Hkv, int N,
                            int D, int win_left, int win_right, int dilation,
                            int dilation_block, const int32_t* global_idx,
                            int n_global, float scale, void* stream);

/*
 * swa_decode -- one new query token per sequence against a ring-buffer KV
 * cache of W slots (bf16).  Sequence b's token is at position pos[b] >= 0;
 * the caller has already written its k/v into slot pos[b] % W.  The query
 * attends positions max(0, pos-W+1) .. pos, i.e. ring slots
 * 0 .. min(pos, W-1) (all W slots once pos >= W-1).  scale is 1/sqrt(D).
 * D must be 128 or 64; H % Hkv == 0 and H / Hkv <= 8.  Launches on
 * `stream`: at D = 128 a tensor-core kernel over parts of about 1024 slots
 * and a kernel merging the parts; at D = 64 the split-KV row kernel.
 * The first call on a device allocates a small library-owned workspace
 * (split partials and counters, kept until swa_release); make that first
 * call before capturing a CUDA graph.  Calls on different streams of one
 * device share that workspace and must not overlap.
 */
SWA_API int swa_decode(const void* q, const void* k_ring, const void* v_ring,
                       void* out, const int64_t* pos, int B, int H, int Hkv,
                       int D, int W, void* stream);

/* swa_decode_ex -- swa_decode that also writes lse [B,H] (fp32, may be NULL)
   and takes a scale (<= 0: 1/sqrt(D)). */
SWA_API int swa_decode_ex(const void* q, const void* k_ring, const void* v_ring,
                          void* out, float* lse, const int64_t* pos, int B, int H,
                          int Hkv, int D, int W, float scale, void* stream);

/*
 * swa_decode_noalloc -- swa_decode for callers that must not have the
 * library allocate device memory.  (No counterpart on the method's pages:
 * this is a deployment variant of swa_decode, same arguments, same result.)
 *
 * Who needs it: callers that route every byte of device memory through
 * their own pre-sized pool or arena (a serving engine with a fixed memory
 * budget, where a library cudaMalloc would break the budget or fragment the
 * pool), and callers on latency-critical paths that cannot accept the
 * device-wide synchronisation a cudaMalloc may imply.  swa_decode keeps its
 * split partials in a workspace it cudaMalloc's on first use; this call
 * instead uses a fixed array compiled into the library
 * (swa_decode_noalloc_scratch_bytes() bytes, 16 MiB), which every GPU that
 * loads the library holds until the process exits.  It calls no cudaMalloc,
 * cudaFree or other allocating routine.  The caller still passes inputs and
 * outputs.
 *
 * Limits and behaviour:
 *  - the array holds the split counters and the split partials: with
 *    S = B * Hkv query sets, nsplit = ceil(W / 1024) key chunks per set and
 *    nq = H/Hkv rounded up to a power of two, a problem with nsplit > 1
 *    needs round_up(S * 4, 256) + S * nsplit * nq * (D + 2) * 4 bytes; one
 *    that needs more than swa_decode_noalloc_scratch_bytes() returns
 *    SWA_ERR_UNSUPPORTED and launches nothing (W <= 1024 needs none);
 *  - the first call on a device looks up the array's device address (once
 *    per device, with that device current); make that first call before
 *    any stream capture;
 *  - every call on a device shares the one array, which keeps the last
 *    call's contents (the call clears the part that must start at zero on
 *    `stream`): calls that overlap on the GPU, e.g. on two streams, race and
 *    must be serialised by the caller.
 */
SWA_API int swa_decode_noalloc(const void* q, const void* k_ring, const void* v_ring,
                               void* out, const int64_t* pos, int B, int H, int Hkv,
                               int D, int W, void* stream);

/* swa_decode_noalloc_scratch_bytes -- size of swa_decode_noalloc's fixed
   device array, per GPU. */
SWA_API size_t swa_decode_noalloc_scratch_bytes(void);

/*
 * swa_decode_paged -- swa_decode over a paged KV cache ("空洞滑窗机制"
 * page, §四: the cache is managed in PagedAttention-style pages, and pages
 * that fall out of the window can be released).
 *   k_pages, v_pages  [num_pages * page_size, Hkv, D] bf16, device: the page
 *                     pool; page p holds rows [p * page_size, (p+1) * page_size)
 *   block_table       [B, max_pages] int32, device: token t of sequence b is
 *                     row t % page_size of page block_table[b, t / page_size]
 *   pos               [B] int64, device: position of the new token (>= 0);
 *                     its k/v are already in the pool
 *   q, out            [B, H, D] bf16; lse [B, H] fp32 natural log (may be NULL)
 * The query attends positions max(0, pos-W+1) .. pos.  Only table entries
 * for those positions are read; an entry outside [0, num_pages), or a
 * logical page >= max_pages, reads as zero keys (a caller error, never an
 * out-of-bounds access).  page_size must be a positive multiple of 64;
 * D in {64, 128}; H % Hkv == 0, H / Hkv <= 8; scale <= 0 means 1/sqrt(D).
 * Workspace, streams and graphs as for swa_decode.
 */
SWA_API int swa_decode_paged(const void* q, const void* k_pages, const void* v_pages, void* out,
                             float* lse, const int32_t* block_table, const int64_t* pos, int B,
                             int H, int Hkv, int D, int page_size, int num_pages, int max_pages,
                             int W, float scale, void* stream);

/*
 * swa_paged_window -- host-only: the logical pages [*first_page,
 * *last_page] that a decode at `pos` with window W reads; every page below
 * *first_page has left the window and can be returned to the pool (and
 * stays out: later tokens only move the window forward).  Returns
 * SWA_ERR_ARG for pos < 0, W < 1 or page_size < 1.
 */
SWA_API int swa_paged_window(int64_t pos, int W, int page_size, int64_t* first_page,
                             int64_t* last_page);

/*
 * swa_append -- a chunk of C new tokens per sequence enters a ring-buffer
 * KV cache (aiqz.cc page, "推理优化策略": streaming inference; page
 * "大模型窗口扩展技术" §3.1: position t lives in slot t % W).
 *   q      [B, C, H, D] bf16: the chunk's queries
 *   k_new, v_new [B, C, Hkv, D] bf16: the chunk's keys and values
 *   k_ring, v_ring [B, W, Hkv, D] bf16: the cache holding positions < pos0;
 *          updated in place: slot (pos0 + c) % W receives token c (of a
 *          chunk longer than W only the last W tokens stay)
 *   pos0   [B] int64, device: position of the chunk's first token (>= 0)
 *   out    [B, C, H, D] bf16; lse [B, H, C] fp32 (may be NULL)
 * Token c (position p = pos0 + c) attends positions max(0, p-W+1) .. p,
 * taking positions >= pos0 from the chunk and the others from the ring as
 * it was before the call.  W must be a positive multiple of 64; 1 <= C <=
 * 65535; D in {64, 128}; H % Hkv == 0, H / Hkv <= 8; scale <= 0 means
 * 1/sqrt(D).  Launches on `stream`: for C >= 32 the tensor-core attention
 * reading ring and chunk in place.  When its work items do not fill the
 * SMs each key walk is split over several CTAs: two parts run as a
 * cluster of two CTAs that merge each other's results on chip and, when
 * the cluster holds every reader of its kv head's ring rows (one query
 * tile, all the kv head's query heads in one item), also store the chunk
 * into the ring, all in one launch; more parts write partial results to a
 * library workspace, merged (with the ring update) by a second kernel.
 * Without a split the ring update is a second kernel.  For shorter chunks:
 * the row-kernel attention, then the ring update.  Workspace, streams and
 * graphs as for swa_decode.
 */
SWA_API int swa_append(const void* q, const void* k_new, const void* v_new, void* k_ring,
                       void* v_ring, void* out, float* lse, const int64_t* pos0, int B, int C,
                       int H, int Hkv, int D, int W, float scale, void* stream);

/*
 * swa_device_error -- synchronises `stream`, then reports (and clears) a
 * device-side timeout: every wait inside the kernels is bounded, and a wait
 * that gives up records an error word instead of hanging.  Returns SWA_OK,
 * SWA_ERR_TIMEOUT or SWA_ERR_CUDA.
 */
SWA_API int swa_device_error(void* stream);

/*
 * swa_selftest_timeout -- launches one tiny kernel that waits on an mbarrier
 * nobody arrives at, with a limit of `limit_us` microseconds, so the bounded
 * wait expires and records its error.  Used by the failure-detection test;
 * follow with swa_device_error(), which then returns SWA_ERR_TIMEOUT.
 */
SWA_API int swa_selftest_timeout(int limit_us, void* stream);

/*
 * swa_schedule -- host-only query of the band-aware tile scheduler (no GPU
 * needed).  For the forward problem (N, win_left, win_right, dilation,
 * dilation_block), writes one record of 6 int32 per query tile:
 *   { residue_class, q_tile, first_row, kv_tile_begin, kv_tile_end, n_edge }
 * where the 128-row query tile covers virtual rows [first_row,
 * first_row+128) of its residue class, it visits kv tiles [begin, end) of
 * 128 keys of the same class, and n_edge of those need the element mask
 * (the rest lie wholly inside every row's window).  Rows of residue class c
 * are the positions c, c+d, c+2d, ... (token-level) or the blocks
 * c, c+d, ... (block-level).  The global-key tiles, if any, follow the band
 * tiles and are not counted.  Returns the number of query tiles (the
 * records written are min(that, cap)), or a negative swa_status.
 * tile_out may be NULL to count only.
 */
SWA_API int swa_schedule(int N, int win_left, int win_right, int dilation,
                         int dilation_block, int32_t* tile_out, int cap);

/* swa_release -- frees every library-owned workspace (the row kernel's
   split workspaces and the backward's accumulators) and the copy streams of
   swa_forward_host on every device that has them, after synchronising that
   device; later calls make them again. */
SWA_API int swa_release(void);

/*
 * Caller-provided allocator for the library-owned workspaces (no
 * counterpart on the method's pages: a deployment hook).  alloc(bytes, user)
 * must return `bytes` of device memory on the calling thread's current
 * device (16-byte aligned) or NULL; free_fn(ptr, user) gives back a block
 * alloc returned.  Both are called with the device current, from inside
 * library calls, on the calling thread, under a library lock (they must not
 * call back into the library).  A serving engine routes the workspaces
 * through its own memory pool this way.
 */
typedef void* (*swa_alloc_fn)(size_t bytes, void* user);
typedef void (*swa_free_fn)(void* ptr, void* user);

/*
 * swa_set_workspace_allocator -- every later workspace allocation and free
 * goes through alloc / free_fn (both NULL: back to cudaMalloc / cudaFree).
 * The workspaces that exist are released first, through the allocator that
 * made them (as swa_release does).  A NULL alloc with a non-NULL free_fn, or
 * the other way round, is SWA_ERR_ARG.  When alloc returns NULL the call
 * that needed the memory returns SWA_ERR_NOMEM and launches nothing.  Call
 * it while no other library call is in progress; alloc, free_fn and user
 * must stay valid until the allocator is replaced.
 */
SWA_API int swa_set_workspace_allocator(swa_alloc_fn alloc, swa_free_fn free_fn, void* user);

/* swa_status_string -- static text for a status code. */
SWA_API const char* swa_status_string(int status);

/* swa_version -- library version, major * 10000 + minor * 100 + patch. */
SWA_API int swa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SWA_H_ */
