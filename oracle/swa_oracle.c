/*
 * swa_oracle.c -- plain, slow, fp64 CPU oracle for sliding-window attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA library; neither includes the
 * other.
 *
 * What it computes (one query at a time, over an explicit key list):
 *
 *   K(i)  = band(i) U G U (all keys if i in G), then, when win_right == 0
 *           (causal), K(i) := K(i) restricted to j <= i.            [as a set]
 *   s_ij  = scale * sum_c q[b,i,h,c] * k[b,j,g,c]      (g = h / (H/Hkv))
 *   m     = max_j s_ij,  l = sum_j exp(s_ij - m)
 *   out   = sum_j exp(s_ij - m) / l * v[b,j,g,:],   lse = m + ln l
 *
 * Sources (page title, section):
 *  - "滑动窗口注意力" (bmjup.com/post/11897), "滑动窗口注意力的核心原理" 1:
 *    window [i-(W-1)/2, i+(W-1)/2] truncated at the sequence edges, and
 *    y_i = sum_j softmax(q_i.k_j/sqrt(d)) v_j over the window only.
 *  - same page, "掩码实现": out-of-window scores become -inf, so excluded keys
 *    carry zero weight (here: they are simply not in the list).
 *  - "滑动窗口注意力：Mistral 的长文本“接力跑”智慧" (aiqz.cc), "Python 演示":
 *    the causal window is the last window_size keys including the current
 *    token, and the softmax subtracts the max before exponentiating.
 *  - same page, "全局注意力token": a global token attends to every key and
 *    every query attends to it.
 *  - "空洞滑窗机制" (mhpn.cn/news/940557), §二.1: dilated window
 *    j = i + k*d, k in [-w, w]; §四: dilation applied to whole 64-token blocks.
 *  - "大模型窗口扩展技术" (intelliparadigm.com), §3.1 RingBuffer: item t of the
 *    stream lives in slot t % size.
 *
 * Readings where the pages are silent or garbled:
 *  - win_left / win_right count dilation steps (tokens when dilation == 1);
 *    a negative value means unbounded on that side; win_right == 0 means
 *    causal, which also clips global keys and global query rows to j <= i.
 *  - block-level dilation (dilation_block = Bs > 1): with b_i = i / Bs the
 *    key set is the union of blocks b_i + m*d for m in
 *    [-(win_left / Bs), win_right / Bs], each block [b*Bs, (b+1)*Bs) cut to
 *    [0, N).  Parity for this reading is pinned only by its special cases.
 *  - decode: the query at position pos sees positions
 *    [max(0, pos-W+1), pos]; position t is read from ring slot t mod W.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef __cplusplus
extern "C" {
#endif

static int cmp_int(const void* a, const void* b) {
  int x = *(const int*)a, y = *(const int*)b;
  return (x > y) - (x < y);
}

static int in_sorted(const int* G, int ng, int x) {
  for (int t = 0; t < ng; ++t)
    if (G[t] == x) return 1;
  return 0;
}

/*
 * Explicit key list K(i) for query i, sorted ascending, no duplicates.
 * keys must have room for N entries plus n_global.  Returns |K(i)|.
 */
int oracle_key_set(int i, int N, int win_left, int win_right, int dilation,
                   int dilation_block, const int* G, int n_global, int* keys) {
  int n = 0;
  int d = dilation;
  if (dilation_block <= 1) {
    /* token-level: j = i + k*d with k in [-win_left, win_right] */
    long kmin = win_left < 0 ? -(long)(i / d) - 1 : -(long)win_left;
    long kmax = win_right < 0 ? (long)((N - 1 - i) / d) + 1 : (long)win_right;
    for (long k = kmin; k <= kmax; ++k) {
      long j = (long)i + k * d;
      if (j >= 0 && j < N) keys[n++] = (int)j;
    }
  } else {
    /* block-level: blocks b_i + m*d, m in [-(win_left/Bs), win_right/Bs] */
    int bs = dilation_block;
    int nb = (N + bs - 1) / bs;
    int bi = i / bs;
    long mmin = win_left < 0 ? -(long)(bi / d) - 1 : -(long)(win_left / bs);
    long mmax = win_right < 0 ? (long)((nb - 1 - bi) / d) + 1 : (long)(win_right / bs);
    for (long m = mmin; m <= mmax; ++m) {
      long b = (long)bi + m * d;
      if (b < 0 || b >= nb) continue;
      for (long j = b * bs; j < (b + 1) * bs && j < N; ++j) keys[n++] = (int)j;
    }
  }
  /* global keys, and every key for a global query */
  for (int t = 0; t < n_global; ++t) keys[n++] = G[t];
  if (in_sorted(G, n_global, i)) {
    n = 0;
    for (int j = 0; j < N; ++j) keys[n++] = j;
  }
  /* set semantics: sort and drop duplicates */
  qsort(keys, (size_t)n, sizeof(int), cmp_int);
  int u = 0;
  for (int t = 0; t < n; ++t)
    if (u == 0 || keys[t] != keys[u - 1]) keys[u++] = keys[t];
  n = u;
  /* causal clip */
  if (win_right == 0) {
    u = 0;
    for (int t = 0; t < n; ++t)
      if (keys[t] <= i) keys[u++] = keys[t];
    n = u;
  }
  return n;
}

/* softmax-weighted sum of the listed value rows, in fp64 */
static void attend(const float* qrow, const float* kbase, const float* vbase,
                   long kv_row_stride, const int* keys, int nk, int D,
                   double scale, double* s, double* out, double* lse) {
  double m = -INFINITY;
  for (int t = 0; t < nk; ++t) {
    const float* kr = kbase + (long)keys[t] * kv_row_stride;
    double acc = 0.0;
    for (int c = 0; c < D; ++c) acc += (double)qrow[c] * (double)kr[c];
    s[t] = scale * acc;
    if (s[t] > m) m = s[t];
  }
  double l = 0.0;
  for (int t = 0; t < nk; ++t) {
    s[t] = exp(s[t] - m);
    l += s[t];
  }
  for (int c = 0; c < D; ++c) out[c] = 0.0;
  for (int t = 0; t < nk; ++t) {
    const float* vr = vbase + (long)keys[t] * kv_row_stride;
    double w = s[t] / l;
    for (int c = 0; c < D; ++c) out[c] += w * (double)vr[c];
  }
  *lse = m + log(l);
}

typedef struct {
  const float *q, *k, *v;
  double *out, *lse;
  int B, H, Hkv, N, D, L, R, d, bs, ng;
  const int* G;
  double scale;
  const int64_t* rows; /* triples (b, h, i) or NULL */
  int64_t nrows;
  int tid, nthreads;
} fwd_job;

static void* fwd_worker(void* arg) {
  fwd_job* J = (fwd_job*)arg;
  int* keys = (int*)malloc(sizeof(int) * (size_t)(J->N + J->ng + 1));
  double* s = (double*)malloc(sizeof(double) * (size_t)(J->N + J->ng + 1));
  int64_t total = J->rows ? J->nrows : (int64_t)J->B * J->H * J->N;
  int grp = J->H / J->Hkv;
  for (int64_t r = J->tid; r < total; r += J->nthreads) {
    int b, h, i;
    if (J->rows) {
      b = (int)J->rows[3 * r];
      h = (int)J->rows[3 * r + 1];
      i = (int)J->rows[3 * r + 2];
    } else {
      b = (int)(r / ((int64_t)J->H * J->N));
      h = (int)((r / J->N) % J->H);
      i = (int)(r % J->N);
    }
    /* destination: listed rows in list order, else the [B,N,H,D] / [B,H,N]
       layouts of the library outputs */
    int64_t o_row = J->rows ? r : ((int64_t)b * J->N + i) * J->H + h;
    int64_t l_row = J->rows ? r : ((int64_t)b * J->H + h) * J->N + i;
    int g = h / grp;
    int nk = oracle_key_set(i, J->N, J->L, J->R, J->d, J->bs, J->G, J->ng, keys);
    const float* qrow = J->q + (((long)b * J->N + i) * J->H + h) * J->D;
    const float* kb = J->k + ((long)b * J->N * J->Hkv + g) * J->D;
    const float* vb = J->v + ((long)b * J->N * J->Hkv + g) * J->D;
    attend(qrow, kb, vb, (long)J->Hkv * J->D, keys, nk, J->D, J->scale, s,
           J->out + o_row * J->D, J->lse + l_row);
  }
  free(keys);
  free(s);
  return NULL;
}

/*
 * Forward oracle.  q [B,N,H,D], k and v [B,N,Hkv,D], all fp32 (bf16 inputs are
 * passed widened, which is exact).  If rows is NULL every (b,h,i) is computed
 * and out is [B,N,H,D], lse [B,H,N]; otherwise out is [nrows,D] and lse
 * [nrows] for the listed (b,h,i) triples.
 */
void oracle_forward(const float* q, const float* k, const float* v, double* out,
                    double* lse, int B, int H, int Hkv, int N, int D,
                    int win_left, int win_right, int dilation, int dilation_block,
                    const int* G, int n_global, double scale, const int64_t* rows,
                    int64_t nrows, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  fwd_job* jobs = (fwd_job*)malloc(sizeof(fwd_job) * (size_t)nthreads);
  for (int t = 0; t < nthreads; ++t) {
    fwd_job J = {q, k, v, out, lse, B, H, Hkv, N, D, win_left, win_right,
                 dilation, dilation_block, n_global, G, scale, rows, nrows,
                 t, nthreads};
    jobs[t] = J;
    pthread_create(&th[t], NULL, fwd_worker, &jobs[t]);
  }
  for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
  free(th);
  free(jobs);
}

typedef struct {
  const float *q, *kr, *vr;
  const int64_t* pos;
  double *out, *lse;
  int B, H, Hkv, D, W;
  double scale;
  int tid, nthreads;
} dec_job;

static void* dec_worker(void* arg) {
  dec_job* J = (dec_job*)arg;
  int* keys = (int*)malloc(sizeof(int) * (size_t)J->W);
  double* s = (double*)malloc(sizeof(double) * (size_t)J->W);
  int grp = J->H / J->Hkv;
  for (int64_t r = J->tid; r < (int64_t)J->B * J->H; r += J->nthreads) {
    int b = (int)(r / J->H), h = (int)(r % J->H), g = h / grp;
    int64_t p = J->pos[b];
    int64_t first = p - J->W + 1 < 0 ? 0 : p - J->W + 1;
    int nk = 0;
    for (int64_t t = first; t <= p; ++t) keys[nk++] = (int)(t % J->W);
    const float* qrow = J->q + ((long)b * J->H + h) * J->D;
    const float* kb = J->kr + ((long)b * J->W * J->Hkv + g) * J->D;
    const float* vb = J->vr + ((long)b * J->W * J->Hkv + g) * J->D;
    attend(qrow, kb, vb, (long)J->Hkv * J->D, keys, nk, J->D, J->scale, s,
           J->out + r * J->D, J->lse + r);
  }
  free(keys);
  free(s);
  return NULL;
}

/*
 * Ring-buffer decode oracle.  q [B,H,D], k_ring and v_ring [B,W,Hkv,D] (fp32),
 * pos [B].  out [B,H,D], lse [B,H].
 */
void oracle_decode(const float* q, const float* k_ring, const float* v_ring,
                   const int64_t* pos, double* out, double* lse, int B, int H,
                   int Hkv, int D, int W, double scale, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  dec_job* jobs = (dec_job*)malloc(sizeof(dec_job) * (size_t)nthreads);
  for (int t = 0; t < nthreads; ++t) {
    dec_job J = {q, k_ring, v_ring, pos, out, lse, B, H, Hkv, D, W, scale,
                 t, nthreads};
    jobs[t] = J;
    pthread_create(&th[t], NULL, dec_worker, &jobs[t]);
  }
  for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
  free(th);
  free(jobs);
}

/*
 * Paged decode oracle ("空洞滑窗机制" page, §四, KV cache management with
 * PagedAttention: the cache lives in fixed-size pages found through a block
 * table, and pages that fall out of the window can be released).  Token t
 * of sequence b sits in row block_table[b * max_pages + t / page_size] *
 * page_size + t % page_size of k_pages / v_pages ([rows, Hkv, D]).  The new
 * token at pos attends positions [max(0, pos - W + 1), pos] (the same key
 * set as the ring decode).  q [B,H,D]; out [B,H,D], lse [B,H].
 */
typedef struct {
  const float *q, *kp, *vp;
  const int32_t* table;
  const int64_t* pos;
  double *out, *lse;
  int B, H, Hkv, D, ps, max_pages, W;
  double scale;
  int tid, nthreads;
} paged_job;

static void* paged_worker(void* arg) {
  paged_job* J = (paged_job*)arg;
  int* keys = (int*)malloc(sizeof(int) * (size_t)J->W);
  double* s = (double*)malloc(sizeof(double) * (size_t)J->W);
  int grp = J->H / J->Hkv;
  for (int64_t r = J->tid; r < (int64_t)J->B * J->H; r += J->nthreads) {
    int b = (int)(r / J->H), h = (int)(r % J->H), g = h / grp;
    int64_t p = J->pos[b];
    int64_t first = p - J->W + 1 < 0 ? 0 : p - J->W + 1;
    int nk = 0;
    for (int64_t t = first; t <= p; ++t) {
      int64_t page = J->table[(int64_t)b * J->max_pages + t / J->ps];
      keys[nk++] = (int)(page * J->ps + t % J->ps);
    }
    const float* qrow = J->q + ((long)b * J->H + h) * J->D;
    attend(qrow, J->kp + (long)g * J->D, J->vp + (long)g * J->D, (long)J->Hkv * J->D, keys, nk,
           J->D, J->scale, s, J->out + r * J->D, J->lse + r);
  }
  free(keys);
  free(s);
  return NULL;
}

void oracle_decode_paged(const float* q, const float* k_pages, const float* v_pages,
                         const int32_t* block_table, const int64_t* pos, double* out,
                         double* lse, int B, int H, int Hkv, int D, int page_size,
                         int max_pages, int W, double scale, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  paged_job* jobs = (paged_job*)malloc(sizeof(paged_job) * (size_t)nthreads);
  for (int t = 0; t < nthreads; ++t) {
    paged_job J = {q, k_pages, v_pages, block_table, pos, out, lse, B, H, Hkv, D,
                   page_size, max_pages, W, scale, t, nthreads};
    jobs[t] = J;
    pthread_create(&th[t], NULL, paged_worker, &jobs[t]);
  }
  for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
  free(th);
  free(jobs);
}

/*
 * Chunked append oracle (aiqz.cc page, "推理优化策略": streaming inference
 * reads new tokens while computing and drops what leaves the window;
 * "大模型窗口扩展技术" page §3.1: position t lives in ring slot t % W).
 * C new tokens of sequence b take positions pos0[b] .. pos0[b] + C - 1.
 * Query c (position p = pos0 + c) attends positions [max(0, p - W + 1), p];
 * position t's key and value are the new token t - pos0 when t >= pos0,
 * else ring slot t % W of the cache as it was before the chunk.
 * q [B,C,H,D], k_ring / v_ring [B,W,Hkv,D], k_new / v_new [B,C,Hkv,D];
 * out [B,C,H,D], lse [B,H,C].
 */
typedef struct {
  const float *q, *kr, *vr, *kn, *vn;
  const int64_t* pos0;
  double *out, *lse;
  int B, C, H, Hkv, D, W;
  double scale;
  int tid, nthreads;
} app_job;

static void* app_worker(void* arg) {
  app_job* J = (app_job*)arg;
  const int D = J->D;
  float* kb = (float*)malloc(sizeof(float) * (size_t)J->W * D);
  float* vb = (float*)malloc(sizeof(float) * (size_t)J->W * D);
  int* keys = (int*)malloc(sizeof(int) * (size_t)J->W);
  double* s = (double*)malloc(sizeof(double) * (size_t)J->W);
  int grp = J->H / J->Hkv;
  for (int64_t r = J->tid; r < (int64_t)J->B * J->C * J->H; r += J->nthreads) {
    int h = (int)(r % J->H);
    int c = (int)((r / J->H) % J->C);
    int b = (int)(r / ((int64_t)J->H * J->C));
    int kvh = h / grp;
    int64_t p = J->pos0[b] + c;
    int64_t first = p - J->W + 1 < 0 ? 0 : p - J->W + 1;
    int nk = 0;
    for (int64_t t = first; t <= p; ++t) {
      const float *ks, *vs;
      if (t >= J->pos0[b]) {
        long row = ((long)b * J->C + (t - J->pos0[b])) * J->Hkv + kvh;
        ks = J->kn + row * D;
        vs = J->vn + row * D;
      } else {
        long row = ((long)b * J->W + t % J->W) * J->Hkv + kvh;
        ks = J->kr + row * D;
        vs = J->vr + row * D;
      }
      memcpy(kb + (size_t)nk * D, ks, sizeof(float) * (size_t)D);
      memcpy(vb + (size_t)nk * D, vs, sizeof(float) * (size_t)D);
      keys[nk] = nk;
      ++nk;
    }
    const float* qrow = J->q + r * D;
    int64_t li = ((int64_t)b * J->H + h) * J->C + c;
    attend(qrow, kb, vb, D, keys, nk, D, J->scale, s, J->out + r * D, J->lse + li);
  }
  free(kb);
  free(vb);
  free(keys);
  free(s);
  return NULL;
}

void oracle_append(const float* q, const float* k_ring, const float* v_ring,
                   const float* k_new, const float* v_new, const int64_t* pos0, double* out,
                   double* lse, int B, int C, int H, int Hkv, int D, int W, double scale,
                   int nthreads) {
  if (nthreads < 1) nthreads = 1;
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  app_job* jobs = (app_job*)malloc(sizeof(app_job) * (size_t)nthreads);
  for (int t = 0; t < nthreads; ++t) {
    app_job J = {q, k_ring, v_ring, k_new, v_new, pos0, out, lse, B, C, H, Hkv, D, W, scale,
                 t, nthreads};
    jobs[t] = J;
    pthread_create(&th[t], NULL, app_worker, &jobs[t]);
  }
  for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
  free(th);
  free(jobs);
}

/*
 * Backward oracle: gradients of the forward definition above with respect to
 * q, k and v, for an upstream gradient dout = dL/dout.  The pages use the
 * method in training but print no backward pass, so this is the derivative
 * of the definition written out (plain calculus, fp64), row by row over the
 * same key sets:
 *   P_ij  = exp(s_ij - lse_i),       s_ij = scale * q_i . k_j,  j in K(i)
 *   dV_j += P_ij dO_i
 *   dP_ij = dO_i . v_j,              D_i = sum_j P_ij dP_ij  (= dO_i . out_i)
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale * sum_j dS_ij k_j, dK_j += scale * dS_ij q_i
 * q, dout [B,N,H,D]; k, v [B,N,Hkv,D] (fp32); dq [B,N,H,D], dk, dv
 * [B,N,Hkv,D] (fp64).  Work is split by (b, kv head) so the dk / dv sums of
 * a GQA group stay in one thread.
 */
typedef struct {
  const float *q, *k, *v, *dout;
  double *dq, *dk, *dv;
  int B, H, Hkv, N, D, L, R, d, bs, ng;
  const int* G;
  double scale;
  int tid, nthreads;
} bwd_job;

static void* bwd_worker(void* arg) {
  bwd_job* J = (bwd_job*)arg;
  const int D = J->D;
  int* keys = (int*)malloc(sizeof(int) * (size_t)(J->N + J->ng + 1));
  double* s = (double*)malloc(sizeof(double) * (size_t)(J->N + J->ng + 1));
  double* dp = (double*)malloc(sizeof(double) * (size_t)(J->N + J->ng + 1));
  double* o = (double*)malloc(sizeof(double) * (size_t)D);
  int grp = J->H / J->Hkv;
  long kvs = (long)J->Hkv * D;
  for (int64_t u = J->tid; u < (int64_t)J->B * J->Hkv; u += J->nthreads) {
    int b = (int)(u / J->Hkv), g = (int)(u % J->Hkv);
    const float* kb = J->k + ((long)b * J->N * J->Hkv + g) * D;
    const float* vb = J->v + ((long)b * J->N * J->Hkv + g) * D;
    double* dkb = J->dk + ((long)b * J->N * J->Hkv + g) * D;
    double* dvb = J->dv + ((long)b * J->N * J->Hkv + g) * D;
    for (int h = g * grp; h < (g + 1) * grp; ++h) {
      for (int i = 0; i < J->N; ++i) {
        int nk = oracle_key_set(i, J->N, J->L, J->R, J->d, J->bs, J->G, J->ng, keys);
        long row = ((long)b * J->N + i) * J->H + h;
        const float* qi = J->q + row * D;
        const float* doi = J->dout + row * D;
        double m = -INFINITY;
        for (int t = 0; t < nk; ++t) {
          const float* kr = kb + (long)keys[t] * kvs;
          double acc = 0.0;
          for (int c = 0; c < D; ++c) acc += (double)qi[c] * (double)kr[c];
          s[t] = J->scale * acc;
          if (s[t] > m) m = s[t];
        }
        double l = 0.0;
        for (int t = 0; t < nk; ++t) l += exp(s[t] - m);
        double lse = m + log(l);
        /* P (in s), out_i, D_i */
        for (int c = 0; c < D; ++c) o[c] = 0.0;
        for (int t = 0; t < nk; ++t) {
          s[t] = exp(s[t] - lse);
          const float* vr = vb + (long)keys[t] * kvs;
          for (int c = 0; c < D; ++c) o[c] += s[t] * (double)vr[c];
        }
        double Di = 0.0;
        for (int c = 0; c < D; ++c) Di += (double)doi[c] * o[c];
        double* dqi = J->dq + row * D;
        for (int t = 0; t < nk; ++t) {
          const float* kr = kb + (long)keys[t] * kvs;
          const float* vr = vb + (long)keys[t] * kvs;
          double a = 0.0;
          for (int c = 0; c < D; ++c) a += (double)doi[c] * (double)vr[c];
          dp[t] = a;
          double ds = s[t] * (dp[t] - Di);
          double* dkr = dkb + (long)keys[t] * kvs;
          double* dvr = dvb + (long)keys[t] * kvs;
          for (int c = 0; c < D; ++c) {
            dqi[c] += J->scale * ds * (double)kr[c];
            dkr[c] += J->scale * ds * (double)qi[c];
            dvr[c] += s[t] * (double)doi[c];
          }
        }
      }
    }
  }
  free(keys);
  free(s);
  free(dp);
  free(o);
  return NULL;
}

void oracle_backward(const float* q, const float* k, const float* v, const float* dout,
                     double* dq, double* dk, double* dv, int B, int H, int Hkv, int N, int D,
                     int win_left, int win_right, int dilation, int dilation_block,
                     const int* G, int n_global, double scale, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  memset(dq, 0, sizeof(double) * (size_t)B * N * H * D);
  memset(dk, 0, sizeof(double) * (size_t)B * N * Hkv * D);
  memset(dv, 0, sizeof(double) * (size_t)B * N * Hkv * D);
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  bwd_job* jobs = (bwd_job*)malloc(sizeof(bwd_job) * (size_t)nthreads);
  for (int t = 0; t < nthreads; ++t) {
    bwd_job J = {q, k, v, dout, dq, dk, dv, B, H, Hkv, N, D, win_left, win_right, dilation,
                 dilation_block, n_global, G, scale, t, nthreads};
    jobs[t] = J;
    pthread_create(&th[t], NULL, bwd_worker, &jobs[t]);
  }
  for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
  free(th);
  free(jobs);
}

#ifdef __cplusplus
}
#endif
