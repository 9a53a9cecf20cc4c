/*
 * sparda_oracle.c -- plain, slow, fp64 CPU oracle for the SparDA hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library, and it includes no CUDA header.
 *
 * Sources (web pages about "SparDA: Sparse Decoupled Attention for Efficient
 * Long-Context LLM Inference", Fu, Xiao, Dong, Han, Villa, arXiv 2606.04511):
 *   [p4]  "SparDA: a fourth projection that lets sparse attention prefetch its
 *         own KV cache" (ai.thesatyajit.com/articles/sparda)
 *   [p1]  deepresearch2agi.pages.dev/sparda_sparse_decoupled_attention,
 *         section "架构细节" (architecture details)
 *
 * Every routine computes the plain definition in double precision, from the
 * exact values of the bf16 inputs (a bf16 is decoded exactly into a double).
 * There is no blocking, fusion or reordering beyond what the definition says.
 *
 * Readings of points the pages leave open:
 *  - block j holds token positions [j*blk, (j+1)*blk); the last block of a
 *    sequence whose length is not a multiple of blk holds fewer tokens and its
 *    compressed key is the mean over the tokens it holds;
 *  - for a query at position p, c = floor(p/blk) is its own block; the local
 *    window is the n_local blocks ending at c, [max(0, c-n_local+1), c]; the
 *    initial blocks are [0, n_init) clipped to the blocks before the window;
 *  - top-k is taken over the candidates that are neither initial nor local
 *    (blocks [n_init, c-n_local+1)), so |set| = k + n_init + n_local whenever
 *    there are at least k candidates;
 *  - the ranking is by raw score, highest first, equal scores going to the
 *    lower block index; no softmax, no scaling (a positive scale or a softmax
 *    cannot change the ranking);
 *  - the output set lists block ids in ascending order, padded with -1 to
 *    S = k + n_init + n_local entries when fewer blocks exist;
 *  - attention over a set is ordinary softmax attention over the keys of its
 *    blocks with key position <= query position (causal), scale 1/sqrt(d)
 *    unless given; query head h belongs to KV group h / (Hq/G).
 *
 * Parallelism: independent problems (one per (batch, query, group) or per
 * (batch, query, head)) are spread over a few POSIX threads; each problem is
 * computed exactly as written, so the thread count never changes a result.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ------------------------------------------------------------------------ */
/* bf16 <-> double                                                          */
/* ------------------------------------------------------------------------ */

/* A bf16 is the top 16 bits of an IEEE binary32; widening is exact. */
static double bf16_to_double(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Round a double to the nearest bf16 (8 significant bits), ties to even,
 * in one step (no intermediate float rounding).  Finite normal range only;
 * values below the bf16 normal range are flushed to signed zero. */
uint16_t oracle_double_to_bf16(double x) {
  if (x == 0.0 || isnan(x)) {
    float z = (float)x;
    uint32_t u;
    memcpy(&u, &z, sizeof u);
    return (uint16_t)(u >> 16);
  }
  int e;
  double m = frexp(x, &e);          /* x = m * 2^e, 0.5 <= |m| < 1 */
  double scaled = ldexp(m, 8);      /* 8 significant bits: |scaled| in [128, 256) */
  double r = nearbyint(scaled);     /* default rounding mode: to nearest, ties to even */
  double v = ldexp(r, e - 8);       /* exactly representable in binary32 (normal range) */
  if (fabs(v) < 1.1754943508222875e-38) v = copysign(0.0, x);
  float f = (float)v;               /* exact */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (uint16_t)(u >> 16);
}

double oracle_bf16_to_double(uint16_t h) { return bf16_to_double(h); }

/* ------------------------------------------------------------------------ */
/* a tiny parallel-for over independent problems                           */
/* ------------------------------------------------------------------------ */

typedef void (*item_fn)(void *ctx, long long item);

typedef struct {
  item_fn fn;
  void *ctx;
  long long n;
  long long next;
  pthread_mutex_t lock;
} pool_t;

static void *pool_worker(void *arg) {
  pool_t *p = (pool_t *)arg;
  for (;;) {
    pthread_mutex_lock(&p->lock);
    long long it = p->next++;
    pthread_mutex_unlock(&p->lock);
    if (it >= p->n) break;
    p->fn(p->ctx, it);
  }
  return NULL;
}

int oracle_num_threads(void) {
  const char *s = getenv("SPARDA_ORACLE_THREADS");
  int n = s ? atoi(s) : (int)sysconf(_SC_NPROCESSORS_ONLN);
  if (n < 1) n = 1;
  if (n > 256) n = 256;
  return n;
}

static void parallel_for(long long n, item_fn fn, void *ctx) {
  int nt = oracle_num_threads();
  if (nt > n) nt = (int)(n > 0 ? n : 1);
  if (nt <= 1) {
    for (long long i = 0; i < n; ++i) fn(ctx, i);
    return;
  }
  pool_t p;
  p.fn = fn;
  p.ctx = ctx;
  p.n = n;
  p.next = 0;
  pthread_mutex_init(&p.lock, NULL);
  pthread_t th[256];
  int started = 0;
  for (int t = 0; t < nt; ++t)
    if (pthread_create(&th[t], NULL, pool_worker, &p) == 0) ++started;
  if (started == 0) pool_worker(&p);
  for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
  pthread_mutex_destroy(&p.lock);
}

/* ------------------------------------------------------------------------ */
/* o1: mean-pooled compressed keys                                          */
/*   [p1] "架构细节": the top-k part scores against the block-mean of the     */
/*   layer's keys; [p4] "The problem InfLLM-V2 leaves on the table": keys    */
/*   are mean-pooled into one compressed representation per block.         */
/*                                                                          */
/*   Kc[b,g,j,:] = (1/n_j) * sum_{t in block j} K[b,g,t,:]                  */
/*   K row (b,g,t) lives at K + (b*G+g)*bg_stride + t*tok_stride (elements) */
/*   Kc is [B][G][NB][d], NB = ceil(T/blk).                                 */
/* ------------------------------------------------------------------------ */

typedef struct {
  int B, G, T, d, blk, NB;
  const uint16_t *K;
  long long bg_stride, tok_stride;
  double *kc;
  uint16_t *kc_bf16;
} compress_ctx;

static void compress_item(void *vctx, long long item) {
  compress_ctx *c = (compress_ctx *)vctx;
  long long bg = item / c->NB;
  int j = (int)(item % c->NB);
  int t0 = j * c->blk;
  int n = c->T - t0 < c->blk ? c->T - t0 : c->blk;
  for (int x = 0; x < c->d; ++x) {
    double s = 0.0;
    for (int t = 0; t < n; ++t)
      s += bf16_to_double(c->K[bg * c->bg_stride + (long long)(t0 + t) * c->tok_stride + x]);
    double mean = s / (double)n;
    long long o = item * c->d + x;
    if (c->kc) c->kc[o] = mean;
    if (c->kc_bf16) c->kc_bf16[o] = oracle_double_to_bf16(mean);
  }
}

/* o1w: the window grid of the real models (f3): compressed key w is the   */
/*   mean of the keys at positions [w*stride, w*stride + win), complete     */
/*   windows only: NW = (T - win) / stride + 1 for T >= win, else 0.        */
/*   [p4] "One Forecast head per GQA group": the test models pool their     */
/*   keys with a 32-token window at stride 16.  kw [B][G][NW][d].           */
typedef struct {
  int T, d, win, stride, NW;
  const uint16_t *K;
  long long bg_stride, tok_stride;
  double *kw;
  uint16_t *kw_bf16;
} window_ctx;

static void window_item(void *vctx, long long item) {
  window_ctx *c = (window_ctx *)vctx;
  long long bg = item / c->NW;
  int w = (int)(item % c->NW);
  int t0 = w * c->stride;
  for (int x = 0; x < c->d; ++x) {
    double s = 0.0;
    for (int t = 0; t < c->win; ++t)
      s += bf16_to_double(c->K[bg * c->bg_stride + (long long)(t0 + t) * c->tok_stride + x]);
    double mean = s / (double)c->win;
    long long o = item * c->d + x;
    if (c->kw) c->kw[o] = mean;
    if (c->kw_bf16) c->kw_bf16[o] = oracle_double_to_bf16(mean);
  }
}

int oracle_window_count(int T, int win, int stride) {
  return T >= win ? (T - win) / stride + 1 : 0;
}

void oracle_compress_windows(int B, int G, int T, int d, int win, int stride, const uint16_t *K,
                             long long bg_stride, long long tok_stride, double *kw,
                             uint16_t *kw_bf16) {
  window_ctx c;
  c.T = T; c.d = d; c.win = win; c.stride = stride;
  c.NW = oracle_window_count(T, win, stride);
  c.K = K; c.bg_stride = bg_stride; c.tok_stride = tok_stride;
  c.kw = kw; c.kw_bf16 = kw_bf16;
  parallel_for((long long)B * G * c.NW, window_item, &c);
}

void oracle_compress_keys(int B, int G, int T, int d, int blk, const uint16_t *K,
                          long long bg_stride, long long tok_stride, double *kc,
                          uint16_t *kc_bf16) {
  compress_ctx c;
  c.B = B; c.G = G; c.T = T; c.d = d; c.blk = blk;
  c.NB = (T + blk - 1) / blk;
  c.K = K; c.bg_stride = bg_stride; c.tok_stride = tok_stride;
  c.kc = kc; c.kc_bf16 = kc_bf16;
  parallel_for((long long)B * G * c.NB, compress_item, &c);
}

/* ------------------------------------------------------------------------ */
/* the three parts of a query's block set                                   */
/*   [p4] "The problem InfLLM-V2 leaves on the table", eq. B_l(i):          */
/*   B(i) = B_init  U  B_local(i)  U  B_topk(i)                             */
/* ------------------------------------------------------------------------ */

typedef struct {
  int c;          /* the query's own block */
  int init_hi;    /* initial blocks are [0, init_hi) */
  int local_lo;   /* local blocks are [local_lo, c] */
  int cand_lo;    /* top-k candidates are [cand_lo, cand_hi) */
  int cand_hi;
} block_parts;

static block_parts parts_for(int pos, int blk, int n_init, int n_local) {
  block_parts r;
  r.c = pos / blk;
  r.local_lo = r.c - n_local + 1;
  if (r.local_lo < 0) r.local_lo = 0;
  r.init_hi = n_init < r.local_lo ? n_init : r.local_lo;
  r.cand_lo = n_init;
  r.cand_hi = r.local_lo;
  if (r.cand_hi < r.cand_lo) r.cand_hi = r.cand_lo;
  return r;
}

/* ------------------------------------------------------------------------ */
/* o2: Forecast block selection (and the multi-head baseline selector)      */
/*   [p4] "The fourth projection", Eq. 4:                                   */
/*        B_{l+1} = B_init U B_local U f_top(F_l Kc_{l+1}^T, k)             */
/*   [p4] "One Forecast head per GQA group": one Forecast vector per GQA    */
/*        group, raw dot products, top-k by score with no softmax.  The     */
/*        baseline selector scores with each of the group's query heads and */
/*        sums the per-head scores before ranking (its softmax is monotone  */
/*        and is not applied: it cannot change the ranking).                */
/*                                                                          */
/*   F  [B][nq][G][nf][d]  (nf = 1: Forecast; nf = heads per group: baseline)*/
/*   Kc [B][G][NB][d]                                                       */
/*   idx [B][nq][G][S], ascending block ids, -1 padded                      */
/*   kth / kth1 [B][nq][G]: score of the k-th and (k+1)-th ranked candidate */
/*   (-inf when it does not exist)                                          */
/* ------------------------------------------------------------------------ */

typedef struct {
  double score;
  int idx;
} scored;

/* higher score first; equal scores: lower block index first */
static int cmp_rank(const void *a, const void *b) {
  const scored *x = (const scored *)a, *y = (const scored *)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  return (x->idx > y->idx) - (x->idx < y->idx);
}

static int cmp_int(const void *a, const void *b) {
  int x = *(const int *)a, y = *(const int *)b;
  return (x > y) - (x < y);
}

typedef struct {
  int B, nq, G, nf, d, blk, NB, k, n_init, n_local, q_start, S;
  int win, stride, NW;   /* window grid (f3); win = 0: one key per block */
  const uint16_t *F, *kc;
  int32_t *idx;
  double *kth, *kth1;
} select_ctx;

/* score of key row r for the scoring vectors f: sum over the nf vectors */
static double row_score(const select_ctx *c, const uint16_t *f, const uint16_t *keys, long long r) {
  double s = 0.0;
  for (int h = 0; h < c->nf; ++h) {
    double dot = 0.0;
    for (int x = 0; x < c->d; ++x)
      dot += bf16_to_double(f[h * c->d + x]) * bf16_to_double(keys[r * c->d + x]);
    s += dot;
  }
  return s;
}

static void select_item(void *vctx, long long item) {
  select_ctx *c = (select_ctx *)vctx;
  int g = (int)(item % c->G);
  long long bi = item / c->G;          /* b * nq + i */
  int i = (int)(bi % c->nq);
  int b = (int)(bi / c->nq);
  int pos = c->q_start + i;
  block_parts bp = parts_for(pos, c->blk, c->n_init, c->n_local);
  int ncand = bp.cand_hi - bp.cand_lo;

  const uint16_t *f = c->F + (((long long)b * c->nq + i) * c->G + g) * c->nf * c->d;
  const long long rows = c->win ? c->NW : c->NB;  /* key rows per (b, g) */
  const uint16_t *kc = c->kc + ((long long)b * c->G + g) * rows * c->d;

  scored *cand = (scored *)malloc(sizeof(scored) * (ncand > 0 ? ncand : 1));
  for (int n = 0; n < ncand; ++n) {
    int j = bp.cand_lo + n;
    double s;
    if (c->win == 0) {
      s = row_score(c, f, kc, j);
    } else {
      /* window grid (f3): the block's score is the largest score of the
         windows lying inside it, [ceil(j*blk/stride), ...) while the window
         ends by the block's end */
      s = -INFINITY;
      for (int w = (j * c->blk + c->stride - 1) / c->stride;
           w < c->NW && w * c->stride + c->win <= (j + 1) * c->blk; ++w) {
        double sw = row_score(c, f, kc, w);
        if (sw > s) s = sw;
      }
    }
    if (s == 0.0) s = 0.0; /* one zero */
    cand[n].score = s;
    cand[n].idx = j;
  }
  qsort(cand, ncand, sizeof(scored), cmp_rank);

  int ntop = ncand < c->k ? ncand : c->k;
  if (c->kth) c->kth[item] = (c->k >= 1 && c->k <= ncand) ? cand[c->k - 1].score : -INFINITY;
  if (c->kth1) c->kth1[item] = (c->k < ncand) ? cand[c->k].score : -INFINITY;

  int *set = (int *)malloc(sizeof(int) * (size_t)(c->S + c->n_init + c->n_local + 1));
  int m = 0;
  for (int j = 0; j < bp.init_hi; ++j) set[m++] = j;
  for (int n = 0; n < ntop; ++n) set[m++] = cand[n].idx;
  for (int j = bp.local_lo; j <= bp.c; ++j) set[m++] = j;
  qsort(set, m, sizeof(int), cmp_int);

  int32_t *out = c->idx + item * c->S;
  for (int s = 0; s < c->S; ++s) out[s] = s < m ? set[s] : -1;
  free(set);
  free(cand);
}

void oracle_select(int B, int nq, int G, int nf, int d, int blk, int NB, int k, int n_init,
                   int n_local, int q_start, const uint16_t *F, const uint16_t *kc,
                   int32_t *idx, double *kth, double *kth1) {
  select_ctx c;
  c.B = B; c.nq = nq; c.G = G; c.nf = nf; c.d = d; c.blk = blk; c.NB = NB; c.k = k;
  c.n_init = n_init; c.n_local = n_local; c.q_start = q_start;
  c.S = k + n_init + n_local;
  c.win = 0; c.stride = 0; c.NW = 0;
  c.F = F; c.kc = kc; c.idx = idx; c.kth = kth; c.kth1 = kth1;
  parallel_for((long long)B * nq * G, select_item, &c);
}

/* o2w: the same selection on the window grid (f3): a candidate block's score
 * is the largest score of the windows lying inside it (max-pooling of the
 * window scores to blocks, [p4] "Training: distilling the selector you
 * already have" names the selector's final max-pooling step).  kw is
 * [B][G][NW][d]; T is the sequence length that sets NB and NW. */
void oracle_select_windows(int B, int nq, int G, int nf, int d, int blk, int win, int stride, int T,
                           int k, int n_init, int n_local, int q_start, const uint16_t *F,
                           const uint16_t *kw, int32_t *idx, double *kth, double *kth1) {
  select_ctx c;
  c.B = B; c.nq = nq; c.G = G; c.nf = nf; c.d = d; c.blk = blk; c.NB = (T + blk - 1) / blk;
  c.k = k; c.n_init = n_init; c.n_local = n_local; c.q_start = q_start;
  c.S = k + n_init + n_local;
  c.win = win; c.stride = stride; c.NW = oracle_window_count(T, win, stride);
  c.F = F; c.kc = kw; c.idx = idx; c.kth = kth; c.kth1 = kth1;
  parallel_for((long long)B * nq * G, select_item, &c);
}

/* ------------------------------------------------------------------------ */
/* o2h: the original selector in its per-head softmax form (f3)             */
/*   [p4] "Training: distilling the selector you already have", Eq. 6: the  */
/*        original selector's shared importance score is, for each query    */
/*        head of the group, a softmax over the compressed keys of its      */
/*        scores divided by a temperature tau, summed over the group's      */
/*        heads; it is taken before the selector's final max-pooling of     */
/*        window scores to blocks.  Its top-k, minus the initial and local  */
/*        blocks, is the selected set (the same section).                   */
/*   [p4] "One Forecast head per GQA group": the baseline scores with every */
/*        query head of the group, combines, then ranks.                    */
/*                                                                          */
/*   Readings taken here:                                                   */
/*   - a head's softmax runs over every key row the query sees: on the      */
/*     block grid blocks 0..c (c = the query's own block), on the window    */
/*     grid the windows complete by the query position                      */
/*     (w*stride + win <= pos + 1).  Initial and local rows count in the    */
/*     normalisation but are not ranked (they are in the set anyway);      */
/*   - on the window grid a block weighs as much as the heaviest window     */
/*     inside it (the map of o2w), -inf when no window of it is complete;   */
/*   - ranking: higher weight first, equal weights to the lower block id.   */
/*                                                                          */
/*   Q  [B][G][nf][d]  the decode query's heads, grouped (one query token)  */
/*   kc [B][G][NR][d]  block keys (win = 0) or window keys                  */
/*   idx [B][G][S]; kth / kth1 [B][G] as o2;                                */
/*   wblk [B][G][NB] (optional): each block's weight (-inf past block c)    */
/* ------------------------------------------------------------------------ */

typedef struct {
  int B, G, nf, d, blk, win, stride, NR, NB, k, n_init, n_local, q_start, S;
  double tau;
  const uint16_t *Q, *kc;
  int32_t *idx;
  double *kth, *kth1, *wblk;
} hsm_ctx;

static void hsm_item(void *vctx, long long item) {
  hsm_ctx *c = (hsm_ctx *)vctx;
  int g = (int)(item % c->G);
  int b = (int)(item / c->G);
  int pos = c->q_start;
  block_parts bp = parts_for(pos, c->blk, c->n_init, c->n_local);
  const uint16_t *q = c->Q + ((long long)b * c->G + g) * c->nf * c->d;
  const uint16_t *kc = c->kc + ((long long)b * c->G + g) * (long long)c->NR * c->d;

  /* the key rows the query sees */
  int rows;
  if (c->win == 0) {
    rows = bp.c + 1;
  } else {
    rows = 0;
    while (rows < c->NR && rows * c->stride + c->win <= pos + 1) ++rows;
  }
  if (rows > c->NR) rows = c->NR;

  /* S[r] = sum_h softmax_r(q_h . kc_r / tau) */
  double *sc = (double *)malloc(sizeof(double) * (rows > 0 ? rows : 1));
  double *w = (double *)calloc(rows > 0 ? rows : 1, sizeof(double));
  for (int h = 0; h < c->nf; ++h) {
    double mx = -INFINITY;
    for (int r = 0; r < rows; ++r) {
      double dot = 0.0;
      for (int x = 0; x < c->d; ++x)
        dot += bf16_to_double(q[h * c->d + x]) * bf16_to_double(kc[(long long)r * c->d + x]);
      sc[r] = dot / c->tau;
      if (sc[r] > mx) mx = sc[r];
    }
    double z = 0.0;
    for (int r = 0; r < rows; ++r) z += exp(sc[r] - mx);
    for (int r = 0; r < rows; ++r) w[r] += exp(sc[r] - mx) / z;
  }

  /* block weights: the row itself, or the heaviest complete window inside */
  double *wb = (double *)malloc(sizeof(double) * (size_t)(bp.c + 1));
  for (int j = 0; j <= bp.c; ++j) {
    double v;
    if (c->win == 0) {
      v = j < rows ? w[j] : -INFINITY;
    } else {
      v = -INFINITY;
      for (int r = (j * c->blk + c->stride - 1) / c->stride;
           r < rows && r * c->stride + c->win <= (j + 1) * c->blk; ++r)
        if (w[r] > v) v = w[r];
    }
    wb[j] = v;
  }
  if (c->wblk) {
    double *o = c->wblk + item * c->NB;
    for (int j = 0; j < c->NB; ++j) o[j] = j <= bp.c ? wb[j] : -INFINITY;
  }

  int ncand = bp.cand_hi - bp.cand_lo;
  scored *cand = (scored *)malloc(sizeof(scored) * (ncand > 0 ? ncand : 1));
  for (int n = 0; n < ncand; ++n) {
    cand[n].score = wb[bp.cand_lo + n];
    cand[n].idx = bp.cand_lo + n;
  }
  qsort(cand, ncand, sizeof(scored), cmp_rank);
  int ntop = ncand < c->k ? ncand : c->k;
  if (c->kth) c->kth[item] = (c->k >= 1 && c->k <= ncand) ? cand[c->k - 1].score : -INFINITY;
  if (c->kth1) c->kth1[item] = (c->k < ncand) ? cand[c->k].score : -INFINITY;

  int *set = (int *)malloc(sizeof(int) * (size_t)(c->S + c->n_init + c->n_local + 1));
  int m = 0;
  for (int j = 0; j < bp.init_hi; ++j) set[m++] = j;
  for (int n = 0; n < ntop; ++n) set[m++] = cand[n].idx;
  for (int j = bp.local_lo; j <= bp.c; ++j) set[m++] = j;
  qsort(set, m, sizeof(int), cmp_int);
  int32_t *out = c->idx + item * c->S;
  for (int s = 0; s < c->S; ++s) out[s] = s < m ? set[s] : -1;
  free(set);
  free(cand);
  free(wb);
  free(w);
  free(sc);
}

/* win = 0: block keys, NR = NB blocks; win > 0: window keys, NR = windows of T
 * tokens.  T sets NB; the query sits at q_start (decode: T - 1). */
void oracle_select_head_softmax(int B, int G, int nf, int d, int blk, int win, int stride, int T,
                                int NR, int k, int n_init, int n_local, int q_start, double tau,
                                const uint16_t *Q, const uint16_t *kc, int32_t *idx, double *kth,
                                double *kth1, double *wblk) {
  hsm_ctx c;
  c.B = B; c.G = G; c.nf = nf; c.d = d; c.blk = blk; c.win = win; c.stride = stride;
  c.NR = NR; c.NB = (T + blk - 1) / blk; c.k = k; c.n_init = n_init; c.n_local = n_local;
  c.q_start = q_start; c.S = k + n_init + n_local; c.tau = tau;
  c.Q = Q; c.kc = kc; c.idx = idx; c.kth = kth; c.kth1 = kth1; c.wblk = wblk;
  parallel_for((long long)B * G, hsm_item, &c);
}

/* ------------------------------------------------------------------------ */
/* o3: gather of selected blocks from the host copy into device slots       */
/*   [p4] "The fourth projection", Algorithm 2: fetch(B_next, src = CPU     */
/*   pinned, dst = GPU).  The result is a byte copy: slot s of (b,g) holds  */
/*   block idx[b,g,s] (its K half then its V half).  Entries equal to -1,   */
/*   and the initial/local entries when skip_resident is set, are left      */
/*   untouched.                                                             */
/*   host_kv [B][G][NB][2][blk][d], slots [B][G][S][2][blk][d]              */
/* ------------------------------------------------------------------------ */

void oracle_gather_blocks(int B, int G, int NB, int S, int blk, int d, int pos, int n_init,
                          int n_local, int skip_resident, const uint16_t *host_kv,
                          const int32_t *idx, uint16_t *slots) {
  block_parts bp = parts_for(pos, blk, n_init, n_local);
  long long blk_elems = 2LL * blk * d;
  for (long long bg = 0; bg < (long long)B * G; ++bg) {
    for (int s = 0; s < S; ++s) {
      int j = idx[bg * S + s];
      if (j < 0 || j >= NB) continue;
      if (skip_resident && !(j >= bp.cand_lo && j < bp.cand_hi)) continue;
      memcpy(slots + (bg * S + s) * blk_elems, host_kv + (bg * NB + j) * blk_elems,
             sizeof(uint16_t) * (size_t)blk_elems);
    }
  }
}

/* ------------------------------------------------------------------------ */
/* o3c: a device slot cache across decode steps (fetch only what is new)    */
/*   [p4] "The fourth projection", Algorithm 2 fetches layer l+1's blocks   */
/*   from CPU pinned memory each step; "What this doesn't fix" notes that   */
/*   the transfer is bounded by the host link.  Blocks that stay selected   */
/*   from one step to the next need no new transfer if they stay in the     */
/*   device slots.  The pages give no policy, so the plainest one is taken: */
/*   each (b,g) owns C slots; block_of[c] is the block slot c holds (-1:    */
/*   empty) and `hand` a clock position.  For one step's list idx:          */
/*    1. an entry whose block is held in some slot c is a hit: phys = c;    */
/*    2. every other valid entry, in list order, is a miss: the hand moves  */
/*       forward (cyclically) past slots holding a block of this step's     */
/*       list, takes the next slot, and moves one further; that slot now    */
/*       holds the entry's block, phys = that slot and fetch = 1.           */
/*   Entries of -1 or outside [0, NB) get phys = -1, fetch = 0.  C >= S is  */
/*   required (a free slot then always exists).                             */
/*   idx [B][G][S]; block_of [B][G][C], hand [B][G] (updated in place);     */
/*   phys, fetch [B][G][S] (out)                                            */
/* ------------------------------------------------------------------------ */

int oracle_cache_plan(int B, int G, int S, int C, int NB, const int32_t *idx, int32_t *block_of,
                      int32_t *hand, int32_t *phys, int32_t *fetch) {
  if (C < S || C < 1) return -1;
  unsigned char *used = (unsigned char *)malloc((size_t)C);
  if (!used) return -1;
  for (long long bg = 0; bg < (long long)B * G; ++bg) {
    const int32_t *row = idx + bg * S;
    int32_t *blk = block_of + bg * C;
    int32_t *ph = phys + bg * S;
    int32_t *fe = fetch + bg * S;
    memset(used, 0, (size_t)C);
    for (int s = 0; s < S; ++s) {
      int j = row[s];
      ph[s] = -1;
      fe[s] = 0;
      if (j < 0 || j >= NB) continue;
      for (int c = 0; c < C; ++c) {
        if (blk[c] == j) {
          ph[s] = c;
          used[c] = 1;
          break;
        }
      }
    }
    for (int s = 0; s < S; ++s) {
      int j = row[s];
      if (j < 0 || j >= NB || ph[s] >= 0) continue;
      while (used[hand[bg]]) hand[bg] = (hand[bg] + 1) % C;
      int v = hand[bg];
      hand[bg] = (v + 1) % C;
      blk[v] = j;
      used[v] = 1;
      ph[s] = v;
      fe[s] = 1;
    }
  }
  free(used);
  return 0;
}

/* the cache side of o3: slot phys[s] of (b,g) receives block idx[s] for   */
/* every entry with fetch[s] set; cache [B][G][C][2][blk][d]               */
void oracle_gather_cached(int B, int G, int NB, int S, int C, int blk, int d,
                          const uint16_t *host_kv, const int32_t *idx, const int32_t *phys,
                          const int32_t *fetch, uint16_t *cache) {
  long long blk_elems = 2LL * blk * d;
  for (long long bg = 0; bg < (long long)B * G; ++bg) {
    for (int s = 0; s < S; ++s) {
      int j = idx[bg * S + s], c = phys[bg * S + s];
      if (!fetch[bg * S + s] || j < 0 || j >= NB || c < 0 || c >= C) continue;
      memcpy(cache + (bg * C + c) * blk_elems, host_kv + (bg * NB + j) * blk_elems,
             sizeof(uint16_t) * (size_t)blk_elems);
    }
  }
}

/* ------------------------------------------------------------------------ */
/* o4: attention of each query head over the keys of its block set          */
/*   [p4] "The fourth projection", Eq. 5 / Algorithm 1:                     */
/*        O_l = attention(Q_l, K_l[B_l], V_l[B_l])                          */
/*   For query token i (position pos = q_start + i) and head h of group g:  */
/*     keys  = { t : t in a block of idx[b,i,g,:], t <= pos, t < T }        */
/*     o     = sum_t softmax_t(scale * q.k_t) v_t                           */
/*   The list is read as a set: -1 entries and repeats are ignored.         */
/*   Q [B][nq][Hq][d]; O [B][nq][Hq][d] (double)                            */
/*   K/V row t of (b,g): base + (b*G+g)*bg_stride + (t/blk)*blk_stride      */
/*                       + (t%blk)*d                                        */
/* ------------------------------------------------------------------------ */

typedef struct {
  int B, nq, Hq, G, d, blk, T, q_start, S;
  double scale;
  const uint16_t *Q, *K, *V;
  long long bg_stride, blk_stride;
  const int32_t *idx;
  double *O;
} attn_ctx;

static const uint16_t *kv_row(const uint16_t *base, long long bg, int t, int blk, int d,
                              long long bg_stride, long long blk_stride) {
  return base + bg * bg_stride + (long long)(t / blk) * blk_stride + (long long)(t % blk) * d;
}

static void attn_item(void *vctx, long long item) {
  attn_ctx *c = (attn_ctx *)vctx;
  int h = (int)(item % c->Hq);
  long long bi = item / c->Hq;
  int i = (int)(bi % c->nq);
  int b = (int)(bi / c->nq);
  int r = c->Hq / c->G;
  int g = h / r;
  int pos = c->q_start + i;
  long long bg = (long long)b * c->G + g;
  const uint16_t *q = c->Q + item * c->d;
  const int32_t *set = c->idx + (bi * c->G + g) * c->S;

  /* distinct valid blocks of the set */
  int *blocks = (int *)malloc(sizeof(int) * (size_t)(c->S > 0 ? c->S : 1));
  int nb = 0;
  for (int s = 0; s < c->S; ++s) {
    int j = set[s];
    if (j < 0) continue;
    int dup = 0;
    for (int u = 0; u < nb; ++u) dup |= (blocks[u] == j);
    if (!dup) blocks[nb++] = j;
  }
  long long nkeys = (long long)nb * c->blk;
  double *logit = (double *)malloc(sizeof(double) * (size_t)(nkeys > 0 ? nkeys : 1));
  int *tok = (int *)malloc(sizeof(int) * (size_t)(nkeys > 0 ? nkeys : 1));
  long long n = 0;
  for (int u = 0; u < nb; ++u) {
    for (int w = 0; w < c->blk; ++w) {
      int t = blocks[u] * c->blk + w;
      if (t > pos || t >= c->T) continue;
      const uint16_t *k = kv_row(c->K, bg, t, c->blk, c->d, c->bg_stride, c->blk_stride);
      double dot = 0.0;
      for (int x = 0; x < c->d; ++x) dot += bf16_to_double(q[x]) * bf16_to_double(k[x]);
      logit[n] = c->scale * dot;
      tok[n] = t;
      ++n;
    }
  }
  double *o = c->O + item * c->d;
  for (int x = 0; x < c->d; ++x) o[x] = 0.0;
  if (n > 0) {
    double mx = -INFINITY;
    for (long long e = 0; e < n; ++e) mx = logit[e] > mx ? logit[e] : mx;
    double den = 0.0;
    for (long long e = 0; e < n; ++e) {
      double p = exp(logit[e] - mx);
      den += p;
      const uint16_t *v = kv_row(c->V, bg, tok[e], c->blk, c->d, c->bg_stride, c->blk_stride);
      for (int x = 0; x < c->d; ++x) o[x] += p * bf16_to_double(v[x]);
    }
    for (int x = 0; x < c->d; ++x) o[x] /= den;
  } else {
    for (int x = 0; x < c->d; ++x) o[x] = NAN; /* attention over an empty set is undefined */
  }
  free(tok);
  free(logit);
  free(blocks);
}

void oracle_sparse_attention(int B, int nq, int Hq, int G, int d, int blk, int T, int q_start,
                             double scale, const uint16_t *Q, const uint16_t *K,
                             const uint16_t *V, long long bg_stride, long long blk_stride,
                             const int32_t *idx, int S, double *O) {
  attn_ctx c;
  c.B = B; c.nq = nq; c.Hq = Hq; c.G = G; c.d = d; c.blk = blk; c.T = T;
  c.q_start = q_start; c.S = S;
  c.scale = scale > 0.0 ? scale : 1.0 / sqrt((double)d);
  c.Q = Q; c.K = K; c.V = V; c.bg_stride = bg_stride; c.blk_stride = blk_stride;
  c.idx = idx; c.O = O;
  parallel_for((long long)B * nq * Hq, attn_item, &c);
}

/* ------------------------------------------------------------------------ */
/* o5: dense causal attention, the textbook form (no blocks at all).        */
/*   When the top-k covers every candidate block, the block set is every    */
/*   block up to the query's own, and Eq. 5 reduces to this.                */
/*   Q [B][nq][Hq][d]; K/V [B][G][T][d] contiguous; O [B][nq][Hq][d]        */
/* ------------------------------------------------------------------------ */

typedef struct {
  int B, nq, Hq, G, d, T, q_start;
  double scale;
  const uint16_t *Q, *K, *V;
  double *O;
} dense_ctx;

static void dense_item(void *vctx, long long item) {
  dense_ctx *c = (dense_ctx *)vctx;
  int h = (int)(item % c->Hq);
  long long bi = item / c->Hq;
  int i = (int)(bi % c->nq);
  int b = (int)(bi / c->nq);
  int g = h / (c->Hq / c->G);
  int pos = c->q_start + i;
  int last = pos < c->T - 1 ? pos : c->T - 1;
  const uint16_t *q = c->Q + item * c->d;
  const uint16_t *K = c->K + ((long long)b * c->G + g) * c->T * c->d;
  const uint16_t *V = c->V + ((long long)b * c->G + g) * c->T * c->d;
  double *w = (double *)malloc(sizeof(double) * (size_t)(last + 1));
  double mx = -INFINITY;
  for (int t = 0; t <= last; ++t) {
    double dot = 0.0;
    for (int x = 0; x < c->d; ++x)
      dot += bf16_to_double(q[x]) * bf16_to_double(K[(long long)t * c->d + x]);
    w[t] = c->scale * dot;
    if (w[t] > mx) mx = w[t];
  }
  double den = 0.0;
  for (int t = 0; t <= last; ++t) {
    w[t] = exp(w[t] - mx);
    den += w[t];
  }
  double *o = c->O + item * c->d;
  for (int x = 0; x < c->d; ++x) {
    double acc = 0.0;
    for (int t = 0; t <= last; ++t) acc += w[t] * bf16_to_double(V[(long long)t * c->d + x]);
    o[x] = acc / den;
  }
  free(w);
}

void oracle_dense_causal_attention(int B, int nq, int Hq, int G, int d, int T, int q_start,
                                   double scale, const uint16_t *Q, const uint16_t *K,
                                   const uint16_t *V, double *O) {
  dense_ctx c;
  c.B = B; c.nq = nq; c.Hq = Hq; c.G = G; c.d = d; c.T = T; c.q_start = q_start;
  c.scale = scale > 0.0 ? scale : 1.0 / sqrt((double)d);
  c.Q = Q; c.K = K; c.V = V; c.O = O;
  parallel_for((long long)B * nq * Hq, dense_item, &c);
}
