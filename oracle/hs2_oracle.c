/*
 * hs2_oracle.c -- plain, slow, fp64 CPU oracle of the HySparse2 hot path.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's CPU
 * baseline call this code. It shares nothing with the CUDA path (no headers, no helpers,
 * no constants) and defines what "correct" means for it.
 *
 * What it computes, from the pages about "HySparse2: Hybrid Sparse Attention with
 * Two-Level KV Sharing":
 *
 *  - full_attn_select: exact causal multi-query attention (many query heads, one K/V head;
 *    arex-research.com article "小米 MiMo 负责人罗福利公开 MiMo-V3 核心架构 HySparse2",
 *    section "三套 80B-A3B 对照模型里算出的数字": 64 Q heads share one KV). The layer is
 *    also the indexer: it uses its exact attention scores to choose tokens for the
 *    following sparse layers (same article, section "外层 KV Bridging，内层 KV Reuse";
 *    toolnavs.com article, section "Was HySparse2 tut"). For every query position t the
 *    most recent `window` tokens t-window+1..t are always selected, plus the `topk`
 *    older tokens (0..t-window) with the highest score (same sections; zgeo.com.cn
 *    article, section "核心技术原理解析": last 128 plus 1,024 earlier tokens).
 *    The pages do not say how per-head scores are combined into one score per token.
 *    Reading used here: score(t, j) = sum over heads of the post-softmax probability
 *    p_h(t, j), where the softmax runs over the whole causal row 0..t; equal scores go to
 *    the lower index.
 *  - sparse_attn: a sparse layer reuses the full layer's K/V cache and selection indices
 *    unchanged and only brings its own Q (arex-research.com, section "外层 KV Bridging，
 *    内层 KV Reuse"; toolnavs.com, section "Was HySparse2 tut"); it is plain softmax
 *    attention restricted to the selected tokens (the separate SWA branch and its gate
 *    are removed, same sections).
 *  - attn_bwd: the gradients of the full layer's and the sparse layers' attention (the full
 *    layers are trained natively as indexers, arex-research.com, section "外层 KV Bridging，
 *    内层 KV Reuse"), i.e. of out = softmax(scale q K_set^T) V_set with respect to Q, K and V for
 *    a given output gradient dO, the key set of a row being its causal row (full layer) or its
 *    selected slots (sparse layer; the selection is a constant: it has no gradient). K and V
 *    gradients sum over every head and every row that reads the key.
 *  - bridge_kv_proj: KV Bridging; each cross-decoder full-attention layer l forms its own
 *    K_l = H W_k^l and V_l = H W_v^l from one shared self-decoder hidden state H
 *    (arex-research.com, section "外层 KV Bridging，内层 KV Reuse"; toolnavs.com,
 *    section "Was HySparse2 tut"). No bias, no normalisation (the pages name none).
 *
 * Causal alignment: query i of Lq sits at position t = Lk - Lq + i (Lq == Lk is prefill,
 * Lq == 1 is one decode step whose own K/V row is already the last cache row).
 *
 * Inputs are bf16 bit patterns (uint16), widened exactly to double. All arithmetic is
 * double; exp/log are libm's. Work is split over POSIX threads by independent rows only;
 * each result is computed by one thread with plain loops.
 */
#include <math.h>
#include <pthread.h>
#include <stdatomic.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORC_OK 0
#define ORC_EINVAL 1
#define ORC_EINDEX 2
#define ORC_ENOMEM 3

static double widen(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* ------------------------------------------------------------------ thread pool */
typedef void (*task_fn)(void* ctx, int64_t task, double* scratch);
typedef struct {
  task_fn fn;
  void* ctx;
  int64_t n_tasks;
  atomic_llong next;
  size_t scratch_doubles;
  atomic_int failed;
} pool_t;

static void* pool_worker(void* arg) {
  pool_t* p = (pool_t*)arg;
  double* scratch = NULL;
  if (p->scratch_doubles) {
    scratch = (double*)malloc(p->scratch_doubles * sizeof(double));
    if (!scratch) {
      atomic_store(&p->failed, 1);
      return NULL;
    }
  }
  for (;;) {
    int64_t t = atomic_fetch_add(&p->next, 1);
    if (t >= p->n_tasks) break;
    p->fn(p->ctx, t, scratch);
  }
  free(scratch);
  return NULL;
}

int oracle_default_threads(void) {
  long n = sysconf(_SC_NPROCESSORS_ONLN);
  return n > 0 ? (int)n : 1;
}

static int run_tasks(task_fn fn, void* ctx, int64_t n_tasks, size_t scratch_doubles, int n_threads) {
  if (n_tasks <= 0) return ORC_OK;
  if (n_threads <= 0) n_threads = oracle_default_threads();
  if (n_threads > n_tasks) n_threads = (int)n_tasks;
  pool_t p;
  p.fn = fn;
  p.ctx = ctx;
  p.n_tasks = n_tasks;
  atomic_init(&p.next, 0);
  p.scratch_doubles = scratch_doubles;
  atomic_init(&p.failed, 0);
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)n_threads);
  if (!th) return ORC_ENOMEM;
  int started = 0;
  for (int i = 0; i < n_threads; ++i) {
    if (pthread_create(&th[i], NULL, pool_worker, &p) == 0) started++;
    else break;
  }
  if (started == 0) pool_worker(&p);
  for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
  free(th);
  return atomic_load(&p.failed) ? ORC_ENOMEM : ORC_OK;
}

/* ------------------------------------------------------------------ full attention + selection */
typedef struct {
  const uint16_t *Q, *K, *V;
  int B, Lq, Lk, H, d, window, topk;
  double scale;
  const int64_t* rows; /* flattened (b * Lq + i) */
  int64_t n_rows;
  double* out;   /* [n_rows, H, d] */
  double* lse;   /* [n_rows, H]    natural log */
  int32_t* idx;  /* [n_rows, window + topk] */
  double* score; /* [n_rows, Lk]   head-summed probability for j <= t, 0 beyond */
  int64_t key_block;
} full_ctx;

/* logits s_j = scale * <q, k_j> for j = 0..t into s[] */
static void logits(const full_ctx* c, int b, const uint16_t* q, int t, double* s) {
  for (int j = 0; j <= t; ++j) {
    const uint16_t* k = c->K + ((int64_t)b * c->Lk + j) * c->d;
    double acc = 0.0;
    for (int x = 0; x < c->d; ++x) acc += widen(q[x]) * widen(k[x]);
    s[j] = c->scale * acc;
  }
}

/* task (row, head): lse and attention output of one head of one query */
static void full_task_head(void* vctx, int64_t task, double* s) {
  const full_ctx* c = (const full_ctx*)vctx;
  const int64_t r = task / c->H;
  const int h = (int)(task % c->H);
  const int64_t flat = c->rows[r];
  const int b = (int)(flat / c->Lq), i = (int)(flat % c->Lq);
  const int t = c->Lk - c->Lq + i;
  const uint16_t* q = c->Q + (((int64_t)b * c->Lq + i) * c->H + h) * c->d;
  logits(c, b, q, t, s);
  double m = -INFINITY;
  for (int j = 0; j <= t; ++j)
    if (s[j] > m) m = s[j];
  double sum = 0.0;
  for (int j = 0; j <= t; ++j) sum += exp(s[j] - m);
  const double lse = m + log(sum);
  c->lse[r * c->H + h] = lse;
  double* o = c->out + (r * c->H + h) * c->d;
  for (int x = 0; x < c->d; ++x) o[x] = 0.0;
  for (int j = 0; j <= t; ++j) {
    const double p = exp(s[j] - lse);
    const uint16_t* v = c->V + ((int64_t)b * c->Lk + j) * c->d;
    for (int x = 0; x < c->d; ++x) o[x] += p * widen(v[x]);
  }
}

/* task (row, key block): head-summed probability score(t, j) = sum_h exp(s_hj - lse_h) */
static void full_task_score(void* vctx, int64_t task, double* unused) {
  (void)unused;
  const full_ctx* c = (const full_ctx*)vctx;
  const int64_t nblk = (c->Lk + c->key_block - 1) / c->key_block;
  const int64_t r = task / nblk;
  const int64_t blk = task % nblk;
  const int64_t flat = c->rows[r];
  const int b = (int)(flat / c->Lq), i = (int)(flat % c->Lq);
  const int t = c->Lk - c->Lq + i;
  const int64_t j0 = blk * c->key_block;
  int64_t j1 = j0 + c->key_block;
  if (j1 > c->Lk) j1 = c->Lk;
  double* sc = c->score + r * c->Lk;
  for (int64_t j = j0; j < j1; ++j) {
    if (j > t) {
      sc[j] = 0.0;
      continue;
    }
    const uint16_t* k = c->K + ((int64_t)b * c->Lk + j) * c->d;
    double total = 0.0;
    for (int h = 0; h < c->H; ++h) {
      const uint16_t* q = c->Q + (((int64_t)b * c->Lq + i) * c->H + h) * c->d;
      double acc = 0.0;
      for (int x = 0; x < c->d; ++x) acc += widen(q[x]) * widen(k[x]);
      total += exp(c->scale * acc - c->lse[r * c->H + h]);
    }
    sc[j] = total;
  }
}

typedef struct {
  double s;
  int32_t j;
} cand_t;

/* score descending, then index ascending */
static int cand_cmp(const void* a, const void* b) {
  const cand_t* x = (const cand_t*)a;
  const cand_t* y = (const cand_t*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->j > y->j) - (x->j < y->j);
}
static int int_cmp(const void* a, const void* b) {
  const int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/* task (row): selection = window + top-k of the older tokens; ascending, -1 padded */
static void full_task_select(void* vctx, int64_t r, double* unused) {
  (void)unused;
  const full_ctx* c = (const full_ctx*)vctx;
  const int S = c->window + c->topk;
  const int64_t flat = c->rows[r];
  const int i = (int)(flat % c->Lq);
  const int t = c->Lk - c->Lq + i;
  int32_t* sel = c->idx + r * S;
  int n = 0;
  const int n_old = t - c->window + 1; /* candidates 0..t-window */
  if (n_old > 0) {
    cand_t* cs = (cand_t*)malloc(sizeof(cand_t) * (size_t)n_old);
    if (!cs) {
      for (int x = 0; x < S; ++x) sel[x] = -2; /* allocation failure marker */
      return;
    }
    const double* sc = c->score + r * c->Lk;
    for (int j = 0; j < n_old; ++j) {
      cs[j].s = sc[j];
      cs[j].j = j;
    }
    qsort(cs, (size_t)n_old, sizeof(cand_t), cand_cmp);
    const int take = n_old < c->topk ? n_old : c->topk;
    for (int x = 0; x < take; ++x) sel[n++] = cs[x].j;
    free(cs);
  }
  for (int j = (t - c->window + 1 > 0 ? t - c->window + 1 : 0); j <= t; ++j) sel[n++] = j;
  qsort(sel, (size_t)n, sizeof(int32_t), int_cmp);
  for (int x = n; x < S; ++x) sel[x] = -1;
}

/*
 * Full causal MQA attention with token selection for the query rows `rows` (flattened
 * b * Lq + i; rows == NULL means all B * Lq rows in order).
 * Q: [B, Lq, H, d]  K, V: [B, Lk, d]  (bf16 bits)
 * out: [n_rows, H, d]; lse: [n_rows, H] (natural log); idx: [n_rows, window + topk]
 * (ascending, -1 padded); score: [n_rows, Lk] (may be NULL).
 */
int oracle_full_attn_select(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int B, int Lq, int Lk, int H,
                            int d, double scale, int window, int topk, const int64_t* rows, int64_t n_rows,
                            double* out, double* lse, int32_t* idx, double* score, int n_threads) {
  if (!Q || !K || !V || !out || !lse || !idx) return ORC_EINVAL;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Lq > Lk || H <= 0 || d <= 0 || window < 0 || topk < 0) return ORC_EINVAL;
  int64_t* all = NULL;
  if (!rows) {
    n_rows = (int64_t)B * Lq;
    all = (int64_t*)malloc(sizeof(int64_t) * (size_t)n_rows);
    if (!all) return ORC_ENOMEM;
    for (int64_t r = 0; r < n_rows; ++r) all[r] = r;
    rows = all;
  }
  for (int64_t r = 0; r < n_rows; ++r)
    if (rows[r] < 0 || rows[r] >= (int64_t)B * Lq) {
      free(all);
      return ORC_EINVAL;
    }
  double* own_score = NULL;
  if (!score) {
    own_score = (double*)malloc(sizeof(double) * (size_t)n_rows * (size_t)Lk);
    if (!own_score) {
      free(all);
      return ORC_ENOMEM;
    }
    score = own_score;
  }
  full_ctx c = {Q, K, V, B, Lq, Lk, H, d, window, topk, scale, rows, n_rows, out, lse, idx, score, 4096};
  int rc = run_tasks(full_task_head, &c, n_rows * H, (size_t)Lk, n_threads);
  if (rc == ORC_OK) {
    const int64_t nblk = (Lk + c.key_block - 1) / c.key_block;
    rc = run_tasks(full_task_score, &c, n_rows * nblk, 0, n_threads);
  }
  if (rc == ORC_OK) rc = run_tasks(full_task_select, &c, n_rows, 0, n_threads);
  if (rc == ORC_OK)
    for (int64_t r = 0; r < n_rows; ++r)
      if (idx[r * (window + topk)] == -2) rc = ORC_ENOMEM;
  free(own_score);
  free(all);
  return rc;
}

/* ------------------------------------------------------------------ sparse attention */
typedef struct {
  const uint16_t *Q, *K, *V;
  const int32_t* idx; /* [B, Lq, S] */
  int B, Lq, Lk, H, d, S;
  double scale;
  const int64_t* rows;
  int64_t n_rows;
  double* out; /* [n_rows, H, d] */
  double* lse; /* [n_rows, H] */
  atomic_int bad;
} sparse_ctx;

static void sparse_task(void* vctx, int64_t task, double* s) {
  sparse_ctx* c = (sparse_ctx*)vctx;
  const int64_t r = task / c->H;
  const int h = (int)(task % c->H);
  const int64_t flat = c->rows[r];
  const int b = (int)(flat / c->Lq), i = (int)(flat % c->Lq);
  const int32_t* sel = c->idx + flat * c->S;
  const uint16_t* q = c->Q + (((int64_t)b * c->Lq + i) * c->H + h) * c->d;
  double m = -INFINITY;
  int n_valid = 0;
  for (int n = 0; n < c->S; ++n) {
    const int32_t j = sel[n];
    if (j == -1) continue;
    if (j < 0 || j >= c->Lk) {
      atomic_store(&c->bad, ORC_EINDEX);
      return;
    }
    const uint16_t* k = c->K + ((int64_t)b * c->Lk + j) * c->d;
    double acc = 0.0;
    for (int x = 0; x < c->d; ++x) acc += widen(q[x]) * widen(k[x]);
    s[n] = c->scale * acc;
    if (s[n] > m) m = s[n];
    n_valid++;
  }
  if (n_valid == 0) {
    atomic_store(&c->bad, ORC_EINDEX);
    return;
  }
  double sum = 0.0;
  for (int n = 0; n < c->S; ++n)
    if (sel[n] != -1) sum += exp(s[n] - m);
  const double lse = m + log(sum);
  c->lse[r * c->H + h] = lse;
  double* o = c->out + (r * c->H + h) * c->d;
  for (int x = 0; x < c->d; ++x) o[x] = 0.0;
  for (int n = 0; n < c->S; ++n) {
    const int32_t j = sel[n];
    if (j == -1) continue;
    const double p = exp(s[n] - lse);
    const uint16_t* v = c->V + ((int64_t)b * c->Lk + j) * c->d;
    for (int x = 0; x < c->d; ++x) o[x] += p * widen(v[x]);
  }
}

/*
 * Sparse attention of query rows `rows` over the tokens listed in idx[b, i, :] (-1 = empty
 * slot). Q: [B, Lq, H, d]; K, V: [B, Lk, d]; idx: [B, Lq, S].
 * Returns ORC_EINDEX if an index is outside [0, Lk) or a row has no valid index.
 */
int oracle_sparse_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const int32_t* idx, int B, int Lq,
                       int Lk, int H, int d, int S, double scale, const int64_t* rows, int64_t n_rows, double* out,
                       double* lse, int n_threads) {
  if (!Q || !K || !V || !idx || !out || !lse) return ORC_EINVAL;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || H <= 0 || d <= 0 || S <= 0) return ORC_EINVAL;
  int64_t* all = NULL;
  if (!rows) {
    n_rows = (int64_t)B * Lq;
    all = (int64_t*)malloc(sizeof(int64_t) * (size_t)n_rows);
    if (!all) return ORC_ENOMEM;
    for (int64_t r = 0; r < n_rows; ++r) all[r] = r;
    rows = all;
  }
  for (int64_t r = 0; r < n_rows; ++r)
    if (rows[r] < 0 || rows[r] >= (int64_t)B * Lq) {
      free(all);
      return ORC_EINVAL;
    }
  sparse_ctx c;
  c.Q = Q;
  c.K = K;
  c.V = V;
  c.idx = idx;
  c.B = B;
  c.Lq = Lq;
  c.Lk = Lk;
  c.H = H;
  c.d = d;
  c.S = S;
  c.scale = scale;
  c.rows = rows;
  c.n_rows = n_rows;
  c.out = out;
  c.lse = lse;
  atomic_init(&c.bad, 0);
  int rc = run_tasks(sparse_task, &c, n_rows * H, (size_t)S, n_threads);
  free(all);
  if (rc != ORC_OK) return rc;
  return atomic_load(&c.bad);
}

/* ------------------------------------------------------------------ attention backward */
/*
 * For one row (query i of sequence b at t = Lk - Lq + i) and head h, with key set J (the
 * causal row 0..t, or the row's selected slots):
 *   s_j = scale <q, k_j>, p_j = exp(s_j - lse), lse = log sum_j exp(s_j)   (the forward)
 *   dP_j = <dO, v_j>,  D = sum_j p_j dP_j,  dS_j = p_j (dP_j - D)
 *   dQ   = scale sum_j dS_j k_j
 *   dK_j += scale dS_j q        dV_j += p_j dO     (summed over every (row, head) reading j)
 */
typedef struct {
  const uint16_t *Q, *K, *V, *dO;
  const int32_t* idx; /* [B, Lq, S] or NULL (causal rows) */
  int B, Lq, Lk, H, d, S;
  double scale;
  const int64_t* rows;
  int64_t n_rows;
  double* dQ;    /* [n_rows, H, d] */
  double* lse;   /* [B * Lq, H] (pass 2: every row) */
  double* D;     /* [B * Lq, H] */
  double *dK, *dV;   /* [B, Lk, d] */
  const int64_t* inv_start; /* [B * Lk + 1] rows reading key (b, j): inv_rows[inv_start[.]..] */
  const int64_t* inv_rows;
  atomic_int bad;
} bwd_ctx;

/* the key of slot n of row `flat` (or -1), causal rows: slot n is key n for n <= t */
static int bwd_key(const bwd_ctx* c, int64_t flat, int n) {
  if (!c->idx) {
    const int t = c->Lk - c->Lq + (int)(flat % c->Lq);
    return n <= t ? n : -1;
  }
  return c->idx[flat * c->S + n];
}

/* task (row, head): lse, D and dQ of one head of one row; s[] holds the slots' logits */
static void bwd_task_row(void* vctx, int64_t task, double* s) {
  bwd_ctx* c = (bwd_ctx*)vctx;
  const int64_t r = task / c->H;
  const int h = (int)(task % c->H);
  const int64_t flat = c->rows[r];
  const int b = (int)(flat / c->Lq);
  const int n_slots = c->idx ? c->S : c->Lk;
  const uint16_t* q = c->Q + (flat * c->H + h) * c->d;
  const uint16_t* g = c->dO + (flat * c->H + h) * c->d;
  double m = -INFINITY;
  int n_valid = 0;
  for (int n = 0; n < n_slots; ++n) {
    const int j = bwd_key(c, flat, n);
    if (j == -1) continue;
    if (j < 0 || j >= c->Lk) {
      atomic_store(&c->bad, ORC_EINDEX);
      return;
    }
    const uint16_t* k = c->K + ((int64_t)b * c->Lk + j) * c->d;
    double acc = 0.0;
    for (int x = 0; x < c->d; ++x) acc += widen(q[x]) * widen(k[x]);
    s[n] = c->scale * acc;
    if (s[n] > m) m = s[n];
    n_valid++;
  }
  if (n_valid == 0) {
    atomic_store(&c->bad, ORC_EINDEX);
    return;
  }
  double sum = 0.0;
  for (int n = 0; n < n_slots; ++n)
    if (bwd_key(c, flat, n) != -1) sum += exp(s[n] - m);
  const double lse = m + log(sum);
  /* dP_j and D = sum_j p_j dP_j */
  double D = 0.0;
  for (int n = 0; n < n_slots; ++n) {
    const int j = bwd_key(c, flat, n);
    if (j == -1) continue;
    const uint16_t* v = c->V + ((int64_t)b * c->Lk + j) * c->d;
    double dp = 0.0;
    for (int x = 0; x < c->d; ++x) dp += widen(g[x]) * widen(v[x]);
    D += exp(s[n] - lse) * dp;
  }
  c->lse[flat * c->H + h] = lse;
  c->D[flat * c->H + h] = D;
  if (!c->dQ) return;
  double* dq = c->dQ + (r * c->H + h) * c->d;
  for (int x = 0; x < c->d; ++x) dq[x] = 0.0;
  for (int n = 0; n < n_slots; ++n) {
    const int j = bwd_key(c, flat, n);
    if (j == -1) continue;
    const uint16_t* k = c->K + ((int64_t)b * c->Lk + j) * c->d;
    const uint16_t* v = c->V + ((int64_t)b * c->Lk + j) * c->d;
    double dp = 0.0;
    for (int x = 0; x < c->d; ++x) dp += widen(g[x]) * widen(v[x]);
    const double ds = exp(s[n] - lse) * (dp - D);
    for (int x = 0; x < c->d; ++x) dq[x] += c->scale * ds * widen(k[x]);
  }
}

/* task (sequence, key): dK and dV of one key, from every (row, head) whose set reads it */
static void bwd_task_key(void* vctx, int64_t task, double* unused) {
  (void)unused;
  bwd_ctx* c = (bwd_ctx*)vctx;
  const int b = (int)(task / c->Lk);
  const int j = (int)(task % c->Lk);
  const uint16_t* k = c->K + ((int64_t)b * c->Lk + j) * c->d;
  const uint16_t* v = c->V + ((int64_t)b * c->Lk + j) * c->d;
  double* dk = c->dK + ((int64_t)b * c->Lk + j) * c->d;
  double* dv = c->dV + ((int64_t)b * c->Lk + j) * c->d;
  for (int x = 0; x < c->d; ++x) dk[x] = dv[x] = 0.0;
  int64_t r0, r1;
  if (c->idx) {
    r0 = c->inv_start[task];
    r1 = c->inv_start[task + 1];
  } else {  /* causal: rows i with t = Lk - Lq + i >= j */
    const int64_t i0 = (int64_t)j - (c->Lk - c->Lq);
    r0 = i0 > 0 ? i0 : 0;
    r1 = c->Lq;
  }
  for (int64_t e = r0; e < r1; ++e) {
    const int64_t flat = c->idx ? c->inv_rows[e] : (int64_t)b * c->Lq + e;
    for (int h = 0; h < c->H; ++h) {
      const uint16_t* q = c->Q + (flat * c->H + h) * c->d;
      const uint16_t* g = c->dO + (flat * c->H + h) * c->d;
      double acc = 0.0, dp = 0.0;
      for (int x = 0; x < c->d; ++x) {
        acc += widen(q[x]) * widen(k[x]);
        dp += widen(g[x]) * widen(v[x]);
      }
      const double p = exp(c->scale * acc - c->lse[flat * c->H + h]);
      const double ds = p * (dp - c->D[flat * c->H + h]);
      for (int x = 0; x < c->d; ++x) {
        dk[x] += c->scale * ds * widen(q[x]);
        dv[x] += p * widen(g[x]);
      }
    }
  }
}

/*
 * Gradients of attention over per-row key sets. Q, dO: [B, Lq, H, d]; K, V: [B, Lk, d] (bf16
 * bits); idx: [B, Lq, S] selected slots (-1 = empty), or NULL for the causal rows (query i at
 * t = Lk - Lq + i reads keys 0..t). dQ: [n_rows, H, d] for the rows `rows` (NULL: every row; dQ
 * may be NULL). dK, dV: [B, Lk, d] (both or neither; they need every row, so rows must then be
 * NULL). Returns ORC_EINDEX for an index outside [0, Lk) or a row without a valid key.
 */
int oracle_attn_bwd(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const uint16_t* dO, const int32_t* idx,
                    int B, int Lq, int Lk, int H, int d, int S, double scale, const int64_t* rows, int64_t n_rows,
                    double* dQ, double* dK, double* dV, int n_threads) {
  if (!Q || !K || !V || !dO || (!dK) != (!dV)) return ORC_EINVAL;
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Lq > Lk || H <= 0 || d <= 0 || (idx && S <= 0)) return ORC_EINVAL;
  if (dK && rows) return ORC_EINVAL;
  const int64_t all_rows = (int64_t)B * Lq;
  int64_t* all = NULL;
  if (!rows) {
    n_rows = all_rows;
    all = (int64_t*)malloc(sizeof(int64_t) * (size_t)n_rows);
    if (!all) return ORC_ENOMEM;
    for (int64_t r = 0; r < n_rows; ++r) all[r] = r;
    rows = all;
  }
  for (int64_t r = 0; r < n_rows; ++r)
    if (rows[r] < 0 || rows[r] >= all_rows) {
      free(all);
      return ORC_EINVAL;
    }
  double* lse = (double*)malloc(sizeof(double) * (size_t)all_rows * H);
  double* Dv = (double*)malloc(sizeof(double) * (size_t)all_rows * H);
  int64_t* inv_start = NULL;
  int64_t* inv_rows = NULL;
  int rc = (lse && Dv) ? ORC_OK : ORC_ENOMEM;
  if (rc == ORC_OK && dK && idx) {
    /* rows reading each key (b, j), one entry per slot, rows ascending */
    inv_start = (int64_t*)calloc((size_t)B * Lk + 1, sizeof(int64_t));
    if (!inv_start) rc = ORC_ENOMEM;
    for (int64_t f = 0; rc == ORC_OK && f < all_rows; ++f)
      for (int n = 0; n < S; ++n) {
        const int32_t j = idx[f * S + n];
        if (j == -1) continue;
        if (j < 0 || j >= Lk) { rc = ORC_EINDEX; break; }
        inv_start[(f / Lq) * Lk + j + 1]++;
      }
    if (rc == ORC_OK) {
      for (int64_t e = 0; e < (int64_t)B * Lk; ++e) inv_start[e + 1] += inv_start[e];
      inv_rows = (int64_t*)malloc(sizeof(int64_t) * (size_t)(inv_start[(int64_t)B * Lk] + 1));
      int64_t* fill = (int64_t*)malloc(sizeof(int64_t) * (size_t)B * Lk);
      if (!inv_rows || !fill) rc = ORC_ENOMEM;
      else {
        memcpy(fill, inv_start, sizeof(int64_t) * (size_t)B * Lk);
        for (int64_t f = 0; f < all_rows; ++f)
          for (int n = 0; n < S; ++n) {
            const int32_t j = idx[f * S + n];
            if (j != -1) inv_rows[fill[(f / Lq) * Lk + j]++] = f;
          }
      }
      free(fill);
    }
  }
  bwd_ctx c;
  c.Q = Q; c.K = K; c.V = V; c.dO = dO; c.idx = idx;
  c.B = B; c.Lq = Lq; c.Lk = Lk; c.H = H; c.d = d; c.S = S;
  c.scale = scale;
  c.rows = rows; c.n_rows = n_rows;
  c.dQ = dQ; c.lse = lse; c.D = Dv; c.dK = dK; c.dV = dV;
  c.inv_start = inv_start; c.inv_rows = inv_rows;
  atomic_init(&c.bad, 0);
  if (rc == ORC_OK) rc = run_tasks(bwd_task_row, &c, n_rows * H, (size_t)(idx ? S : Lk), n_threads);
  if (rc == ORC_OK) rc = atomic_load(&c.bad);
  if (rc == ORC_OK && dK) rc = run_tasks(bwd_task_key, &c, (int64_t)B * Lk, 0, n_threads);
  free(inv_rows);
  free(inv_start);
  free(Dv);
  free(lse);
  free(all);
  return rc;
}

/* ------------------------------------------------------------------ KV Bridging projection */
typedef struct {
  const uint16_t *Hs, *W;
  int T, hidden, n_layers, d;
  const int64_t* rows;
  int64_t n_rows;
  double* KV; /* [n_layers, 2, n_rows, d] */
} bridge_ctx;

static void bridge_task(void* vctx, int64_t task, double* unused) {
  (void)unused;
  const bridge_ctx* c = (const bridge_ctx*)vctx;
  const int64_t r = task / (2 * c->n_layers);
  const int lk = (int)(task % (2 * c->n_layers)); /* l * 2 + (0: K, 1: V) */
  const uint16_t* hrow = c->Hs + c->rows[r] * c->hidden;
  const uint16_t* w = c->W + (int64_t)lk * c->hidden * c->d;
  double* o = c->KV + ((int64_t)lk * c->n_rows + r) * c->d;
  for (int x = 0; x < c->d; ++x) {
    double acc = 0.0;
    for (int y = 0; y < c->hidden; ++y) acc += widen(hrow[y]) * widen(w[(int64_t)y * c->d + x]);
    o[x] = acc;
  }
}

/*
 * KV Bridging: for rows r of H [T, hidden] and every layer l, K_l[r] = H[r] W[l, 0] and
 * V_l[r] = H[r] W[l, 1]. W: [n_layers, 2, hidden, d]; KV: [n_layers, 2, n_rows, d].
 */
int oracle_bridge_kv_proj(const uint16_t* Hs, int T, int hidden, const uint16_t* W, int n_layers, int d,
                          const int64_t* rows, int64_t n_rows, double* KV, int n_threads) {
  if (!Hs || !W || !KV || T <= 0 || hidden <= 0 || n_layers <= 0 || d <= 0) return ORC_EINVAL;
  int64_t* all = NULL;
  if (!rows) {
    n_rows = T;
    all = (int64_t*)malloc(sizeof(int64_t) * (size_t)n_rows);
    if (!all) return ORC_ENOMEM;
    for (int64_t r = 0; r < n_rows; ++r) all[r] = r;
    rows = all;
  }
  for (int64_t r = 0; r < n_rows; ++r)
    if (rows[r] < 0 || rows[r] >= T) {
      free(all);
      return ORC_EINVAL;
    }
  bridge_ctx c = {Hs, W, T, hidden, n_layers, d, rows, n_rows, KV};
  int rc = run_tasks(bridge_task, &c, n_rows * 2 * n_layers, 0, n_threads);
  free(all);
  return rc;
}
