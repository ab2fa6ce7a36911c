/*
 * lh_oracle.c -- plain, slow CPU oracle for one Lighthouse Attention layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this file:
 * only the tests, the package's smoke check and the CPU-baseline leg of the
 * benchmark load it.  It shares no code, header, table or helper with the CUDA
 * library; it is written from the method's description, step by step, in the
 * order the pages give it.
 *
 * Pages cited (title, then section):
 *   [ES]  gist.science/es, "Resumen Técnico: Pre-entrenamiento con Contexto Largo
 *         mediante Atención Lighthouse", §2 Metodología (A pirámide, B puntuación
 *         y selección, C sub-secuencia densa).
 *   [PT]  bitsgeniais.com.br, "Adeus Custo Quadrático! Como a Lighthouse Attention
 *         Vai TURBINAR o Treinamento de LLMs!", section "A Grande Sacada: Lighthouse
 *         Attention em Quatro Fases!" (phases 1-4).
 *   [JA]  gist.science/ja, "技術的サマリー：Lighthouse Attention による長文脈前学習",
 *         §2 (mirror of [ES]).
 *
 * Notation (per independent unit u = (b,h)):
 *   n_l = N / p^l entries at level l, off_l = sum_{m<l} n_m, M = off_L.
 *   Entry e = (l, j) has global id gid = off_l + j, covers tokens
 *   span(e) = [j p^l, (j+1) p^l - 1] and is placed at pos(e) = (j+1) p^l - 1.
 *   Row-major tensors with the head dimension d innermost.
 *
 * Precision: every floating-point step is fp64 except the score (c.3), which
 * decides an integer result (the selected set) and is therefore computed in
 * fp32 in one fixed, documented order that the GPU path also uses.
 *
 * Threads: units (or rows of one unit) are spread over POSIX threads; each work
 * item is computed by one thread, so results do not depend on the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int64_t B, H, N;
  int32_t d, p, L, S;
} lho_shape;

/* ------------------------------------------------------------------ helpers */

static int64_t ipow(int64_t base, int e) {
  int64_t r = 1;
  for (int i = 0; i < e; ++i) r *= base;
  return r;
}

static int64_t level_len(const lho_shape* s, int l) { return s->N / ipow(s->p, l); }

static int64_t level_off(const lho_shape* s, int l) {
  int64_t off = 0;
  for (int m = 0; m < l; ++m) off += level_len(s, m);
  return off;
}

int64_t lho_num_entries(const lho_shape* s) { return level_off(s, s->L); }

/* level of a global id */
static int gid_level(const lho_shape* s, int64_t gid) {
  int l = 0;
  while (l + 1 < s->L && gid >= level_off(s, l + 1)) ++l;
  return l;
}

/* Parallel-for over [0, n) using up to nthreads POSIX threads. */
typedef void (*lho_item_fn)(void* ctx, int64_t i);
typedef struct {
  lho_item_fn fn;
  void* ctx;
  int64_t n;
  int64_t next;
  pthread_mutex_t mu;
} lho_pool;

static void* lho_worker(void* arg) {
  lho_pool* pool = (lho_pool*)arg;
  for (;;) {
    pthread_mutex_lock(&pool->mu);
    int64_t i = pool->next++;
    pthread_mutex_unlock(&pool->mu);
    if (i >= pool->n) break;
    pool->fn(pool->ctx, i);
  }
  return NULL;
}

static void lho_parallel_for(int64_t n, int nthreads, lho_item_fn fn, void* ctx) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if ((int64_t)nthreads > n) nthreads = (int)(n > 0 ? n : 1);
  lho_pool pool;
  pool.fn = fn;
  pool.ctx = ctx;
  pool.n = n;
  pool.next = 0;
  pthread_mutex_init(&pool.mu, NULL);
  if (nthreads == 1) {
    lho_worker(&pool);
  } else {
    pthread_t th[256];
    for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, lho_worker, &pool);
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
  }
  pthread_mutex_destroy(&pool.mu);
}

/* ------------------------------------------------------------ c.2 pyramid
 * [ES] §2.A, [JA] §2.A: level 0 is the full-resolution sequence; every level l
 * summarises p consecutive entries of level l-1; Q, K and V are pooled alike.
 * [PT] phase 1 ("Pyramid Pool"): the summary is an average.
 * Written out: X^(l)[j] = (1/p) * sum_{i<p} X^(l-1)[p j + i], in fp64.
 * Input: level 0 widened to fp64 (exact for bf16 and fp32 inputs), [U, N, d].
 * Output: levels 1..L-1 concatenated, [U, M-N, d].  Level 0 is the input.     */
typedef struct {
  const lho_shape* s;
  const double* x;
  double* pyr;
} pyr_ctx;

static void pyr_unit(void* vctx, int64_t u) {
  pyr_ctx* c = (pyr_ctx*)vctx;
  const lho_shape* s = c->s;
  const int64_t N = s->N, M = lho_num_entries(s);
  const int d = s->d, p = s->p;
  const double* x0 = c->x + u * N * d;
  double* out = c->pyr + u * (M - N) * d;
  for (int l = 1; l < s->L; ++l) {
    int64_t nl = level_len(s, l);
    double* dst = out + (level_off(s, l) - N) * d;
    for (int64_t j = 0; j < nl; ++j) {
      for (int c2 = 0; c2 < d; ++c2) {
        double acc = 0.0;
        for (int i = 0; i < p; ++i) {
          int64_t child = p * j + i;
          double v = (l == 1) ? x0[child * d + c2]
                              : out[(level_off(s, l - 1) - N + child) * d + c2];
          acc += v;
        }
        dst[j * d + c2] = acc / (double)p;
      }
    }
  }
}

void lho_pyramid(const lho_shape* s, const double* x, double* pyr, int nthreads) {
  pyr_ctx c = {s, x, pyr};
  lho_parallel_for(s->B * s->H, nthreads, pyr_unit, &c);
}

/* --------------------------------------------------- c.3/c.4 score (fp32)
 * [ES] §2.B, [JA] §2.B: the scorer has no parameters; for each entry it takes
 * the l2 norm of the projected Q and K vectors; coarser levels inherit scores
 * from finer ones by max-pooling.  [PT] phase 2: two scores per entry (query
 * score, key score), per head.
 * Readings fixed here: the entry score is the SUM of the two norms; norms are
 * taken at level 0 only and inherited upward by max over the p children.
 * The squared norm uses one fixed fp32 order (the selection is an integer
 * result decided in fp32):
 *   a_b = fmaf chain over x[8b+0..7]^2 starting from 0, for b < d/8;
 *   pairwise tree: for w = 1, 2, 4, ...: a_b <- a_b + a_{b+w} for b = 0 mod 2w;
 *   ss = a_0;  norm = sqrtf(ss)  (IEEE correctly rounded).                     */
static float ss_canonical(const float* x, int d) {
  float a[32];
  int nb = d / 8;
  for (int b = 0; b < nb; ++b) {
    float acc = 0.0f;
    for (int i = 0; i < 8; ++i) acc = fmaf(x[8 * b + i], x[8 * b + i], acc);
    a[b] = acc;
  }
  for (int w = 1; w < nb; w *= 2)
    for (int b = 0; b + w < nb; b += 2 * w) a[b] = a[b] + a[b + w];
  return a[0];
}

typedef struct {
  const lho_shape* s;
  const float *q, *k;
  float* score;
  int mode; /* 0 sum of the norms (default), 1 their product, 2 norm of [q; k] */
} score_ctx;

static void score_unit(void* vctx, int64_t u) {
  score_ctx* c = (score_ctx*)vctx;
  const lho_shape* s = c->s;
  const int64_t N = s->N, M = lho_num_entries(s);
  const int d = s->d;
  const float* q = c->q + u * N * d;
  const float* k = c->k + u * N * d;
  float* sc = c->score + u * M;
  for (int64_t t = 0; t < N; ++t) {
    float sq = ss_canonical(q + t * d, d);
    float sk = ss_canonical(k + t * d, d);
    if (c->mode == 1)
      sc[t] = sqrtf(sq) * sqrtf(sk);
    else if (c->mode == 2)
      sc[t] = sqrtf(sq + sk);
    else
      sc[t] = sqrtf(sq) + sqrtf(sk);
  }
  for (int l = 1; l < s->L; ++l) {
    int64_t nl = level_len(s, l), o = level_off(s, l), oc = level_off(s, l - 1);
    for (int64_t j = 0; j < nl; ++j) {
      float m = sc[oc + s->p * j];
      for (int i = 1; i < s->p; ++i) {
        float v = sc[oc + s->p * j + i];
        if (v > m) m = v;
      }
      sc[o + j] = m;
    }
  }
}

/* Ablations of the reading above (how the two norms combine), same fp32 order
 * for the squared norms: mode 1 = sqrtf(ss(q)) * sqrtf(ss(k)), mode 2 =
 * sqrtf(ss(q) + ss(k)), the norm of the concatenated vector [q; k].          */
void lho_score_mode(const lho_shape* s, const float* q, const float* k, float* score, int mode,
                    int nthreads) {
  score_ctx c = {s, q, k, score, mode};
  lho_parallel_for(s->B * s->H, nthreads, score_unit, &c);
}

void lho_score(const lho_shape* s, const float* q, const float* k, float* score, int nthreads) {
  lho_score_mode(s, q, k, score, 0, nthreads);
}

/* ------------------------------------------- c.5/c.6 joint top-K + order
 * [ES] §2.B: one top-K over all levels jointly.  [ES] §2.C, [PT] phase 3: the
 * selected triplets are sorted topologically into one contiguous, hole-free,
 * causally consistent sequence of length S.
 * Readings fixed here: K = S; ties between equal scores go to the lower level,
 * then the lower index (i.e. the lower gid), which makes the selection unique;
 * the sequence is ordered by (pos ascending, level ascending).
 * Brute force: sort all M entries by (score desc, gid asc) with qsort, keep the
 * first S, then sort those by (pos asc, level asc).                           */
typedef struct {
  float score;
  int64_t gid;
  int64_t pos;
  int level;
} sel_item;

static int cmp_rank(const void* a, const void* b) {
  const sel_item* x = (const sel_item*)a;
  const sel_item* y = (const sel_item*)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  return (x->gid < y->gid) ? -1 : (x->gid > y->gid);
}

static int cmp_order(const void* a, const void* b) {
  const sel_item* x = (const sel_item*)a;
  const sel_item* y = (const sel_item*)b;
  if (x->pos != y->pos) return (x->pos < y->pos) ? -1 : 1;
  return (x->level < y->level) ? -1 : (x->level > y->level);
}

typedef struct {
  const lho_shape* s;
  const float* score;
  int32_t *idx, *pos, *slot;
  int keep_coarsest;
} sel_ctx;

static void select_unit(void* vctx, int64_t u) {
  sel_ctx* c = (sel_ctx*)vctx;
  const lho_shape* s = c->s;
  const int64_t M = lho_num_entries(s);
  const int S = s->S;
  const float* sc = c->score + u * M;
  sel_item* items = (sel_item*)malloc(sizeof(sel_item) * (size_t)M);
  for (int64_t g = 0; g < M; ++g) {
    int l = gid_level(s, g);
    int64_t j = g - level_off(s, l);
    /* keep-coarsest-level variant ([PT] phase 1: the coarsest level keeps a
     * contributor for every position): its entries rank above every score */
    items[g].score = (c->keep_coarsest && l == s->L - 1) ? INFINITY : sc[g];
    items[g].gid = g;
    items[g].level = l;
    items[g].pos = (j + 1) * ipow(s->p, l) - 1;
  }
  qsort(items, (size_t)M, sizeof(sel_item), cmp_rank);
  qsort(items, (size_t)S, sizeof(sel_item), cmp_order);
  int32_t* slot = c->slot + u * M;
  for (int64_t g = 0; g < M; ++g) slot[g] = -1;
  for (int k = 0; k < S; ++k) {
    c->idx[u * S + k] = (int32_t)items[k].gid;
    c->pos[u * S + k] = (int32_t)items[k].pos;
    slot[items[k].gid] = k;
  }
  free(items);
}

void lho_select_opt(const lho_shape* s, const float* score, int32_t* idx, int32_t* pos,
                    int32_t* slot, int keep_coarsest, int nthreads) {
  sel_ctx c = {s, score, idx, pos, slot, keep_coarsest};
  lho_parallel_for(s->B * s->H, nthreads, select_unit, &c);
}

void lho_select(const lho_shape* s, const float* score, int32_t* idx, int32_t* pos, int32_t* slot,
                int nthreads) {
  lho_select_opt(s, score, idx, pos, slot, 0, nthreads);
}

/* ------------------------------------------------------------ c.7 gather
 * [ES] §2.C: the selected entries are collected into the dense sub-sequence.
 * xs[k] = X^(l_k)[j_k]: level 0 from the input, coarser levels from the
 * pyramid.  fp64, no rounding.                                                */
void lho_gather(const lho_shape* s, const double* x, const double* pyr, const int32_t* idx,
                double* xs) {
  const int64_t U = s->B * s->H, N = s->N, M = lho_num_entries(s);
  const int d = s->d, S = s->S;
  for (int64_t u = 0; u < U; ++u) {
    for (int k = 0; k < S; ++k) {
      int64_t g = idx[u * S + k];
      double* dst = xs + (u * S + k) * d;
      if (g < N) {
        for (int c2 = 0; c2 < d; ++c2) dst[c2] = x[(u * N + g) * d + c2];
      } else {
        for (int c2 = 0; c2 < d; ++c2) dst[c2] = pyr[(u * (M - N) + (g - N)) * d + c2];
      }
    }
  }
}

/* ----------------------------------------------- c.8 attention forward
 * [ES] §2.C: stock causal SDPA on the dense sub-sequence.  Causality is on the
 * slot index (row k sees columns k' <= k), as causal SDPA does on any sequence.
 * Textbook softmax with max subtraction, fp64:
 *   z_kk' = scale <q_k, k_k'>,  m_k = max_k' z,  l_k = sum exp(z - m_k),
 *   o_k = sum exp(z - m_k) v_k' / l_k,  lse_k = m_k + ln l_k.
 * Work item = one (unit, row); rows may be a subset (rows != NULL).          */
typedef struct {
  const lho_shape* s;
  const double *qs, *ks, *vs;
  double scale;
  double *os, *lse;
  const int32_t* rows;
  int64_t nrows;
} attn_ctx;

static void attn_fwd_row(const attn_ctx* c, int64_t u, int64_t r, double* z, double* orow,
                         double* lse_out) {
  const int d = c->s->d, S = c->s->S;
  const double* q = c->qs + (u * S + r) * d;
  double m = -INFINITY;
  for (int64_t j = 0; j <= r; ++j) {
    const double* kk = c->ks + (u * S + j) * d;
    double dot = 0.0;
    for (int i = 0; i < d; ++i) dot += q[i] * kk[i];
    z[j] = c->scale * dot;
    if (z[j] > m) m = z[j];
  }
  double l = 0.0;
  for (int i = 0; i < d; ++i) orow[i] = 0.0;
  for (int64_t j = 0; j <= r; ++j) {
    double e = exp(z[j] - m);
    l += e;
    const double* vv = c->vs + (u * S + j) * d;
    for (int i = 0; i < d; ++i) orow[i] += e * vv[i];
  }
  for (int i = 0; i < d; ++i) orow[i] /= l;
  *lse_out = m + log(l);
}

static void attn_fwd_item(void* vctx, int64_t it) {
  attn_ctx* c = (attn_ctx*)vctx;
  const int S = c->s->S, d = c->s->d;
  int64_t u = it / c->nrows, ri = it % c->nrows;
  int64_t r = c->rows ? c->rows[ri] : ri;
  double* z = (double*)malloc(sizeof(double) * (size_t)S);
  attn_fwd_row(c, u, r, z, c->os + (u * c->nrows + ri) * d, c->lse + u * c->nrows + ri);
  free(z);
}

/* os/lse are [U, nrows(,d)]; rows == NULL means all S rows in order. */
void lho_attn_fwd(const lho_shape* s, const double* qs, const double* ks, const double* vs,
                  double scale, const int32_t* rows, int64_t nrows, double* os, double* lse,
                  int nthreads) {
  if (!rows) nrows = s->S;
  attn_ctx c = {s, qs, ks, vs, scale, os, lse, rows, nrows};
  lho_parallel_for(s->B * s->H * nrows, nthreads, attn_fwd_item, &c);
}

/* ---------------------------------------------- c.10 attention backward
 * [ES] §2.B: gradients flow through gather, the attention and scatter-back
 * only.  The attention backward is the textbook softmax adjoint, fp64:
 *   P_ij = exp(scale <q_i,k_j> - lse_i)  (j <= i),
 *   dP_ij = <do_i, v_j>,  D_i = sum_j P_ij dP_ij,  dS_ij = P_ij (dP_ij - D_i),
 *   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,
 *   dv_j = sum_i P_ij do_i.
 * Three passes: lse_i and D_i for every row; dq rows; dk/dv columns.        */
typedef struct {
  const lho_shape* s;
  const double *qs, *ks, *vs, *dos;
  double scale;
  double *lse, *D;
  double *dqs, *dks, *dvs;
} bwd_ctx;

static double bwd_p(const bwd_ctx* c, int64_t u, int64_t i, int64_t j) {
  const int d = c->s->d, S = c->s->S;
  const double* q = c->qs + (u * S + i) * d;
  const double* kk = c->ks + (u * S + j) * d;
  double dot = 0.0;
  for (int t = 0; t < d; ++t) dot += q[t] * kk[t];
  return exp(c->scale * dot - c->lse[u * S + i]);
}

static double bwd_dp(const bwd_ctx* c, int64_t u, int64_t i, int64_t j) {
  const int d = c->s->d, S = c->s->S;
  const double* g = c->dos + (u * S + i) * d;
  const double* vv = c->vs + (u * S + j) * d;
  double dot = 0.0;
  for (int t = 0; t < d; ++t) dot += g[t] * vv[t];
  return dot;
}

static void bwd_stats_item(void* vctx, int64_t it) {
  bwd_ctx* c = (bwd_ctx*)vctx;
  const int S = c->s->S, d = c->s->d;
  int64_t u = it / S, i = it % S;
  /* lse_i by definition (fp64, max-subtracted) */
  double* z = (double*)malloc(sizeof(double) * (size_t)(i + 1));
  const double* q = c->qs + (u * S + i) * d;
  double m = -INFINITY;
  for (int64_t j = 0; j <= i; ++j) {
    const double* kk = c->ks + (u * S + j) * d;
    double dot = 0.0;
    for (int t = 0; t < d; ++t) dot += q[t] * kk[t];
    z[j] = c->scale * dot;
    if (z[j] > m) m = z[j];
  }
  double l = 0.0;
  for (int64_t j = 0; j <= i; ++j) l += exp(z[j] - m);
  c->lse[u * S + i] = m + log(l);
  free(z);
  double D = 0.0;
  for (int64_t j = 0; j <= i; ++j) D += bwd_p(c, u, i, j) * bwd_dp(c, u, i, j);
  c->D[u * S + i] = D;
}

static void bwd_dq_item(void* vctx, int64_t it) {
  bwd_ctx* c = (bwd_ctx*)vctx;
  const int S = c->s->S, d = c->s->d;
  int64_t u = it / S, i = it % S;
  double* out = c->dqs + (u * S + i) * d;
  for (int t = 0; t < d; ++t) out[t] = 0.0;
  for (int64_t j = 0; j <= i; ++j) {
    double ds = bwd_p(c, u, i, j) * (bwd_dp(c, u, i, j) - c->D[u * S + i]);
    const double* kk = c->ks + (u * S + j) * d;
    for (int t = 0; t < d; ++t) out[t] += ds * kk[t];
  }
  for (int t = 0; t < d; ++t) out[t] *= c->scale;
}

static void bwd_dkv_item(void* vctx, int64_t it) {
  bwd_ctx* c = (bwd_ctx*)vctx;
  const int S = c->s->S, d = c->s->d;
  int64_t u = it / S, j = it % S;
  double* dk = c->dks + (u * S + j) * d;
  double* dv = c->dvs + (u * S + j) * d;
  for (int t = 0; t < d; ++t) dk[t] = dv[t] = 0.0;
  for (int64_t i = j; i < S; ++i) {
    double P = bwd_p(c, u, i, j);
    double ds = P * (bwd_dp(c, u, i, j) - c->D[u * S + i]);
    const double* q = c->qs + (u * S + i) * d;
    const double* g = c->dos + (u * S + i) * d;
    for (int t = 0; t < d; ++t) {
      dk[t] += ds * q[t];
      dv[t] += P * g[t];
    }
  }
  for (int t = 0; t < d; ++t) dk[t] *= c->scale;
}

void lho_attn_bwd(const lho_shape* s, const double* qs, const double* ks, const double* vs,
                  const double* dos, double scale, double* dqs, double* dks, double* dvs,
                  int nthreads) {
  const int64_t U = s->B * s->H;
  double* lse = (double*)malloc(sizeof(double) * (size_t)(U * s->S));
  double* D = (double*)malloc(sizeof(double) * (size_t)(U * s->S));
  bwd_ctx c = {s, qs, ks, vs, dos, scale, lse, D, dqs, dks, dvs};
  lho_parallel_for(U * s->S, nthreads, bwd_stats_item, &c);
  lho_parallel_for(U * s->S, nthreads, bwd_dq_item, &c);
  lho_parallel_for(U * s->S, nthreads, bwd_dkv_item, &c);
  free(lse);
  free(D);
}

/* -------------------------------------------------- c.9 scatter-back
 * [ES] §2.C, [PT] phase 4: a deterministic kernel puts each output back at the
 * original positions it stands for, giving a fully dense output.  [PT] phase 1
 * speaks of "contributors" per original position.
 * Readings fixed here: a selected entry contributes its output to every token
 * of its span; a token's output is the mean over its contributors (the selected
 * entries whose span covers it), summed in ascending level; a token with no
 * contributor gets 0.  slot_l(t) = slot[off_l + floor(t / p^l)].              */
static int contributors(const lho_shape* s, const int32_t* slot_u, int64_t t, int32_t* sl) {
  int c = 0;
  for (int l = 0; l < s->L; ++l) {
    sl[l] = slot_u[level_off(s, l) + t / ipow(s->p, l)];
    if (sl[l] >= 0) ++c;
  }
  return c;
}

/* Ablations of reading (i) above (how a coarse output spreads over its span):
 *   mode 0 (default) mean over the contributors covering t;
 *   mode 1 their sum (no division);
 *   mode 2 last token only: an entry delivers its output only to pos(e), the
 *          last token of its span (the strictly causal reading of [PT] phase 4,
 *          "the output does not see the future"), and a token takes the mean of
 *          what is delivered to it.
 * delivered() gives the slots that reach token t under the mode (-1 = none). */
static int delivered(const lho_shape* s, const int32_t* slot_u, int64_t t, int mode, int32_t* sl) {
  int c = contributors(s, slot_u, t, sl);
  if (mode != 2) return c;
  c = 0;
  for (int l = 0; l < s->L; ++l) {
    if ((t + 1) % ipow(s->p, l) != 0) sl[l] = -1;  /* the entry's span ends later */
    if (sl[l] >= 0) ++c;
  }
  return c;
}

void lho_scatter_mode(const lho_shape* s, const double* os, const int32_t* slot, double* o,
                      int mode) {
  const int64_t U = s->B * s->H, N = s->N, M = lho_num_entries(s);
  const int d = s->d, S = s->S;
  int32_t sl[64];
  for (int64_t u = 0; u < U; ++u) {
    for (int64_t t = 0; t < N; ++t) {
      double* dst = o + (u * N + t) * d;
      int cnt = delivered(s, slot + u * M, t, mode, sl);
      for (int i = 0; i < d; ++i) dst[i] = 0.0;
      if (cnt == 0) continue;
      for (int l = 0; l < s->L; ++l) {
        if (sl[l] < 0) continue;
        const double* src = os + (u * S + sl[l]) * d;
        for (int i = 0; i < d; ++i) dst[i] += src[i];
      }
      if (mode != 1)
        for (int i = 0; i < d; ++i) dst[i] /= (double)cnt;
    }
  }
}

void lho_scatter(const lho_shape* s, const double* os, const int32_t* slot, double* o) {
  lho_scatter_mode(s, os, slot, o, 0);
}

/* Adjoint of lho_scatter_mode: dos[k] = sum over the tokens t of span(e_k) that
 * e_k reaches of dO[t] / c_t (/ 1 for the sum), t ascending. */
void lho_scatter_bwd_mode(const lho_shape* s, const double* dO, const int32_t* idx,
                          const int32_t* slot, double* dos, int mode) {
  const int64_t U = s->B * s->H, N = s->N, M = lho_num_entries(s);
  const int d = s->d, S = s->S;
  int32_t sl[64];
  for (int64_t u = 0; u < U; ++u) {
    for (int k = 0; k < S; ++k) {
      int64_t g = idx[u * S + k];
      int l = gid_level(s, g);
      int64_t j = g - level_off(s, l), w = ipow(s->p, l);
      double* dst = dos + (u * S + k) * d;
      for (int i = 0; i < d; ++i) dst[i] = 0.0;
      for (int64_t t = j * w; t < (j + 1) * w; ++t) {
        int cnt = delivered(s, slot + u * M, t, mode, sl);
        if (sl[l] != k) continue;  /* this entry does not reach t (last-token mode) */
        const double* g0 = dO + (u * N + t) * d;
        const double c = (mode == 1) ? 1.0 : (double)cnt;
        for (int i = 0; i < d; ++i) dst[i] += g0[i] / c;
      }
    }
  }
}

void lho_scatter_bwd(const lho_shape* s, const double* dO, const int32_t* idx,
                     const int32_t* slot, double* dos) {
  lho_scatter_bwd_mode(s, dO, idx, slot, dos, 0);
}

/* Adjoint of pyramid + gather (pooling is linear, the mean's adjoint is 1/p^l):
 *   dX[t] = sum_{l ascending, slot_l(t) >= 0} dxs[slot_l(t)] / p^l.          */
void lho_gather_bwd(const lho_shape* s, const double* dxs, const int32_t* slot, double* dx) {
  const int64_t U = s->B * s->H, N = s->N, M = lho_num_entries(s);
  const int d = s->d, S = s->S;
  int32_t sl[64];
  for (int64_t u = 0; u < U; ++u) {
    for (int64_t t = 0; t < N; ++t) {
      double* dst = dx + (u * N + t) * d;
      contributors(s, slot + u * M, t, sl);
      for (int i = 0; i < d; ++i) dst[i] = 0.0;
      for (int l = 0; l < s->L; ++l) {
        if (sl[l] < 0) continue;
        const double* src = dxs + (u * S + sl[l]) * d;
        double w = (double)ipow(s->p, l);
        for (int i = 0; i < d; ++i) dst[i] += src[i] / w;
      }
    }
  }
}
