/*
 * synth_host.c -- host side of the seeded input generator.
 *
 * Builds the normal-quantile table, fills whole tensors on the host (split
 * over threads; results do not depend on the split), and implements the two
 * msk_source providers the oracle reads from.  Compile with
 * -ffp-contract=off so the float steps in msk_synth.h round exactly as the
 * device fill kernels do.
 */
#include "msk_synth.h"
#include "msk_source.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ---- normal quantile table ---------------------------------------------- */
/* Upper-tail probability of the standard normal. */
static double upper_tail(double z) { return 0.5 * erfc(z / sqrt(2.0)); }

/* z >= 0 with upper_tail(z) = q, 0 < q <= 0.5, by bisection to full double. */
static double upper_quantile(double q) {
  double lo = 0.0, hi = 40.0;
  for (int it = 0; it < 200; ++it) {
    double mid = 0.5 * (lo + hi);
    if (mid == lo || mid == hi) break;
    if (upper_tail(mid) > q) lo = mid; else hi = mid;
  }
  return 0.5 * (lo + hi);
}

static sy_gtab g_tab;
static int g_tab_ready = 0;
static pthread_mutex_t g_tab_mu = PTHREAD_MUTEX_INITIALIZER;

const sy_gtab* sy_table(void) {
  pthread_mutex_lock(&g_tab_mu);
  if (!g_tab_ready) {
    const double two32 = 4294967296.0;
    for (int r = 0; r < SY_GT_LOW; ++r) g_tab.low[r] = (float)upper_quantile((r + 0.5) / two32);
    for (int b = 6; b <= 30; ++b)
      for (int j = 0; j <= SY_GT_SEG; ++j) {
        double rn = ldexp(1.0, b) + (double)j * ldexp(1.0, b - 6);
        g_tab.oct[b - 6][j] = (float)upper_quantile((rn + 0.5) / two32);
      }
    g_tab_ready = 1;
  }
  pthread_mutex_unlock(&g_tab_mu);
  return &g_tab;
}

/* ---- model-level tensor parameters ------------------------------------- */
static uint32_t role_kind(int role) {
  static const uint32_t k[7] = {SY_WQ, SY_WK, SY_WV, SY_WO, SY_WGATE, SY_WUP, SY_WDOWN};
  return k[role];
}

void sy_nvfp4_shape(const sy_model* m, int role, int64_t* rows, int64_t* K) {
  int qd = m->n_q_heads * m->head_dim, kvd = m->n_kv_heads * m->head_dim;
  switch (role) {
    case SRC_WQ: *rows = qd; *K = m->d_model; break;
    case SRC_WK: case SRC_WV: *rows = kvd; *K = m->d_model; break;
    case SRC_WO: *rows = m->d_model; *K = qd; break;
    case SRC_WGATE: case SRC_WUP: *rows = m->expert_dim; *K = m->d_model; break;
    default: *rows = m->d_model; *K = m->expert_dim; break;
  }
}

/* sigma = 1/sqrt(fan_in) rounded to float; global scale a power of two. */
void sy_nvfp4_params(const sy_model* m, int role, float* sigma, float* gs) {
  int64_t rows, K;
  sy_nvfp4_shape(m, role, &rows, &K);
  double s = 1.0 / sqrt((double)K);
  *sigma = (float)s;
  if (m->use_global_scale) {
    double t = 8.0 * s / 6.0 / 448.0;
    *gs = (float)ldexp(1.0, (int)ceil(log2(t)));
  } else {
    *gs = 1.0f;
  }
}

uint64_t sy_nvfp4_key(const sy_model* m, int role, int layer, int expert) {
  int e = role >= SRC_WGATE ? expert : 0;
  return sy_key(m->seed, sy_stream(role_kind(role), (uint32_t)layer, (uint32_t)e, 0));
}

/* ---- threaded fills ------------------------------------------------------ */
typedef struct fill_job {
  void (*fn)(struct fill_job*, int64_t, int64_t);
  int64_t n;
  const sy_model* m;
  uint64_t key, key2;
  uint32_t K;
  float sigma, gs, lo, span;
  uint8_t *codes, *scales, *b0, *b1;
  float* f;
  int64_t row0;
} fill_job;

typedef struct { fill_job* job; int64_t a, b; } fill_part;

static void* fill_thread(void* p) {
  fill_part* fp = (fill_part*)p;
  fp->job->fn(fp->job, fp->a, fp->b);
  return NULL;
}

static int g_threads = 0;
void sy_set_threads(int n) { g_threads = n; }

static void run_fill(fill_job* job) {
  int nt = g_threads > 0 ? g_threads : 8;
  if (job->n < 4096 || nt <= 1) { job->fn(job, 0, job->n); return; }
  if (nt > 64) nt = 64;
  pthread_t th[64];
  fill_part parts[64];
  for (int i = 0; i < nt; ++i) {
    parts[i].job = job;
    parts[i].a = job->n * i / nt;
    parts[i].b = job->n * (i + 1) / nt;
    pthread_create(&th[i], NULL, fill_thread, &parts[i]);
  }
  for (int i = 0; i < nt; ++i) pthread_join(th[i], NULL);
}

static void nvfp4_part(fill_job* j, int64_t a, int64_t b) {
  const sy_gtab* T = sy_table();
  uint32_t nkb = j->K / 16;
  for (int64_t blk = a; blk < b; ++blk) {
    int64_t r = blk / nkb;
    uint32_t kb = (uint32_t)(blk % nkb);
    uint8_t c8[8];
    uint8_t sc = sy_nvfp4_gen_block(T, j->key, (uint64_t)(j->row0 + r), j->K, kb, j->sigma, j->gs, c8);
    memcpy(j->codes + r * (j->K / 2) + kb * 8, c8, 8);
    j->scales[r * nkb + kb] = sc;
  }
}

/* Rows [row0, row0+nrows) of an NVFP4 tensor into codes[nrows][K/2],
 * scales[nrows][K/16]; returns the global scale. */
float sy_fill_nvfp4(const sy_model* m, int role, int layer, int expert, int64_t row0,
                    int64_t nrows, uint8_t* codes, uint8_t* scales) {
  int64_t rows, K;
  sy_nvfp4_shape(m, role, &rows, &K);
  fill_job j;
  memset(&j, 0, sizeof j);
  j.fn = nvfp4_part;
  j.m = m;
  j.key = sy_nvfp4_key(m, role, layer, expert);
  j.K = (uint32_t)K;
  sy_nvfp4_params(m, role, &j.sigma, &j.gs);
  j.codes = codes;
  j.scales = scales;
  j.row0 = row0;
  j.n = nrows * (K / 16);
  run_fill(&j);
  return j.gs;
}

static void gauss_part(fill_job* j, int64_t a, int64_t b) {
  const sy_gtab* T = sy_table();
  for (int64_t i = a; i < b; ++i) j->f[i] = SY_MUL(j->sigma, sy_gauss(T, sy_u64(j->key, (uint64_t)i)));
}
static void unif_part(fill_job* j, int64_t a, int64_t b) {
  for (int64_t i = a; i < b; ++i) j->f[i] = sy_uniform(sy_u64(j->key, (uint64_t)i), j->lo, j->span);
}

/* Gains U(0.8, 1.2); router N(0, 1/d) fp32 [E][d]. */
void sy_vec_params(const sy_model* m, int role, int layer, uint64_t* key, int64_t* n, int* gauss,
                   float* sigma) {
  static const uint32_t kinds[5] = {SY_ATTN_G, SY_Q_G, SY_K_G, SY_MOE_G, SY_ROUTER};
  *key = sy_key(m->seed, sy_stream(kinds[role], (uint32_t)layer, 0, 0));
  *gauss = role == SRC_ROUTER;
  *sigma = (float)(1.0 / sqrt((double)m->d_model));
  switch (role) {
    case SRC_Q_G: case SRC_K_G: *n = m->head_dim; break;
    case SRC_ROUTER: *n = (int64_t)m->n_experts * m->d_model; break;
    default: *n = m->d_model; break;
  }
}

void sy_fill_vec(const sy_model* m, int role, int layer, float* out) {
  fill_job j;
  memset(&j, 0, sizeof j);
  int gauss;
  sy_vec_params(m, role, layer, &j.key, &j.n, &gauss, &j.sigma);
  j.f = out;
  j.lo = 0.8f;
  j.span = 0.4f;
  j.fn = gauss ? gauss_part : unif_part;
  run_fill(&j);
}

/* bf16 N(0,1) hidden rows of (seq, token in seq): out[d] */
uint64_t sy_hidden_key(const sy_model* m, int seq, int tok) {
  return sy_key(m->seed, sy_stream(SY_HIDDEN, 0, (uint32_t)seq, (uint32_t)tok));
}
void sy_fill_hidden(const sy_model* m, int seq, int tok, uint16_t* out) {
  const sy_gtab* T = sy_table();
  uint64_t key = sy_hidden_key(m, seq, tok);
  for (int i = 0; i < m->d_model; ++i) out[i] = sy_bf16(sy_gauss(T, sy_u64(key, (uint64_t)i)));
}

/* past K/V: fp8 e4m3 of N(0,1), element (pos, i) at index pos*hd + i */
uint64_t sy_past_key(const sy_model* m, int kv, int layer, int seq, int head) {
  return sy_key(m->seed, sy_stream(kv ? SY_PAST_V : SY_PAST_K, (uint32_t)layer, (uint32_t)seq, (uint32_t)head));
}
static void past_part(fill_job* j, int64_t a, int64_t b) {
  const sy_gtab* T = sy_table();
  for (int64_t i = a; i < b; ++i) {
    uint64_t idx = (uint64_t)(j->row0 + i);
    j->b0[i] = sy_e4m3(sy_gauss(T, sy_u64(j->key, idx)));
    j->b1[i] = sy_e4m3(sy_gauss(T, sy_u64(j->key2, idx)));
  }
}
void sy_fill_past(const sy_model* m, int layer, int seq, int head, int64_t pos0, int64_t n,
                  uint8_t* k, uint8_t* v) {
  fill_job j;
  memset(&j, 0, sizeof j);
  j.fn = past_part;
  j.key = sy_past_key(m, 0, layer, seq, head);
  j.key2 = sy_past_key(m, 1, layer, seq, head);
  j.row0 = pos0 * m->head_dim;
  j.n = n * m->head_dim;
  j.b0 = k;
  j.b1 = v;
  run_fill(&j);
}

/* ---- lazy generating source ---------------------------------------------- */
typedef struct lazy_src {
  msk_source src;
  sy_model m;
  msk_src_nvfp4* w; /* [L][7][E] (dense roles use expert 0) */
  float** vec;      /* [L][5] */
  int64_t bytes;
} lazy_src;

static int lazy_nvfp4(void* ctx, int layer, int role, int expert, msk_src_nvfp4* out) {
  lazy_src* s = (lazy_src*)ctx;
  const sy_model* m = &s->m;
  if (layer < 0 || layer >= m->n_layers || role < 0 || role > 6) return -1;
  if (role < SRC_WGATE) expert = 0;
  if (expert < 0 || expert >= m->n_experts) return -1;
  msk_src_nvfp4* w = &s->w[((int64_t)layer * 7 + role) * m->n_experts + expert];
  if (!w->codes) {
    int64_t rows, K;
    sy_nvfp4_shape(m, role, &rows, &K);
    uint8_t* c = (uint8_t*)malloc((size_t)(rows * K / 2));
    uint8_t* sc = (uint8_t*)malloc((size_t)(rows * K / 16));
    if (!c || !sc) { free(c); free(sc); return -2; }
    w->global_scale = sy_fill_nvfp4(m, role, layer, expert, 0, rows, c, sc);
    w->codes = c;
    w->scales = sc;
    s->bytes += rows * K / 2 + rows * K / 16;
  }
  *out = *w;
  return 0;
}

static int lazy_vec(void* ctx, int layer, int role, const float** out) {
  lazy_src* s = (lazy_src*)ctx;
  const sy_model* m = &s->m;
  if (layer < 0 || layer >= m->n_layers || role < 0 || role > 4) return -1;
  float** v = &s->vec[layer * 5 + role];
  if (!*v) {
    uint64_t key; int64_t n; int g; float sg;
    sy_vec_params(m, role, layer, &key, &n, &g, &sg);
    *v = (float*)malloc((size_t)n * sizeof(float));
    if (!*v) return -2;
    sy_fill_vec(m, role, layer, *v);
    s->bytes += n * 4;
  }
  *out = *v;
  return 0;
}

static int lazy_past(void* ctx, int layer, int seq, int head, int64_t pos0, int64_t n, uint8_t* k,
                     uint8_t* v) {
  lazy_src* s = (lazy_src*)ctx;
  if (layer < 0 || layer >= s->m.n_layers || head < 0 || head >= s->m.n_kv_heads || pos0 < 0 || n < 0)
    return -1;
  sy_fill_past(&s->m, layer, seq, head, pos0, n, k, v);
  return 0;
}

msk_source* sy_lazy_source_create(const sy_model* m) {
  lazy_src* s = (lazy_src*)calloc(1, sizeof(lazy_src));
  if (!s) return NULL;
  s->m = *m;
  s->w = (msk_src_nvfp4*)calloc((size_t)m->n_layers * 7 * m->n_experts, sizeof(msk_src_nvfp4));
  s->vec = (float**)calloc((size_t)m->n_layers * 5, sizeof(float*));
  if (!s->w || !s->vec) { free(s->w); free(s->vec); free(s); return NULL; }
  s->src.ctx = s;
  s->src.nvfp4 = lazy_nvfp4;
  s->src.vec = lazy_vec;
  s->src.past_kv = lazy_past;
  return &s->src;
}

int64_t sy_lazy_source_bytes(msk_source* src) { return ((lazy_src*)src->ctx)->bytes; }

void sy_lazy_source_destroy(msk_source* src) {
  if (!src) return;
  lazy_src* s = (lazy_src*)src->ctx;
  int64_t nw = (int64_t)s->m.n_layers * 7 * s->m.n_experts;
  for (int64_t i = 0; i < nw; ++i) { free((void*)s->w[i].codes); free((void*)s->w[i].scales); }
  for (int i = 0; i < s->m.n_layers * 5; ++i) free(s->vec[i]);
  free(s->w);
  free(s->vec);
  free(s);
}

/* ---- array source over borrowed host arrays ------------------------------ */
typedef struct arr_past { const uint8_t *k, *v; int64_t n; } arr_past;
typedef struct arr_src {
  msk_source src;
  int L, E, S, H, hd;
  msk_src_nvfp4* w; /* [L][7][E] */
  const float** vec; /* [L][5] */
  arr_past* past;    /* [L][S][H] */
} arr_src;

static int arr_nvfp4(void* ctx, int layer, int role, int expert, msk_src_nvfp4* out) {
  arr_src* s = (arr_src*)ctx;
  if (layer < 0 || layer >= s->L || role < 0 || role > 6) return -1;
  if (role < SRC_WGATE) expert = 0;
  if (expert < 0 || expert >= s->E) return -1;
  msk_src_nvfp4* w = &s->w[((int64_t)layer * 7 + role) * s->E + expert];
  if (!w->codes) return -3;
  *out = *w;
  return 0;
}
static int arr_vec(void* ctx, int layer, int role, const float** out) {
  arr_src* s = (arr_src*)ctx;
  if (layer < 0 || layer >= s->L || role < 0 || role > 4) return -1;
  if (!s->vec[layer * 5 + role]) return -3;
  *out = s->vec[layer * 5 + role];
  return 0;
}
static int arr_past_kv(void* ctx, int layer, int seq, int head, int64_t pos0, int64_t n, uint8_t* k,
                       uint8_t* v) {
  arr_src* s = (arr_src*)ctx;
  if (layer < 0 || layer >= s->L || seq < 0 || seq >= s->S || head < 0 || head >= s->H) return -1;
  arr_past* p = &s->past[((int64_t)layer * s->S + seq) * s->H + head];
  if (pos0 < 0 || pos0 + n > p->n) return -4;
  memcpy(k, p->k + pos0 * s->hd, (size_t)(n * s->hd));
  memcpy(v, p->v + pos0 * s->hd, (size_t)(n * s->hd));
  return 0;
}

msk_source* sy_array_source_create(int L, int E, int S, int H, int hd) {
  arr_src* s = (arr_src*)calloc(1, sizeof(arr_src));
  if (!s) return NULL;
  s->L = L; s->E = E; s->S = S; s->H = H; s->hd = hd;
  s->w = (msk_src_nvfp4*)calloc((size_t)L * 7 * E, sizeof(msk_src_nvfp4));
  s->vec = (const float**)calloc((size_t)L * 5, sizeof(float*));
  s->past = (arr_past*)calloc((size_t)L * S * H, sizeof(arr_past));
  s->src.ctx = s;
  s->src.nvfp4 = arr_nvfp4;
  s->src.vec = arr_vec;
  s->src.past_kv = arr_past_kv;
  return &s->src;
}
void sy_array_set_nvfp4(msk_source* src, int layer, int role, int expert, const uint8_t* codes,
                        const uint8_t* scales, float gs) {
  arr_src* s = (arr_src*)src->ctx;
  if (role < SRC_WGATE) expert = 0;
  msk_src_nvfp4* w = &s->w[((int64_t)layer * 7 + role) * s->E + expert];
  w->codes = codes; w->scales = scales; w->global_scale = gs;
}
void sy_array_set_vec(msk_source* src, int layer, int role, const float* v) {
  arr_src* s = (arr_src*)src->ctx;
  s->vec[layer * 5 + role] = v;
}
void sy_array_set_past(msk_source* src, int layer, int seq, int head, const uint8_t* k, const uint8_t* v,
                       int64_t n) {
  arr_src* s = (arr_src*)src->ctx;
  arr_past* p = &s->past[((int64_t)layer * s->S + seq) * s->H + head];
  p->k = k; p->v = v; p->n = n;
}
void sy_array_source_destroy(msk_source* src) {
  if (!src) return;
  arr_src* s = (arr_src*)src->ctx;
  free(s->w); free((void*)s->vec); free(s->past); free(s);
}

/* Copy the quantile table out (the device fill kernels take it verbatim). */
void sy_table_copy(sy_gtab* out) { *out = *sy_table(); }
int sy_table_bytes(void) { return (int)sizeof(sy_gtab); }
