/*
 * msk_oracle.c -- TEST INFRASTRUCTURE.  A plain, slow, fp64 CPU reference of
 * one decode/verify step of the QK-normed MoE decoder stack.  Only the tests,
 * the package's smoke check and the benchmark's CPU-baseline leg call it; the
 * product path never does.  It shares no code with the CUDA path: its
 * decoders, encoders and arithmetic are written here from the definitions.
 *
 * What it computes, per layer, in the order of the step (the pages are the
 * PyTorch blog post "Optimizing Muse Spark Open on TPU v7 with
 * SGLang-TorchTPU" and its restatements; section names below are theirs):
 *   x    = RMSNorm(h) * g_attn
 *   q,k,v = x . deq(W_q|k|v)^T          NVFP4: e2m1 code * e4m3 scale per 16
 *                                       inputs * fp32 global scale
 *                                       ("Expert Weight Quantization")
 *   q,k  <- per-head RMSNorm * g_q|g_k  (QK-norm, "Removing Attention
 *                                       Bottlenecks")
 *   k,v  -> fp8 e4m3 (RNE, saturating)  written to the cache, read back
 *                                       (fp8 KV cache, "Key points")
 *   o    = softmax(q.k_j / sqrt(hd)) . v_j over keys j <= pos, and
 *          pos - j < 2048 on sliding-window layers ("Model Architecture
 *          Details": 2,048-token window, full-context layers).  This is the
 *          ordinary max-subtracted softmax; the fixed-bound form the kernel
 *          uses is equal to it by shift invariance.
 *   h   += o . deq(W_o)^T
 *   x2   = RMSNorm(h) * g_moe ; logits = x2 . W_r^T (fp32 router)
 *   top-8 of 256 by (logit desc, index asc), weights = softmax over the 8
 *          ("One program replaces many kernel boundaries": 8 of 256 experts)
 *   h   += sum_slot w_slot * (silu(x2.Wg^T) * (x2.Wu^T)) . Wd^T, slot order
 *   out  = bf16(h), round to nearest even.
 * Readings where the pages are silent (no RoPE, eps = 1e-6, gains shared
 * across heads, GQA groups contiguous) are the plainest ones and are listed
 * with the design notes.  Every function is pinned by tests under tests/.
 */
#include "msk_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ---- formats, from their definitions ------------------------------------- */
/* e2m1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; no inf/NaN. */
double msk_or_e2m1_decode(int nib) {
  int s = (nib >> 3) & 1, e = (nib >> 1) & 3, m = nib & 1;
  double v = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return s ? -v : v;
}

/* e4m3fn: 1 sign, 4 exponent (bias 7), 3 mantissa bits; S.1111.111 is NaN,
 * no infinities; largest finite 448. */
double msk_or_e4m3_decode(int code) {
  int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
  if (e == 15 && m == 7) return NAN;
  double v = e == 0 ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
  return s ? -v : v;
}

static double g_e4m3[256];
static double g_e2m1[16];
static pthread_once_t g_tab_once = PTHREAD_ONCE_INIT;
static void build_tables(void) {
  for (int c = 0; c < 256; ++c) g_e4m3[c] = msk_or_e4m3_decode(c);
  for (int c = 0; c < 16; ++c) g_e2m1[c] = msk_or_e2m1_decode(c);
}

/* Round x to a grid of `bits` significant bits, nearest even (default FP
 * rounding mode of nearbyint). */
static double round_sig(double x, int bits) {
  if (x == 0.0) return 0.0;
  int e;
  double m = frexp(x, &e); /* |m| in [0.5, 1) */
  return ldexp(nearbyint(ldexp(m, bits)), e - bits);
}

/* fp64 -> e4m3fn code: nearest even, saturating to +-448.  The sign bit is
 * the operand's (so -0 and negative values that round to zero give the
 * signed zero S.0000.000 = 0x80, as IEEE rounding keeps the operand's sign);
 * NaN gives the NaN code S.1111.111. */
int msk_or_e4m3_encode(double x) {
  double a = fabs(x), r;
  int base = signbit(x) ? 128 : 0;
  if (isnan(x)) return base | 0x7F;
  if (a < ldexp(1.0, -6)) r = ldexp(nearbyint(ldexp(a, 9)), -9); /* subnormal spacing 2^-9 */
  else r = round_sig(a, 4);
  if (r > 448.0) r = 448.0;
  if (r == 0.0) return base;
  pthread_once(&g_tab_once, build_tables);
  for (int c = 1; c < 127; ++c)
    if (g_e4m3[c] == r) return base | c;
  return -1; /* unreachable */
}

/* msk_or_e4m3_encode over an array (codes of n values). */
void msk_or_e4m3_encode_n(const double* x, int64_t n, uint8_t* codes) {
  for (int64_t i = 0; i < n; ++i) codes[i] = (uint8_t)msk_or_e4m3_encode(x[i]);
}

/* fp64 -> bf16 bits: nearest even (finite, normal-range inputs). */
uint16_t msk_or_bf16_encode(double x) {
  float f = (float)round_sig(x, 8); /* exact in float */
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}
double msk_or_bf16_decode(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* ---- small building blocks ------------------------------------------------ */
void msk_or_rmsnorm(const double* x, const float* g, int n, double eps, double* y) {
  double ss = 0.0;
  for (int i = 0; i < n; ++i) ss += x[i] * x[i];
  double r = 1.0 / sqrt(ss / n + eps);
  for (int i = 0; i < n; ++i) y[i] = x[i] * r * (double)g[i];
}

double msk_or_silu(double a) { return a / (1.0 + exp(-a)); }

/* Dequantised row n of an NVFP4 [rows][K] tensor. */
static void deq_row(const msk_src_nvfp4* w, int64_t K, int64_t n, double* out) {
  const uint8_t* c = w->codes + n * (K / 2);
  const uint8_t* s = w->scales + n * (K / 16);
  for (int64_t k = 0; k < K; ++k) {
    int nib = (c[k / 2] >> (4 * (k & 1))) & 15;
    out[k] = g_e2m1[nib] * g_e4m3[s[k / 16]] * (double)w->global_scale;
  }
}

/* top-k of n logits by (value desc, index asc); weights = softmax over the
 * selected; gap = k-th minus (k+1)-th value (inf if k == n). */
static const double* g_sort_vals;
static int cmp_desc(const void* a, const void* b) {
  int i = *(const int*)a, j = *(const int*)b;
  double vi = g_sort_vals[i], vj = g_sort_vals[j];
  if (vi > vj) return -1;
  if (vi < vj) return 1;
  return i < j ? -1 : (i > j);
}
static pthread_mutex_t g_sort_mu = PTHREAD_MUTEX_INITIALIZER;

void msk_or_topk(const double* logits, int n, int k, int16_t* ids, double* w, double* gap) {
  int* idx = (int*)malloc(sizeof(int) * (size_t)n);
  for (int i = 0; i < n; ++i) idx[i] = i;
  pthread_mutex_lock(&g_sort_mu);
  g_sort_vals = logits;
  qsort(idx, (size_t)n, sizeof(int), cmp_desc);
  pthread_mutex_unlock(&g_sort_mu);
  for (int i = 0; i < k; ++i) ids[i] = (int16_t)idx[i];
  if (gap) *gap = k < n ? logits[idx[k - 1]] - logits[idx[k]] : INFINITY;
  free(idx);
  msk_or_route_weights(logits, ids, k, w);
}

void msk_or_route_weights(const double* logits, const int16_t* ids, int k, double* w) {
  double mx = -INFINITY, sum = 0.0;
  for (int i = 0; i < k; ++i) mx = fmax(mx, logits[ids[i]]);
  for (int i = 0; i < k; ++i) { w[i] = exp(logits[ids[i]] - mx); sum += w[i]; }
  for (int i = 0; i < k; ++i) w[i] /= sum;
}

/* One attention row: o = sum_j softmax(s)_j v_j, s_j = scale * q.k_j, over
 * n keys given as rows of decoded K, V [n][hd]; max-subtracted softmax. */
void msk_or_attend(const double* q, const double* K, const double* V, int64_t n, int hd, double scale,
                   double* o, double* s_max) {
  double* s = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  double m = -INFINITY;
  for (int64_t j = 0; j < n; ++j) {
    double acc = 0.0;
    for (int i = 0; i < hd; ++i) acc += q[i] * K[j * hd + i];
    s[j] = scale * acc;
    m = fmax(m, s[j]);
  }
  double l = 0.0;
  for (int i = 0; i < hd; ++i) o[i] = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    double p = exp(s[j] - m);
    l += p;
    for (int i = 0; i < hd; ++i) o[i] += p * V[j * hd + i];
  }
  for (int i = 0; i < hd; ++i) o[i] = n > 0 ? o[i] / l : 0.0;
  if (s_max) *s_max = m;
  free(s);
}

/* ---- parallel for ----------------------------------------------------------- */
typedef void (*par_fn)(void* ctx, int64_t i);
typedef struct { par_fn fn; void* ctx; int64_t a, b; } par_part;
static void* par_thread(void* p) {
  par_part* pp = (par_part*)p;
  for (int64_t i = pp->a; i < pp->b; ++i) pp->fn(pp->ctx, i);
  return NULL;
}
static void par_for(int64_t n, int nt, par_fn fn, void* ctx) {
  if (nt > 128) nt = 128;
  if (nt <= 1 || n <= 1) { for (int64_t i = 0; i < n; ++i) fn(ctx, i); return; }
  if (nt > n) nt = (int)n;
  pthread_t th[128];
  par_part pp[128];
  for (int t = 0; t < nt; ++t) {
    pp[t].fn = fn; pp[t].ctx = ctx;
    pp[t].a = n * t / nt; pp[t].b = n * (t + 1) / nt;
    pthread_create(&th[t], NULL, par_thread, &pp[t]);
  }
  for (int t = 0; t < nt; ++t) pthread_join(th[t], NULL);
}

/* y[t][n] (+)= sum_k x[t][k] * deq(W)[n][k] for all T tokens, rows in parallel */
typedef struct { const msk_src_nvfp4* w; int64_t K, N; int T; const double* x; double* y; int accumulate; } mm_ctx;
static void mm_row(void* p, int64_t n) {
  mm_ctx* c = (mm_ctx*)p;
  double* row = (double*)malloc(sizeof(double) * (size_t)c->K);
  deq_row(c->w, c->K, n, row);
  for (int t = 0; t < c->T; ++t) {
    double acc = 0.0;
    const double* xt = c->x + (int64_t)t * c->K;
    for (int64_t k = 0; k < c->K; ++k) acc += xt[k] * row[k];
    if (c->accumulate) c->y[(int64_t)t * c->N + n] += acc;
    else c->y[(int64_t)t * c->N + n] = acc;
  }
  free(row);
}
static void matmul_nvfp4(const msk_src_nvfp4* w, int64_t K, int64_t N, int T, const double* x, double* y,
                         int accumulate, int nt) {
  mm_ctx c = {w, K, N, T, x, y, accumulate};
  par_for(N, nt, mm_row, &c);
}

/* attention of one (token, q head) */
typedef struct {
  const msk_or_cfg* cfg;
  int T, tps, layer;
  const int32_t* positions;
  const double* q;      /* [T][hq*hd] normalised */
  const uint8_t* knew;  /* [T][hkv][hd] codes */
  const uint8_t* vnew;
  uint8_t** past_k;     /* [S*hkv] codes [pos0_b][hd] */
  uint8_t** past_v;
  double* o;            /* [T][hq*hd] */
  double* smax;         /* [T*hq] */
} at_ctx;
static void attend_one(void* p, int64_t i) {
  at_ctx* c = (at_ctx*)p;
  const msk_or_cfg* g = c->cfg;
  int hd = g->head_dim, hq = g->n_q_heads, hkv = g->n_kv_heads;
  int t = (int)(i / hq), h = (int)(i % hq), kvh = h / (hq / hkv);
  int b = t / c->tps;
  int64_t pos = c->positions[t], pos0 = c->positions[b * c->tps];
  int64_t lo = 0;
  if (g->is_sliding[c->layer]) { lo = pos - g->window + 1; if (lo < 0) lo = 0; }
  int64_t n = pos - lo + 1;
  double* K = (double*)malloc(sizeof(double) * (size_t)(n * hd));
  double* V = (double*)malloc(sizeof(double) * (size_t)(n * hd));
  for (int64_t j = lo; j <= pos; ++j) {
    const uint8_t *kc, *vc;
    if (j >= pos0) { /* a key of this block: written by this step, token index j - pos0 */
      int64_t tt = (int64_t)b * c->tps + (j - pos0);
      kc = c->knew + (tt * hkv + kvh) * hd;
      vc = c->vnew + (tt * hkv + kvh) * hd;
    } else {
      kc = c->past_k[b * hkv + kvh] + j * hd;
      vc = c->past_v[b * hkv + kvh] + j * hd;
    }
    for (int d = 0; d < hd; ++d) { K[(j - lo) * hd + d] = g_e4m3[kc[d]]; V[(j - lo) * hd + d] = g_e4m3[vc[d]]; }
  }
  msk_or_attend(c->q + (int64_t)t * hq * hd + (int64_t)h * hd, K, V, n, hd, 1.0 / sqrt((double)hd),
                c->o + (int64_t)t * hq * hd + (int64_t)h * hd, &c->smax[i]);
  free(K);
  free(V);
}

/* one expert over its tokens */
typedef struct {
  const msk_or_cfg* cfg;
  int n_used;
  const int* used;          /* expert ids */
  const msk_src_nvfp4* wg;  /* per used expert */
  const msk_src_nvfp4* wu;
  const msk_src_nvfp4* wd;
  int T;
  const int16_t* ids;       /* [T][k] */
  const double* x2;         /* [T][d] */
  double* y;                /* [T][k][d] */
} ex_ctx;
static void expert_one(void* p, int64_t ui) {
  ex_ctx* c = (ex_ctx*)p;
  const msk_or_cfg* g = c->cfg;
  int d = g->d_model, f = g->expert_dim, k = g->top_k, e = c->used[ui];
  double* gate = (double*)malloc(sizeof(double) * (size_t)f);
  double* up = (double*)malloc(sizeof(double) * (size_t)f);
  double* a = (double*)malloc(sizeof(double) * (size_t)f);
  double* row = (double*)malloc(sizeof(double) * (size_t)(d > f ? d : f));
  for (int t = 0; t < c->T; ++t)
    for (int s = 0; s < k; ++s) {
      if (c->ids[t * k + s] != e) continue;
      const double* x = c->x2 + (int64_t)t * d;
      for (int n = 0; n < f; ++n) {
        double ag = 0.0, au = 0.0;
        deq_row(&c->wg[ui], d, n, row);
        for (int i = 0; i < d; ++i) ag += x[i] * row[i];
        deq_row(&c->wu[ui], d, n, row);
        for (int i = 0; i < d; ++i) au += x[i] * row[i];
        gate[n] = ag; up[n] = au;
        a[n] = msk_or_silu(ag) * au;
      }
      double* y = c->y + ((int64_t)t * k + s) * d;
      for (int m = 0; m < d; ++m) {
        deq_row(&c->wd[ui], f, m, row);
        double acc = 0.0;
        for (int n = 0; n < f; ++n) acc += a[n] * row[n];
        y[m] = acc;
      }
    }
  free(gate); free(up); free(a); free(row);
}

/* ---- the step ------------------------------------------------------------------ */
int msk_oracle_step(const msk_or_cfg* g, const msk_source* src, int n_seqs, int tps,
                    const int32_t* seq_ids, const int32_t* positions, const uint16_t* hidden_in,
                    const msk_or_force* force, int n_threads, msk_or_out* out) {
  const int16_t* forced_ids = force ? force->ids : NULL;
  pthread_once(&g_tab_once, build_tables);
  const int L = g->n_layers, d = g->d_model, hq = g->n_q_heads, hkv = g->n_kv_heads, hd = g->head_dim;
  const int E = g->n_experts, k = g->top_k, f = g->expert_dim;
  const int T = n_seqs * tps, qd = hq * hd, kvd = hkv * hd;
  if (L < 1 || L > SY_MAX_LAYERS || d % 16 || qd % 16 || f % 16 || hq % hkv || k < 1 || k > E || T < 1)
    return MSK_OR_EINVAL;
  for (int b = 0; b < n_seqs; ++b)
    for (int i = 0; i < tps; ++i)
      if (positions[b * tps + i] != positions[b * tps] + i || positions[b * tps] < 0) return MSK_OR_EPOS;

  double* h = (double*)malloc(sizeof(double) * (size_t)T * d);
  double* x = (double*)malloc(sizeof(double) * (size_t)T * d);
  double* q = (double*)malloc(sizeof(double) * (size_t)T * qd);
  double* kk = (double*)malloc(sizeof(double) * (size_t)T * kvd);
  double* vv = (double*)malloc(sizeof(double) * (size_t)T * kvd);
  double* o = (double*)malloc(sizeof(double) * (size_t)T * qd);
  double* tmp = (double*)malloc(sizeof(double) * (size_t)(qd > d ? qd : d));
  double* logits = (double*)malloc(sizeof(double) * (size_t)T * E);
  double* rw = (double*)malloc(sizeof(double) * (size_t)T * k);
  int16_t* ids = (int16_t*)malloc(sizeof(int16_t) * (size_t)T * k);
  double* y = (double*)malloc(sizeof(double) * (size_t)T * k * d);
  double* smax = (double*)malloc(sizeof(double) * (size_t)T * hq);
  uint8_t* knew = (uint8_t*)malloc((size_t)T * kvd);
  uint8_t* vnew = (uint8_t*)malloc((size_t)T * kvd);
  uint8_t** past_k = (uint8_t**)calloc((size_t)n_seqs * hkv, sizeof(uint8_t*));
  uint8_t** past_v = (uint8_t**)calloc((size_t)n_seqs * hkv, sizeof(uint8_t*));
  int* used = (int*)malloc(sizeof(int) * (size_t)E);
  msk_src_nvfp4* wexp = (msk_src_nvfp4*)malloc(sizeof(msk_src_nvfp4) * 3 * (size_t)E);
  int rc = MSK_OR_OK;
  if (!h || !x || !q || !kk || !vv || !o || !tmp || !logits || !rw || !ids || !y || !smax || !knew || !vnew ||
      !past_k || !past_v || !used || !wexp) { rc = MSK_OR_ENOMEM; goto done; }

  for (int64_t i = 0; i < (int64_t)T * d; ++i) h[i] = msk_or_bf16_decode(hidden_in[i]);

  for (int l = 0; l < L; ++l) {
    const float *g_attn, *g_q, *g_k, *g_moe, *wr;
    msk_src_nvfp4 wq, wk, wv, wo;
    if (src->vec(src->ctx, l, SRC_ATTN_G, &g_attn) || src->vec(src->ctx, l, SRC_Q_G, &g_q) ||
        src->vec(src->ctx, l, SRC_K_G, &g_k) || src->vec(src->ctx, l, SRC_MOE_G, &g_moe) ||
        src->vec(src->ctx, l, SRC_ROUTER, &wr) || src->nvfp4(src->ctx, l, SRC_WQ, 0, &wq) ||
        src->nvfp4(src->ctx, l, SRC_WK, 0, &wk) || src->nvfp4(src->ctx, l, SRC_WV, 0, &wv) ||
        src->nvfp4(src->ctx, l, SRC_WO, 0, &wo)) { rc = MSK_OR_ESRC; goto done; }

    /* attention block */
    for (int t = 0; t < T; ++t) msk_or_rmsnorm(h + (int64_t)t * d, g_attn, d, g->rms_eps, x + (int64_t)t * d);
    matmul_nvfp4(&wq, d, qd, T, x, q, 0, n_threads);
    matmul_nvfp4(&wk, d, kvd, T, x, kk, 0, n_threads);
    matmul_nvfp4(&wv, d, kvd, T, x, vv, 0, n_threads);
    for (int t = 0; t < T; ++t) {
      for (int hh = 0; hh < hq; ++hh) {
        double* p = q + (int64_t)t * qd + hh * hd;
        msk_or_rmsnorm(p, g_q, hd, g->rms_eps, tmp);
        memcpy(p, tmp, sizeof(double) * hd);
      }
      for (int hh = 0; hh < hkv; ++hh) {
        double* p = kk + (int64_t)t * kvd + hh * hd;
        msk_or_rmsnorm(p, g_k, hd, g->rms_eps, tmp);
        memcpy(p, tmp, sizeof(double) * hd);
      }
    }
    for (int64_t i = 0; i < (int64_t)T * kvd; ++i) {
      knew[i] = (uint8_t)msk_or_e4m3_encode(kk[i]);
      vnew[i] = (uint8_t)msk_or_e4m3_encode(vv[i]);
      if (force && force->k && force->k[(int64_t)l * T * kvd + i] >= 0) knew[i] = (uint8_t)force->k[(int64_t)l * T * kvd + i];
      if (force && force->v && force->v[(int64_t)l * T * kvd + i] >= 0) vnew[i] = (uint8_t)force->v[(int64_t)l * T * kvd + i];
    }
    if (out->k_pre) memcpy(out->k_pre + (int64_t)l * T * kvd, kk, sizeof(double) * (size_t)T * kvd);
    if (out->v_pre) memcpy(out->v_pre + (int64_t)l * T * kvd, vv, sizeof(double) * (size_t)T * kvd);
    if (out->k_new) memcpy(out->k_new + (int64_t)l * T * kvd, knew, (size_t)T * kvd);
    if (out->v_new) memcpy(out->v_new + (int64_t)l * T * kvd, vnew, (size_t)T * kvd);

    /* past keys each (seq, kv head) needs: [lo of its first token, pos0) */
    for (int b = 0; b < n_seqs; ++b) {
      int64_t pos0 = positions[b * tps];
      int64_t lo = 0;
      if (g->is_sliding[l]) { lo = pos0 - g->window + 1; if (lo < 0) lo = 0; }
      for (int hh = 0; hh < hkv; ++hh) {
        free(past_k[b * hkv + hh]); free(past_v[b * hkv + hh]);
        past_k[b * hkv + hh] = (uint8_t*)malloc((size_t)(pos0 * hd + 1));
        past_v[b * hkv + hh] = (uint8_t*)malloc((size_t)(pos0 * hd + 1));
        if (!past_k[b * hkv + hh] || !past_v[b * hkv + hh]) { rc = MSK_OR_ENOMEM; goto done; }
        if (pos0 > lo &&
            src->past_kv(src->ctx, l, seq_ids ? seq_ids[b] : b, hh, lo, pos0 - lo,
                         past_k[b * hkv + hh] + lo * hd, past_v[b * hkv + hh] + lo * hd)) {
          rc = MSK_OR_ESRC; goto done;
        }
      }
    }
    at_ctx ac = {g, T, tps, l, positions, q, knew, vnew, past_k, past_v, o, smax};
    par_for((int64_t)T * hq, n_threads, attend_one, &ac);
    if (out->attn_out) memcpy(out->attn_out + (int64_t)l * T * qd, o, sizeof(double) * (size_t)T * qd);
    if (out->s_max_minus_bound) {
      double gq = 0, gk = 0, mx = -INFINITY;
      for (int i = 0; i < hd; ++i) { gq = fmax(gq, fabs(g_q[i])); gk = fmax(gk, fabs(g_k[i])); }
      for (int i = 0; i < T * hq; ++i) mx = fmax(mx, smax[i]);
      out->s_max_minus_bound[l] = mx - sqrt((double)hd) * gq * gk;
    }
    matmul_nvfp4(&wo, qd, d, T, o, h, 1, n_threads);

    /* MoE block */
    for (int t = 0; t < T; ++t) msk_or_rmsnorm(h + (int64_t)t * d, g_moe, d, g->rms_eps, x + (int64_t)t * d);
    for (int t = 0; t < T; ++t)
      for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int i = 0; i < d; ++i) acc += x[(int64_t)t * d + i] * (double)wr[(int64_t)e * d + i];
        logits[(int64_t)t * E + e] = acc;
      }
    for (int t = 0; t < T; ++t) {
      double gap;
      msk_or_topk(logits + (int64_t)t * E, E, k, ids + t * k, rw + t * k, &gap);
      if (out->route_gap) out->route_gap[(int64_t)l * T + t] = gap;
      const int16_t* fr = forced_ids ? forced_ids + ((int64_t)l * T + t) * k : NULL;
      if (fr && fr[0] >= 0) {
        for (int s = 0; s < k; ++s) ids[t * k + s] = fr[s];
        msk_or_route_weights(logits + (int64_t)t * E, ids + t * k, k, rw + t * k);
      }
    }
    if (out->logits) memcpy(out->logits + (int64_t)l * T * E, logits, sizeof(double) * (size_t)T * E);
    if (out->route_ids) memcpy(out->route_ids + (int64_t)l * T * k, ids, sizeof(int16_t) * (size_t)T * k);
    if (out->route_w) memcpy(out->route_w + (int64_t)l * T * k, rw, sizeof(double) * (size_t)T * k);

    int n_used = 0;
    for (int e = 0; e < E; ++e) {
      int hit = 0;
      for (int i = 0; i < T * k && !hit; ++i) hit = ids[i] == e;
      if (hit) {
        if (src->nvfp4(src->ctx, l, SRC_WGATE, e, &wexp[n_used]) ||
            src->nvfp4(src->ctx, l, SRC_WUP, e, &wexp[E + n_used]) ||
            src->nvfp4(src->ctx, l, SRC_WDOWN, e, &wexp[2 * E + n_used])) { rc = MSK_OR_ESRC; goto done; }
        used[n_used++] = e;
      }
    }
    if (out->n_distinct) out->n_distinct[l] = n_used;
    ex_ctx ec = {g, n_used, used, wexp, wexp + E, wexp + 2 * E, T, ids, x, y};
    par_for(n_used, n_threads, expert_one, &ec);
    for (int t = 0; t < T; ++t)
      for (int s = 0; s < k; ++s) {
        const double* ys = y + ((int64_t)t * k + s) * d;
        double w = rw[t * k + s];
        for (int i = 0; i < d; ++i) h[(int64_t)t * d + i] += w * ys[i];
      }
  }
  if (out->h_out) memcpy(out->h_out, h, sizeof(double) * (size_t)T * d);
  if (out->hidden_out)
    for (int64_t i = 0; i < (int64_t)T * d; ++i) out->hidden_out[i] = msk_or_bf16_encode(h[i]);

done:
  if (past_k) for (int i = 0; i < n_seqs * hkv; ++i) free(past_k[i]);
  if (past_v) for (int i = 0; i < n_seqs * hkv; ++i) free(past_v[i]);
  free(h); free(x); free(q); free(kk); free(vv); free(o); free(tmp); free(logits); free(rw); free(ids);
  free(y); free(smax); free(knew); free(vnew); free(past_k); free(past_v); free(used); free(wexp);
  return rc;
}
