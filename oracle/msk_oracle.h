/*
 * msk_oracle.h -- TEST INFRASTRUCTURE: fp64 CPU reference of one
 * decode/verify step.  Only tests, the smoke check and the benchmark's CPU
 * baseline use it; the product library never links or calls it.
 */
#ifndef MSK_ORACLE_H
#define MSK_ORACLE_H

#include <stdint.h>

#include "../synth/msk_source.h"

#ifdef __cplusplus
extern "C" {
#endif

enum { MSK_OR_OK = 0, MSK_OR_EINVAL = 1, MSK_OR_EPOS = 2, MSK_OR_ENOMEM = 3, MSK_OR_ESRC = 4 };

typedef struct msk_or_cfg {
  int32_t n_layers, d_model, n_q_heads, n_kv_heads, head_dim;
  int32_t n_experts, top_k, expert_dim, window;
  uint8_t is_sliding[SY_MAX_LAYERS];
  double rms_eps;
} msk_or_cfg;

/* Outputs; any pointer may be NULL.  T = n_seqs * tokens_per_seq. */
typedef struct msk_or_out {
  uint16_t* hidden_out;      /* [T][d] bf16 bits */
  double* h_out;             /* [T][d] final residual before rounding */
  int16_t* route_ids;        /* [L][T][k] */
  double* route_w;           /* [L][T][k] */
  double* route_gap;         /* [L][T] k-th minus (k+1)-th logit */
  double* logits;            /* [L][T][E] */
  double* attn_out;          /* [L][T][Hq*hd] pre-W_o attention output */
  uint8_t* k_new;            /* [L][T][Hkv][hd] fp8 codes written this step */
  uint8_t* v_new;
  double* s_max_minus_bound; /* [L] max score minus sqrt(hd) max|g_q| max|g_k| */
  int32_t* n_distinct;       /* [L] distinct experts selected */
  double* k_pre;             /* [L][T][Hkv][hd] K after QK-norm, before fp8 */
  double* v_pre;             /* [L][T][Hkv][hd] V before fp8 */
} msk_or_out;

/* Optional replacements for decisions with two valid answers (NULL = none).
 *  ids[L][T][k]:   a token's expert set where ids[..][0] >= 0 (near-tied
 *                  routing); weights are the softmax of those experts' logits
 *  k, v[L][T][Hkv*hd]: an fp8 code where >= 0 (a value at an e4m3 rounding
 *                  midpoint, up to the compared implementation's error) */
typedef struct msk_or_force {
  const int16_t* ids;
  const int16_t* k;
  const int16_t* v;
} msk_or_force;

/* One step.  positions[n_seqs][tps] must be contiguous per sequence; keys
 * below a sequence's first position come from src->past_kv with sequence id
 * seq_ids[b] (or b if seq_ids is NULL).  `force` may be NULL. */
int msk_oracle_step(const msk_or_cfg* cfg, const msk_source* src, int n_seqs, int tps,
                    const int32_t* seq_ids, const int32_t* positions, const uint16_t* hidden_in,
                    const msk_or_force* force, int n_threads, msk_or_out* out);

/* building blocks, exported for the pin tests */
double msk_or_e2m1_decode(int nib);
double msk_or_e4m3_decode(int code);
int msk_or_e4m3_encode(double x);
void msk_or_e4m3_encode_n(const double* x, int64_t n, uint8_t* codes);
uint16_t msk_or_bf16_encode(double x);
double msk_or_bf16_decode(uint16_t b);
void msk_or_rmsnorm(const double* x, const float* g, int n, double eps, double* y);
double msk_or_silu(double a);
void msk_or_topk(const double* logits, int n, int k, int16_t* ids, double* w, double* gap);
void msk_or_route_weights(const double* logits, const int16_t* ids, int k, double* w);
void msk_or_attend(const double* q, const double* K, const double* V, int64_t n, int hd, double scale,
                   double* o, double* s_max);

#ifdef __cplusplus
}
#endif
#endif /* MSK_ORACLE_H */
