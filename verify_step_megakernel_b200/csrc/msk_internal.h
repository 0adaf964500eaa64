/*
 * msk_internal.h -- structures shared by the host launcher and the
 * persistent step kernel (not part of the public ABI).
 */
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "../../include/msk.h"

/* CTA shape: warpgroup 0 is the producer (one thread issues the bulk/TMA
 * copies into the ring; the group gives its registers back), warpgroups 1-2
 * are MSK_NCW consumer warps (tensor-core tiles, norms, routing). */
#define MSK_NCW 8
#define MSK_NTHREADS ((MSK_NCW + 4) * 32)
#define MSK_NST 5            /* ring stages */
#define MSK_STAGE 36864      /* bytes per stage: 16 rows x 4096 NVFP4 + scales */
#define MSK_SCR 32768        /* consumer scratch: split-K / key-split reductions */
#define MSK_NT_DENSE 8       /* n-tiles of 8 tokens: dense projections, T <= 64 */
#define MSK_UNIT_TOK 8       /* tokens of an expert unit (one 8-column n-tile) */
#define MSK_MAX_UNITS 512    /* expert units per layer (T*k <= 512) */
#define MSK_MAX_PAIRS 64     /* (sequence, kv-head) attention pairs */

#define MSK_MAP_DENSE 6
#define MSK_MAP_GUSW 14 /* gate and up codes as 128-byte-swizzled 128 x 128-byte boxes */
#define MSK_NMAPS 16
#define MSK_XQ_BYTES(d) ((size_t)(d) * 4 + 16)

/* control words, zeroed per step: the grid barrier's counter, the abort
 * word, from CTRL_PAIR0 one counter per attention pair (the CTAs that have
 * written their part of the pair's attention in the current layer), and
 * from CTRL_UT0 one word per (token, expert) pair: the last layer + 1 whose
 * SwiGLU term row of the pair is written */
enum { CTRL_BARRIER = 0, CTRL_ABORT = 1, CTRL_PAIR0 = 32, CTRL_UT0 = 32 + MSK_MAX_PAIRS,
       CTRL_WORDS = CTRL_UT0 + MSK_MAX_TOKENS * 8 };
/* persistent status words (cleared by msk_step_status) */
enum { ST_CODE = 0, ST_WHERE = 1, ST_WORDS = 4 };

typedef struct MskNv {
  const uint8_t* codes;
  const uint8_t* scales;
  float gs;
  int32_t pad;
} MskNv;

typedef struct MskLayer {
  const float* g_attn;
  const float* g_q;
  const float* g_k;
  const float* g_moe;
  const float* router;
  MskNv wq, wk, wv, wo, wg, wu, wd;
  /* 2-D tensor maps of the weights (device), MSK_NMAPS of them: gate
   * codes, gate scales, up codes, up scales, down codes, down scales, then
   * (from MSK_MAP_DENSE) codes and scales of wq, wk, wv, wo */
  const CUtensorMap* emap;
  /* expert weights repacked (library-owned) into slot images, one
   * contiguous bulk copy per K chunk: gate/up tiles of the block-scaled path
   * [E][f/128][d/256][36 KB] (swizzled codes of both matrices, then their
   * scale-factor atoms), down tiles of the CUDA-core path
   * [E][d/128][f/KC][128 (KC/2 + 32 + KC/16)] (null when K is not a
   * multiple of 256: whole rows are copied then) */
  const uint8_t* xtgu;
  const uint8_t* xtdn;
  /* down tiles of the block-scaled path [E][d/128][f/512][36 KB]: per 512-wide
   * K chunk the swizzled codes of its two 256-wide halves, then their
   * scale-factor atoms (the gate/up tile layout with the halves in place of
   * the two matrices); null when no unit takes that path or f is not a
   * multiple of 512 */
  const uint8_t* xtdt;
  float bound_log2; /* M * log2(e), M = sqrt(hd) max|g_q| max|g_k| */
  int32_t sliding;
} MskLayer;

typedef struct MskParams {
  int32_t L, d, hq, hkv, hd, E, k, f, W, G, qd, kvd;
  int32_t ncta, max_T;
  float eps, scale_log2; /* 1/sqrt(hd) * log2(e) */
  int64_t timeout_ns;
  uint32_t flags;
  int32_t tau;      /* expert units with at least tau tokens: gate/up on the block-scaled tensor cores */
  /* scratch (device) */
  float* h;         /* [T][d] residual */
  uint16_t* x;      /* [T][d] f16 attention-norm input of the projections */
  float* qkv;       /* split-K partials of the projections: QKV [S][T][qd + 2 kvd], W_o [S][T][d] */
  uint16_t* qs;     /* [T][qd] f16 normalised queries */
  float* part;      /* [slots][R_max][hd + 4] attention partials */
  uint16_t* o;      /* [T][qd] f16 attention output */
  float* x2f;       /* [T][d] moe-norm output, fp32 (router) */
  uint16_t* x2h;    /* [T][d] same, f16 (gate/up on the CUDA-core path) */
  uint8_t* xq;      /* [T] the same row as eight e2m1 terms for the gate/up tensor cores, MSK_XQ_BYTES(d) each:
                       codes [d/32][8 term rows][16 B], then the fp32 factor */
  float* logits;    /* [T][E] */
  uint16_t* u;      /* [T*k][f] f16 SwiGLU activations */
  uint8_t* ut;      /* [T*k] the same row as eight e2m1 terms for the down projection on the block-scaled
                       tensor cores, MSK_XQ_BYTES(f) each (layout of xq) */
  float* y;         /* [T*k][d] expert outputs */
  uint32_t* ctrl;   /* CTRL_WORDS, zeroed per step */
  uint32_t* status; /* ST_WORDS */
  int32_t* n_distinct; /* [L] */
  int32_t* last_shape; /* [2 + MSK_MAX_TOKENS]: S, Tq, first position of each sequence */
  int32_t part_stride; /* floats per partial slot */
  /* debug capture (may be null) */
  int16_t* dbg_ids;
  float* dbg_w;
  float* dbg_logits;
  float* dbg_attn;
  uint64_t* dbg_trace;
  float* dbg_kpre;  /* [L][T][kvd] keys after QK-norm, before fp8 */
  float* dbg_vpre;  /* [L][T][kvd] values before fp8 */
  int32_t dbg_hold; /* > 0: CTA 0 withholds its arrival at grid barrier number dbg_hold (test hook) */
  int32_t dbg_pad;
  MskLayer layers[MSK_MAX_LAYERS];
} MskParams;

typedef struct MskStep {
  const uint16_t* hidden_in;
  const int32_t* positions;
  uint16_t* hidden_out;
  uint8_t* kv_base;        /* K region; V region starts kv_half_rows rows later */
  int64_t kv_cap;
  int64_t kv_half_rows;    /* L * kv_seqs * hkv * cap */
  int32_t kv_seqs;
  int32_t S, Tq, T;
} MskStep;
