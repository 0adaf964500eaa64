/*
 * msk_source.h -- how a consumer (the oracle) reads the step's inputs.
 *
 * A source hands out the model's tensors one at a time, in the stored
 * formats the step consumes: NVFP4 weights (e2m1 codes, two per byte, low
 * nibble = even index; one e4m3 scale per 16 consecutive inputs; an fp32
 * per-tensor global scale), fp32 gain vectors and router, and fp8-e4m3 past
 * K/V codes.  Two implementations live in synth_host.c: a lazy generator
 * that regenerates any tensor bit-identically from the seed, and an array
 * source over caller-filled host arrays (hand-built test cases).
 *
 * Sources are not thread-safe: call them from one thread.
 */
#ifndef MSK_SOURCE_H
#define MSK_SOURCE_H

#include <stdint.h>

#define SY_MAX_LAYERS 64

/* NVFP4 tensors by role */
enum { SRC_WQ = 0, SRC_WK = 1, SRC_WV = 2, SRC_WO = 3, SRC_WGATE = 4, SRC_WUP = 5, SRC_WDOWN = 6 };
/* fp32 vectors by role: gains [d] / [hd] / [hd] / [d], router [E][d] */
enum { SRC_ATTN_G = 0, SRC_Q_G = 1, SRC_K_G = 2, SRC_MOE_G = 3, SRC_ROUTER = 4 };

typedef struct sy_model {
  uint64_t seed;
  int32_t n_layers, d_model, n_q_heads, n_kv_heads, head_dim;
  int32_t n_experts, top_k, expert_dim, window;
  uint8_t is_sliding[SY_MAX_LAYERS];
  /* 0: literal reading, every global scale = 1; 1: per-tensor power-of-two
   * global scale from the fan-in */
  int32_t use_global_scale;
} sy_model;

typedef struct msk_src_nvfp4 {
  const uint8_t* codes;  /* [rows][K/2] */
  const uint8_t* scales; /* [rows][K/16] e4m3 codes */
  float global_scale;
} msk_src_nvfp4;

typedef struct msk_source {
  void* ctx;
  /* expert is ignored for the dense roles; returns 0 on success */
  int (*nvfp4)(void* ctx, int layer, int role, int expert, msk_src_nvfp4* out);
  int (*vec)(void* ctx, int layer, int role, const float** out);
  /* past K/V codes of (layer, seq, kv head) for positions [pos0, pos0+n),
   * written as k[n][head_dim], v[n][head_dim] */
  int (*past_kv)(void* ctx, int layer, int seq, int head, int64_t pos0, int64_t n,
                 uint8_t* k, uint8_t* v);
} msk_source;

#endif /* MSK_SOURCE_H */
