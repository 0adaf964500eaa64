/*
 * msk.h -- C ABI of the B200 decode/verify-step megakernel for QK-normed
 * mixture-of-experts decoder stacks.
 *
 * The operation is one decode or speculative-verify step of the decoder
 * stack described in the PyTorch blog post "Optimizing Muse Spark Open on
 * TPU v7 with SGLang-TorchTPU" (sections "One program replaces many kernel
 * boundaries", "Removing Attention Bottlenecks", "Model Architecture
 * Details", "Expert Weight Quantization"): for every layer, RMSNorm, QK-norm
 * attention over an fp8-e4m3 KV cache (sliding-window-2048 or full-context
 * layers), RMSNorm, top-k-of-E routing, NVFP4 SwiGLU experts and a weighted
 * combine, all in one persistent cooperative kernel launch.  Embedding, LM
 * head, draft model and sampling stay with the caller, as the post places
 * them in the serving layer.
 *
 * Conventions
 *  - Every call returns msk_status_t; none throws, aborts or exits.
 *  - "dev" pointers are CUDA device pointers on the handle's device; "host"
 *    pointers are read during the call only.
 *  - Weight pointers are BORROWED: they must stay valid and unchanged until
 *    msk_destroy.  All of them must be 16-byte aligned.  msk_create reads
 *    the expert weights once, to repack them into library-owned tiles that
 *    each K chunk's weights stream from as one contiguous copy
 *    (msk_query().repacked_bytes); the step reads those tiles.
 *  - msk_step enqueues work on the caller's stream and never synchronises the
 *    host.  Errors the device detects (a wait that gave up, a position
 *    outside the cache) are recorded in a device status word that
 *    msk_step_status returns after the caller has synchronised the stream.
 *  - A handle is not thread-safe; use one handle per thread and device.
 */
#ifndef MSK_H
#define MSK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MSK_MAX_LAYERS 64
#define MSK_MAX_TOKENS 64 /* n_seqs * tokens_per_seq per step */

typedef enum msk_status {
  MSK_OK = 0,
  MSK_ERR_INVALID_ARG = 1, /* a null pointer, bad shape, misaligned pointer */
  MSK_ERR_UNSUPPORTED = 2, /* not an sm_100 device, no cooperative launch, or
                              a shape outside the supported set */
  MSK_ERR_OOM = 3,         /* device allocation failed */
  MSK_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed */
  MSK_ERR_BOUND = 5,       /* 2*M >= 80 for some layer: the fixed softmax
                              shift would underflow fp32 exp */
  MSK_ERR_KV_RANGE = 6,    /* positions not contiguous per sequence, negative,
                              or beyond the cache capacity (device-detected) */
  MSK_ERR_TIMEOUT = 7,     /* a device-side wait exceeded its limit; the
                              step's outputs are undefined */
  MSK_ERR_DEVICE = 8       /* another device-side check failed */
} msk_status_t;

/* An NVFP4 tensor [rows][K] (device memory, borrowed):
 *  codes  [rows][K/2]  e2m1 codes, two per byte, low nibble = even column
 *  scales [rows][K/16] e4m3 scale codes, one per 16 consecutive columns
 *  value(r, c) = e2m1(code) * e4m3(scale[r][c/16]) * global_scale
 * (the post's "NVFP4 ... one scale per 16 values"; the fp32 per-tensor
 * global scale is the usual NVFP4 second level and may be 1). */
typedef struct msk_nvfp4 {
  const uint8_t* codes;
  const uint8_t* scales;
  float global_scale;
} msk_nvfp4_t;

typedef struct msk_config {
  int32_t n_layers;       /* 1 .. MSK_MAX_LAYERS */
  int32_t d_model;        /* multiple of 256, <= 4096; above 512 a multiple of 512 */
  int32_t n_q_heads;      /* n_q_heads * head_dim: multiple of 256, <= 4096;
                             above 512 a multiple of 512 */
  int32_t n_kv_heads;     /* divides n_q_heads */
  int32_t head_dim;       /* 64 or 128 */
  int32_t n_experts;      /* multiple of 32, <= 256 */
  int32_t top_k;          /* 1 .. 8, <= n_experts */
  int32_t expert_dim;     /* multiple of 128, <= 4096; above 512 a multiple of 512 */
  int32_t window;         /* sliding-window length in keys, >= 1 */
  uint8_t layer_is_sliding[MSK_MAX_LAYERS]; /* 1: sliding-window layer */
  float rms_eps;          /* RMSNorm epsilon (all four norms) */
  int32_t max_seqs;       /* largest n_seqs a step may pass */
  int32_t max_tokens_per_seq; /* largest tokens_per_seq a step may pass;
                                 max_seqs * max_tokens_per_seq <= 64 and
                                 max_tokens_per_seq * (n_q_heads/n_kv_heads)
                                 <= 64 */
  uint32_t flags;         /* MSK_F_* */
  int32_t wait_timeout_us; /* limit of every device wait; 0 = 2,000,000 */
  int32_t expert_mma_min_tokens; /* tau: the gate/up projection of an expert
                             unit (up to 8 of an expert's tokens) with at
                             least tau tokens runs on the block-scaled tensor
                             cores, the others on the CUDA-core path (the
                             post's "Expert Weight Quantization": NVFP4 GEMV
                             at one token, a dense contraction where several
                             tokens share an expert).  0 = the library's
                             default, MSK_TAU_DEFAULT; above 8 = never (the
                             CUDA-core path for every unit); 1 = always */
} msk_config_t;

#define MSK_F_TRACE 1u /* record per-phase %globaltimer stamps (msk_query) */
/* Gate/up projections of every expert unit on the block-scaled tensor cores
 * (tcgen05.mma kind::mxf4nvf4), the same as expert_mma_min_tokens = 1: the
 * NVFP4 weights are consumed as stored (their block scales from a copy
 * msk_create repacks into the tensor cores' layout), the moe-norm
 * activations as eight e2m1 terms (relative error ~1e-5 of the row's
 * largest value). */
#define MSK_F_TC_EXPERTS 2u
/* expert_mma_min_tokens when the config leaves it 0: every unit on the
 * block-scaled tensor cores (measured faster than the CUDA-core decode at
 * every unit size the workloads produce, 1-8 tokens) */
#define MSK_TAU_DEFAULT 1
#define MSK_TAU_NEVER 0x7FFFFFFF

/* Per-layer weights, all device pointers, borrowed.
 *  attn_norm_g [d], moe_norm_g [d]      RMSNorm gains (fp32)
 *  q_norm_g [head_dim], k_norm_g [head_dim]  QK-norm gains shared by heads
 *  router [n_experts][d] fp32
 *  wq [Hq*hd][d], wk, wv [Hkv*hd][d], wo [d][Hq*hd]          NVFP4
 *  w_gate, w_up [n_experts][expert_dim][d], w_down [n_experts][d][expert_dim]
 *    NVFP4, experts contiguous; one global scale per tensor. */
typedef struct msk_layer_weights {
  const float* attn_norm_g;
  const float* q_norm_g;
  const float* k_norm_g;
  const float* moe_norm_g;
  const float* router;
  msk_nvfp4_t wq, wk, wv, wo;
  msk_nvfp4_t w_gate, w_up, w_down;
} msk_layer_weights_t;

typedef struct msk_handle msk_handle_t;
typedef struct msk_kv msk_kv_t;

/* Optional capture of intermediate results by the next steps (device
 * pointers, any may be NULL; T = n_seqs * tokens_per_seq of the step):
 *  route_ids [L][T][top_k] int16, route_w [L][T][top_k] fp32,
 *  logits [L][T][n_experts] fp32, attn_out [L][T][Hq*hd] fp32 (attention
 *  output before W_o), trace [L][16] uint64 %globaltimer stamps of CTA 0,
 *  k_pre, v_pre [L][T][Hkv*hd] fp32: this step's keys after QK-norm and
 *  values, each exactly as the step holds it just before the fp8 e4m3
 *  encoding that writes it into the cache.
 * hold_barrier (a test hook of this library, not part of the method): when
 * n > 0, CTA 0 withholds its arrival at the step's n-th grid barrier, so
 * every CTA's wait there runs out after wait_timeout_us and the step ends
 * with MSK_ERR_TIMEOUT (no trap, no fault: copies in flight land first and
 * the kernel returns).  0 = off. */
typedef struct msk_debug {
  int16_t* route_ids;
  float* route_w;
  float* logits;
  float* attn_out;
  uint64_t* trace;
  float* k_pre;
  float* v_pre;
  int32_t hold_barrier;
} msk_debug_t;

typedef struct msk_stats {
  int32_t n_layers;
  int32_t n_distinct[MSK_MAX_LAYERS]; /* distinct experts per layer, last step */
  int64_t algorithmic_bytes;  /* HBM bytes the last step must stream: dense
                                 NVFP4 + router + distinct experts' NVFP4 +
                                 KV read over distinct positions + KV write +
                                 hidden in/out */
  int64_t weight_bytes;       /* the weight part of algorithmic_bytes */
  int64_t kv_bytes;           /* the KV part */
  int64_t scratch_bytes;      /* device scratch the handle owns */
  int64_t repacked_bytes;     /* library-owned copies of weight data in
                                 another layout (the gate/up block scales in
                                 the block-scaled tensor cores' layout, when
                                 that expert path is enabled) */
} msk_stats_t;

/* Create a handle on `device`: validates the shapes, computes the per-layer
 * softmax bound M = sqrt(head_dim) * max|q_norm_g| * max|k_norm_g| (reads
 * the gains once, synchronously) and rejects 2*M >= 80 with MSK_ERR_BOUND,
 * allocates scratch, and copies the weight descriptors (not the weights).
 * `layers` is a host array of n_layers entries. */
msk_status_t msk_create(const msk_config_t* config, const msk_layer_weights_t* layers, int device,
                        msk_handle_t** out);
void msk_destroy(msk_handle_t* h);

/* Library-owned fp8-e4m3 KV cache for n_seqs sequences of `capacity`
 * positions each, layout [K|V][layer][seq][kv_head][position][head_dim],
 * zero-initialised.  capacity is rounded up to a multiple of 16. */
msk_status_t msk_kv_create(msk_handle_t* h, int n_seqs, int64_t capacity, msk_kv_t** out);
void msk_kv_destroy(msk_kv_t* kv);

/* Copy n positions [pos0, pos0+n) of sequence `seq`, layer `layer` into the
 * cache from device arrays k_fp8, v_fp8 laid out [n][n_kv_heads][head_dim]
 * (e4m3 codes; 0x7F/0xFF NaN codes are not allowed).  Async on `stream`. */
msk_status_t msk_kv_append(msk_handle_t* h, msk_kv_t* kv, int layer, int seq, int64_t pos0, int64_t n,
                           const uint8_t* k_fp8, const uint8_t* v_fp8, void* stream);

/* Encode n fp32 values into fp8 e4m3 codes with the rounding the step uses
 * when it writes this step's keys and values into the cache: round to
 * nearest, ties to even, saturating to +-448 (the OFP8 "E4M3" format the
 * post's fp8 KV cache stores; NaN stays NaN).  in: dev fp32 [n], out: dev
 * uint8 [n]; both 16-byte aligned, on the current device.  For callers
 * that build past K/V for msk_kv_append from wider values.  Async on
 * `stream`. */
msk_status_t msk_kv_encode(const float* in, uint8_t* out, int64_t n, void* stream);

/* Read n positions back out of the cache into device or host arrays
 * laid out [n][n_kv_heads][head_dim]; synchronous. */
msk_status_t msk_kv_read(msk_handle_t* h, msk_kv_t* kv, int layer, int seq, int64_t pos0, int64_t n,
                         uint8_t* k_out, uint8_t* v_out);

/* One decode (tokens_per_seq == 1) or verify (tokens_per_seq > 1) step.
 *  hidden_in  dev bf16 [n_seqs*tokens_per_seq][d_model]
 *  positions  dev int32 [n_seqs][tokens_per_seq], contiguous per sequence
 *             (p, p+1, ...); keys at positions below p must already be in
 *             the cache; this step writes K/V at its own positions
 *             (overwriting: rolling back a draft is passing earlier positions)
 *  hidden_out dev bf16 [n_seqs*tokens_per_seq][d_model]
 *  stream     cudaStream_t (NULL = legacy default stream)
 * Enqueues one cooperative kernel launch (plus a small memset); no host
 * synchronisation.  Sequence b of the step is sequence b of the cache. */
msk_status_t msk_step(msk_handle_t* h, const uint16_t* hidden_in, const int32_t* positions, int n_seqs,
                      int tokens_per_seq, msk_kv_t* kv, uint16_t* hidden_out, void* stream);

/* Size of the working-memory array built into the library for
 * msk_step_static (8 MiB per device). */
#define MSK_STATIC_SCRATCH_BYTES (8u << 20)

/* msk_step with no allocation behind it.  The blog post has no counterpart
 * of this call: it is an integration aid of this library.
 *
 * Who needs it: a caller that must not let the library allocate device
 * memory at step time or tie a step's working memory to one handle -- for
 * instance a serving engine that hands all free HBM to its own KV-block
 * pool after start-up (so any later cudaMalloc fails or fragments the pool)
 * and wants the step's footprint fixed and known when the library loads.
 *
 * Same arguments, same results and same kernel as msk_step; the difference
 * is where the step's working buffers (residual, projections, attention
 * partials, expert activations, barrier words) and the kernel's copy of the
 * parameter block live: in one array of MSK_STATIC_SCRATCH_BYTES compiled
 * into the library, shared by every handle on a device.  The call allocates
 * nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *  - First call on a device: looks the array's device address up
 *    (cudaGetSymbolAddress) with that device current; later calls reuse it.
 *    A lookup that fails is not remembered: the call returns MSK_ERR_CUDA
 *    and the next call tries again.  Make the first call before any stream
 *    capture begins.
 *  - Enqueues one small kernel that copies the handle's parameter block into
 *    the array and zeroes the barrier words (the only bytes that must start
 *    at zero), then the step kernel; no host synchronisation.
 *  - Device status and statistics still go to the handle: msk_step_status
 *    and msk_query work after it as after msk_step.
 *  - Returns MSK_ERR_UNSUPPORTED, before any device work, when the handle's
 *    shapes need more working memory than the array holds (about 6.7 MiB for
 *    16 tokens of d_model 2048; 64 tokens of d_model 4096 do not fit), or the
 *    device index is 64 or more; MSK_ERR_CUDA if the lookup fails.
 *  - All calls on a device share the array: two such steps in flight at the
 *    same time on one device (other streams, handles or threads) race and
 *    corrupt each other.  Order them on one stream, or use msk_step. */
msk_status_t msk_step_static(msk_handle_t* h, const uint16_t* hidden_in, const int32_t* positions, int n_seqs,
                             int tokens_per_seq, msk_kv_t* kv, uint16_t* hidden_out, void* stream);

/* Device status of the steps since the last call (call after synchronising
 * the stream); clears it. */
msk_status_t msk_step_status(msk_handle_t* h);

/* msk_step_status, plus where the device recorded its first error: the
 * layer, the phase (0 input norm, 1 QKV projection, 2 QK-norm and KV write,
 * 3 attention, 4 attention combine, 5 W_o, 6 MoE norm, 7 router, 8 top-k,
 * 9 gate/up, 10 down, 11 combine, 12 the wait for a (token, expert) pair's
 * SwiGLU row as e2m1 terms, read by the block-scaled down projection) and
 * the CTA; all -1 when the status is
 * MSK_OK or the error carries no site (positions refused before the layer
 * loop).  Any out pointer may be NULL.  Clears the status like
 * msk_step_status. */
msk_status_t msk_step_status_at(msk_handle_t* h, int32_t* layer, int32_t* phase, int32_t* cta);

/* Set (or, with NULL, clear) the capture buffers used by later steps. */
msk_status_t msk_set_debug(msk_handle_t* h, const msk_debug_t* dbg);

/* Statistics of the last completed step (synchronises the device). */
msk_status_t msk_query(msk_handle_t* h, msk_stats_t* out);

const char* msk_status_string(msk_status_t s);

#ifdef __cplusplus
}
#endif
#endif /* MSK_H */
