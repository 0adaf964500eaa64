/*
 * msk_synth.h -- seeded synthetic inputs for the MoE decode/verify step.
 *
 * This header is the whole input recipe: a counter-based generator
 * (splitmix64, Steele/Lea/Flood 2014) keyed by (seed, tensor stream,
 * element index), a table-driven standard normal, and the encoders that turn
 * those normals into the stored input formats (bf16 hidden states, fp32
 * router, fp8-e4m3 past KV, NVFP4 weights).  It is compiled both by the host
 * C compiler (for the oracle's on-demand regeneration) and by nvcc (for the
 * device fill kernels), and every operation in it is either integer or an
 * IEEE correctly rounded float operation that is never fused, so the two
 * sides produce bit-identical tensors.
 *
 * It holds none of the step's arithmetic: the encoders here prepare inputs
 * (weight quantisation happens offline in the pages' system), they are not
 * used by the step itself.
 */
#ifndef MSK_SYNTH_H
#define MSK_SYNTH_H

#include <stdint.h>

#if defined(__CUDACC__)
#define SY_FN static __host__ __device__ __forceinline__
#else
#define SY_FN static inline
#endif

/* Correctly rounded, never-contracted float arithmetic on both sides.  The
 * host side must be compiled with -ffp-contract=off on an SSE2 target. */
#if defined(__CUDA_ARCH__)
#define SY_ADD(a, b) __fadd_rn((a), (b))
#define SY_SUB(a, b) __fsub_rn((a), (b))
#define SY_MUL(a, b) __fmul_rn((a), (b))
#define SY_DIV(a, b) __fdiv_rn((a), (b))
#else
#define SY_ADD(a, b) ((float)((float)(a) + (float)(b)))
#define SY_SUB(a, b) ((float)((float)(a) - (float)(b)))
#define SY_MUL(a, b) ((float)((float)(a) * (float)(b)))
#define SY_DIV(a, b) ((float)((float)(a) / (float)(b)))
#endif

SY_FN uint32_t sy_f2u(float f) {
#if defined(__CUDA_ARCH__)
  return __float_as_uint(f);
#else
  union { float f; uint32_t u; } c; c.f = f; return c.u;
#endif
}
SY_FN float sy_u2f(uint32_t u) {
#if defined(__CUDA_ARCH__)
  return __uint_as_float(u);
#else
  union { float f; uint32_t u; } c; c.u = u; return c.f;
#endif
}
SY_FN int sy_clz32(uint32_t x) {
#if defined(__CUDA_ARCH__)
  return __clz((int)x);
#else
  return x ? __builtin_clz(x) : 32;
#endif
}

/* ---- counter-based generator: splitmix64 ------------------------------- */
#define SY_GAMMA 0x9E3779B97F4A7C15ull
SY_FN uint64_t sy_fmix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
/* Key of one tensor stream under one seed. */
SY_FN uint64_t sy_key(uint64_t seed, uint64_t stream) {
  return sy_fmix64(sy_fmix64(seed + SY_GAMMA) ^ (stream * 0xD1B54A32D192ED03ull + 0x632BE59BD9B4E019ull));
}
/* i-th output of splitmix64 started at state `key`. */
SY_FN uint64_t sy_u64(uint64_t key, uint64_t idx) {
  return sy_fmix64(key + (idx + 1ull) * SY_GAMMA);
}

/* Tensor streams: one per (kind, layer, a, b). */
enum {
  SY_HIDDEN = 1, SY_ATTN_G = 2, SY_Q_G = 3, SY_K_G = 4, SY_MOE_G = 5, SY_ROUTER = 6,
  SY_WQ = 7, SY_WK = 8, SY_WV = 9, SY_WO = 10, SY_WGATE = 11, SY_WUP = 12, SY_WDOWN = 13,
  SY_PAST_K = 14, SY_PAST_V = 15
};
SY_FN uint64_t sy_stream(uint32_t kind, uint32_t layer, uint32_t a, uint32_t b) {
  return ((uint64_t)kind << 56) | ((uint64_t)(layer & 0xFFFu) << 44) |
         ((uint64_t)(a & 0x3FFFFFu) << 22) | (uint64_t)(b & 0x3FFFFFu);
}

/* ---- standard normal by table-interpolated inverse CDF ----------------- *
 * The top 32 bits u of a draw give a sign (bit 31) and r in [0, 2^31); the
 * magnitude is z = Phi^-1(1 - q), q = (r + 0.5) / 2^32.  For r < 64 the
 * table holds z exactly; above, r falls in the octave [2^b, 2^(b+1)),
 * b = 6..30, split into 64 equal segments with z interpolated linearly
 * between the segment nodes.  The table is built once on the host (double
 * precision bisection on erfc) and passed to the device unchanged. */
#define SY_GT_LOW 64
#define SY_GT_OCT 25
#define SY_GT_SEG 64
typedef struct sy_gtab {
  float low[SY_GT_LOW];
  float oct[SY_GT_OCT][SY_GT_SEG + 1];
} sy_gtab;

SY_FN float sy_pow2i(int e) { /* 2^e for -126 <= e <= 127 */
  return sy_u2f((uint32_t)(e + 127) << 23);
}

SY_FN float sy_gauss(const sy_gtab* T, uint64_t h) {
  uint32_t u = (uint32_t)(h >> 32);
  uint32_t r = u & 0x7FFFFFFFu;
  float z;
  if (r < SY_GT_LOW) {
    z = T->low[r];
  } else {
    int b = 31 - sy_clz32(r);
    int sh = b - 6;
    uint32_t off = r - (1u << b);
    uint32_t j = off >> sh;
    uint32_t rem = off & ((1u << sh) - 1u);
    float fr = SY_MUL((float)rem, sy_pow2i(-sh));
    float a = T->oct[b - 6][j], c = T->oct[b - 6][j + 1];
    z = SY_ADD(a, SY_MUL(fr, SY_SUB(c, a)));
  }
  return (u >> 31) ? -z : z;
}

/* Uniform in [lo, lo + span) from 24 bits. */
SY_FN float sy_uniform(uint64_t h, float lo, float span) {
  float u = SY_MUL((float)(uint32_t)(h >> 40), sy_pow2i(-24));
  return SY_ADD(lo, SY_MUL(u, span));
}

/* ---- input encoders ------------------------------------------------------ */
/* float -> bf16 bits, round to nearest even (finite inputs). */
SY_FN uint16_t sy_bf16(float f) {
  uint32_t u = sy_f2u(f);
  uint32_t lsb = (u >> 16) & 1u;
  return (uint16_t)((u + 0x7FFFu + lsb) >> 16);
}

/* round-half-even of 0 <= y < 2^22 to an integer, exactly, via 2^23 */
SY_FN float sy_rint_small(float y) {
  return SY_SUB(SY_ADD(y, 8388608.0f), 8388608.0f);
}

/* float -> fp8 e4m3fn, round to nearest even, saturating to +-448. */
SY_FN uint8_t sy_e4m3(float f) {
  uint32_t u = sy_f2u(f);
  uint8_t sign = (uint8_t)((u >> 24) & 0x80u);
  float a = sy_u2f(u & 0x7FFFFFFFu);
  if (!(a == a)) return (uint8_t)(sign | 0x7Eu); /* NaN input never occurs */
  if (a < 0.015625f) { /* below 2^-6: subnormal grid of 2^-9 */
    float m = sy_rint_small(SY_MUL(a, 512.0f)); /* 0..8, 8 is 2^-6 = code 8 */
    return (uint8_t)(sign | (uint8_t)m);
  }
  uint32_t ab = u & 0x7FFFFFFFu;
  int e = (int)(ab >> 23) - 127; /* >= -6 */
  if (e > 8) return (uint8_t)(sign | 0x7Eu);
  uint32_t mant = ab & 0x7FFFFFu;
  uint32_t keep = mant >> 20, rest = mant & 0xFFFFFu;
  if (rest > 0x80000u || (rest == 0x80000u && (keep & 1u))) keep++;
  if (keep == 8u) { keep = 0; e++; }
  int code = ((e + 7) << 3) | (int)keep;
  if (code > 0x7E) code = 0x7E;
  return (uint8_t)(sign | (uint8_t)code);
}

/* fp8 e4m3fn code -> float (exact), for finite codes. */
SY_FN float sy_e4m3_value(uint8_t c) {
  int e = (c >> 3) & 0xF, m = c & 7;
  float v = e ? SY_MUL((float)(8 + m), sy_pow2i(e - 10)) : SY_MUL((float)m, sy_pow2i(-9));
  return (c & 0x80) ? -v : v;
}

/* float -> e2m1 nibble, round to nearest even on the grid
 * {0, .5, 1, 1.5, 2, 3, 4, 6}, saturating to +-6. */
SY_FN uint8_t sy_e2m1(float f) {
  uint32_t u = sy_f2u(f);
  uint8_t sign = (uint8_t)((u >> 28) & 0x8u);
  float a = sy_u2f(u & 0x7FFFFFFFu);
  uint8_t m;
  if (a <= 0.25f) m = 0;
  else if (a < 0.75f) m = 1;
  else if (a <= 1.25f) m = 2;
  else if (a < 1.75f) m = 3;
  else if (a <= 2.5f) m = 4;
  else if (a < 3.5f) m = 5;
  else if (a <= 5.0f) m = 6;
  else m = 7;
  return (uint8_t)(sign | m);
}

/* Per-tensor power-of-two global scale for NVFP4 weights of standard
 * deviation sigma: 2^ceil(log2(8 sigma / 6 / 448)), so the largest block
 * scales land near the top of the e4m3 range.  Computed on the host only. */

/* Quantise one block of 16 values to NVFP4: writes 8 code bytes (low nibble
 * = even index) and returns the e4m3 scale code.  gs is the tensor's global
 * scale (a power of two). */
SY_FN uint8_t sy_nvfp4_block(const float* w, float gs, uint8_t* codes8) {
  float amax = 0.0f;
  for (int i = 0; i < 16; ++i) {
    float a = w[i] < 0.0f ? -w[i] : w[i];
    amax = a > amax ? a : amax;
  }
  uint8_t sc = sy_e4m3(SY_DIV(SY_DIV(amax, 6.0f), gs));
  float s = SY_MUL(sy_e4m3_value(sc), gs);
  for (int i = 0; i < 8; ++i) {
    uint8_t lo = 0, hi = 0;
    if (s > 0.0f) {
      lo = sy_e2m1(SY_DIV(w[2 * i], s));
      hi = sy_e2m1(SY_DIV(w[2 * i + 1], s));
    }
    codes8[i] = (uint8_t)(lo | (hi << 4));
  }
  return sc;
}

/* One NVFP4 block (row, kb) of a [rows][K] weight of standard deviation sigma. */
SY_FN uint8_t sy_nvfp4_gen_block(const sy_gtab* T, uint64_t key, uint64_t row, uint32_t K,
                                 uint32_t kb, float sigma, float gs, uint8_t* codes8) {
  float w[16];
  uint64_t base = row * (uint64_t)K + (uint64_t)kb * 16u;
  for (int i = 0; i < 16; ++i) w[i] = SY_MUL(sigma, sy_gauss(T, sy_u64(key, base + (uint64_t)i)));
  return sy_nvfp4_block(w, gs, codes8);
}

#endif /* MSK_SYNTH_H */
