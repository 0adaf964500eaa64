/*
 * synth_dev.cu -- device fill kernels of the seeded input generator.
 *
 * Same recipe as synth_host.c, element for element: the kernels include
 * msk_synth.h, whose float steps map to __f*_rn intrinsics on the device, so
 * a tensor filled here equals the host fill bit for bit.  Used to put the
 * large workloads (tens of GB of weights and KV) on the GPU in seconds.
 */
#include <cuda_runtime.h>
#include <stdint.h>

#include "msk_synth.h"
#include "msk_source.h"

extern "C" {
const sy_gtab* sy_table(void);
void sy_nvfp4_shape(const sy_model* m, int role, int64_t* rows, int64_t* K);
void sy_nvfp4_params(const sy_model* m, int role, float* sigma, float* gs);
uint64_t sy_nvfp4_key(const sy_model* m, int role, int layer, int expert);
void sy_vec_params(const sy_model* m, int role, int layer, uint64_t* key, int64_t* n, int* gauss,
                   float* sigma);
uint64_t sy_hidden_key(const sy_model* m, int seq, int tok);
uint64_t sy_past_key(const sy_model* m, int kv, int layer, int seq, int head);
}

__device__ sy_gtab g_dev_tab;

static __global__ void k_fill_nvfp4(uint64_t key, uint32_t K, int64_t nblocks, float sigma, float gs,
                                    uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const uint32_t nkb = K / 16;
  for (int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; blk < nblocks;
       blk += (int64_t)gridDim.x * blockDim.x) {
    int64_t r = blk / nkb;
    uint32_t kb = (uint32_t)(blk - r * nkb);
    uint8_t c8[8];
    uint8_t sc = sy_nvfp4_gen_block(&g_dev_tab, key, (uint64_t)r, K, kb, sigma, gs, c8);
    uint2 w;
    w.x = (uint32_t)c8[0] | ((uint32_t)c8[1] << 8) | ((uint32_t)c8[2] << 16) | ((uint32_t)c8[3] << 24);
    w.y = (uint32_t)c8[4] | ((uint32_t)c8[5] << 8) | ((uint32_t)c8[6] << 16) | ((uint32_t)c8[7] << 24);
    *reinterpret_cast<uint2*>(codes + r * (K / 2) + (int64_t)kb * 8) = w;
    scales[blk] = sc;
  }
}

/* the same fill for n experts' tensors stacked [E][rows][K]: expert e's
 * blocks use keys[e] (one launch for a whole expert role) */
static __global__ void k_fill_nvfp4_experts(const uint64_t* __restrict__ keys, uint32_t K, int64_t blocks_per_expert,
                                            int64_t nblocks, float sigma, float gs, uint8_t* __restrict__ codes,
                                            uint8_t* __restrict__ scales) {
  const uint32_t nkb = K / 16;
  for (int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; blk < nblocks;
       blk += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e = blk / blocks_per_expert, in_e = blk - e * blocks_per_expert;
    const int64_t r = in_e / nkb;
    const uint32_t kb = (uint32_t)(in_e - r * nkb);
    uint8_t c8[8];
    uint8_t sc = sy_nvfp4_gen_block(&g_dev_tab, keys[e], (uint64_t)r, K, kb, sigma, gs, c8);
    uint2 w;
    w.x = (uint32_t)c8[0] | ((uint32_t)c8[1] << 8) | ((uint32_t)c8[2] << 16) | ((uint32_t)c8[3] << 24);
    w.y = (uint32_t)c8[4] | ((uint32_t)c8[5] << 8) | ((uint32_t)c8[6] << 16) | ((uint32_t)c8[7] << 24);
    *reinterpret_cast<uint2*>(codes + blk * 8) = w;
    scales[blk] = sc;
  }
}

static __global__ void k_fill_vec(uint64_t key, int64_t n, int gauss, float sigma, float* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    uint64_t h = sy_u64(key, (uint64_t)i);
    out[i] = gauss ? SY_MUL(sigma, sy_gauss(&g_dev_tab, h)) : sy_uniform(h, 0.8f, 0.4f);
  }
}

static __global__ void k_fill_hidden(const uint64_t* __restrict__ keys, int d, int64_t n,
                                     uint16_t* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    int64_t t = i / d;
    out[i] = sy_bf16(sy_gauss(&g_dev_tab, sy_u64(keys[t], (uint64_t)(i - t * d))));
  }
}

/* 16 consecutive codes of K and of V per thread; row p of the range goes to
 * byte offset p * row_stride */
static __global__ void k_fill_past(uint64_t kk, uint64_t kv, int64_t idx0, int64_t n16, int hd,
                                   int64_t row_stride, uint8_t* __restrict__ k, uint8_t* __restrict__ v) {
  for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < n16; c += (int64_t)gridDim.x * blockDim.x) {
    uint32_t a[4] = {0, 0, 0, 0}, b[4] = {0, 0, 0, 0};
    for (int i = 0; i < 16; ++i) {
      uint64_t idx = (uint64_t)(idx0 + c * 16 + i);
      a[i >> 2] |= (uint32_t)sy_e4m3(sy_gauss(&g_dev_tab, sy_u64(kk, idx))) << (8 * (i & 3));
      b[i >> 2] |= (uint32_t)sy_e4m3(sy_gauss(&g_dev_tab, sy_u64(kv, idx))) << (8 * (i & 3));
    }
    int64_t p = (c * 16) / hd, off = p * row_stride + (c * 16 - p * hd);
    *reinterpret_cast<uint4*>(k + off) = make_uint4(a[0], a[1], a[2], a[3]);
    *reinterpret_cast<uint4*>(v + off) = make_uint4(b[0], b[1], b[2], b[3]);
  }
}

static int grid_for(int64_t n) {
  int64_t g = (n + 255) / 256;
  if (g > 148 * 64) g = 148 * 64;
  return (int)(g < 1 ? 1 : g);
}

extern "C" {

/* Upload the quantile table to the current device. */
int sy_dev_init(void) {
  cudaError_t e = cudaMemcpyToSymbol(g_dev_tab, sy_table(), sizeof(sy_gtab));
  return e == cudaSuccess ? 0 : (int)e;
}

/* Whole NVFP4 tensor: codes[rows][K/2], scales[rows][K/16]; *gs_out gets the
 * global scale. */
int sy_dev_fill_nvfp4(const sy_model* m, int role, int layer, int expert, void* codes, void* scales,
                      float* gs_out, void* stream) {
  int64_t rows, K;
  float sigma, gs;
  sy_nvfp4_shape(m, role, &rows, &K);
  sy_nvfp4_params(m, role, &sigma, &gs);
  if (K % 16) return -1;
  if (((uintptr_t)codes & 7u) != 0) return -2;
  int64_t nb = rows * (K / 16);
  k_fill_nvfp4<<<grid_for(nb), 256, 0, (cudaStream_t)stream>>>(sy_nvfp4_key(m, role, layer, expert),
                                                                (uint32_t)K, nb, sigma, gs,
                                                                (uint8_t*)codes, (uint8_t*)scales);
  if (gs_out) *gs_out = gs;
  return (int)cudaGetLastError();
}

/* Every expert of one role: codes[E][rows][K/2], scales[E][rows][K/16] in
 * one launch.  keys_dev is caller-provided device scratch of n_experts
 * uint64. */
int sy_dev_fill_nvfp4_experts(const sy_model* m, int role, int layer, int n_experts, void* keys_dev, void* codes,
                              void* scales, float* gs_out, void* stream) {
  int64_t rows, K;
  float sigma, gs;
  sy_nvfp4_shape(m, role, &rows, &K);
  sy_nvfp4_params(m, role, &sigma, &gs);
  if (K % 16 || n_experts < 1) return -1;
  if (((uintptr_t)codes & 7u) != 0) return -2;
  uint64_t* hk = (uint64_t*)malloc(sizeof(uint64_t) * (size_t)n_experts);
  if (!hk) return -3;
  for (int e = 0; e < n_experts; ++e) hk[e] = sy_nvfp4_key(m, role, layer, e);
  cudaError_t err = cudaMemcpyAsync(keys_dev, hk, sizeof(uint64_t) * (size_t)n_experts, cudaMemcpyHostToDevice,
                                    (cudaStream_t)stream);
  if (err == cudaSuccess) err = cudaStreamSynchronize((cudaStream_t)stream);
  free(hk);
  if (err != cudaSuccess) return (int)err;
  const int64_t per = rows * (K / 16), nb = per * n_experts;
  k_fill_nvfp4_experts<<<grid_for(nb), 256, 0, (cudaStream_t)stream>>>((const uint64_t*)keys_dev, (uint32_t)K, per,
                                                                      nb, sigma, gs, (uint8_t*)codes,
                                                                      (uint8_t*)scales);
  if (gs_out) *gs_out = gs;
  return (int)cudaGetLastError();
}

int sy_dev_fill_vec(const sy_model* m, int role, int layer, void* out, void* stream) {
  uint64_t key;
  int64_t n;
  int gauss;
  float sigma;
  sy_vec_params(m, role, layer, &key, &n, &gauss, &sigma);
  k_fill_vec<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(key, n, gauss, sigma, (float*)out);
  return (int)cudaGetLastError();
}

/* hidden[n_seqs*tps][d] bf16; row (s, t) uses the key of (seq0 + s, t).
 * keys_dev is caller-provided device scratch of n_seqs*tps uint64. */
int sy_dev_fill_hidden(const sy_model* m, int seq0, int n_seqs, int tps, void* keys_dev, void* out,
                       void* stream) {
  int T = n_seqs * tps;
  uint64_t* hk = (uint64_t*)malloc(sizeof(uint64_t) * (size_t)T);
  if (!hk) return -1;
  for (int s = 0; s < n_seqs; ++s)
    for (int t = 0; t < tps; ++t) hk[s * tps + t] = sy_hidden_key(m, seq0 + s, t);
  cudaError_t e = cudaMemcpyAsync(keys_dev, hk, sizeof(uint64_t) * (size_t)T, cudaMemcpyHostToDevice,
                                  (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  free(hk);
  if (e != cudaSuccess) return (int)e;
  int64_t n = (int64_t)T * m->d_model;
  k_fill_hidden<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>((const uint64_t*)keys_dev, m->d_model, n,
                                                               (uint16_t*)out);
  return (int)cudaGetLastError();
}

/* Past K/V codes of (layer, seq, head) for positions [pos0, pos0+n): row p
 * (head_dim codes) at k + p*row_stride and v + p*row_stride (16-byte aligned
 * device memory; row_stride a multiple of 16, >= head_dim). */
int sy_dev_fill_past(const sy_model* m, int layer, int seq, int head, int64_t pos0, int64_t n, void* k,
                     void* v, int64_t row_stride, void* stream) {
  int64_t elems = n * m->head_dim;
  if (m->head_dim % 16 || row_stride % 16 || row_stride < m->head_dim || ((uintptr_t)k & 15u) ||
      ((uintptr_t)v & 15u))
    return -1;
  int64_t n16 = elems / 16;
  k_fill_past<<<grid_for(n16), 256, 0, (cudaStream_t)stream>>>(sy_past_key(m, 0, layer, seq, head),
                                                               sy_past_key(m, 1, layer, seq, head),
                                                               pos0 * m->head_dim, n16, m->head_dim,
                                                               row_stride, (uint8_t*)k, (uint8_t*)v);
  return (int)cudaGetLastError();
}

}  // extern "C"
