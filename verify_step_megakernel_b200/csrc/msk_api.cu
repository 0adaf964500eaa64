/*
 * msk_api.cu -- the C ABI declared in include/msk.h: argument checks,
 * scratch allocation, the KV cache object with its tensor map, and the
 * cooperative launch of the step kernel.
 */
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <new>

#include "msk_internal.h"

extern "C" size_t msk_kernel_smem_bytes();
extern "C" cudaError_t msk_kernel_setup(int hd, int* ctas_per_sm);
extern "C" size_t msk_kernel_xtile_gu_bytes(int E, int f, int d);
extern "C" size_t msk_kernel_xtile_dn_bytes(int E, int rows_per_expert, int K);
extern "C" size_t msk_kernel_xtile_dt_bytes(int E, int rows_per_expert, int K);
extern "C" cudaError_t msk_kernel_xtile(int kind, const uint8_t* c0, const uint8_t* c1, const uint8_t* s0, const uint8_t* s1,
                                        uint8_t* out, int E, int rows_per_expert, int K, cudaStream_t st);
extern "C" cudaError_t msk_kernel_kv_encode(const float* in, uint8_t* out, int64_t n, cudaStream_t stream);
extern "C" cudaError_t msk_kernel_launch(int hd, const MskParams* P_dev, const MskStep* st, const CUtensorMap* map,
                                         int ncta, cudaStream_t stream);

struct msk_handle {
  int device;
  int ncta;
  msk_config_t cfg;
  msk_layer_weights_t layers[MSK_MAX_LAYERS];
  MskParams host;   /* mirror of the device copy */
  MskParams* dev;   /* device copy */
  void* scratch;    /* one allocation for every scratch buffer */
  CUtensorMap* emaps; /* [L][MSK_NMAPS] weight tensor maps (device) */
  uint8_t* repack;    /* gate/up scale-factor atoms of every layer (block-scaled expert path), or null */
  size_t repack_bytes;
  size_t scratch_bytes;
  uint32_t* words;  /* ctrl + status */
  msk_debug_t dbg;
  int have_last;
};

struct msk_kv {
  msk_handle_t* h;
  int n_seqs;
  int64_t cap;
  int64_t half_rows;
  uint8_t* base;
  CUtensorMap map;
};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

/* floats per token of the projections' split-K partials: K slices of 512
 * (one slice for K <= 512) times the output rows, QKV or W_o */
static size_t proj_floats(const MskParams& P) {
  const size_t sq = P.d <= 512 ? 1 : P.d / 512, so = P.qd <= 512 ? 1 : P.qd / 512;
  const size_t a = sq * (size_t)(P.qd + 2 * P.kvd), b = so * (size_t)P.d;
  return a > b ? a : b;
}

static msk_status_t check_nv(const msk_nvfp4_t& w) {
  if (!w.codes || !w.scales || !aligned16(w.codes) || !aligned16(w.scales)) return MSK_ERR_INVALID_ARG;
  if (!(w.global_scale > 0.0f) || !isfinite(w.global_scale)) return MSK_ERR_INVALID_ARG;
  return MSK_OK;
}

static msk_status_t check_config(const msk_config_t* c) {
  if (c->n_layers < 1 || c->n_layers > MSK_MAX_LAYERS) return MSK_ERR_INVALID_ARG;
  if (c->head_dim != 64 && c->head_dim != 128) return MSK_ERR_UNSUPPORTED;
  if (c->n_kv_heads < 1 || c->n_q_heads < 1 || c->n_q_heads % c->n_kv_heads) return MSK_ERR_INVALID_ARG;
  const int qd = c->n_q_heads * c->head_dim;
  /* the projections' K dimensions (d_model, qd) split into slices of 512
   * (or one slice of 256 or 512) read as 2-D tensor boxes */
  if (c->d_model < 256 || c->d_model % 256 || c->d_model > 4096) return MSK_ERR_UNSUPPORTED;
  if (qd < 256 || qd % 256 || qd > 4096 || (qd > 512 && qd % 512)) return MSK_ERR_UNSUPPORTED;
  if (c->expert_dim < 128 || c->expert_dim % 128 || c->expert_dim > 4096) return MSK_ERR_UNSUPPORTED;
  /* expert tiles stream K in chunks of 512: longer rows must split evenly */
  if ((c->d_model > 512 && c->d_model % 512) || (c->expert_dim > 512 && c->expert_dim % 512))
    return MSK_ERR_UNSUPPORTED;
  if (c->n_experts < 32 || c->n_experts % 32 || c->n_experts > 256) return MSK_ERR_UNSUPPORTED;
  if (c->top_k < 1 || c->top_k > 8 || c->top_k > c->n_experts) return MSK_ERR_INVALID_ARG;
  if (c->window < 1) return MSK_ERR_INVALID_ARG;
  if (!(c->rms_eps >= 0.0f)) return MSK_ERR_INVALID_ARG;
  if (c->max_seqs < 1 || c->max_tokens_per_seq < 1) return MSK_ERR_INVALID_ARG;
  if (c->max_seqs * c->max_tokens_per_seq > MSK_MAX_TOKENS) return MSK_ERR_UNSUPPORTED;
  if (c->max_tokens_per_seq * (c->n_q_heads / c->n_kv_heads) > 64) return MSK_ERR_UNSUPPORTED;
  if (c->max_seqs * c->n_kv_heads > MSK_MAX_PAIRS) return MSK_ERR_UNSUPPORTED;
  if (c->wait_timeout_us < 0 || c->expert_mma_min_tokens < 0) return MSK_ERR_INVALID_ARG;
  return MSK_OK;
}

/* ---- working memory compiled into the library (msk_step_static) -------------------------
 * msk_step_static runs the same step kernel as msk_step, but its per-step
 * working buffers and its copy of the parameter block live in this fixed
 * array instead of the handle's allocation.  The array is zero when the
 * module loads; only the control words (barrier counter, abort word) must be
 * zero when a step starts, and the parameter kernel below clears them before
 * every step.  Every call on a device uses the same bytes, so two such steps
 * in flight at once on one device (two streams, two handles, two threads)
 * overwrite each other's buffers. */
static __device__ __align__(256) uint8_t g_static_scratch[MSK_STATIC_SCRATCH_BYTES];

#define MSK_STATIC_MAX_DEVICES 64
/* the array's device address per device, found on the first call that
 * succeeds in looking it up (a failed lookup leaves the slot empty, so a
 * later call tries again) */
static std::mutex g_static_mu;
static uint8_t* g_static_ptr[MSK_STATIC_MAX_DEVICES];

/* where the step's buffers sit inside g_static_scratch */
struct StaticLayout {
  size_t params, h, x, qkv, qs, part, o, x2f, x2h, xq, logits, u, ut, y, ctrl, total;
};

static StaticLayout static_layout(const msk_handle_t* h) {
  const MskParams& P = h->host;
  const msk_config_t& c = h->cfg;
  const size_t T = (size_t)P.max_T, d = P.d, qd = P.qd;
  const size_t slots = (size_t)h->ncta + (size_t)c.max_seqs * P.hkv;
  StaticLayout L;
  size_t at = 0;
  auto take = [&at](size_t bytes) { const size_t o = at; at += (bytes + 255) & ~(size_t)255; return o; };
  L.params = take(sizeof(MskParams));
  L.h = take(T * d * 4);
  L.x = take(T * d * 2);
  L.qkv = take(T * proj_floats(P) * 4);
  L.qs = take(T * qd * 2);
  L.part = take(slots * (size_t)P.part_stride * 4);
  L.o = take(T * qd * 2);
  L.x2f = take(T * d * 4);
  L.x2h = take(T * d * 2);
  L.xq = take(T * MSK_XQ_BYTES(d));
  L.logits = take(T * P.E * 4);
  L.u = take(T * P.k * P.f * 2);
  L.ut = take(T * P.k * MSK_XQ_BYTES(P.f));
  L.y = take(T * P.k * d * 4);
  L.ctrl = take(CTRL_WORDS * 4);
  L.total = at;
  return L;
}

struct StaticPtrs {
  float* h;
  uint16_t* x;
  float* qkv;
  uint16_t* qs;
  float* part;
  uint16_t* o;
  float* x2f;
  uint16_t* x2h;
  uint8_t* xq;
  float* logits;
  uint16_t* u;
  uint8_t* ut;
  float* y;
  uint32_t* ctrl;
};

/* copy the handle's parameter block into the array, point its working
 * buffers at the array and zero the control words (one CTA) */
__global__ void msk_static_params(const MskParams* src, MskParams* dst, StaticPtrs p) {
  const unsigned long long* s = (const unsigned long long*)src;
  unsigned long long* t = (unsigned long long*)dst;
  for (size_t i = threadIdx.x; i < sizeof(MskParams) / 8; i += blockDim.x) t[i] = s[i];
  for (int i = threadIdx.x; i < CTRL_WORDS; i += blockDim.x) p.ctrl[i] = 0u;
  __syncthreads();
  if (threadIdx.x == 0) {
    dst->h = p.h;
    dst->x = p.x;
    dst->qkv = p.qkv;
    dst->qs = p.qs;
    dst->part = p.part;
    dst->o = p.o;
    dst->x2f = p.x2f;
    dst->x2h = p.x2h;
    dst->xq = p.xq;
    dst->logits = p.logits;
    dst->u = p.u;
    dst->ut = p.ut;
    dst->y = p.y;
    dst->ctrl = p.ctrl;
  }
}

extern "C" {

const char* msk_status_string(msk_status_t s) {
  switch (s) {
    case MSK_OK: return "ok";
    case MSK_ERR_INVALID_ARG: return "invalid argument";
    case MSK_ERR_UNSUPPORTED: return "unsupported device or shape";
    case MSK_ERR_OOM: return "out of device memory";
    case MSK_ERR_CUDA: return "CUDA error";
    case MSK_ERR_BOUND: return "softmax bound 2M >= 80";
    case MSK_ERR_KV_RANGE: return "positions outside the KV cache or not contiguous";
    case MSK_ERR_TIMEOUT: return "device wait timed out";
    case MSK_ERR_DEVICE: return "device-side check failed";
  }
  return "unknown status";
}

msk_status_t msk_create(const msk_config_t* config, const msk_layer_weights_t* layers, int device,
                        msk_handle_t** out) {
  if (!config || !layers || !out) return MSK_ERR_INVALID_ARG;
  *out = nullptr;
  msk_status_t st = check_config(config);
  if (st) return st;
  for (int l = 0; l < config->n_layers; ++l) {
    const msk_layer_weights_t& w = layers[l];
    if (!w.attn_norm_g || !w.q_norm_g || !w.k_norm_g || !w.moe_norm_g || !w.router) return MSK_ERR_INVALID_ARG;
    if (!aligned16(w.attn_norm_g) || !aligned16(w.moe_norm_g) || !aligned16(w.router) || !aligned16(w.q_norm_g) ||
        !aligned16(w.k_norm_g))
      return MSK_ERR_INVALID_ARG;
    const msk_nvfp4_t* nvs[7] = {&w.wq, &w.wk, &w.wv, &w.wo, &w.w_gate, &w.w_up, &w.w_down};
    for (auto* nv : nvs)
      if ((st = check_nv(*nv))) return st;
  }
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) return MSK_ERR_UNSUPPORTED;
  int prev = 0;
  cudaGetDevice(&prev);
  if (cudaSetDevice(device) != cudaSuccess) return MSK_ERR_CUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) { cudaSetDevice(prev); return MSK_ERR_CUDA; }
  if (prop.major != 10 || !prop.cooperativeLaunch) { cudaSetDevice(prev); return MSK_ERR_UNSUPPORTED; }
  int per_sm = 0;
  if (msk_kernel_setup(config->head_dim, &per_sm) != cudaSuccess || per_sm < 1) { cudaSetDevice(prev); return MSK_ERR_UNSUPPORTED; }

  msk_handle_t* h = new (std::nothrow) msk_handle_t();
  if (!h) { cudaSetDevice(prev); return MSK_ERR_OOM; }
  h->device = device;
  h->ncta = prop.multiProcessorCount; /* one persistent CTA per SM */
  h->cfg = *config;
  memcpy(h->layers, layers, sizeof(msk_layer_weights_t) * config->n_layers);

  MskParams& P = h->host;
  memset(&P, 0, sizeof P);
  const msk_config_t& c = *config;
  P.L = c.n_layers; P.d = c.d_model; P.hq = c.n_q_heads; P.hkv = c.n_kv_heads; P.hd = c.head_dim;
  P.E = c.n_experts; P.k = c.top_k; P.f = c.expert_dim; P.W = c.window; P.G = c.n_q_heads / c.n_kv_heads;
  P.qd = P.hq * P.hd; P.kvd = P.hkv * P.hd;
  P.ncta = h->ncta;
  P.max_T = c.max_seqs * c.max_tokens_per_seq;
  P.eps = c.rms_eps;
  P.scale_log2 = (float)(1.4426950408889634 / sqrt((double)P.hd));
  P.timeout_ns = (int64_t)(c.wait_timeout_us ? c.wait_timeout_us : 2000000) * 1000;
  P.flags = c.flags;
  /* tau: 0 = the default, above the unit size = never, MSK_F_TC_EXPERTS = every unit */
  P.tau = (c.flags & MSK_F_TC_EXPERTS) ? 1 : (c.expert_mma_min_tokens > 0 ? c.expert_mma_min_tokens : MSK_TAU_DEFAULT);
  if (P.tau > MSK_UNIT_TOK) P.tau = MSK_TAU_NEVER;

  /* the fixed softmax shift of each layer, from its QK-norm gains */
  float* gq = (float*)malloc(sizeof(float) * P.hd);
  float* gk = (float*)malloc(sizeof(float) * P.hd);
  st = MSK_OK;
  for (int l = 0; l < P.L && st == MSK_OK; ++l) {
    if (cudaMemcpy(gq, layers[l].q_norm_g, sizeof(float) * P.hd, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(gk, layers[l].k_norm_g, sizeof(float) * P.hd, cudaMemcpyDeviceToHost) != cudaSuccess) {
      st = MSK_ERR_CUDA;
      break;
    }
    double mq = 0, mk = 0;
    for (int i = 0; i < P.hd; ++i) { mq = fmax(mq, fabs(gq[i])); mk = fmax(mk, fabs(gk[i])); }
    const double M = sqrt((double)P.hd) * mq * mk;
    if (!(2.0 * M < 80.0)) st = MSK_ERR_BOUND;
    MskLayer& Ly = P.layers[l];
    const msk_layer_weights_t& w = layers[l];
    Ly.g_attn = w.attn_norm_g; Ly.g_q = w.q_norm_g; Ly.g_k = w.k_norm_g; Ly.g_moe = w.moe_norm_g; Ly.router = w.router;
    auto nv = [](const msk_nvfp4_t& x) { MskNv r; r.codes = x.codes; r.scales = x.scales; r.gs = x.global_scale; r.pad = 0; return r; };
    Ly.wq = nv(w.wq); Ly.wk = nv(w.wk); Ly.wv = nv(w.wv); Ly.wo = nv(w.wo);
    Ly.wg = nv(w.w_gate); Ly.wu = nv(w.w_up); Ly.wd = nv(w.w_down);
    Ly.bound_log2 = (float)(M * 1.4426950408889634);
    Ly.sliding = c.layer_is_sliding[l] ? 1 : 0;
  }
  free(gq);
  free(gk);
  if (st) { delete h; cudaSetDevice(prev); return st; }

  /* scratch */
  const size_t T = (size_t)P.max_T, d = P.d, qd = P.qd;
  const size_t R_max = (size_t)c.max_tokens_per_seq * P.G;
  P.part_stride = (int32_t)(R_max * (P.hd + 4));
  const size_t slots = (size_t)h->ncta + (size_t)c.max_seqs * P.hkv;
  size_t sizes[] = {
      T * d * 4,                 /* h */
      T * d * 2,                 /* x */
      T * proj_floats(P) * 4,    /* split-K partials of the projections */
      T * qd * 2,                /* qs */
      slots * P.part_stride * 4, /* part */
      T * qd * 2,                /* o */
      T * d * 4,                 /* x2f */
      T * d * 2,                 /* x2h */
      T * MSK_XQ_BYTES(d),       /* xq */
      T * P.E * 4,               /* logits */
      T * P.k * P.f * 2,         /* u */
      T * P.k * MSK_XQ_BYTES(P.f), /* ut */
      T * P.k * d * 4,           /* y */
      (CTRL_WORDS + ST_WORDS) * 4,
      (size_t)P.L * 4,           /* n_distinct */
      (2 + MSK_MAX_TOKENS) * 4,  /* last_shape */
  };
  const int nbuf = sizeof(sizes) / sizeof(sizes[0]);
  size_t off[20], total = 0;
  for (int i = 0; i < nbuf; ++i) { off[i] = total; total += (sizes[i] + 255) & ~(size_t)255; }
  if (cudaMalloc(&h->scratch, total) != cudaSuccess) { delete h; cudaSetDevice(prev); return MSK_ERR_OOM; }
  cudaMemset(h->scratch, 0, total);
  h->scratch_bytes = total;
  uint8_t* b = (uint8_t*)h->scratch;
  P.h = (float*)(b + off[0]);
  P.x = (uint16_t*)(b + off[1]);
  P.qkv = (float*)(b + off[2]);
  P.qs = (uint16_t*)(b + off[3]);
  P.part = (float*)(b + off[4]);
  P.o = (uint16_t*)(b + off[5]);
  P.x2f = (float*)(b + off[6]);
  P.x2h = (uint16_t*)(b + off[7]);
  P.xq = b + off[8];
  P.logits = (float*)(b + off[9]);
  P.u = (uint16_t*)(b + off[10]);
  P.ut = b + off[11];
  P.y = (float*)(b + off[12]);
  P.ctrl = (uint32_t*)(b + off[13]);
  P.status = P.ctrl + CTRL_WORDS;
  P.n_distinct = (int32_t*)(b + off[14]);
  P.last_shape = (int32_t*)(b + off[15]);
  h->words = P.ctrl;
  /* tensor maps of the expert tensors, for the K-chunked expert tiles */
  {
    EncodeTiledFn enc = encode_fn();
    CUtensorMap* hm = (CUtensorMap*)calloc((size_t)P.L * MSK_NMAPS, sizeof(CUtensorMap));
    bool ok = enc != nullptr && hm != nullptr && cudaMalloc(&h->emaps, sizeof(CUtensorMap) * MSK_NMAPS * P.L) == cudaSuccess;
    for (int l = 0; l < P.L && ok; ++l) {
      const msk_layer_weights_t& w = layers[l];
      const msk_nvfp4_t* mats[3] = {&w.w_gate, &w.w_up, &w.w_down};
      for (int m = 0; m < 3 && ok; ++m) {
        const int64_t K = m < 2 ? P.d : P.f, rows = (int64_t)P.E * (m < 2 ? P.f : P.d);
        /* K chunks: 256 for gate/up on the tensor cores, else 512 (or all of K) */
        const int KC = K <= 512 ? (int)K : 512; /* the CUDA-core path's chunks */
        /* K not a multiple of 256 (128, 384): whole rows go as bulk copies
         * and the maps stay zero */
        if (K % 256) continue;
        for (int part = 0; part < 2 && ok; ++part) {
          /* codes as 16-bit pairs [rows][K/4], a 128-row box 32 bytes wider
           * than the K chunk; scales [rows][K/16], a 128-row box of the chunk */
          const bool codes = part == 0;
          cuuint64_t dims[2] = {(cuuint64_t)(codes ? K / 4 : K / 16), (cuuint64_t)rows};
          cuuint64_t strides[1] = {(cuuint64_t)(codes ? K / 2 : K / 16)};
          cuuint32_t box[2] = {(cuuint32_t)(codes ? KC / 4 + 16 : KC / 16), 128};
          cuuint32_t estr[2] = {1, 1};
          void* base = (void*)(codes ? mats[m]->codes : mats[m]->scales);
          ok = enc(&hm[l * MSK_NMAPS + m * 2 + part], codes ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                   base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
        }
      }
      /* the dense projections: 16-row boxes of a K slice (512, or all of
       * K <= 512), codes 32 bytes wider than the slice as for the experts */
      const msk_nvfp4_t* dm[4] = {&w.wq, &w.wk, &w.wv, &w.wo};
      for (int m = 0; m < 4 && ok; ++m) {
        const int64_t K = m < 3 ? P.d : P.qd, rows = m == 0 ? P.qd : (m < 3 ? P.kvd : P.d);
        const int KS = K <= 512 ? (int)K : 512;
        for (int part = 0; part < 2 && ok; ++part) {
          const bool codes = part == 0;
          cuuint64_t dims[2] = {(cuuint64_t)(codes ? K / 4 : K / 16), (cuuint64_t)rows};
          cuuint64_t strides[1] = {(cuuint64_t)(codes ? K / 2 : K / 16)};
          cuuint32_t box[2] = {(cuuint32_t)(codes ? KS / 4 + 16 : KS / 16), 16};
          cuuint32_t estr[2] = {1, 1};
          void* base = (void*)(codes ? dm[m]->codes : dm[m]->scales);
          ok = enc(&hm[l * MSK_NMAPS + MSK_MAP_DENSE + m * 2 + part],
                   codes ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
        }
      }
      /* gate and up codes for the block-scaled tensor cores: 128 rows x 128
       * bytes (256 codes) per box, 128-byte swizzle */
      for (int m = 0; m < 2 && ok; ++m) {
        const int64_t K = P.d, rows = (int64_t)P.E * P.f;
        cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
        cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
        cuuint32_t box[2] = {128, 128};
        cuuint32_t estr[2] = {1, 1};
        ok = enc(&hm[l * MSK_NMAPS + MSK_MAP_GUSW + m], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, (void*)mats[m]->codes, dims,
                 strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
      }
      P.layers[l].emap = h->emaps + l * MSK_NMAPS;
    }
    if (ok) ok = cudaMemcpy(h->emaps, hm, sizeof(CUtensorMap) * MSK_NMAPS * P.L, cudaMemcpyHostToDevice) == cudaSuccess;
    free(hm);
    if (!ok) {
      if (h->emaps) cudaFree(h->emaps);
      cudaFree(h->scratch);
      delete h;
      cudaSetDevice(prev);
      return MSK_ERR_CUDA;
    }
  }
  /* the expert weights as slot images, one contiguous bulk copy per K
   * chunk (library-owned copies; the borrowed weights are not touched):
   * gate/up for the block-scaled path when some unit can take it, down for
   * that path too when f is 512 or 1024, and down for the CUDA-core path
   * when some unit takes it and its K is a multiple of 256.  (With at most
   * two 512-wide chunks per down item, an issuing warp reuses a chunk's
   * scale-factor columns four fills later, after the slot chain has seen
   * that chunk's products complete; longer items would reuse them within
   * one item, ordered only by the tensor pipe's issue order.) */
  {
    const bool gu = P.tau <= MSK_UNIT_TOK, dt = gu && (P.f == 512 || P.f == 1024);
    const bool dn = (P.f % 256) == 0 && (!dt || P.tau > 1); /* tau 1: every unit (>= 1 token) is block-scaled */
    const size_t gub = gu ? msk_kernel_xtile_gu_bytes(P.E, P.f, P.d) : 0;
    const size_t dtb = dt ? msk_kernel_xtile_dt_bytes(P.E, P.d, P.f) : 0;
    const size_t dnb = dn ? msk_kernel_xtile_dn_bytes(P.E, P.d, P.f) : 0;
    h->repack_bytes = (gub + dtb + dnb) * P.L;
    bool ok = h->repack_bytes == 0 || cudaMalloc(&h->repack, h->repack_bytes) == cudaSuccess;
    for (int l = 0; l < P.L && ok && h->repack_bytes; ++l) {
      uint8_t* g = h->repack + (gub + dtb + dnb) * l;
      const msk_layer_weights_t& w = layers[l];
      if (gu)
        ok = msk_kernel_xtile(0, w.w_gate.codes, w.w_up.codes, w.w_gate.scales, w.w_up.scales, g, P.E, P.f, P.d, 0) ==
             cudaSuccess;
      if (ok && dt)
        ok = msk_kernel_xtile(2, w.w_down.codes, nullptr, w.w_down.scales, nullptr, g + gub, P.E, P.d, P.f, 0) ==
             cudaSuccess;
      if (ok && dn)
        ok = msk_kernel_xtile(1, w.w_down.codes, nullptr, w.w_down.scales, nullptr, g + gub + dtb, P.E, P.d, P.f, 0) ==
             cudaSuccess;
      P.layers[l].xtgu = gu ? g : nullptr;
      P.layers[l].xtdt = dt ? g + gub : nullptr;
      P.layers[l].xtdn = dn ? g + gub + dtb : nullptr;
    }
    if (ok) ok = cudaDeviceSynchronize() == cudaSuccess;
    if (!ok) {
      if (h->repack) cudaFree(h->repack);
      cudaFree(h->emaps);
      cudaFree(h->scratch);
      delete h;
      cudaSetDevice(prev);
      return MSK_ERR_OOM;
    }
  }
  if (cudaMalloc(&h->dev, sizeof(MskParams)) != cudaSuccess) {
    if (h->repack) cudaFree(h->repack);
    cudaFree(h->emaps);
    cudaFree(h->scratch);
    delete h;
    cudaSetDevice(prev);
    return MSK_ERR_OOM;
  }
  if (cudaMemcpy(h->dev, &P, sizeof(MskParams), cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess) {
    cudaFree(h->dev);
    if (h->repack) cudaFree(h->repack);
    cudaFree(h->emaps);
    cudaFree(h->scratch);
    delete h;
    cudaSetDevice(prev);
    return MSK_ERR_CUDA;
  }
  cudaSetDevice(prev);
  *out = h;
  return MSK_OK;
}

void msk_destroy(msk_handle_t* h) {
  if (!h) return;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(h->device);
  cudaDeviceSynchronize();
  cudaFree(h->dev);
  cudaFree(h->scratch);
  cudaFree(h->emaps);
  if (h->repack) cudaFree(h->repack);
  cudaSetDevice(prev);
  delete h;
}

msk_status_t msk_kv_create(msk_handle_t* h, int n_seqs, int64_t capacity, msk_kv_t** out) {
  if (!h || !out || n_seqs < 1 || capacity < 1) return MSK_ERR_INVALID_ARG;
  *out = nullptr;
  if (n_seqs > h->cfg.max_seqs) return MSK_ERR_INVALID_ARG;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return MSK_ERR_CUDA;
  const MskParams& P = h->host;
  const int64_t cap = (capacity + 15) / 16 * 16;
  const int64_t half_rows = (int64_t)P.L * n_seqs * P.hkv * cap;
  if (2 * half_rows >= ((int64_t)1 << 31)) return MSK_ERR_UNSUPPORTED; /* tensor-copy coordinates are int32 */
  const size_t bytes = (size_t)(2 * half_rows) * P.hd;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(h->device);
  msk_kv_t* kv = new (std::nothrow) msk_kv_t();
  if (!kv) { cudaSetDevice(prev); return MSK_ERR_OOM; }
  kv->h = h;
  kv->n_seqs = n_seqs;
  kv->cap = cap;
  kv->half_rows = half_rows;
  if (cudaMalloc(&kv->base, bytes) != cudaSuccess) { delete kv; cudaSetDevice(prev); return MSK_ERR_OOM; }
  /* zero: unwritten positions must decode to finite values (masked keys
   * still pass through the tensor-core tile as 0 * v) */
  if (cudaMemset(kv->base, 0, bytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
    cudaFree(kv->base);
    delete kv;
    cudaSetDevice(prev);
    return MSK_ERR_CUDA;
  }
  /* head dim 64: one box per attention stage, C positions of one (layer,
   * sequence, kv head) row range with K and V together (the third
   * dimension steps from the K half of the cache to the V half), 32 KB.
   * Head dim 128: one box is K or V of 128 positions (16 KB); the two go to
   * separate rings. */
  const int C = P.hd == 128 ? 128 : 256;
  const cuuint32_t rank = P.hd == 128 ? 2 : 3;
  cuuint64_t dims[3] = {(cuuint64_t)P.hd, (cuuint64_t)half_rows, 2};
  cuuint64_t strides[2] = {(cuuint64_t)P.hd, (cuuint64_t)half_rows * (cuuint64_t)P.hd};
  cuuint32_t box[3] = {(cuuint32_t)P.hd, (cuuint32_t)C, 2};
  cuuint32_t estr[3] = {1, 1, 1};
  if (rank == 2) dims[1] = (cuuint64_t)(2 * half_rows);
  CUresult r = enc(&kv->map, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, kv->base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE,
                   P.hd == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  cudaSetDevice(prev);
  if (r != CUDA_SUCCESS) {
    cudaFree(kv->base);
    delete kv;
    return MSK_ERR_CUDA;
  }
  *out = kv;
  return MSK_OK;
}

void msk_kv_destroy(msk_kv_t* kv) {
  if (!kv) return;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(kv->h->device);
  cudaDeviceSynchronize();
  cudaFree(kv->base);
  cudaSetDevice(prev);
  delete kv;
}

static int64_t kv_row(const msk_kv_t* kv, int layer, int seq, int head, int64_t pos) {
  const MskParams& P = kv->h->host;
  return (((int64_t)layer * kv->n_seqs + seq) * P.hkv + head) * kv->cap + pos;
}

msk_status_t msk_kv_append(msk_handle_t* h, msk_kv_t* kv, int layer, int seq, int64_t pos0, int64_t n,
                           const uint8_t* k_fp8, const uint8_t* v_fp8, void* stream) {
  if (!h || !kv || kv->h != h || !k_fp8 || !v_fp8) return MSK_ERR_INVALID_ARG;
  const MskParams& P = h->host;
  if (layer < 0 || layer >= P.L || seq < 0 || seq >= kv->n_seqs || pos0 < 0 || n < 0) return MSK_ERR_INVALID_ARG;
  if (pos0 + n > kv->cap) return MSK_ERR_KV_RANGE;
  if (n == 0) return MSK_OK;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(h->device);
  cudaError_t e = cudaSuccess;
  for (int hh = 0; hh < P.hkv && e == cudaSuccess; ++hh) {
    for (int kvsel = 0; kvsel < 2 && e == cudaSuccess; ++kvsel) {
      uint8_t* dst = kv->base + (kv_row(kv, layer, seq, hh, pos0) + (kvsel ? kv->half_rows : 0)) * P.hd;
      const uint8_t* src = (kvsel ? v_fp8 : k_fp8) + (size_t)hh * P.hd;
      e = cudaMemcpy2DAsync(dst, P.hd, src, (size_t)P.hkv * P.hd, P.hd, (size_t)n, cudaMemcpyDefault,
                            (cudaStream_t)stream);
    }
  }
  cudaSetDevice(prev);
  return e == cudaSuccess ? MSK_OK : MSK_ERR_CUDA;
}

msk_status_t msk_kv_encode(const float* in, uint8_t* out, int64_t n, void* stream) {
  if (n < 0 || (n > 0 && (!in || !out || !aligned16(in) || !aligned16(out)))) return MSK_ERR_INVALID_ARG;
  if (n == 0) return MSK_OK;
  return msk_kernel_kv_encode(in, out, n, (cudaStream_t)stream) == cudaSuccess ? MSK_OK : MSK_ERR_CUDA;
}

msk_status_t msk_kv_read(msk_handle_t* h, msk_kv_t* kv, int layer, int seq, int64_t pos0, int64_t n, uint8_t* k_out,
                         uint8_t* v_out) {
  if (!h || !kv || kv->h != h || !k_out || !v_out) return MSK_ERR_INVALID_ARG;
  const MskParams& P = h->host;
  if (layer < 0 || layer >= P.L || seq < 0 || seq >= kv->n_seqs || pos0 < 0 || n < 0) return MSK_ERR_INVALID_ARG;
  if (pos0 + n > kv->cap) return MSK_ERR_KV_RANGE;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(h->device);
  cudaError_t e = cudaDeviceSynchronize();
  for (int hh = 0; hh < P.hkv && e == cudaSuccess; ++hh) {
    for (int kvsel = 0; kvsel < 2 && e == cudaSuccess; ++kvsel) {
      const uint8_t* src = kv->base + (kv_row(kv, layer, seq, hh, pos0) + (kvsel ? kv->half_rows : 0)) * P.hd;
      uint8_t* dst = (kvsel ? v_out : k_out) + (size_t)hh * P.hd;
      e = cudaMemcpy2D(dst, (size_t)P.hkv * P.hd, src, P.hd, P.hd, (size_t)n, cudaMemcpyDefault);
    }
  }
  cudaSetDevice(prev);
  return e == cudaSuccess ? MSK_OK : MSK_ERR_CUDA;
}

msk_status_t msk_step(msk_handle_t* h, const uint16_t* hidden_in, const int32_t* positions, int n_seqs,
                      int tokens_per_seq, msk_kv_t* kv, uint16_t* hidden_out, void* stream) {
  if (!h || !hidden_in || !positions || !kv || !hidden_out || kv->h != h) return MSK_ERR_INVALID_ARG;
  if (n_seqs < 1 || tokens_per_seq < 1 || n_seqs > h->cfg.max_seqs || tokens_per_seq > h->cfg.max_tokens_per_seq ||
      n_seqs > kv->n_seqs)
    return MSK_ERR_INVALID_ARG;
  if (!aligned16(hidden_in) || !aligned16(hidden_out) || ((uintptr_t)positions & 3u)) return MSK_ERR_INVALID_ARG;
  const MskParams& P = h->host;
  MskStep st;
  st.hidden_in = hidden_in;
  st.positions = positions;
  st.hidden_out = hidden_out;
  st.kv_base = kv->base;
  st.kv_cap = kv->cap;
  st.kv_half_rows = kv->half_rows;
  st.kv_seqs = kv->n_seqs;
  st.S = n_seqs;
  st.Tq = tokens_per_seq;
  st.T = n_seqs * tokens_per_seq;
  int prev = 0;
  cudaGetDevice(&prev);
  if (prev != h->device) cudaSetDevice(h->device);
  cudaError_t e = cudaMemsetAsync(P.ctrl, 0, CTRL_WORDS * 4, (cudaStream_t)stream);
  if (e == cudaSuccess) e = msk_kernel_launch(P.hd, h->dev, &st, &kv->map, h->ncta, (cudaStream_t)stream);
  if (prev != h->device) cudaSetDevice(prev);
  h->have_last = 1;
  return e == cudaSuccess ? MSK_OK : MSK_ERR_CUDA;
}

msk_status_t msk_step_status_at(msk_handle_t* h, int32_t* layer, int32_t* phase, int32_t* cta) {
  if (layer) *layer = -1;
  if (phase) *phase = -1;
  if (cta) *cta = -1;
  if (!h) return MSK_ERR_INVALID_ARG;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(h->device);
  uint32_t w[ST_WORDS];
  cudaError_t e = cudaMemcpy(w, h->host.status, sizeof w, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(h->host.status, 0, sizeof w);
  cudaSetDevice(prev);
  if (e != cudaSuccess) return MSK_ERR_CUDA;
  /* the site word is (layer << 16) | (phase << 8) | cta, plus one in the top
   * bit when set (a site-less error leaves it zero) */
  if (w[ST_CODE] != 0 && (w[ST_WHERE] & 0x80000000u)) {
    if (layer) *layer = (int32_t)((w[ST_WHERE] >> 16) & 0x7FFF);
    if (phase) *phase = (int32_t)((w[ST_WHERE] >> 8) & 0xFF);
    if (cta) *cta = (int32_t)(w[ST_WHERE] & 0xFF);
  }
  return (msk_status_t)w[ST_CODE];
}

msk_status_t msk_step_status(msk_handle_t* h) { return msk_step_status_at(h, nullptr, nullptr, nullptr); }

msk_status_t msk_set_debug(msk_handle_t* h, const msk_debug_t* dbg) {
  if (!h) return MSK_ERR_INVALID_ARG;
  MskParams& P = h->host;
  msk_debug_t z;
  memset(&z, 0, sizeof z);
  const msk_debug_t& d = dbg ? *dbg : z;
  P.dbg_ids = d.route_ids;
  P.dbg_w = d.route_w;
  P.dbg_logits = d.logits;
  P.dbg_attn = d.attn_out;
  P.dbg_trace = d.trace;
  P.dbg_kpre = d.k_pre;
  P.dbg_vpre = d.v_pre;
  P.dbg_hold = d.hold_barrier > 0 ? d.hold_barrier : 0;
  h->dbg = d;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(h->device);
  cudaError_t e = cudaMemcpy(h->dev, &P, sizeof(MskParams), cudaMemcpyHostToDevice);
  cudaSetDevice(prev);
  return e == cudaSuccess ? MSK_OK : MSK_ERR_CUDA;
}

msk_status_t msk_query(msk_handle_t* h, msk_stats_t* out) {
  if (!h || !out) return MSK_ERR_INVALID_ARG;
  memset(out, 0, sizeof *out);
  const MskParams& P = h->host;
  out->n_layers = P.L;
  out->scratch_bytes = (int64_t)h->scratch_bytes;
  out->repacked_bytes = (int64_t)h->repack_bytes;
  if (!h->have_last) return MSK_OK;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(h->device);
  cudaError_t e = cudaDeviceSynchronize();
  int32_t shape[2 + MSK_MAX_TOKENS];
  if (e == cudaSuccess) e = cudaMemcpy(out->n_distinct, P.n_distinct, sizeof(int32_t) * P.L, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(shape, P.last_shape, sizeof shape, cudaMemcpyDeviceToHost);
  cudaSetDevice(prev);
  if (e != cudaSuccess) return MSK_ERR_CUDA;
  /* bytes the step must move at least once: each weight it uses, each KV
   * position it attends (the union over a sequence's rows) and writes, and
   * the hidden states in and out */
  const int64_t d = P.d, qd = P.qd, kvd = P.kvd, f = P.f;
  auto nvb = [](int64_t n) { return n / 2 + n / 16; }; /* NVFP4 bytes of n values */
  int64_t wbytes = 0, kvbytes = 0;
  const int S = shape[0], Tq = shape[1], T = S * Tq;
  for (int l = 0; l < P.L; ++l) {
    wbytes += nvb(qd * d) + 2 * nvb(kvd * d) + nvb(d * qd) + (int64_t)P.E * d * 4;
    wbytes += (int64_t)out->n_distinct[l] * (3 * nvb(d * f));
    for (int b_ = 0; b_ < S; ++b_) {
      const int64_t p0 = shape[2 + b_], last = p0 + Tq - 1;
      int64_t lo = 0;
      if (P.layers[l].sliding) { lo = p0 - P.W + 1; if (lo < 0) lo = 0; }
      kvbytes += P.hkv * (last - lo + 1) * 2 * P.hd; /* K and V read */
    }
    kvbytes += (int64_t)T * 2 * kvd; /* K and V written */
  }
  out->weight_bytes = wbytes;
  out->kv_bytes = kvbytes;
  out->algorithmic_bytes = wbytes + kvbytes + (int64_t)T * d * 2 * 2;
  return MSK_OK;
}

msk_status_t msk_step_static(msk_handle_t* h, const uint16_t* hidden_in, const int32_t* positions, int n_seqs,
                             int tokens_per_seq, msk_kv_t* kv, uint16_t* hidden_out, void* stream) {
  if (!h || !hidden_in || !positions || !kv || !hidden_out || kv->h != h) return MSK_ERR_INVALID_ARG;
  if (n_seqs < 1 || tokens_per_seq < 1 || n_seqs > h->cfg.max_seqs || tokens_per_seq > h->cfg.max_tokens_per_seq ||
      n_seqs > kv->n_seqs)
    return MSK_ERR_INVALID_ARG;
  if (!aligned16(hidden_in) || !aligned16(hidden_out) || ((uintptr_t)positions & 3u)) return MSK_ERR_INVALID_ARG;
  /* the handle's shapes must fit the array: refused before any device work */
  const StaticLayout Lo = static_layout(h);
  if (Lo.total > (size_t)MSK_STATIC_SCRATCH_BYTES) return MSK_ERR_UNSUPPORTED;
  if (h->device < 0 || h->device >= MSK_STATIC_MAX_DEVICES) return MSK_ERR_UNSUPPORTED;
  int prev = 0;
  cudaGetDevice(&prev);
  if (prev != h->device && cudaSetDevice(h->device) != cudaSuccess) return MSK_ERR_CUDA;
  /* with the device current: the array's device address, looked up on the
   * first call that succeeds */
  uint8_t* base = nullptr;
  cudaError_t e = cudaSuccess;
  {
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_ptr[h->device]) {
      uint8_t* p = nullptr;
      e = cudaGetSymbolAddress((void**)&p, g_static_scratch);
      if (e == cudaSuccess && p) g_static_ptr[h->device] = p;
      else if (e == cudaSuccess) e = cudaErrorInvalidSymbol;
    }
    base = g_static_ptr[h->device];
  }
  if (e == cudaSuccess) {
    uint8_t* b = base;
    StaticPtrs p;
    p.h = (float*)(b + Lo.h);
    p.x = (uint16_t*)(b + Lo.x);
    p.qkv = (float*)(b + Lo.qkv);
    p.qs = (uint16_t*)(b + Lo.qs);
    p.part = (float*)(b + Lo.part);
    p.o = (uint16_t*)(b + Lo.o);
    p.x2f = (float*)(b + Lo.x2f);
    p.x2h = (uint16_t*)(b + Lo.x2h);
    p.xq = b + Lo.xq;
    p.logits = (float*)(b + Lo.logits);
    p.u = (uint16_t*)(b + Lo.u);
    p.ut = b + Lo.ut;
    p.y = (float*)(b + Lo.y);
    p.ctrl = (uint32_t*)(b + Lo.ctrl);
    MskParams* Pd = (MskParams*)(b + Lo.params);
    msk_static_params<<<1, 256, 0, (cudaStream_t)stream>>>(h->dev, Pd, p);
    e = cudaGetLastError();
    if (e == cudaSuccess) {
      MskStep st;
      st.hidden_in = hidden_in;
      st.positions = positions;
      st.hidden_out = hidden_out;
      st.kv_base = kv->base;
      st.kv_cap = kv->cap;
      st.kv_half_rows = kv->half_rows;
      st.kv_seqs = kv->n_seqs;
      st.S = n_seqs;
      st.Tq = tokens_per_seq;
      st.T = n_seqs * tokens_per_seq;
      e = msk_kernel_launch(h->host.hd, Pd, &st, &kv->map, h->ncta, (cudaStream_t)stream);
    }
  }
  if (prev != h->device) cudaSetDevice(prev);
  if (e != cudaSuccess) return MSK_ERR_CUDA;
  h->have_last = 1;
  return MSK_OK;
}

}  // extern "C"
