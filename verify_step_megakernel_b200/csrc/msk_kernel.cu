/*
 * msk_kernel.cu -- the persistent, cooperative decode/verify-step kernel.
 *
 * One launch runs every layer of the step (the pages' "one program replaces
 * many kernel boundaries"): one CTA per SM, each with one producer warp that
 * streams weight tiles (cp.async.bulk), KV stages (tensor copies, 128-byte
 * swizzle) and expert tiles into shared-memory rings guarded by mbarriers,
 * two warps that issue the tcgen05 tensor-core products (attention at head
 * dim 128, the block-scaled experts), and eight consumer warps that run the
 * rest of the math.  The producer runs ahead across phase and layer
 * boundaries: the next phase's dense weights and the past keys are in
 * flight while the consumers wait at a grid barrier; expert tiles are
 * issued as soon as this CTA has resolved the top-k routing (the pages'
 * "dense weights are streamed through a ring of tiles, selected expert
 * weights are requested as soon as routing finishes").
 *
 * Per layer (grid barriers marked |):
 *   QKV projection | QK-norm + fp8 KV write | split-sequence attention with
 *   the fixed softmax bound (at head dim 128 with its chunk combine) |
 *   (head dim 64: chunk combine |) W_o + residual | MoE RMSNorm | router
 *   logits | top-k (every CTA, redundantly) + gate/up + SwiGLU | SwiGLU
 *   terms + down projection | weighted combine + next RMSNorm |
 * NVFP4 products: the experts of units with at least tau tokens on the
 * block-scaled tensor cores (tcgen05.mma kind::mxf4nvf4, the activations as
 * eight e2m1 terms), the projections and the other units on mma.sync
 * m16n8k16 (f16 operands, fp32 accumulate: each e2m1 code times its e4m3
 * block scale is exact in f16); the fp32 global scale is applied to the
 * accumulator.
 *
 * Every wait is bounded by params.timeout_ns; a wait that gives up records
 * MSK_ERR_TIMEOUT and sets an abort word every other wait polls, so the
 * kernel always returns.
 */
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "msk_device.cuh"
#include "msk_internal.h"

namespace {

constexpr int NCW = MSK_NCW;
constexpr int NCT = MSK_NCW * 32;  /* consumer threads */
constexpr int BAR_CONS = 1;        /* named barrier of the consumer warps */
constexpr int CONS_WARP0 = 4;      /* warpgroup 0 produces, warpgroups 1-2 consume */
constexpr int CONS0 = CONS_WARP0 * 32;
/* registers per thread after the split; 128*64 + 256*208 must not exceed
 * the launch pool 384 * (launch registers), checked by the host */
constexpr int REGS_PRODUCER = 64;
constexpr int REGS_CONSUMER = 208;

enum Phase {
  PH_IN = 0, PH_QKV, PH_QKNORM, PH_ATT, PH_ATTC, PH_WO, PH_MOENORM, PH_ROUTER, PH_TOPK, PH_GU, PH_DN, PH_COMB,
  PH_UT /* the SwiGLU rows as e2m1 terms (block-scaled down projection) */
};

struct Route {
  int n_units, n_distinct;
  int n_units_tc; /* units [0, n_units_tc) take the block-scaled gate/up path, the rest the CUDA-core path */
  int16_t ids[MSK_MAX_TOKENS * 8];
  float w[MSK_MAX_TOKENS * 8];
  int16_t cnt[256];
  int16_t start[257];
  int16_t pairs[MSK_MAX_TOKENS * 8];  /* (token*k + slot), grouped by expert */
  int16_t unit_e[MSK_MAX_UNITS];
  int16_t unit_start[MSK_MAX_UNITS];  /* into pairs[] */
  int16_t unit_n[MSK_MAX_UNITS];
};

/* expert phases: a work item is 128 rows (16 per consumer warp) of the
 * selected expert matrices for one unit of <= 8 tokens; K streams in chunks
 * of <= 512 through a ring of slots (in the stage ring's memory) that the
 * producer thread fills */
constexpr int XROWS = 16 * MSK_NCW;
constexpr int XKC_MAX = 512;
constexpr int XNS_MAX = 4;

struct AttGeo {
  int npairs;
  int nparts; /* CTAs that take part: each gets >= 2 stages of keys when possible */
  int64_t N;
  int64_t lo[MSK_MAX_PAIRS];  /* first key position of the pair */
  int64_t off[MSK_MAX_PAIRS + 1]; /* prefix sums of key counts */
};
struct Smem {
  uint64_t full[MSK_NST];
  uint64_t empty[MSK_NST];
  uint64_t dfull[MSK_NCW][2];  /* dense weight slot of a warp landed */
  uint64_t dempty[MSK_NCW][2]; /* dense weight slot read by its warp */
  uint64_t bfull;              /* dense activation slice landed */
  uint64_t rfull;              /* the step's router logits landed (top-k) */
  uint64_t dfull2[2];       /* accumulator buffer 0/1 holds a finished item */
  uint64_t dempty2[2];      /* accumulator buffer 0/1 read by every consumer warp */
  uint64_t tfin;            /* every tensor-core op issued complete */
  uint32_t tmem_base;
  AttGeo ag;                /* this layer's attention key split (consumers) */
  AttGeo agp;               /* the producer warp's copy */
  uint4 sfb_one[64];        /* per issuing role: 128 rows x 4 ue4m3 scales of 1.0, the activation terms' scales */
  volatile int issuer_done; /* MMA-issuing warps that have committed their last work */
  uint64_t xfull[XNS_MAX];  /* expert slot landed (producer's expect-tx) */
  uint64_t xempty[XNS_MAX]; /* block-scaled expert slot consumed (both issuing roles' commits) */
  uint64_t xempty_cc[XNS_MAX]; /* CUDA-core expert slot consumed (each consumer warp arrives) */
  volatile int kv_ready;    /* layer+1 whose KV writes all CTAs finished */
  volatile int route_ready; /* layer+1 whose routing this CTA resolved */
  volatile int ring_free;   /* layer+1 whose expert phases released the ring */
  volatile int dn_ready;    /* layer+1 whose gate/up outputs all CTAs finished */
  volatile int dense_done;  /* dense phases this CTA finished (2 per layer) */
  volatile int abort;
  /* attention on the tensor cores (head dim 128): stage ring, score and
   * probability buffers, Q terms, output accumulator handoff */
  uint64_t kfull[6];        /* a stage's K landed (producer's expect-tx) */
  uint64_t kempty[6];       /* its QK products completed (tensor-core commit) */
  uint64_t vfull[6];        /* a stage's V landed */
  uint64_t vempty[6];       /* its P.V products completed */
  uint64_t s_ready[2];      /* scores S^T of buffer b computed */
  uint64_t s_free[2];       /* S^T of buffer b read by every consumer warp */
  uint64_t p_ready[3];      /* P^T of buffer b (stage mod 3) and the stage's bf16 V written by every consumer warp */
  uint64_t pv_done[3];      /* the P.V products of P^T buffer b completed */
  uint64_t q_ready;         /* the segment's Q terms written */
  uint64_t o_free;          /* the segment's output accumulator read */
  volatile int ag_ready;    /* layer+1 whose attention key split (ag) the consumers computed */
  volatile int attc_last;   /* this CTA wrote the last part of a pair: it combines the pair */
  float qfac[64];           /* per query row: softmax scale / its Q-term factor */
  int pos0[MSK_MAX_TOKENS];
  float lbuf[4][32][2];
  float red8[MSK_NCW];
  Route route;
};

constexpr size_t SMEM_BYTES = 1024 + (size_t)MSK_NST * MSK_STAGE + MSK_SCR + sizeof(Smem);
static_assert(SMEM_BYTES <= 232448, "227 KB of shared memory per CTA");

/* ---- context ---------------------------------------------------------------------- */
struct Ctx {
  const MskParams* P;
  MskStep st;
  const CUtensorMap* kvmap;
  uint8_t* ring;
  float* scr;
  Smem* S;
  int cta, ncta;
  uint32_t nbar; /* grid barriers passed */
};

MSK_DEV bool aborted(const Ctx& c) {
  return c.S->abort || ld_volatile_u32(&c.P->ctrl[CTRL_ABORT]) != 0;
}

MSK_DEV void raise_err(const Ctx& c, uint32_t code, int layer, int phase) {
  if (atomicCAS(&c.P->status[ST_CODE], 0u, code) == 0u)
    c.P->status[ST_WHERE] =
        0x80000000u | ((uint32_t)(layer & 0x7FFF) << 16) | ((uint32_t)phase << 8) | (uint32_t)(c.cta & 0xFF);
  atomicExch(&c.P->ctrl[CTRL_ABORT], 1u);
  c.S->abort = 1;
}

/* Waits consult the abort word and the timer only every WAIT_POLL SM
 * cycles (about 2 us): the abort word is in global memory, and a global
 * load behind a full copy stream takes about a microsecond, during which a
 * wait could not see its barrier complete.  A wait therefore runs up to
 * WAIT_POLL cycles past its limit. */
constexpr long long WAIT_POLL = 4096;

/* bounded mbarrier wait; false on timeout or abort.  `mult` scales the
 * limit: the producer's waits on the consumers' progress take twice the
 * limit of the consumers' own waits, so that when a step stalls, the wait
 * nearest the cause gives up first and its site is the one recorded. */
MSK_DEV bool wait_bar(const Ctx& c, uint64_t* bar, uint32_t parity, int layer, int phase, uint32_t mult = 1) {
  if (mbar_try(bar, parity)) return true;
  long long next = clock64() + WAIT_POLL;
  uint64_t t0 = 0;
  for (;;) {
    if (mbar_try(bar, parity)) return true;
    const long long now = clock64();
    if (now >= next) {
      if (aborted(c)) return false;
      const uint64_t t = gtimer();
      if (t0 == 0) t0 = t;
      else if (t - t0 > mult * (uint64_t)c.P->timeout_ns) {
        raise_err(c, MSK_ERR_TIMEOUT, layer, phase);
        return false;
      }
      next = now + WAIT_POLL;
    }
  }
}

/* consumer-only grid barrier; false if the step is being aborted */
MSK_DEV bool grid_sync(Ctx& c, int layer, int phase) {
  named_sync(BAR_CONS, NCT);
  __shared__ int s_ok;
  if (threadIdx.x == CONS0) {
    int ok = !c.S->abort;
    if (ok) {
      /* release: the CTA's writes (ordered before this thread by the CTA
       * barrier above) become visible before the count moves; acquire on
       * the poll orders the other CTAs' writes before ours.  The test hook
       * dbg_hold makes CTA 0 withhold one arrival, so that every wait at
       * that barrier runs out. */
      if (!(c.cta == 0 && c.P->dbg_hold > 0 && c.nbar + 1 == (uint32_t)c.P->dbg_hold))
        red_release_add_u32(&c.P->ctrl[CTRL_BARRIER], 1u);
      const uint32_t target = (c.nbar + 1) * (uint32_t)c.ncta;
      uint64_t t0 = 0;
      for (uint32_t it = 0; ld_acquire_u32(&c.P->ctrl[CTRL_BARRIER]) < target; ++it) {
        if ((it & 15) == 15) { /* the abort word and the clock, now and then */
          if (ld_volatile_u32(&c.P->ctrl[CTRL_ABORT])) { ok = 0; break; }
          if (t0 == 0) t0 = gtimer();
          else if (gtimer() - t0 > (uint64_t)c.P->timeout_ns) {
            raise_err(c, MSK_ERR_TIMEOUT, layer, phase);
            ok = 0;
            break;
          }
        }
      }
    }
    if (!ok) c.S->abort = 1;
    s_ok = ok;
  }
  named_sync(BAR_CONS, NCT);
  c.nbar++;
  if (c.P->dbg_trace && c.cta == 0 && threadIdx.x == CONS0 && layer >= 0)
    c.P->dbg_trace[layer * 16 + phase] = gtimer();
  return s_ok != 0;
}

/* ---- work split ------------------------------------------------------------------- */
MSK_DEV void item_range(int n, int cta, int ncta, int* a, int* b) {
  *a = (int)((int64_t)n * cta / ncta);
  *b = (int)((int64_t)n * (cta + 1) / ncta);
}

/* Slot layout of an expert chunk, the same for the producer and consumers.
 * Per matrix: codes [128][cpitch] then scales [128][spitch]; then the
 * unit's activation rows [8][bpitch] (f16).  Where K is a multiple of 256
 * the codes come as one 2-D tensor box 32 bytes wider than the chunk (the
 * next chunk's first bytes, or zero fill past the row), so that rows sit 32
 * bytes off the 128-byte bank period; with the lanes' interleaved block
 * order below, the warp's shared loads are then free of bank conflicts.
 * Other K (128, 384) take whole rows as single bulk copies. */
/* gate/up on the block-scaled tensor cores: K chunks of 256, slot layout
 * (1024-byte aligned, four slots in the ring):
 * [GU_A]  codes of gate, up: one 128-row x 128-byte box each (256 codes per
 *         row), 128-byte swizzled — the K-major SW128 layout
 * [GU_AS] scales of gate, up: their scale-factor atoms [matrix][4 k steps][512 B]
 * [GU_B]  the unit's tokens' activation terms: token t at t*1024, its chunk's
 *         [8 core-matrix columns][8 term rows][16 B] (all term scales are 1) */
constexpr int GU_KC = 256;
constexpr uint32_t GU_A = 0, GU_AS = 32768, GU_B = 36864, GU_SLOT = 45056;
constexpr uint32_t GU_AS_END = GU_B; /* codes and scale atoms of a chunk: one repacked tile */
/* block-scaled down slot: one repacked 512-wide K chunk (the gate/up tile
 * layout, its halves in place of the matrices), then per half the unit's
 * pairs' SwiGLU terms (8 pairs x 1 KB) */
constexpr uint32_t DT_B = GU_AS_END, DT_SLOT = DT_B + 2 * 8192;
/* TMEM columns: two buffers of gate and up accumulators (128 lanes x 64
 * each), then the scale factors of two chunks in flight */
constexpr uint32_t TM_D = 0, TM_DU = 64, TM_SFA = 256, TM_SFB = 384, TM_COLS = 512;
/* scale-factor buffers in TMEM: four chunks in rotation */
constexpr int NSF = 4;
constexpr uint32_t TM_SFA_BUF = 32; /* columns per buffer: 2 matrices x 4 steps x 4; SFB: 4 columns of ones */
static_assert(TM_SFA + NSF * TM_SFA_BUF <= TM_SFB && TM_SFB + 8 <= TM_COLS, "TMEM columns");

struct XGeo {
  int K, KC, nkc, rows_unit, ngroups, NM, tma, ns;
  uint32_t cpitch, spitch, bpitch, mat_bytes, b_off, slot_bytes;
  int u0;   /* first unit of the part */
  int a, b; /* this CTA's items [a, b) of the part (item i: unit u0 + i / ngroups) */
};

/* some expert unit can take the block-scaled gate/up path */
MSK_DEV bool tc_experts(const MskParams* P) { return P->tau <= MSK_UNIT_TOK; }
/* the block-scaled units take the block-scaled down projection too (the
 * host repacked the down tiles for it) */
MSK_DEV bool tc_down(const MskParams* P) { return P->layers[0].xtdt != nullptr; }

/* the parts of an expert phase: gate/up of the block-scaled units, gate/up
 * of the CUDA-core units, the down projection on the CUDA-core path (every
 * unit, or the CUDA-core units when tc_down), the block-scaled down
 * projection of the block-scaled units */
enum { XP_TC = 0, XP_CC = 1, XP_DN = 2, XP_DT = 3 };

MSK_DEV void xgeo(const Ctx& c, int part, XGeo& x) {
  const MskParams* P = c.P;
  const Route& R = c.S->route;
  if (part == XP_DT) {
    x.K = P->f;
    x.rows_unit = P->d;
    x.KC = 512;
    x.nkc = x.K / x.KC;
    x.tma = 1;
    x.cpitch = x.spitch = x.bpitch = 0;
    x.NM = 1;
    x.mat_bytes = x.b_off = DT_B;
    x.slot_bytes = DT_SLOT;
    x.ns = min(XNS_MAX, (int)((uint32_t)(MSK_NST * MSK_STAGE) / DT_SLOT));
    x.ngroups = x.rows_unit / XROWS;
    x.u0 = 0;
    item_range(R.n_units_tc * x.ngroups, c.cta, c.ncta, &x.a, &x.b);
    return;
  }
  const bool gu = part != XP_DN, tc = part == XP_TC;
  x.K = gu ? P->d : P->f;
  x.rows_unit = gu ? P->f : P->d;
  x.KC = tc ? GU_KC : (x.K <= XKC_MAX ? x.K : XKC_MAX);
  x.nkc = x.K / x.KC;
  x.tma = (x.K % 256) == 0;
  x.cpitch = (uint32_t)(x.tma ? x.KC / 2 + 32 : x.KC / 2);
  x.spitch = (uint32_t)(x.KC / 16);
  x.bpitch = (uint32_t)(2 * x.KC + 16);
  x.NM = gu ? 2 : 1;
  x.mat_bytes = XROWS * (x.cpitch + x.spitch);
  x.b_off = x.NM * x.mat_bytes;
  x.slot_bytes = tc ? GU_SLOT : (x.b_off + MSK_UNIT_TOK * x.bpitch + 127) & ~127u;
  x.ns = min(XNS_MAX, (int)((uint32_t)(MSK_NST * MSK_STAGE) / x.slot_bytes));
  x.ngroups = x.rows_unit / XROWS;
  x.u0 = (part == XP_CC || (part == XP_DN && tc_down(P))) ? R.n_units_tc : 0;
  const int nu = part == XP_TC ? R.n_units_tc : R.n_units - x.u0;
  item_range(nu * x.ngroups, c.cta, c.ncta, &x.a, &x.b);
}
/* bit s set where the phase's fills of expert slot s are odd in number */
MSK_DEV uint32_t fill_parity(const XGeo& x) {
  const int n = (x.b - x.a) * x.nkc;
  uint32_t m = 0;
  for (int s = 0; s < x.ns; ++s)
    if (((n / x.ns) + (s < n % x.ns ? 1 : 0)) & 1) m |= 1u << s;
  return m;
}
/* the slot parities flipped by the fills of item i (0-based in this CTA's
 * range): chunks i nkc .. (i+1) nkc - 1 of the phase */
MSK_DEV uint32_t fill_parity_run(const XGeo& x, int i) {
  uint32_t m = 0;
  for (int j = i * x.nkc; j < (i + 1) * x.nkc; ++j) m ^= 1u << (j % x.ns);
  return m;
}
/* gate+up with K = 512 is the largest slot: two must fit the ring */
static_assert(2 * ((2 * XROWS * (XKC_MAX / 2 + 32 + XKC_MAX / 16) + MSK_UNIT_TOK * (2 * XKC_MAX + 16) + 127) & ~127) <=
                  MSK_NST * MSK_STAGE,
              "two gate+up slots of the CUDA-core path fit the stage ring");
static_assert(XNS_MAX * GU_SLOT <= MSK_NST * MSK_STAGE, "four gate/up slots fit the stage ring");
static_assert(3 * DT_SLOT <= MSK_NST * MSK_STAGE && DT_SLOT % 1024 == 0, "three block-scaled down slots fit the ring");

/* Dense projections (QKV, W_o) with T <= 64 tokens: split-K over CTAs.  A
 * unit is one 16-row m-tile of the output rows times one K slice of 512 (or
 * all of K <= 512); units run slice-major and each CTA takes a contiguous
 * range, so it holds one activation slice [T][slice] in shared memory while
 * its warps stream weight m-tiles against it (unit i of the range goes to
 * warp i mod 8, through that warp's 2-slot ring).  Each unit writes its
 * fp32 partial; the next phase adds the slices in order. */
constexpr int DKS_MAX = 512;
constexpr int MAX_KS = 8; /* K slices of a projection of K <= 4096 */
constexpr int TOPK_MAX = 8; /* experts per token */
constexpr int DNS = 2;
constexpr uint32_t DB_BYTES = MSK_MAX_TOKENS * (2 * DKS_MAX + 16);   /* activation slice */
constexpr uint32_t DSLOT = 16 * (DKS_MAX / 2 + 32 + DKS_MAX / 16); /* one weight m-tile */
static_assert(DB_BYTES + MSK_NCW * DNS * DSLOT <= MSK_NST * MSK_STAGE, "dense buffers fit the stage ring");

struct DGeo {
  int K, rows, KS, S, MT, a, b;
  uint32_t cpitch, spitch, bpitch;
};

MSK_DEV void dgeo(const Ctx& c, bool qkv, DGeo& g) {
  const MskParams* P = c.P;
  g.K = qkv ? P->d : P->qd;
  g.rows = qkv ? P->qd + 2 * P->kvd : P->d;
  g.KS = g.K <= DKS_MAX ? g.K : DKS_MAX;
  g.S = g.K / g.KS;
  g.MT = g.rows / 16;
  g.cpitch = (uint32_t)(g.KS / 2 + 32);
  g.spitch = (uint32_t)(g.KS / 16);
  g.bpitch = (uint32_t)(2 * g.KS + 16);
  item_range(g.S * g.MT, c.cta, c.ncta, &g.a, &g.b);
}

/* matrix of output row `row` (QKV rows are q, then k, then v): its map
 * index, local row and global scale */
MSK_DEV void dense_mat(const MskParams* P, const MskLayer& Ly, bool qkv, int row, int* map, int* lrow, float* gs) {
  if (!qkv) { *map = MSK_MAP_DENSE + 6; *lrow = row; *gs = Ly.wo.gs; }
  else if (row < P->qd) { *map = MSK_MAP_DENSE; *lrow = row; *gs = Ly.wq.gs; }
  else if (row < P->qd + P->kvd) { *map = MSK_MAP_DENSE + 2; *lrow = row - P->qd; *gs = Ly.wk.gs; }
  else { *map = MSK_MAP_DENSE + 4; *lrow = row - P->qd - P->kvd; *gs = Ly.wv.gs; }
}

/* attention key space of one layer: pairs (seq, kv head) in order, each
 * with the union of its rows' key ranges; CTA c owns [c N / n, (c+1) N / n) */
/* the same geometry computed by one warp into shared memory (per-thread
 * copies of the arrays would live in local memory): att_geo_shared for the
 * consumers (warp 0 computes, every consumer warp passes the barrier); the
 * producer warp keeps its own copy, as it runs ahead of them */
MSK_DEV void att_geo_warp(const Ctx& c, int layer, AttGeo& g) {
  const MskParams* P = c.P;
  const int lane = threadIdx.x & 31;
  {
    const int npairs = c.st.S * P->hkv;
    const bool sliding = P->layers[layer].sliding != 0;
    int64_t run = 0;
    for (int base = 0; base < npairs; base += 32) {
      const int p = base + lane;
      int64_t lo = 0, cnt = 0;
      if (p < npairs) {
        const int b = p / P->hkv;
        const int64_t first = c.S->pos0[b], last = first + c.st.Tq - 1;
        if (sliding) { lo = first - P->W + 1; if (lo < 0) lo = 0; }
        cnt = last - lo + 1;
      }
      int64_t x = cnt; /* inclusive scan over the lanes */
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (p < npairs) {
        g.lo[p] = lo;
        g.off[p + 1] = run + x;
      }
      run += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) {
      g.npairs = npairs;
      g.off[0] = 0;
      g.N = run;
      const int64_t C = P->hd == 128 ? 128 : 256;
      const int64_t parts = (run + 2 * C - 1) / (2 * C);
      g.nparts = (int)(parts < 1 ? 1 : (parts > c.ncta ? c.ncta : parts));
    }
  }
  __syncwarp();
}
MSK_DEV void att_geo_shared(const Ctx& c, int layer) {
  if ((threadIdx.x >> 5) == CONS_WARP0) att_geo_warp(c, layer, c.S->ag);
  named_sync(BAR_CONS, NCT);
}
MSK_DEV int att_owner(const AttGeo& g, int64_t x) {
  return (int)(((x + 1) * (int64_t)g.nparts - 1) / g.N);
}
MSK_DEV int att_keys_per_stage(int hd) { return hd == 128 ? 128 : 256; }

/* Calls f(pair, slot, key0, nkeys, first_of_segment, last_of_segment) for
 * this CTA's attention stages. */
template <class F>
MSK_DEV void for_each_att_stage(const Ctx& c, const AttGeo& g, F&& f) {
  const int C = att_keys_per_stage(c.P->hd);
  if (c.cta >= g.nparts) return;
  int64_t A = g.N * c.cta / g.nparts, B = g.N * (c.cta + 1) / g.nparts;
  for (int p = 0; p < g.npairs; ++p) {
    int64_t a = max(A, g.off[p]), b = min(B, g.off[p + 1]);
    if (a >= b) continue;
    int64_t k0 = g.lo[p] + (a - g.off[p]), k1 = g.lo[p] + (b - g.off[p]);
    for (int64_t x = k0; x < k1; x += C) {
      int n = (int)min((int64_t)C, k1 - x);
      if (!f(p, c.cta + p, x, n, x == k0, x + C >= k1)) return;
    }
  }
}

/* tensor-core attention geometry (see attention_phase_tc) */
constexpr uint32_t ATC_HALF = 16384; /* K or V of a stage: 128 keys x 128 bytes */
/* TMEM columns: O^T, two S^T buffers, the V scale factors (all 1), and three
 * buffers of the P^T scale factors (two terms, 4 columns each: a block-scaled
 * MMA takes scale-factor addresses that are multiples of 4 columns) */
constexpr uint32_t ATC_TM_O = 0, ATC_TM_S = 64, ATC_TM_SSTRIDE = 192, ATC_TM_SFA = 448, ATC_TM_SFB = 452;
static_assert(ATC_TM_S + 2 * ATC_TM_SSTRIDE <= ATC_TM_SFA && ATC_TM_SFB + 3 * 8 <= 512 && ATC_TM_SFB % 4 == 0, "TMEM");
/* K and V come in separate rings (K is free once its QK products are
 * done, two stages before V): slots per ring by RP */
MSK_DEV int atc_nk(int RP) { return RP > 32 ? 4 : (RP > 16 ? 4 : 5); }
MSK_DEV int atc_nv(int RP) { return RP > 32 ? 4 : 6; }
MSK_DEV uint32_t atc_v_off(int RP) { return (uint32_t)atc_nk(RP) * ATC_HALF; }
MSK_DEV uint32_t atc_pt_off(int RP) { return (uint32_t)(atc_nk(RP) + atc_nv(RP)) * ATC_HALF; }
MSK_DEV uint32_t atc_q_off(int RP) { return atc_pt_off(RP) + 3u * (uint32_t)RP * 256u; }
/* scale-factor atoms: [3 buffers][2 terms][32 rows][16 B], then 512 B of ue8m0 1.0 */
MSK_DEV uint32_t atc_sf_off(int RP) { return atc_q_off(RP) + 3u * (uint32_t)RP * 128u; }
constexpr uint32_t ATC_SF_BYTES = 3 * 1024 + 512;
MSK_DEV int atc_rp(int R) { return R <= 16 ? 16 : (R <= 32 ? 32 : 64); }
static_assert(8 * ATC_HALF + 3 * 64 * 256 + 3 * 64 * 128 + ATC_SF_BYTES <= MSK_NST * MSK_STAGE + MSK_SCR, "RP 64 fits");
static_assert(10 * ATC_HALF + 3 * 32 * 256 + 3 * 32 * 128 + ATC_SF_BYTES <= MSK_NST * MSK_STAGE + MSK_SCR, "RP 32 fits");
static_assert(11 * ATC_HALF + 3 * 16 * 256 + 3 * 16 * 128 + ATC_SF_BYTES <= MSK_NST * MSK_STAGE + MSK_SCR, "RP 16 fits");
/* instruction descriptors, M = 128, fp32 accumulators.  QK: kind::f8f6f4,
 * e4m3 x e4m3, both K-major, N = 3 RP.  PV: kind::mxf8f6f4 block32, e4m3 x
 * e4m3, both MN-major, ue8m0 scales, N = RP, scale byte kk of B's words. */
MSK_DEV uint32_t atc_idesc_qk(int RP) { return (1u << 4) | ((uint32_t)((3 * RP) >> 3) << 17) | ((128u >> 4) << 24); }
MSK_DEV uint32_t atc_idesc_pv(int RP, uint32_t kk) {
  return (kk << 4) | (1u << 15) | (1u << 16) | ((uint32_t)(RP >> 3) << 17) | (1u << 23) | ((128u >> 4) << 24);
}

/* ---- producer ---------------------------------------------------------------------- */
struct Prod {
  Ctx* c;
  uint32_t it;
  uint32_t ait;   /* tensor-core attention stages issued (their K boxes) */
  uint32_t avt;   /* their V boxes issued */
  uint32_t xpar;  /* bit s: parity of the fills of expert slot s so far */
  uint32_t xused; /* bit s: expert slot s filled at least once */
  uint32_t xptc;  /* bit s: parity of its block-scaled fills (released by the issuers' commits) */
  uint32_t xpcc;  /* bit s: parity of its CUDA-core fills (released by the eight consumer warps) */
  uint32_t xlast; /* bit s: its last fill was a block-scaled one */
  uint32_t dpar;  /* bit 2w+s: parity of the fills of warp w's dense slot s */
  uint32_t dused; /* bit 2w+s: that slot filled at least once */
  bool ok;
};

/* The producer is one warp: every lane keeps the same schedule state and
 * waits itself; a failed wait anywhere fails the whole warp, so its control
 * flow stays uniform.  Lane 0 posts each barrier's byte count, then the
 * lanes issue the copies in parallel. */
MSK_DEV bool pwait_bar(const Ctx& c, uint64_t* bar, uint32_t parity, int layer, int phase) {
  return __all_sync(0xffffffffu, wait_bar(c, bar, parity, layer, phase, 2)) != 0;
}

MSK_DEV bool prod_acquire(Prod& p, int layer, int phase, uint8_t** stg, uint64_t** bar) {
  Ctx& c = *p.c;
  uint32_t slot = p.it % MSK_NST, round = p.it / MSK_NST;
  if (round > 0 && !pwait_bar(c, &c.S->empty[slot], (round - 1) & 1, layer, phase)) return false;
  *stg = c.ring + (size_t)slot * MSK_STAGE;
  *bar = &c.S->full[slot];
  p.it++;
  return true;
}

/* wait until every stage issued so far has been released by the consumers */
MSK_DEV bool prod_drain(Prod& p, int layer, int phase) {
  Ctx& c = *p.c;
  const uint32_t n = p.it < MSK_NST ? p.it : MSK_NST;
  for (uint32_t i = p.it - n; i < p.it; ++i)
    if (!pwait_bar(c, &c.S->empty[i % MSK_NST], (i / MSK_NST) & 1, layer, phase)) return false;
  return true;
}

/* a flag the consumers set: twice the consumers' limit (see wait_bar) */
MSK_DEV bool wait_flag(const Ctx& c, volatile int* flag, int want, int layer, int phase) {
  long long next = clock64() + WAIT_POLL;
  uint64_t t0 = 0;
  while (*flag < want) {
    const long long now = clock64();
    if (now >= next) {
      if (aborted(c)) return false;
      const uint64_t t = gtimer();
      if (t0 == 0) t0 = t;
      else if (t - t0 > 2 * (uint64_t)c.P->timeout_ns) {
        raise_err(c, MSK_ERR_TIMEOUT, layer, phase);
        return false;
      }
      next = now + WAIT_POLL;
    }
    __nanosleep(20);
  }
  __threadfence_block();
  return true;
}
/* wait until a global ready word reaches want (acquire), the abort word and
 * the clock checked now and then; false on abort or timeout (recorded) */
MSK_DEV bool wait_gword(const Ctx& c, const uint32_t* word, uint32_t want, int layer, int phase) {
  uint64_t t0 = 0;
  for (uint32_t it = 0; ld_acquire_u32(word) < want; ++it) {
    if ((it & 15) == 15) {
      if (ld_volatile_u32(&c.P->ctrl[CTRL_ABORT])) return false;
      if (t0 == 0) {
        t0 = gtimer();
      } else if (gtimer() - t0 > (uint64_t)c.P->timeout_ns) {
        raise_err(c, MSK_ERR_TIMEOUT, layer, phase);
        return false;
      }
    }
  }
  return true;
}

MSK_DEV bool pwait_flag(const Ctx& c, volatile int* flag, int want, int layer, int phase) {
  return __all_sync(0xffffffffu, wait_flag(c, flag, want, layer, phase)) != 0;
}

/* Feed the warps' dense weight rings for one projection: this CTA's units
 * in order, unit i of the range into warp i mod 8's next slot. */
MSK_DEV bool prod_dense(Prod& p, int layer, bool qkv) {
  Ctx& c = *p.c;
  const MskParams* P = c.P;
  const MskLayer& Ly = P->layers[layer];
  const int phase = qkv ? PH_QKV : PH_WO;
  DGeo g;
  dgeo(c, qkv, g);
  const uint32_t bytes = 16 * (g.cpitch + g.spitch);
  for (int i = g.a; i < g.b; ++i) {
    const int w = (i - g.a) % NCW, sl = ((i - g.a) / NCW) % DNS, bit = w * DNS + sl;
    if ((p.dused >> bit) & 1u) {
      if (!pwait_bar(c, &c.S->dempty[w][sl], ((p.dpar >> bit) & 1u) ^ 1u, layer, phase)) return false;
    }
    p.dpar ^= 1u << bit;
    p.dused |= 1u << bit;
    const int s = i / g.MT;
    int map, lrow;
    float gs;
    dense_mat(P, Ly, qkv, (i % g.MT) * 16, &map, &lrow, &gs);
    uint8_t* dst = c.ring + DB_BYTES + (size_t)bit * DSLOT;
    uint64_t* bar = &c.S->dfull[w][sl];
    const int lane = threadIdx.x & 31;
    if (lane == 0) mbar_arrive_tx(bar, bytes);
    __syncwarp();
    if (lane == 0) tma_2d_g2s(dst, Ly.emap + map, s * (g.KS / 4), lrow, bar);
    else if (lane == 1) tma_2d_g2s(dst + 16 * g.cpitch, Ly.emap + map + 1, s * (g.KS / 16), lrow, bar);
  }
  return true;
}

/* pull this CTA's weight tiles of a projection of `layer` into L2 */
MSK_DEV void prefetch_dense(const Ctx& c, int layer, bool qkv) {
  const MskParams* P = c.P;
  const MskLayer& Ly = P->layers[layer];
  DGeo g;
  dgeo(c, qkv, g);
  for (int i = g.a + (int)(threadIdx.x & 31); i < g.b; i += 32) {
    int map, lrow;
    float gs;
    dense_mat(P, Ly, qkv, (i % g.MT) * 16, &map, &lrow, &gs);
    const int s = i / g.MT;
    tma_prefetch_2d(Ly.emap + map, s * (g.KS / 4), lrow);
    tma_prefetch_2d(Ly.emap + map + 1, s * (g.KS / 16), lrow);
  }
}

/* Fill the expert ring for one phase: for each of this CTA's items and
 * each K chunk, the 128-row tiles of the unit's expert (gate and up, or
 * down) and the unit's activation rows, all on the slot's full barrier. */
MSK_DEV bool prod_xslot(Prod& p, int s, bool tc, int layer, int phase);

MSK_DEV bool prod_experts(Prod& p, int layer, int part) {
  Ctx& c = *p.c;
  const MskParams* P = c.P;
  const MskLayer& Ly = P->layers[layer];
  const Route& R = c.S->route;
  const bool gu = part != XP_DN;
  const int phase = gu ? PH_GU : PH_DN;
  XGeo x;
  xgeo(c, part, x);
  const MskNv* mat[2] = {gu ? &Ly.wg : &Ly.wd, &Ly.wu};
  const CUtensorMap* cmap[2] = {Ly.emap + (gu ? 0 : 4), Ly.emap + 2};
  const CUtensorMap* smap[2] = {Ly.emap + (gu ? 1 : 5), Ly.emap + 3};
  const int lane = threadIdx.x & 31;
  int j = 0;
  if (part == XP_DT) { /* block-scaled down: one repacked tile per 512-wide chunk, the pairs' SwiGLU terms */
    const size_t utb = MSK_XQ_BYTES(P->f);
    int wunit = -1; /* the unit whose pairs' terms were last waited for */
    for (int item = x.a; item < x.b; ++item) {
      const int unit = x.u0 + item / x.ngroups, grp = item % x.ngroups;
      const int n = R.unit_n[unit], st0 = R.unit_start[unit];
      const int64_t tile0 = ((int64_t)R.unit_e[unit] * x.ngroups + grp) * x.nkc;
      const int tl = lane - 8; /* lanes 8-15 copy pair tl's terms */
      const uint8_t* tq = nullptr;
      if (lane >= 8 && tl < n) tq = P->ut + (size_t)R.pairs[st0 + tl] * utb;
      const uint32_t bytes = DT_B + (uint32_t)n * 2048u;
      for (int kc = 0; kc < x.nkc; ++kc, ++j) {
        const int s = j % x.ns;
        if (!prod_xslot(p, s, true, layer, PH_DN)) return false;
        uint8_t* dst = c.ring + (size_t)s * x.slot_bytes;
        uint64_t* bar = &c.S->xfull[s];
        if (lane == 0) mbar_arrive_tx(bar, bytes);
        __syncwarp();
        bool ok = true;
        if (lane == 0) {
          bulk_g2s(dst, Ly.xtdt + (tile0 + kc) * DT_B, DT_B, bar);
        } else if (tq) { /* per 256-wide half: the pair's kilobyte of terms, once some CTA has written them */
          if (unit != wunit) {
            ok = wait_gword(c, &P->ctrl[CTRL_UT0 + R.pairs[st0 + tl]], (uint32_t)(layer + 1), layer, PH_UT);
            fence_proxy_async_global();
          }
          if (ok) {
            bulk_g2s(dst + DT_B + tl * 1024, tq + (size_t)(2 * kc) * 1024, 1024, bar);
            bulk_g2s(dst + DT_B + 8192 + tl * 1024, tq + (size_t)(2 * kc + 1) * 1024, 1024, bar);
          }
        }
        if (!__all_sync(0xffffffffu, ok)) return false;
        wunit = unit;
      }
    }
    return true;
  }
  if (part == XP_TC) { /* block-scaled tensor cores: swizzled code boxes, scale atoms, the tokens' terms */
    const size_t xqb = MSK_XQ_BYTES(P->d);
    for (int item = x.a; item < x.b; ++item) {
      const int unit = x.u0 + item / x.ngroups, grp = item % x.ngroups;
      const int n = R.unit_n[unit], st0 = R.unit_start[unit];
      const int64_t grow = (int64_t)R.unit_e[unit] * x.rows_unit + (int64_t)grp * XROWS;
      const int tl = lane - 8; /* lanes 8-15 copy token tl's terms */
      const uint8_t* tq = nullptr;
      if (lane >= 8 && tl < n) tq = P->xq + (size_t)(R.pairs[st0 + tl] / P->k) * xqb;
      const uint32_t bytes = (uint32_t)(2 * 16384 + 2 * XROWS * (GU_KC / 16) + n * 8 * (GU_KC / 2));
      for (int kc = 0; kc < x.nkc; ++kc, ++j) {
        const int s = j % x.ns;
        if (!prod_xslot(p, s, true, layer, phase)) return false;
        uint8_t* dst = c.ring + (size_t)s * x.slot_bytes;
        uint64_t* bar = &c.S->xfull[s];
        if (lane == 0) mbar_arrive_tx(bar, bytes);
        __syncwarp();
        if (lane == 0) { /* the chunk's codes and scale atoms of both matrices: one tile, one copy */
          const int64_t tile = (grow / XROWS) * (P->d / GU_KC) + kc;
          bulk_g2s(dst, Ly.xtgu + tile * GU_AS_END, GU_AS_END, bar);
        } else if (tq) {
          bulk_g2s(dst + GU_B + tl * (8 * GU_KC / 2), tq + (size_t)kc * (8 * GU_KC / 2), 8 * GU_KC / 2, bar);
        }
      }
    }
    return true;
  }
  const uint16_t* act = gu ? P->x2h : P->u;
  const int act_ld = gu ? P->d : P->f;
  const uint32_t brow = (uint32_t)(2 * x.KC);
  for (int item = x.a; item < x.b; ++item) {
    const int unit = x.u0 + item / x.ngroups, grp = item % x.ngroups;
    const int n = R.unit_n[unit], st0 = R.unit_start[unit];
    const int64_t grow = (int64_t)R.unit_e[unit] * x.rows_unit + (int64_t)grp * XROWS;
    int my_row = 0; /* lanes 8.. : the activation row of the unit's entry lane-8 (token, or pair) */
    if (lane >= 8 && lane < 8 + n) {
      const int pair = R.pairs[st0 + lane - 8];
      my_row = gu ? pair / P->k : pair;
    }
    for (int kc = 0; kc < x.nkc; ++kc, ++j) {
      const int s = j % x.ns;
      if (!prod_xslot(p, s, false, layer, phase)) return false;
      uint8_t* dst = c.ring + (size_t)s * x.slot_bytes;
      uint64_t* bar = &c.S->xfull[s];
      if (lane == 0) mbar_arrive_tx(bar, x.b_off + (uint32_t)n * brow);
      __syncwarp();
      if (!gu && Ly.xtdn && x.tma) { /* the down chunk's codes and scales: one repacked tile, one copy */
        if (lane == 0) bulk_g2s(dst, Ly.xtdn + ((grow / XROWS) * x.nkc + kc) * (int64_t)x.mat_bytes, x.mat_bytes, bar);
        else if (lane >= 8 && lane < 8 + n)
          bulk_g2s(dst + x.b_off + (lane - 8) * x.bpitch, act + (size_t)my_row * act_ld + (size_t)kc * x.KC, brow, bar);
      } else if (lane < 2 * x.NM) { /* lane 2m: codes of matrix m, lane 2m+1: its scales */
        const int m = lane >> 1;
        uint8_t* md = dst + (size_t)m * x.mat_bytes;
        if (x.tma) {
          if (lane & 1) tma_2d_g2s(md + XROWS * x.cpitch, smap[m], kc * (x.KC / 16), (int32_t)grow, bar);
          else tma_2d_g2s(md, cmap[m], kc * (x.KC / 4), (int32_t)grow, bar);
        } else {
          if (lane & 1) bulk_g2s(md + XROWS * x.cpitch, mat[m]->scales + grow * (x.K / 16), XROWS * x.spitch, bar);
          else bulk_g2s(md, mat[m]->codes + grow * (x.K / 2), XROWS * x.cpitch, bar);
        }
      } else if (lane >= 8 && lane < 8 + n) { /* one activation row per lane */
        bulk_g2s(dst + x.b_off + (lane - 8) * x.bpitch, act + (size_t)my_row * act_ld + (size_t)kc * x.KC, brow, bar);
      }
    }
  }
  return true;
}

/* Before filling expert slot s: wait (if it was filled before) until its
 * last fill was released, by the barrier of that fill's kind, then record
 * this fill (tc: a block-scaled fill). */
MSK_DEV bool prod_xslot(Prod& p, int s, bool tc, int layer, int phase) {
  Ctx& c = *p.c;
  if ((p.xused >> s) & 1u) {
    const bool ltc = (p.xlast >> s) & 1u;
    if (!pwait_bar(c, ltc ? &c.S->xempty[s] : &c.S->xempty_cc[s], (((ltc ? p.xptc : p.xpcc) >> s) & 1u) ^ 1u, layer,
                   phase))
      return false;
  }
  p.xpar ^= 1u << s;
  p.xused |= 1u << s;
  if (tc) {
    p.xptc ^= 1u << s;
    p.xlast |= 1u << s;
  } else {
    p.xpcc ^= 1u << s;
    p.xlast &= ~(1u << s);
  }
  return true;
}

/* wait until the last fill of every expert slot has been released */
MSK_DEV bool prod_xdrain(Prod& p, int layer) {
  Ctx& c = *p.c;
  for (int s = 0; s < XNS_MAX; ++s)
    if ((p.xused >> s) & 1u) {
      const bool tc = (p.xlast >> s) & 1u;
      if (!pwait_bar(c, tc ? &c.S->xempty[s] : &c.S->xempty_cc[s], (((tc ? p.xptc : p.xpcc) >> s) & 1u) ^ 1u, layer, PH_GU))
        return false;
    }
  return true;
}

/* The attention products of one layer at head dim 128 (QK for role 0, P.V
 * for role 1), defined with the attention phase. */
MSK_DEV bool issuer_att(Ctx& c, int layer, int role, uint32_t& ait, uint32_t& aseg);

/* The two MMA-issuing warps (warps 1 and 2; lane 0 issues), role 0 and 1:
 * attention QK and PV products respectively; the gate and the up matrix of
 * the block-scaled gate/up items respectively (each copies its matrix's
 * scale atoms into TMEM and issues its MMAs; the slot and the accumulator
 * buffer complete when both have committed); and every other item of the
 * block-scaled down projection each.  Per chunk: wait for the slot's fill
 * and (first chunk of an item) for the consumers' release of the item's
 * accumulator buffer, copy the scales, issue the MMAs, commit. */
MSK_DEV void issuer(Ctx& c, int role) {
  const MskParams* P = c.P;
  const int lane = threadIdx.x & 31;
  const uint32_t idesc = (1u << 7) | (1u << 10) | ((uint32_t)(64 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
  uint32_t bits = 0; /* 0-3 expert-slot fill parities, 4-5 dempty parities, 6-7 accumulator buffer used */
  bool ok = true;
  uint32_t tb = 0;
  uint32_t ait = 0, aseg = 0; /* attention stages and segments issued */
  for (int l = 0; l < P->L && ok; ++l) {
    if (P->hd == 128 && !issuer_att(c, l, role, ait, aseg)) { ok = false; break; }
    if (!tc_experts(P)) continue;
    if (!pwait_flag(c, &c.S->route_ready, l + 1, l, PH_GU)) { ok = false; break; }
    tb = c.S->tmem_base;
    /* the activation terms' block scales, all 1.0 (ue4m3 0x38), into TMEM
     * each layer (the attention phase reuses those columns); each role
     * copies its own, so its MMAs follow the copy in its issue order */
    if (l == 0) {
      c.S->sfb_one[role * 32 + lane] = make_uint4(0x38383838u, 0x38383838u, 0x38383838u, 0x38383838u);
      fence_proxy_async_shared();
      __syncwarp();
    }
    if (lane == 0) {
      tc_fence_after();
      tc_cp_sf(tb + TM_SFB + 4 * role, umma_desc(smem_u32(c.S->sfb_one + role * 32), 16, 128, 0));
    }
    __syncwarp();
    XGeo x, xc, xd, xt;
    xgeo(c, XP_TC, x);
    xgeo(c, XP_CC, xc); /* (read while this layer's routing is current) */
    xgeo(c, XP_DN, xd);
    const bool dt = tc_down(P) && c.S->route.n_units_tc > 0;
    xgeo(c, XP_DT, xt);
    const uint32_t ring = smem_u32(c.ring);
    int j = 0;
    for (int item = x.a; item < x.b && ok; ++item) {
      const int db = (item - x.a) & 1;
      for (int kc = 0; kc < x.nkc; ++kc, ++j) {
        const int s = j % x.ns, buf = j & (NSF - 1);
        if (!pwait_bar(c, &c.S->xfull[s], (bits >> s) & 1u, l, PH_GU)) { ok = false; break; }
        bits ^= 1u << s;
        if (kc == 0 && ((bits >> (6 + db)) & 1u)) {
          if (!pwait_bar(c, &c.S->dempty2[db], (bits >> (4 + db)) & 1u, l, PH_GU)) { ok = false; break; }
          bits ^= 1u << (4 + db);
        }
        if (lane == 0) {
          tc_fence_after();
          const uint32_t slot = ring + (uint32_t)s * x.slot_bytes;
          const uint64_t sd = umma_desc(slot + GU_AS, 16, 128, 0), ad = umma_desc(slot + GU_A, 16, 1024, 2),
                         bd = umma_desc(slot + GU_B, 128, 8 * GU_KC / 2, 0);
          /* this role's matrix: its scale atoms (4 steps) into its TMEM
           * columns, then its 4 MMAs; descriptors advance by adding to their
           * address field (16-byte units) */
          const uint32_t sfa = tb + TM_SFA + buf * TM_SFA_BUF + 16 * role, sfb = tb + TM_SFB + 4 * role;
          const uint32_t dg = tb + TM_D + db * 128 + TM_DU * role;
          const uint64_t sdr = sd + (uint64_t)(128 * role), adr = ad + (uint64_t)(1024 * role);
#pragma unroll
          for (int st = 0; st < GU_KC / 64; ++st) tc_cp_sf(sfa + 4 * st, sdr + (uint64_t)(st * 32));
#pragma unroll
          for (int st = 0; st < GU_KC / 64; ++st)
            tc_mma_nvf4(dg, adr + (uint64_t)(2 * st), bd + (uint64_t)(16 * st), idesc, (kc > 0 || st > 0) ? 1u : 0u,
                        sfa + 4 * st, sfb);
          tc_commit(&c.S->xempty[s]);
          if (kc == x.nkc - 1) tc_commit(&c.S->dfull2[db]);
        }
        __syncwarp();
        if (kc == x.nkc - 1) bits |= 1u << (6 + db);
      }
    }
    /* the producer fills the same slots for the CUDA-core units and the
     * down projection: count those fills too, so the later waits take the
     * right parity */
    bits ^= fill_parity(xc);
    /* block-scaled down: the items alternate between the roles (item i on
     * accumulator buffer i mod 2 and role i mod 2); a role issues both
     * halves of each of its chunks and commits twice for the slot's and the
     * buffer's two-arrival barriers; it follows the other role's slot fills
     * and buffer releases in its parities without waiting on them */
    int jr = 0; /* chunks this role issued */
    /* a slot's full barrier only tells parities apart: wait until the
     * CUDA-core fills counted above have all landed (every CTA is past
     * gate/up) before waiting on the fills that follow them, so no wait can
     * match a fill two phases early */
    if (dt && ok && !pwait_flag(c, &c.S->dn_ready, l + 1, l, PH_DN)) ok = false;
    for (int item = xt.a; dt && ok && item < xt.b; ++item) {
      const int db = (item - xt.a) & 1;
      const bool mine = db == role;
      for (int kc = 0; kc < xt.nkc; ++kc) {
        const int s = ((item - xt.a) * xt.nkc + kc) % xt.ns;
        if (mine && !pwait_bar(c, &c.S->xfull[s], (bits >> s) & 1u, l, PH_DN)) { ok = false; break; }
        bits ^= 1u << s;
        if (kc == 0 && ((bits >> (6 + db)) & 1u)) {
          if (mine && !pwait_bar(c, &c.S->dempty2[db], (bits >> (4 + db)) & 1u, l, PH_DN)) { ok = false; break; }
          bits ^= 1u << (4 + db);
        }
        if (mine) {
          if (lane == 0) {
            tc_fence_after();
            const uint32_t slot = ring + (uint32_t)s * xt.slot_bytes;
            const uint64_t sd = umma_desc(slot + GU_AS, 16, 128, 0), ad = umma_desc(slot + GU_A, 16, 1024, 2);
            /* two scale buffers per role, alternating by chunk */
            const uint32_t sbuf = tb + TM_SFA + (uint32_t)(2 * (jr & 1) + role) * TM_SFA_BUF;
            const uint32_t dg = tb + TM_D + db * 128, sfb = tb + TM_SFB + 4 * role;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint32_t sfa = sbuf + 16 * h;
              const uint64_t bd = umma_desc(slot + DT_B + 8192 * h, 128, 8 * GU_KC / 2, 0);
#pragma unroll
              for (int st = 0; st < GU_KC / 64; ++st) tc_cp_sf(sfa + 4 * st, sd + (uint64_t)(128 * h + st * 32));
#pragma unroll
              for (int st = 0; st < GU_KC / 64; ++st)
                tc_mma_nvf4(dg, ad + (uint64_t)(1024 * h + 2 * st), bd + (uint64_t)(16 * st), idesc,
                            (kc > 0 || h > 0 || st > 0) ? 1u : 0u, sfa + 4 * st, sfb);
            }
            tc_commit(&c.S->xempty[s]);
            tc_commit(&c.S->xempty[s]);
            if (kc == xt.nkc - 1) {
              tc_commit(&c.S->dfull2[db]);
              tc_commit(&c.S->dfull2[db]);
            }
          }
          __syncwarp();
          ++jr;
        }
        if (kc == xt.nkc - 1) bits |= 1u << (6 + db);
      }
    }
    bits ^= fill_parity(xd);
  }
  if (lane == 0) {
    tc_commit(&c.S->tfin);
    __threadfence_block();
    atomicAdd((int*)&c.S->issuer_done, 1);
  }
}

MSK_DEV bool prod_att_tc(Prod& p, int layer, uint32_t& ait);
MSK_DEV bool prod_att_tc_drain(Prod& p, int layer, uint32_t ait);

MSK_DEV void producer(Ctx& c) {
  const MskParams* P = c.P;
  Prod p;
  p.c = &c;
  p.it = 0;
  p.ait = 0;
  p.avt = 0;
  p.xpar = 0;
  p.xused = 0;
  p.xptc = 0;
  p.xpcc = 0;
  p.xlast = 0;
  p.dpar = 0;
  p.dused = 0;
  p.ok = true;
  const int hd = P->hd;
  const int C = att_keys_per_stage(hd);
  for (int l = 0; l < P->L && p.ok; ++l) {
    /* QKV weight tiles; the ring memory is free once the previous layer's
     * expert phases released it */
    if (!prod_dense(p, l, true)) { p.ok = false; break; }
    /* attention stages reuse the memory once this CTA's QKV units are done:
     * past keys stream at once, chunks holding this step's keys wait until
     * every CTA has written them */
    if (!pwait_flag(c, &c.S->dense_done, 2 * l + 1, l, PH_ATT)) { p.ok = false; break; }
    att_geo_warp(c, l, c.S->agp);
    const AttGeo& g = c.S->agp;
    if (hd == 128) {
      /* tensor-core attention: its own stage ring; W_o tiles once every
       * stage's products have completed */
      if (!prod_att_tc(p, l, p.ait) || !prod_att_tc_drain(p, l, p.ait)) { p.ok = false; break; }
    } else {
    for_each_att_stage(c, g, [&](int pr, int slot, int64_t k0, int n, bool, bool) {
      int b = pr / P->hkv, h = pr % P->hkv;
      if (k0 + C > c.S->pos0[b]) {
        if (!pwait_flag(c, &c.S->kv_ready, l + 1, l, PH_ATT)) { p.ok = false; return false; }
        fence_proxy_async_global();
      }
      uint8_t* stg;
      uint64_t* bar;
      if (!prod_acquire(p, l, PH_ATT, &stg, &bar)) { p.ok = false; return false; }
      int64_t row = (((int64_t)l * c.st.kv_seqs + b) * P->hkv + h) * c.st.kv_cap + k0;
      const int lane = threadIdx.x & 31;
      if (lane == 0) {
        mbar_arrive_tx(bar, (uint32_t)(2 * C * hd));
        tma_3d_g2s(stg, c.kvmap, 0, (int32_t)row, 0, bar); /* K at 0, V at C hd */
      }
      __syncwarp();
      (void)slot;
      (void)n;
      return true;
    });
    }
    if (!p.ok) break;
    /* W_o tiles once every attention stage has been read */
    if (!prod_drain(p, l, PH_WO) || !prod_dense(p, l, false)) { p.ok = false; break; }
    /* pull this CTA's next-layer dense tiles into L2, then feed the expert
     * phases once this layer's routing (and later its gate/up outputs) is
     * known */
    if (l + 1 < P->L) {
      prefetch_dense(c, l + 1, true);
      prefetch_dense(c, l + 1, false);
    }
    if (!pwait_flag(c, &c.S->route_ready, l + 1, l, PH_GU)) { p.ok = false; break; }
    fence_proxy_async_global();
    {
      const Route& R = c.S->route;
      if (R.n_units_tc > 0 && !prod_experts(p, l, XP_TC)) { p.ok = false; break; }
      /* the CUDA-core units' slots are laid out differently: every
       * block-scaled slot must be free first */
      if (R.n_units_tc > 0 && R.n_units > R.n_units_tc && !prod_xdrain(p, l)) { p.ok = false; break; }
      if (R.n_units > R.n_units_tc && !prod_experts(p, l, XP_CC)) { p.ok = false; break; }
    }
    if (!pwait_flag(c, &c.S->dn_ready, l + 1, l, PH_DN)) { p.ok = false; break; }
    fence_proxy_async_global();
    {
      const Route& R = c.S->route;
      const bool dt = tc_down(P) && R.n_units_tc > 0;
      if (dt) { /* every previous slot released, then the block-scaled down units (each pair's terms waited for) */
        if (!prod_xdrain(p, l) || !prod_experts(p, l, XP_DT)) { p.ok = false; break; }
      }
      if (R.n_units > (dt ? R.n_units_tc : 0)) {
        if (dt && !prod_xdrain(p, l)) { p.ok = false; break; }
        if (!prod_experts(p, l, XP_DN)) { p.ok = false; break; }
      }
    }
    if (!pwait_flag(c, &c.S->ring_free, l + 1, l, PH_DN)) { p.ok = false; break; }
  }
  if (!p.ok && (threadIdx.x & 31) == 0) {
    /* let every copy already issued land before the CTA may exit */
    for (int bit = 0; bit < NCW * DNS; ++bit) {
      if (!((p.dused >> bit) & 1u)) continue;
      const uint32_t par = ((p.dpar >> bit) & 1u) ^ 1u;
      uint64_t t0 = gtimer();
      while (!mbar_try(&c.S->dfull[bit / DNS][bit % DNS], par)) {
        if (gtimer() - t0 > 2 * (uint64_t)P->timeout_ns) break;
      }
    }
    for (int sl = 0; sl < XNS_MAX; ++sl) {
      if (!((p.xused >> sl) & 1u)) continue;
      const uint32_t par = ((p.xpar >> sl) & 1u) ^ 1u; /* the slot's latest fill */
      uint64_t t0 = gtimer();
      while (!mbar_try(&c.S->xfull[sl], par)) {
        if (gtimer() - t0 > 2 * (uint64_t)P->timeout_ns) break;
      }
    }
    uint32_t n = p.it < MSK_NST ? p.it : MSK_NST;
    for (uint32_t i = p.it - n; i < p.it; ++i) {
      uint32_t slot = i % MSK_NST;
      uint64_t t0 = gtimer();
      while (!mbar_try(&c.S->full[slot], (i / MSK_NST) & 1)) {
        if (gtimer() - t0 > 2 * (uint64_t)P->timeout_ns) break;
      }
    }
    if (hd == 128) { /* every K and V copy issued */
      const int RP = atc_rp(c.st.Tq * P->G);
      for (int kv = 0; kv < 2; ++kv) {
        const uint32_t ns = (uint32_t)(kv ? atc_nv(RP) : atc_nk(RP)), it = kv ? p.avt : p.ait, na = it < ns ? it : ns;
        for (uint32_t i = it - na; i < it; ++i) {
          uint64_t t0 = gtimer();
          while (!mbar_try(kv ? &c.S->vfull[i % ns] : &c.S->kfull[i % ns], (i / ns) & 1)) {
            if (gtimer() - t0 > 2 * (uint64_t)P->timeout_ns) break;
          }
        }
      }
    }
  }
}

/* ---- consumer: weight stages on the tensor cores ----------------------------------- */
struct Cons {
  Ctx* c;
  uint32_t it;
};

MSK_DEV uint8_t* cons_wait(Cons& q, int layer, int phase, uint32_t* slot_out) {
  Ctx& c = *q.c;
  uint32_t slot = q.it % MSK_NST, round = q.it / MSK_NST;
  if (!wait_bar(c, &c.S->full[slot], round & 1, layer, phase)) return nullptr;
  *slot_out = slot;
  q.it++;
  return c.ring + (size_t)slot * MSK_STAGE;
}
MSK_DEV void cons_release(Cons& q, uint32_t slot) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&q.c->S->empty[slot]);
}

/* split of a weight stage over the consumer warps: mt m-tiles x ks K-slices */
/* ---- consumer: dense projections ------------------------------------------------------ */
/*
 * One warp's 16-row m-tile (codes and scales in its ring slot) times up to
 * NT 8-column tiles of the activation slice in shared memory, over one K
 * slice.  Same lane layout as the expert tiles: lane (g, cq) owns the NVFP4
 * blocks 4 qb + cq, decodes them once and feeds every column tile.
 */
template <int NT, bool FULL>
MSK_DEV void dgemm(uint32_t codes, uint32_t scales, uint32_t cpitch, uint32_t spitch, uint32_t bsm, uint32_t bpitch,
                   int KS, int ntl, float (*acc)[4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, cq = lane & 3;
  const uint32_t sel = (uint32_t)(cq | (cq << 4) | ((cq + 4) << 8) | ((cq + 4) << 12));
  const uint32_t a0 = codes + g * cpitch + 8 * cq, a1 = a0 + 8 * cpitch;
  const uint32_t s0 = scales + g * spitch, s1 = s0 + 8 * spitch;
  const uint32_t b = bsm + g * bpitch + 32 * cq;
  const int nq = KS / 64;
  for (int qb = 0; qb < nq; ++qb) {
    const uint2 c0 = lds64(a0 + 32 * qb), c1 = lds64(a1 + 32 * qb);
    const uint32_t w0 = lds32(s0 + 4 * qb), w1 = lds32(s1 + 4 * qb);
    uint32_t sc[2];
    e4m3x4_to_f16x2x2(__byte_perm(w0, w1, sel), sc);
    uint32_t r0[8], r1[8];
    e2m1x8_to_f16x2x4(c0.x, r0);
    e2m1x8_to_f16x2x4(c0.y, r0 + 4);
    e2m1x8_to_f16x2x4(c1.x, r1);
    e2m1x8_to_f16x2x4(c1.y, r1 + 4);
    uint32_t a[4][4];
#pragma unroll
    for (int st = 0; st < 4; ++st) {
      a[st][0] = hmul2(r0[2 * st], sc[0]);
      a[st][1] = hmul2(r1[2 * st], sc[1]);
      a[st][2] = hmul2(r0[2 * st + 1], sc[0]);
      a[st][3] = hmul2(r1[2 * st + 1], sc[1]);
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      if (FULL || nt < ntl) {
        const uint32_t bt = b + nt * 8 * bpitch + 128 * qb;
        const uint4 b0 = lds128(bt), b1 = lds128(bt + 16);
        mma_f16(acc[nt], a[0], b0.x, b0.y);
        mma_f16(acc[nt], a[1], b0.z, b0.w);
        mma_f16(acc[nt], a[2], b1.x, b1.y);
        mma_f16(acc[nt], a[3], b1.z, b1.w);
      }
    }
  }
}

/* QKV or W_o for this step's T tokens: this CTA's units, slice by slice.
 * dpar bits 0-1: this warp's parities of its two weight slots; bit 8: the
 * activation slice barrier's parity.  Every warp takes part in every slice
 * (the CTA-wide barriers keep one sequence even after a failed wait). */
template <bool QKV>
MSK_DEV bool dense_phase(Ctx& c, int layer, uint32_t& dpar) {
  const MskParams* P = c.P;
  const MskLayer& Ly = P->layers[layer];
  const int cw = (threadIdx.x >> 5) - CONS_WARP0, lane = threadIdx.x & 31, g = lane >> 2, cq = lane & 3;
  const int ctid = threadIdx.x - CONS0;
  const int phase = QKV ? PH_QKV : PH_WO;
  DGeo G;
  dgeo(c, QKV, G);
  const int T = c.st.T, ntl = (T + 7) >> 3;
  const uint16_t* act = QKV ? P->x : P->o;
  float* out = P->qkv;
  const uint32_t ring = smem_u32(c.ring);
  bool ok = true;
  for (int i0 = G.a; i0 < G.b;) {
    const int s = i0 / G.MT;
    const int i1 = min(G.b, (s + 1) * G.MT);
    /* the activation slice: the byte count is posted first, the copies go
     * out once every warp is done with the region */
    const uint32_t bpar = (dpar >> 8) & 1u;
    dpar ^= 1u << 8;
    if (ok && ctid == 0) mbar_arrive_tx(&c.S->bfull, (uint32_t)(T * 2 * G.KS));
    named_sync(BAR_CONS, NCT);
    const bool issued = ok && ctid < T;
    if (issued) {
      fence_proxy_async_global();
      bulk_g2s(c.ring + (size_t)ctid * G.bpitch, act + (size_t)ctid * G.K + (size_t)s * G.KS, (uint32_t)(2 * G.KS),
               &c.S->bfull);
    }
    if (ok && !wait_bar(c, &c.S->bfull, bpar, layer, phase)) ok = false;
    if (!ok && issued) { /* this thread's copy must land before the CTA may exit */
      const uint64_t t0 = gtimer();
      while (!mbar_try(&c.S->bfull, bpar) && gtimer() - t0 < 2 * (uint64_t)P->timeout_ns) {
      }
    }
    const int first = i0 + ((cw - (i0 - G.a)) % NCW + NCW) % NCW;
    for (int i = first; ok && i < i1; i += NCW) {
      const int sl = ((i - G.a) / NCW) % DNS;
      if (!wait_bar(c, &c.S->dfull[cw][sl], (dpar >> sl) & 1u, layer, phase)) { ok = false; break; }
      dpar ^= 1u << sl;
      float acc[MSK_NT_DENSE][4];
#pragma unroll
      for (int nt = 0; nt < MSK_NT_DENSE; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
      const uint32_t slot = ring + DB_BYTES + (uint32_t)(cw * DNS + sl) * DSLOT;
      /* all n-tiles present: a copy without the per-tile guard, which the
       * compiler can schedule across tiles */
      if (ntl == MSK_NT_DENSE)
        dgemm<MSK_NT_DENSE, true>(slot, slot + 16 * G.cpitch, G.cpitch, G.spitch, ring, G.bpitch, G.KS, ntl, acc);
      else
        dgemm<MSK_NT_DENSE, false>(slot, slot + 16 * G.cpitch, G.cpitch, G.spitch, ring, G.bpitch, G.KS, ntl, acc);
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.S->dempty[cw][sl]);
      int map, lrow;
      float gs;
      const int row0 = (i % G.MT) * 16;
      dense_mat(P, Ly, QKV, row0, &map, &lrow, &gs);
      float* dst = out + (size_t)s * T * G.rows;
#pragma unroll
      for (int nt = 0; nt < MSK_NT_DENSE; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = nt * 8 + 2 * cq + (e & 1), row = row0 + g + 8 * (e >> 1);
          if (nt < ntl && col < T) dst[(size_t)col * G.rows + row] = acc[nt][e] * gs;
        }
      }
    }
    i0 = i1;
  }
  if (!ok) c.S->abort = 1;
  const bool aborting = named_sync_or(BAR_CONS, NCT, c.S->abort != 0);
  if (ctid == 0) {
    __threadfence_block();
    c.S->dense_done = 2 * layer + (QKV ? 1 : 2);
  }
  return !aborting;
}

/* ---- consumer: attention stages ------------------------------------------------------ */
MSK_DEV uint32_t swz(uint32_t off, int hd) {
  return hd == 128 ? (off ^ (((off >> 7) & 7u) << 4)) : (off ^ (((off >> 7) & 3u) << 4));
}

template <int HD, int MT>
struct AttState {
  float o[MT][HD / 8][4];
  float l[MT][2];
  int lo[MT][2], hi[MT][2]; /* key window of rows g and g+8 of each m-tile (empty if lo > hi) */
  int lo_max, hi_min;       /* every valid row sees [lo_max, hi_min] */
};

/* Q of the segment's rows as A fragments in the scratch, fragment order:
 * qf[m-tile][step][lane] = 16 bytes (a0a1, a2a3, a4a5, a6a7).  Warps with
 * ki == 0 fill their MT m-tiles; every consumer warp passes the barrier. */
template <int HD, int MT>
MSK_DEV void att_begin(const Ctx& c, AttState<HD, MT>& A, int pair, int mg, bool writer, bool sliding) {
  const MskParams* P = c.P;
  const int lane = threadIdx.x & 31, g = lane >> 2, cq = lane & 3;
  const int b = pair / P->hkv, kvh = pair % P->hkv;
  const int R = c.st.Tq * P->G;
  A.lo_max = -1;
  A.hi_min = 0x7FFFFFFF;
#pragma unroll
  for (int m = 0; m < MT; ++m) {
#pragma unroll
    for (int j = 0; j < HD / 8; ++j) A.o[m][j][0] = A.o[m][j][1] = A.o[m][j][2] = A.o[m][j][3] = 0.f;
    A.l[m][0] = A.l[m][1] = 0.f;
    const int mi = mg * MT + m;
    uint32_t* qfw = reinterpret_cast<uint32_t*>(reinterpret_cast<uint4*>(c.scr) + (size_t)mi * (HD / 16) * 32);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int rho = mi * 16 + g + 8 * half;
      int lo = 1, hi = 0;
      uint32_t qw[HD / 8];
#pragma unroll
      for (int i = 0; i < HD / 8; ++i) qw[i] = 0;
      if (rho < R) {
        const int ti = rho / P->G, h = kvh * P->G + rho % P->G;
        const int t = b * c.st.Tq + ti;
        hi = c.S->pos0[b] + ti;
        lo = sliding ? max(0, hi - P->W + 1) : 0;
        if (writer) {
          const uint16_t* qrow = P->qs + (size_t)t * P->qd + h * HD + cq * (HD / 4);
#pragma unroll
          for (int i = 0; i < HD / 32; ++i) {
            uint4 v = ldg128(qrow + 8 * i);
            qw[4 * i] = v.x; qw[4 * i + 1] = v.y; qw[4 * i + 2] = v.z; qw[4 * i + 3] = v.w;
          }
        }
      }
      A.lo[m][half] = lo;
      A.hi[m][half] = hi;
      if (writer) {
        /* step s uses q[c*HD/4 + 4s .. +4): words 2s (a0a1 / a2a3) and 2s+1 (a4a5 / a6a7) */
#pragma unroll
        for (int s = 0; s < HD / 16; ++s) {
          qfw[(s * 32 + lane) * 4 + half] = qw[2 * s];
          qfw[(s * 32 + lane) * 4 + 2 + half] = qw[2 * s + 1];
        }
      }
    }
  }
  /* the window every valid row of the pair shares (rows differ only in the
   * draft-block position) */
  {
    const int T0 = c.S->pos0[b], T1 = T0 + c.st.Tq - 1;
    A.hi_min = T0;
    A.lo_max = sliding ? max(0, T1 - P->W + 1) : 0;
  }
  named_sync(BAR_CONS, NCT);
}

template <int HD, int MT>
MSK_DEV void att_stage(const Ctx& c, AttState<HD, MT>& A, const uint8_t* stg, int k0, int nkeys, int ks, int mg,
                       int ki, float scale_log2, float bound_log2) {
  const int lane = threadIdx.x & 31, g = lane >> 2, cq = lane & 3;
  const uint32_t kbase = smem_u32(stg);
  const int C = (HD == 128) ? 128 : 256;
  const uint32_t vbase = kbase + C * HD;
  const uint32_t qfb = smem_u32(c.scr) + (uint32_t)(mg * MT * (HD / 16) * 32 + lane) * 16;
  const float two120 = 1.329227995784916e36f; /* 2^120 */
  for (int kb = ki; kb * 16 < nkeys; kb += ks) {
    const int kp0 = k0 + kb * 16;
    const bool full = kb * 16 + 16 <= nkeys && kp0 >= A.lo_max && kp0 + 15 <= A.hi_min;
    uint32_t kw[2][HD / 16];
#pragma unroll
    for (int n2 = 0; n2 < 2; ++n2) {
      const uint32_t row = kb * 16 + n2 * 8 + g;
#pragma unroll
      for (int i = 0; i < HD / 64; ++i) {
        uint4 v = lds128(kbase + swz(row * HD + cq * (HD / 4) + 16 * i, HD));
        kw[n2][4 * i] = v.x; kw[n2][4 * i + 1] = v.y; kw[n2][4 * i + 2] = v.z; kw[n2][4 * i + 3] = v.w;
      }
    }
    float sacc[MT][2][4];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
      for (int n2 = 0; n2 < 2; ++n2) sacc[m][n2][0] = sacc[m][n2][1] = sacc[m][n2][2] = sacc[m][n2][3] = 0.f;
#pragma unroll
    for (int s = 0; s < HD / 16; ++s) {
      uint32_t kf0[2], kf1[2];
      e4m3x4_to_f16x2x2(kw[0][s], kf0);
      e4m3x4_to_f16x2x2(kw[1][s], kf1);
      const uint32_t k00 = kf0[0], k01 = kf0[1], k10 = kf1[0], k11 = kf1[1];
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const uint4 qv = lds128(qfb + (uint32_t)(m * (HD / 16) + s) * 32 * 16);
        const uint32_t qa[4] = {qv.x, qv.y, qv.z, qv.w};
        mma_f16(sacc[m][0], qa, k00, k01);
        mma_f16(sacc[m][1], qa, k10, k11);
      }
    }
    /* p = exp(s - M) under the key windows; l in fp32, P as bf16 scaled by
     * 2^120 to match V's 2^-120 */
    uint32_t pa[MT][4];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
#pragma unroll
      for (int n2 = 0; n2 < 2; ++n2) {
        float p[4];
        if (full) { /* the whole block inside every row's window: no per-score test */
#pragma unroll
          for (int e = 0; e < 4; ++e) p[e] = fast_exp2(sacc[m][n2][e] * scale_log2 - bound_log2);
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int kl = kb * 16 + n2 * 8 + 2 * cq + (e & 1);
            const int kp = k0 + kl, hf = e >> 1;
            const bool ok = kl < nkeys && kp >= A.lo[m][hf] && kp <= A.hi[m][hf];
            p[e] = ok ? fast_exp2(sacc[m][n2][e] * scale_log2 - bound_log2) : 0.f;
          }
        }
        A.l[m][0] += p[0] + p[1];
        A.l[m][1] += p[2] + p[3];
        pa[m][2 * n2] = f32x2_to_bf16x2(p[0] * two120, p[1] * two120);
        pa[m][2 * n2 + 1] = f32x2_to_bf16x2(p[2] * two120, p[3] * two120);
      }
    }
    /* V: lane (g, c) holds columns g*HD/8 .. +HD/8 of keys 2c, 2c+1, 2c+8,
     * 2c+9 (its mma k-slots: keys 2c, 2c+1 from S tile 0, 8+2c, 9+2c from S
     * tile 1); read 8 columns at a time; each converted fragment feeds MT
     * m-tiles */
    const uint32_t rA = kb * 16 + 2 * cq;
#pragma unroll
    for (int hv = 0; hv < HD / 64; ++hv) {
      uint32_t vw[4][2];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t row = rA + (kk & 1) + 8 * (kk >> 1);
        uint2 v = lds64(vbase + swz(row * HD + g * (HD / 8) + 8 * hv, HD));
        vw[kk][0] = v.x; vw[kk][1] = v.y;
      }
#pragma unroll
      for (int wi = 0; wi < 2; ++wi) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t sel = (uint32_t)(j | (j << 4) | ((j + 4) << 8) | ((j + 4) << 12));
          const uint32_t b0 = e4m3pair_to_bf16x2_scaled(vw[0][wi], vw[1][wi], sel);
          const uint32_t b1 = e4m3pair_to_bf16x2_scaled(vw[2][wi], vw[3][wi], sel);
#pragma unroll
          for (int m = 0; m < MT; ++m) mma_bf16(A.o[m][(hv * 2 + wi) * 4 + j], pa[m], b0, b1);
        }
      }
    }
  }
}

/* Reduce the key-split warps of each m-tile group (fixed order, one m-tile
 * at a time through the scratch) and write the segment's partial
 * (o[rho][0..hd), l at [hd]) to slot `slot`. */
template <int HD, int MT>
MSK_DEV void att_end(const Ctx& c, AttState<HD, MT>& A, int slot, int ngroups, int ks) {
  const MskParams* P = c.P;
  const int cw = (threadIdx.x >> 5) - CONS_WARP0, lane = threadIdx.x & 31, g = lane >> 2, cq = lane & 3;
  const bool active = cw < ngroups * ks;
  const int mg = active ? cw / ks : 0, ki = active ? cw % ks : 0;
  /* quad-reduce the row sums first (each lane summed its own key columns) */
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      A.l[m][hf] += __shfl_xor_sync(0xffffffffu, A.l[m][hf], 1);
      A.l[m][hf] += __shfl_xor_sync(0xffffffffu, A.l[m][hf], 2);
    }
  named_sync(BAR_CONS, NCT); /* every warp is done with the Q fragments */
  float* buf = c.scr;
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    for (int step = ks / 2; step >= 1; step >>= 1) {
      if (active && ki >= step && ki < 2 * step) {
        const int bi = mg * step + (ki - step);
        float* dst = buf + (size_t)bi * (HD / 8) * 128;
#pragma unroll
        for (int j = 0; j < HD / 8; ++j)
          *reinterpret_cast<float4*>(&dst[(j * 32 + lane) * 4]) =
              make_float4(A.o[m][j][0], A.o[m][j][1], A.o[m][j][2], A.o[m][j][3]);
        c.S->lbuf[bi][lane][0] = A.l[m][0];
        c.S->lbuf[bi][lane][1] = A.l[m][1];
      }
      named_sync(BAR_CONS, NCT);
      if (active && ki < step) {
        const int bi = mg * step + ki;
        const float* src = buf + (size_t)bi * (HD / 8) * 128;
#pragma unroll
        for (int j = 0; j < HD / 8; ++j) {
          float4 v = *reinterpret_cast<const float4*>(&src[(j * 32 + lane) * 4]);
          A.o[m][j][0] += v.x; A.o[m][j][1] += v.y; A.o[m][j][2] += v.z; A.o[m][j][3] += v.w;
        }
        A.l[m][0] += c.S->lbuf[bi][lane][0];
        A.l[m][1] += c.S->lbuf[bi][lane][1];
      }
      named_sync(BAR_CONS, NCT);
    }
  }
  if (active && ki == 0) {
    const int R = c.st.Tq * P->G;
    float* base = P->part + (size_t)slot * P->part_stride;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int rho = (mg * MT + m) * 16 + g + 8 * half;
        if (rho >= R) continue;
        float* row = base + (size_t)rho * (HD + 4);
#pragma unroll
        for (int j = 0; j < HD / 8; ++j) {
          /* C-fragment column 2c+e of n-tile j is head dim (2c+e)*HD/8 + j */
          row[(2 * cq) * (HD / 8) + j] = A.o[m][j][2 * half];
          row[(2 * cq + 1) * (HD / 8) + j] = A.o[m][j][2 * half + 1];
        }
        if (cq == 0) row[HD] = A.l[m][half];
      }
    }
  }
}

template <int HD, int MT>
MSK_DEV bool attention_phase_mt(Cons& q, int layer) {
  Ctx& c = *q.c;
  const MskParams* P = c.P;
  const MskLayer& Ly = P->layers[layer];
  att_geo_shared(c, layer);
  const AttGeo& g = c.S->ag;
  const int R = c.st.Tq * P->G;
  const int mt = (R + 15) / 16;
  const int ngroups = (mt + MT - 1) / MT; /* 1 or 2 */
  const int ks = NCW / ngroups;
  const int cw = (threadIdx.x >> 5) - CONS_WARP0;
  const bool active = cw < ngroups * ks;
  const int mg = active ? cw / ks : 0, ki = active ? cw % ks : 0;
  const int C = att_keys_per_stage(HD);
  const float scale_log2 = P->scale_log2, bound_log2 = Ly.bound_log2;
  if (c.cta < g.nparts) {
    const int64_t A0 = g.N * c.cta / g.nparts, B0 = g.N * (c.cta + 1) / g.nparts;
    for (int p = 0; p < g.npairs; ++p) {
      const int64_t a = max(A0, g.off[p]), b = min(B0, g.off[p + 1]);
      if (a >= b) continue;
      const int k0 = (int)(g.lo[p] + (a - g.off[p])), k1 = (int)(g.lo[p] + (b - g.off[p]));
      AttState<HD, MT> A;
      att_begin<HD, MT>(c, A, p, mg, active && ki == 0, Ly.sliding != 0);
      for (int x = k0; x < k1; x += C) {
        uint32_t sl;
        const uint8_t* stg = cons_wait(q, layer, PH_ATT, &sl);
        if (stg) {
          if (active) att_stage<HD, MT>(c, A, stg, x, min(C, k1 - x), ks, mg, ki, scale_log2, bound_log2);
          cons_release(q, sl);
        }
      }
      att_end<HD, MT>(c, A, c.cta + p, ngroups, ks);
    }
  }
  /* one answer for every warp, even if the abort word changes meanwhile */
  return !named_sync_or(BAR_CONS, NCT, c.S->abort != 0);
}

/* one warp owns up to two 16-row tiles of a pair (their keys are converted
 * once); more rows split the warps into two groups */
template <int HD>
MSK_DEV bool attention_phase(Cons& q, int layer) {
  const int R = q.c->st.Tq * q.c->P->G;
  return R <= 16 ? attention_phase_mt<HD, 1>(q, layer) : attention_phase_mt<HD, 2>(q, layer);
}

/* One (token t, head hh) item of the projections' output, by one warp
 * (heads: q heads, then k, then v): its K slices' split-K partials added
 * in slice order into v[0..per), per = hd / 32 values per lane; q and k
 * heads then RMS-normalised with their gains (QK-norm). */
MSK_DEV void qkv_head(const Ctx& c, const MskLayer& Ly, int t, int hh, float* v) {
  const MskParams* P = c.P;
  const int lane = threadIdx.x & 31;
  const int hd = P->hd, nqkv = P->qd + 2 * P->kvd, per = hd / 32;
  const int S = P->d <= DKS_MAX ? 1 : P->d / DKS_MAX;
  v[0] = v[1] = v[2] = v[3] = 0.f;
  /* every slice's load issued before the first add (S <= 8 for d <= 4096) */
  float4 q[MAX_KS];
#pragma unroll
  for (int sl = 0; sl < MAX_KS; ++sl) {
    const float* raw = P->qkv + ((size_t)sl * c.st.T + t) * nqkv + hh * hd + lane * per;
    q[sl] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (sl < S) {
      if (per == 4) {
        q[sl] = *reinterpret_cast<const float4*>(raw);
      } else {
        const float2 h2 = *reinterpret_cast<const float2*>(raw);
        q[sl].x = h2.x; q[sl].y = h2.y;
      }
    }
  }
#pragma unroll
  for (int sl = 0; sl < MAX_KS; ++sl)
    if (sl < S) { v[0] += q[sl].x; v[1] += q[sl].y; v[2] += q[sl].z; v[3] += q[sl].w; }
  if (hh < P->hq + P->hkv) {
    float ss = 0.f;
    for (int i = 0; i < per; ++i) ss += v[i] * v[i];
    ss = warp_sum(ss);
    const float r = 1.0f / sqrtf(ss / hd + P->eps);
    const float* gain = (hh < P->hq ? Ly.g_q : Ly.g_k) + lane * per;
    for (int i = 0; i < per; ++i) v[i] = v[i] * r * gain[i];
  }
}

/* This step's key or value of (token t, kv head kvh) as fp8 e4m3 into the
 * cache (and, if captured, its fp32 value before the encode). */
MSK_DEV void kv_store(const Ctx& c, int layer, int t, int kvh, bool isv, const float* v) {
  const MskParams* P = c.P;
  const int lane = threadIdx.x & 31, hd = P->hd, per = hd / 32;
  const int b = t / c.st.Tq, ti = t % c.st.Tq;
  float* pre = isv ? P->dbg_vpre : P->dbg_kpre;
  if (pre) {
    pre += ((size_t)layer * c.st.T + t) * P->kvd + kvh * hd + lane * per;
    for (int i = 0; i < per; ++i) pre[i] = v[i];
  }
  const int64_t pos = c.S->pos0[b] + ti;
  int64_t row = (((int64_t)layer * c.st.kv_seqs + b) * P->hkv + kvh) * c.st.kv_cap + pos;
  if (isv) row += c.st.kv_half_rows;
  uint8_t* dst = c.st.kv_base + row * hd + lane * per;
  if (per == 4) {
    uint32_t lo = f32x2_to_e4m3x2(v[0], v[1]), hi = f32x2_to_e4m3x2(v[2], v[3]);
    *reinterpret_cast<uint32_t*>(dst) = lo | (hi << 16);
  } else {
    *reinterpret_cast<uint16_t*>(dst) = (uint16_t)f32x2_to_e4m3x2(v[0], v[1]);
  }
}

/* ---- attention on the 5th-generation tensor cores (head dim 128) ------------------------ */
/*
 * Per (sequence, kv head) segment of keys, with R = Tq * G query rows padded
 * to RP in {16, 32, 64}:
 *   S^T[128 keys][3 RP] = K Q^T: tcgen05.mma kind::f8f6f4, A = the stage's
 *     K exactly as the tensor copy lands it (e4m3, 128 keys x 128 bytes,
 *     128-byte swizzle: the K-major canonical layout), B = Q as three e4m3
 *     terms per value (q f = t0 + t1 + t2 with a power-of-two row factor f;
 *     about 12 significant bits, as f16) stacked along N, so one MMA per
 *     32-wide K step covers all three: 4 MMAs of N = 3 RP per stage (an MMA
 *     costs about the same up to N = 128, and K is read once); the consumer
 *     adds a row's three term columns.
 *   p = exp(s - M) under the key windows, on CUDA cores: each consumer
 *     lane holds one key (TMEM lane), its rows' scores; l += p per lane.
 *     P^T goes to shared memory as two e4m3 terms per value under one ue8m0
 *     scale per (row, 32-key block): the block's largest p sets the scale
 *     so that p / scale lies below 256; t0 = e4m3(p / scale) and t1 =
 *     e4m3(16 (p / scale - t0)) with scale / 16 (about 9 significant bits,
 *     as bf16; p spans up to 2^-116 .. 1, which one fixed e4m3 scale cannot).
 *   O^T[128 hd][RP] += V^T P^T: kind::mxf8f6f4 block32, A = the stage's V
 *     exactly as the tensor copy lands it (e4m3, key rows of 128 bytes,
 *     128-byte swizzle), read MN-major (head-dim contiguous); B = a P^T term,
 *     MN-major without swizzle (core matrices [8 keys][16 rows]); V's
 *     scales all 1.  8 MMAs of K = 32 keys per stage (2 terms x 4 key
 *     blocks), accumulated in TMEM over the segment.
 * The QK issuer runs one stage ahead: the QK products of stage j+1 are in
 * flight while the consumer warps turn the scores of stage j into
 * probabilities.  Parties and barriers per stage j (b = j mod 2, b3 = j mod 3):
 *   producer -> kfull -> issuer: QK(j) -> s_ready[b] (consumers) and kempty
 *   (K refill) -> consumers: read S^T -> s_free[b] -> issuer (QK(j+2));
 *   consumers: write P^T terms and their scales -> p_ready[b3], producer ->
 *   vfull -> issuer: scales into TMEM, PV(j) -> vempty (V refill) and
 *   pv_done[b3] (P^T buffer reuse; the segment's output read).  The
 *   consumers never touch K or V.  K and V have rings of their own because
 *   K is released two stages before V: with one 32 KB stage per slot, too
 *   few bytes were left in flight to cover the copy latency.
 * Shared memory (from the ring base): NK K slots and NV V slots of 16 KB,
 * then three P^T buffers (stage mod 3) [2 terms][16 key groups][RP / 16 row
 * groups][8 keys][16 rows] e4m3, the Q terms [3][RP rows][128 B], then the
 * scale-factor atoms [3][2 terms][32 rows][16 B] (row n: atom row n mod 32,
 * word n / 32, byte = key block) and 512 bytes of ue8m0 1.0 for V.  TMEM:
 * O^T at column 0, S^T buffers at 64 and 256, V scales at 448, P^T scales
 * at 452 + 8 b3 + 4 term.
 */
/* One issuing warp's part of one layer's attention (lane 0 issues): role 0
 * issues every stage's QK products, role 1 its PV products, so the two
 * streams of MMAs are issued by two threads at once (a single thread issues
 * a tcgen05.mma about every 70 cycles, two together every 45).  ait / aseg:
 * stages and segments this role issued so far (the consumers count the
 * same). */
MSK_DEV bool issuer_att(Ctx& c, int layer, int role, uint32_t& ait, uint32_t& aseg) {
  const MskParams* P = c.P;
  const int lane = threadIdx.x & 31;
  if (!pwait_flag(c, &c.S->ag_ready, layer + 1, layer, PH_ATT)) return false;
  const AttGeo& g = c.S->ag;
  const int RP = atc_rp(c.st.Tq * P->G);
  const uint32_t NK = (uint32_t)atc_nk(RP), NV = (uint32_t)atc_nv(RP);
  const uint32_t tb = c.S->tmem_base, ring = smem_u32(c.ring), vring = ring + atc_v_off(RP);
  const uint32_t qoff = ring + atc_q_off(RP), ptoff = ring + atc_pt_off(RP), sfoff = ring + atc_sf_off(RP);
  const uint32_t id_qk = atc_idesc_qk(RP);
  const uint64_t qb = umma_desc(qoff, 16, 1024, 2);
  bool ok = true, sfa = false;
  for_each_att_stage(c, g, [&](int, int, int64_t, int, bool first, bool last) {
    const uint32_t j = ait;
    if (role == 0) {
      if (first && !pwait_bar(c, &c.S->q_ready, aseg & 1u, layer, PH_ATT)) { ok = false; return false; }
      if (!pwait_bar(c, &c.S->kfull[j % NK], (j / NK) & 1u, layer, PH_ATT)) { ok = false; return false; }
      if (j >= 2 && !pwait_bar(c, &c.S->s_free[j & 1u], ((j >> 1) - 1u) & 1u, layer, PH_ATT)) { ok = false; return false; }
      if (lane == 0) {
        tc_fence_after();
        const uint32_t d = tb + ATC_TM_S + ATC_TM_SSTRIDE * (j & 1u);
        const uint64_t ka = umma_desc(ring + (j % NK) * ATC_HALF, 16, 1024, 2);
#pragma unroll
        for (int s = 0; s < 4; ++s) tc_mma_f8(d, ka + (uint64_t)(2 * s), qb + (uint64_t)(2 * s), id_qk, s > 0 ? 1u : 0u);
        tc_commit(&c.S->s_ready[j & 1u]);
        tc_commit(&c.S->kempty[j % NK]);
      }
      __syncwarp();
    } else {
      if (!pwait_bar(c, &c.S->p_ready[j % 3u], (j / 3u) & 1u, layer, PH_ATT)) { ok = false; return false; }
      if (!pwait_bar(c, &c.S->vfull[j % NV], (j / NV) & 1u, layer, PH_ATT)) { ok = false; return false; }
      if (first && aseg > 0 && !pwait_bar(c, &c.S->o_free, (aseg - 1u) & 1u, layer, PH_ATT)) { ok = false; return false; }
      if (lane == 0) {
        tc_fence_after();
        const uint32_t b3 = j % 3u, pt = ptoff + b3 * (uint32_t)RP * 256u, sfb = tb + ATC_TM_SFB + 8u * b3;
        /* the scale factors into TMEM (V's once per layer), in issue order
         * before the MMAs that read them */
        if (!sfa) tc_cp_sf(tb + ATC_TM_SFA, umma_desc(sfoff + 3072u, 16, 128, 0));
        /* A: V, one 128-byte atom along the head dim, 8-key groups 1 KB apart */
        const uint64_t va = umma_desc(vring + (j % NV) * ATC_HALF, 8192, 1024, 2);
        if (RP <= 32) {
          /* B: both terms stacked along N (2 RP rows), key groups 2 RP * 8
           * bytes apart, 16-row groups 128 bytes; one scale atom */
          tc_cp_sf(sfb, umma_desc(sfoff + b3 * 1024u, 16, 128, 0));
          const uint64_t pbs = umma_desc(pt, 16u * (uint32_t)RP, 128, 0);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_mx8(tb + ATC_TM_O, va + (uint64_t)(256 * kk), pbs + (uint64_t)(4 * RP * kk),
                       atc_idesc_pv(2 * RP, (uint32_t)kk), (first && kk == 0) ? 0u : 1u, tb + ATC_TM_SFA, sfb);
        } else {
          /* B: term t, key groups RP * 8 bytes apart, 16-row groups 128
           * bytes; a scale atom per term; both terms into the same columns */
          tc_cp_sf(sfb, umma_desc(sfoff + b3 * 1024u, 16, 128, 0));
          tc_cp_sf(sfb + 4u, umma_desc(sfoff + b3 * 1024u + 512u, 16, 128, 0));
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const uint64_t pbt = umma_desc(pt + (uint32_t)(t * RP * 128), (uint32_t)RP * 8u, 128, 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc_mma_mx8(tb + ATC_TM_O, va + (uint64_t)(256 * kk), pbt + (uint64_t)(2 * RP * kk),
                         atc_idesc_pv(RP, (uint32_t)kk), (first && t == 0 && kk == 0) ? 0u : 1u, tb + ATC_TM_SFA,
                         sfb + 4u * (uint32_t)t);
          }
        }
        tc_commit(&c.S->vempty[j % NV]);
        tc_commit(&c.S->pv_done[b3]);
      }
      sfa = true;
      __syncwarp();
    }
    ait++;
    if (last) aseg++;
    return true;
  });
  return ok;
}

/* The producer's part: this CTA's K and V boxes (16 KB each) into their
 * rings, K of stage j before V of stage j - 1, so that K, which is needed
 * first, runs a stage ahead.  p.avt counts the V boxes issued. */
MSK_DEV bool prod_att_tc(Prod& p, int layer, uint32_t& ait) {
  Ctx& c = *p.c;
  const MskParams* P = c.P;
  const AttGeo& g = c.S->agp;
  const int RP = atc_rp(c.st.Tq * P->G);
  const uint32_t NK = (uint32_t)atc_nk(RP), NV = (uint32_t)atc_nv(RP);
  uint8_t* vring = c.ring + atc_v_off(RP);
  const int lane = threadIdx.x & 31;
  bool ok = true;
  int64_t vrow = -1; /* the V row of the previous stage, still to issue */
  auto issue_v = [&](int64_t row) -> bool {
    const uint32_t j = p.avt, s = j % NV;
    if (j >= NV && !pwait_bar(c, &c.S->vempty[s], ((j / NV) - 1u) & 1u, layer, PH_ATT)) return false;
    if (lane == 0) {
      mbar_arrive_tx(&c.S->vfull[s], ATC_HALF);
      tma_2d_g2s(vring + (size_t)s * ATC_HALF, c.kvmap, 0, (int32_t)(row + c.st.kv_half_rows), &c.S->vfull[s]);
    }
    __syncwarp();
    p.avt++;
    return true;
  };
  for_each_att_stage(c, g, [&](int pr, int, int64_t k0, int, bool, bool) {
    const int b = pr / P->hkv, h = pr % P->hkv;
    if (k0 + 128 > c.S->pos0[b]) {
      if (!pwait_flag(c, &c.S->kv_ready, layer + 1, layer, PH_ATT)) { ok = false; return false; }
      fence_proxy_async_global();
    }
    const uint32_t j = ait, s = j % NK;
    if (j >= NK && !pwait_bar(c, &c.S->kempty[s], ((j / NK) - 1u) & 1u, layer, PH_ATT)) { ok = false; return false; }
    const int64_t row = (((int64_t)layer * c.st.kv_seqs + b) * P->hkv + h) * c.st.kv_cap + k0;
    if (lane == 0) {
      mbar_arrive_tx(&c.S->kfull[s], ATC_HALF);
      tma_2d_g2s(c.ring + (size_t)s * ATC_HALF, c.kvmap, 0, (int32_t)row, &c.S->kfull[s]);
    }
    __syncwarp();
    ait++;
    if (vrow >= 0 && !issue_v(vrow)) { ok = false; return false; }
    vrow = row;
    return true;
  });
  if (ok && vrow >= 0 && !issue_v(vrow)) ok = false;
  return ok;
}

/* wait (bounded) until every K and V slot issued so far is free again */
MSK_DEV bool prod_att_tc_drain(Prod& p, int layer, uint32_t ait) {
  Ctx& c = *p.c;
  const int RP = atc_rp(c.st.Tq * c.P->G);
  const uint32_t NK = (uint32_t)atc_nk(RP), NV = (uint32_t)atc_nv(RP);
  for (uint32_t i = ait - (ait < NK ? ait : NK); i < ait; ++i)
    if (!pwait_bar(c, &c.S->kempty[i % NK], (i / NK) & 1u, layer, PH_WO)) return false;
  for (uint32_t i = p.avt - (p.avt < NV ? p.avt : NV); i < p.avt; ++i)
    if (!pwait_bar(c, &c.S->vempty[i % NV], (i / NV) & 1u, layer, PH_WO)) return false;
  return true;
}

/* Q of the pair's R rows (QK-normed, f16) as three e4m3 terms (B operand
 * rows t RP + rho, 128-byte swizzle) and each row's softmax factor; one
 * warp per row. */
MSK_DEV void atc_q_terms(const Ctx& c, int pair, int RP, uint32_t qoff) {
  const MskParams* P = c.P;
  const int cw = (threadIdx.x >> 5) - CONS_WARP0, lane = threadIdx.x & 31;
  const int b = pair / P->hkv, kvh = pair % P->hkv;
  const int R = c.st.Tq * P->G;
  /* this warp's rows (at most 64 / 8): every load issued first */
  uint2 wq[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int rho = cw + u * NCW;
    wq[u] = make_uint2(0u, 0u);
    if (rho < R && rho < RP) {
      const int t = b * c.st.Tq + rho / P->G, h = kvh * P->G + rho % P->G;
      wq[u] = *reinterpret_cast<const uint2*>(P->qs + (size_t)t * P->qd + h * 128 + lane * 4);
    }
  }
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int rho = cw + u * NCW;
    if (rho >= RP) break;
    float x[4] = {f16lo_f32(wq[u].x), f16hi_f32(wq[u].x), f16lo_f32(wq[u].y), f16hi_f32(wq[u].y)};
    float mx = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    /* f = 2^e with mx f in (224, 448] */
    int e = 0;
    if (mx > 0.f) e = max(-100, min(100, (int)floorf(log2f(448.0f / mx))));
    const float f = __int_as_float((127 + e) << 23);
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] *= f;
    const uint32_t chunk = (uint32_t)(lane >> 2), within = 4u * (uint32_t)(lane & 3);
#pragma unroll
    for (int t = 0; t < 3; ++t) {
      const uint32_t c01 = f32x2_to_e4m3x2(x[0], x[1]), c23 = f32x2_to_e4m3x2(x[2], x[3]);
      x[0] -= e4m3_to_f32(c01);
      x[1] -= e4m3_to_f32(c01 >> 8);
      x[2] -= e4m3_to_f32(c23);
      x[3] -= e4m3_to_f32(c23 >> 8);
      const uint32_t n = (uint32_t)(t * RP + rho);
      sts32(qoff + n * 128u + ((chunk ^ (n & 7u)) << 4) + within, c01 | (c23 << 16));
    }
    if (lane == 0) c.S->qfac[rho] = rho < R ? P->scale_log2 / f : 0.f;
  }
}

template <int RP>
MSK_DEV bool attention_phase_tc(Ctx& c, int layer, uint32_t& ait, uint32_t& aseg) {
  const MskParams* P = c.P;
  const MskLayer& Ly = P->layers[layer];
  constexpr int NR = RP / 2; /* query rows per consumer warp */
  att_geo_shared(c, layer);
  if (threadIdx.x == CONS0) {
    __threadfence_block();
    c.S->ag_ready = layer + 1;
  }
  const AttGeo& g = c.S->ag;
  const int cw = (threadIdx.x >> 5) - CONS_WARP0, lane = threadIdx.x & 31, ctid = threadIdx.x - CONS0;
  const int qd = cw & 3, hh = cw >> 2; /* TMEM lane quadrant (keys 32 qd ..), row half */
  const int R = c.st.Tq * P->G;
  const uint32_t ring = smem_u32(c.ring), tb = c.S->tmem_base;
  const uint32_t ptoff = ring + atc_pt_off(RP), qoff = ring + atc_q_off(RP), sfoff = ring + atc_sf_off(RP);
  const float bound_log2 = Ly.bound_log2;
  const bool sliding = Ly.sliding != 0;
  float* lred = reinterpret_cast<float*>(c.S->lbuf); /* [4 quadrants][64 rows] */
  bool ok = true;
  /* V's block scales, ue8m0 1.0 (published with the first segment's Q terms) */
  if (ctid < 128) sts32(sfoff + 3072u + 4u * (uint32_t)ctid, 0x7F7F7F7Fu);
  if (c.cta < g.nparts) {
    const int64_t A0 = g.N * c.cta / g.nparts, B0 = g.N * (c.cta + 1) / g.nparts;
    for (int pr = 0; pr < g.npairs; ++pr) {
      const int64_t a = max(A0, g.off[pr]), bb = min(B0, g.off[pr + 1]);
      if (a >= bb) continue;
      const int k0 = (int)(g.lo[pr] + (a - g.off[pr])), k1 = (int)(g.lo[pr] + (bb - g.off[pr]));
      const int b = pr / P->hkv;
      const int T0 = c.S->pos0[b];
      /* the window every valid row shares: [lo_max, hi_min] */
      const int hi_min = T0, lo_max = sliding ? max(0, T0 + c.st.Tq - 1 - P->W + 1) : 0;
      if (ok) atc_q_terms(c, pr, RP, qoff);
      fence_proxy_async_shared();
      named_sync(BAR_CONS, NCT);
      if (ctid == 0) mbar_arrive(&c.S->q_ready);
      float l[NR], qf[NR];
#pragma unroll
      for (int i = 0; i < NR; ++i) {
        l[i] = 0.f;
        qf[i] = c.S->qfac[hh * NR + i]; /* softmax scale / the row's Q-term factor */
      }
      const int nvalid = min(NR, max(0, R - hh * NR)); /* this warp's rows below R */
      for (int x = k0; x < k1; x += 128) {
        const uint32_t j = ait, bf = j & 1u, pb = j % 3u;
        const int nkeys = min(128, k1 - x);
        /* P^T buffer pb and its scale atoms: free once the products of stage j - 3 completed */
        if (ok && j >= 3 && !wait_bar(c, &c.S->pv_done[pb], ((j / 3u) - 1u) & 1u, layer, PH_ATT)) ok = false;
        if (ok && !wait_bar(c, &c.S->s_ready[bf], (j >> 1) & 1u, layer, PH_ATT)) ok = false;
        ok = __all_sync(0xffffffffu, ok) != 0; /* warp-uniform: the TMEM loads below are warp-collective */
        tc_fence_after();
        /* this warp's scores: its quadrant's 32 keys, its NR rows, the sum
         * of each row's three term columns */
        float sr[NR];
        if (ok) {
          const uint32_t ta = tb + ATC_TM_S + ATC_TM_SSTRIDE * bf + (uint32_t)(hh * NR) + ((uint32_t)(qd * 32) << 16);
          constexpr int NB = NR < 16 ? NR : 16;
#pragma unroll
          for (int i = 0; i < NR; i += NB) {
            uint32_t t0[NB], t1[NB], t2[NB];
            if constexpr (NB == 16) {
              tc_ld16(ta + (uint32_t)i, t0);
              tc_ld16(ta + (uint32_t)(RP + i), t1);
              tc_ld16(ta + (uint32_t)(2 * RP + i), t2);
            } else {
              tc_ld8(ta + (uint32_t)i, t0);
              tc_ld8(ta + (uint32_t)(RP + i), t1);
              tc_ld8(ta + (uint32_t)(2 * RP + i), t2);
            }
            tc_wait_ld();
#pragma unroll
            for (int e = 0; e < NB; ++e) sr[i + e] = __uint_as_float(t0[e]) + __uint_as_float(t1[e]) + __uint_as_float(t2[e]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.S->s_free[bf]);
        if (ok) {
          const int key = qd * 32 + lane, kp = x + key;
          const bool full = nkeys == 128 && x >= lo_max && x + 127 <= hi_min;
          float pv[NR];
          if (full) {
#pragma unroll
            for (int i = 0; i < NR; ++i) pv[i] = i < nvalid ? fast_exp2(fmaf(sr[i], qf[i], -bound_log2)) : 0.f;
          } else {
            const int G = P->G, W = P->W;
#pragma unroll
            for (int i = 0; i < NR; ++i) {
              const int hi = T0 + (hh * NR + i) / G, lo = sliding ? max(0, hi - W + 1) : 0;
              const bool valid = i < nvalid && key < nkeys && kp >= lo && kp <= hi;
              pv[i] = valid ? fast_exp2(fmaf(sr[i], qf[i], -bound_log2)) : 0.f;
            }
          }
          /* each row's block scale from its largest p over the warp's 32 keys
           * (one key block): biased exponent E of the maximum, p 2^(134 - E)
           * below 256, ue8m0 code E - 7 (E >= 11 keeps the second term's code
           * E - 11 valid; p >= 2^-116 under the bound wherever it is not 0) */
          uint32_t code = 0; /* lane i < NR: row hh NR + i */
#pragma unroll
          for (int i = 0; i < NR; ++i) {
            l[i] += pv[i];
            const uint32_t m = __reduce_max_sync(0xffffffffu, __float_as_uint(pv[i]));
            const int E = max((int)(m >> 23), 11);
            pv[i] *= __uint_as_float((uint32_t)(261 - E) << 23);
            if (lane == i) code = (uint32_t)(E - 7);
          }
          /* t0 = e4m3(x), t1 = e4m3(16 (x - t0)), x via f16 (exact differences) */
          uint32_t w0[NR / 4], w1[NR / 4];
#pragma unroll
          for (int i = 0; i < NR; i += 2) {
            const uint32_t h = f32x2_to_f16x2(pv[i], pv[i + 1]);
            const uint32_t a = f16x2_to_e4m3x2(h);
            const uint32_t r = f16x2_to_e4m3x2(hmul2(hsub2(h, e4m3x2_to_f16x2(a)), 0x4C004C00u)); /* x 16 */
            if ((i & 2) == 0) {
              w0[i >> 2] = a;
              w1[i >> 2] = r;
            } else {
              w0[i >> 2] |= a << 16;
              w1[i >> 2] |= r << 16;
            }
          }
          /* the key's 16-byte row in its core matrices: key group key / 8,
           * row group, key mod 8.  RP <= 32: the terms stacked as rows
           * (term t, row n at t RP + n), key groups 2 RP * 8 bytes apart;
           * RP = 64: a block of RP * 128 bytes per term. */
          constexpr bool STK = RP <= 32;
          constexpr uint32_t LBO = STK ? 16u * RP : 8u * RP, P1 = STK ? 8u * RP : 128u * RP; /* term 1 */
          const uint32_t pt = ptoff + pb * (uint32_t)RP * 256u + (uint32_t)(key >> 3) * LBO + (uint32_t)(key & 7) * 16u;
          if constexpr (NR == 8) {
            sts64(pt + 8u * (uint32_t)hh, w0[0], w0[1]);
            sts64(pt + P1 + 8u * (uint32_t)hh, w1[0], w1[1]);
          } else {
#pragma unroll
            for (int gq = 0; gq < NR / 16; ++gq) {
              const uint32_t o = (uint32_t)(hh * (NR / 16) + gq) * 128u;
              sts128(pt + o, w0[4 * gq], w0[4 * gq + 1], w0[4 * gq + 2], w0[4 * gq + 3]);
              sts128(pt + P1 + o, w1[4 * gq], w1[4 * gq + 1], w1[4 * gq + 2], w1[4 * gq + 3]);
            }
          }
          if (lane < NR) { /* the scales of row n' (t RP + n stacked, n per term): atom row n' mod 32, word n' / 32, byte qd */
            const int n = hh * NR + lane;
            const uint32_t sa = sfoff + pb * 1024u + (uint32_t)qd;
            if constexpr (STK) {
              const int n1 = RP + n;
              sts8(sa + (uint32_t)(n & 31) * 16u + (uint32_t)(n >> 5) * 4u, code);
              sts8(sa + (uint32_t)(n1 & 31) * 16u + (uint32_t)(n1 >> 5) * 4u, code - 4u);
            } else {
              sts8(sa + (uint32_t)(n & 31) * 16u + (uint32_t)(n >> 5) * 4u, code);
              sts8(sa + 512u + (uint32_t)(n & 31) * 16u + (uint32_t)(n >> 5) * 4u, code - 4u);
            }
          }
        }
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.S->p_ready[pb]);
        ait++;
      }
      /* segment end: the output accumulator after the last stage's products */
      const uint32_t jl = ait - 1u;
      if (ok && !wait_bar(c, &c.S->pv_done[jl % 3u], (jl / 3u) & 1u, layer, PH_ATT)) ok = false;
      ok = __all_sync(0xffffffffu, ok) != 0;
      tc_fence_after();
      const int slotp = c.cta + pr;
      float* base = P->part + (size_t)slotp * P->part_stride;
      if (ok) {
        /* O^T: with the terms stacked (RP <= 32) the sum of the two term columns */
        uint32_t orr[NR], or1[RP <= 32 ? NR : 1];
        const uint32_t ta = tb + ATC_TM_O + (uint32_t)(hh * NR) + ((uint32_t)(qd * 32) << 16);
#pragma unroll
        for (int i = 0; i < NR; i += 8) {
          tc_ld8(ta + (uint32_t)i, orr + i);
          if constexpr (RP <= 32) tc_ld8(ta + (uint32_t)(RP + i), or1 + i);
        }
        tc_wait_ld();
#pragma unroll
        for (int i = 0; i < NR; ++i) {
          const int rho = hh * NR + i;
          float o = __uint_as_float(orr[i]);
          if constexpr (RP <= 32) o += __uint_as_float(or1[i]);
          if (rho < R) base[(size_t)rho * (128 + 4) + qd * 32 + lane] = o;
        }
      }
      /* row sums: over the warp's 32 keys, then the four quadrants */
#pragma unroll
      for (int i = 0; i < NR; ++i) {
        float v = l[i];
#pragma unroll
        for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) lred[qd * 64 + hh * NR + i] = v;
      }
      tc_fence_before();
      named_sync(BAR_CONS, NCT);
      if (ctid < R && ok)
        base[(size_t)ctid * (128 + 4) + 128] = lred[ctid] + lred[64 + ctid] + lred[128 + ctid] + lred[192 + ctid];
      if (ctid == 0) mbar_arrive(&c.S->o_free);
      aseg++;
      /* the pair's parts are combined by the CTA that writes the last one
       * (a counter per pair; the others' parts are visible to it after
       * their fence and its acquire), so no separate phase and grid barrier
       * is needed: o = sum of the parts' O / sum of their l, parts in CTA
       * order, f16 into the W_o projection's input */
      __threadfence();
      named_sync(BAR_CONS, NCT);
      if (ctid == 0) {
        const int cf = att_owner(g, g.off[pr]), cl = att_owner(g, g.off[pr + 1] - 1);
        const uint32_t old = atomicAdd(&P->ctrl[CTRL_PAIR0 + pr], 1u);
        const int last = ok && (int)old + 1 == cl - cf + 1;
        if (last) P->ctrl[CTRL_PAIR0 + pr] = 0u; /* every part arrived: ready for the next layer */
        c.S->attc_last = last;
      }
      named_sync(BAR_CONS, NCT);
      if (c.S->attc_last) {
        __threadfence();
        const int cf = att_owner(g, g.off[pr]), cl = att_owner(g, g.off[pr + 1] - 1);
        for (int item = ctid; item < R * 32; item += NCT) {
          const int rho = item >> 5, c4 = item & 31;
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
          float lsum = 0.f;
          for (int cc = cf; cc <= cl; ++cc) {
            const float* row = P->part + (size_t)(cc + pr) * P->part_stride + (size_t)rho * (128 + 4);
            const float4 q = *reinterpret_cast<const float4*>(row + 4 * c4);
            acc.x += q.x; acc.y += q.y; acc.z += q.z; acc.w += q.w;
            lsum += row[128];
          }
          const float inv = 1.0f / lsum;
          const int t = b * c.st.Tq + rho / P->G, h = (pr % P->hkv) * P->G + rho % P->G;
          uint16_t* dst = P->o + (size_t)t * P->qd + h * 128 + 4 * c4;
          *reinterpret_cast<uint2*>(dst) = make_uint2(f32x2_to_f16x2(acc.x * inv, acc.y * inv), f32x2_to_f16x2(acc.z * inv, acc.w * inv));
          if (P->dbg_attn) {
            float* dbg = P->dbg_attn + ((size_t)layer * c.st.T + t) * P->qd + h * 128 + 4 * c4;
            *reinterpret_cast<float4*>(dbg) = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
          }
        }
      }
      named_sync(BAR_CONS, NCT); /* lred reused by the next segment */
    }
  }
  if (!ok) c.S->abort = 1;
  return !named_sync_or(BAR_CONS, NCT, c.S->abort != 0);
}

/* ---- consumer: small phases (warp per item over the whole grid) --------------------- */
MSK_DEV int gwarp(const Ctx& c) { return c.cta * NCW + (threadIdx.x >> 5) - CONS_WARP0; }
MSK_DEV int nwarps(const Ctx& c) { return c.ncta * NCW; }

/* Row work of one token by a whole CTA: the consumer warps split d into
 * NCW slices (lane-strided float4), the row's sum of squares is reduced in
 * shared memory in fixed order. */
constexpr int ROWV = 4; /* float4 per lane per slice: d <= 4096 */

MSK_DEV float cta_sum(const Ctx& c, float part) {
  const int cw = (threadIdx.x >> 5) - CONS_WARP0, lane = threadIdx.x & 31;
  part = warp_sum(part);
  if (lane == 0) c.S->red8[cw] = part;
  named_sync(BAR_CONS, NCT);
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < NCW; ++i) t += c.S->red8[i];
  named_sync(BAR_CONS, NCT);
  return t;
}

/* xh[i] = f16(v[i] * r * g[i]) (and xf = fp32 copy) over this lane's slice */
MSK_DEV void row_norm_store(const float4* v, int d, float r, const float* gain, uint16_t* xh, float* xf) {
  const int cw = (threadIdx.x >> 5) - CONS_WARP0, lane = threadIdx.x & 31;
  const int sl = d / NCW, base = cw * sl + lane * 4;
#pragma unroll
  for (int u = 0; u < ROWV; ++u) {
    const int i = base + u * 128;
    if (i < (cw + 1) * sl) {
      const float4 gg = *reinterpret_cast<const float4*>(gain + i);
      const float a = v[u].x * r * gg.x, b = v[u].y * r * gg.y, cc = v[u].z * r * gg.z, dd = v[u].w * r * gg.w;
      if (xf) *reinterpret_cast<float4*>(xf + i) = make_float4(a, b, cc, dd);
      if (xh) *reinterpret_cast<uint2*>(xh + i) = make_uint2(f32x2_to_f16x2(a, b), f32x2_to_f16x2(cc, dd));
    }
  }
}

MSK_DEV float cta_max(const Ctx& c, float part) {
  const int cw = (threadIdx.x >> 5) - CONS_WARP0, lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16; o; o >>= 1) part = fmaxf(part, __shfl_xor_sync(0xffffffffu, part, o));
  if (lane == 0) c.S->red8[cw] = part;
  named_sync(BAR_CONS, NCT);
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < NCW; ++i) t = fmaxf(t, c.S->red8[i]);
  named_sync(BAR_CONS, NCT);
  return t;
}

/* The moe-norm row of a token as eight e2m1 terms for the block-scaled
 * tensor cores, all with block scale 1: with f0 the power of two that
 * brings the row's largest magnitude into (3, 6], term j codes the
 * residual the previous terms left, scaled by f0 4^j, rounded to nearest
 * on the e2m1 grid.  Each term leaves at most one grid unit of its scale,
 * which the next (4x finer) term still represents without clipping, so
 * eight terms reach about 6^-1 4^-7 (~1e-5) of the row's largest value.
 * Layout per token (xq): codes [d/32][8 term rows][16 B] (one 8-row
 * core-matrix group per token, any 256-wide K chunk one contiguous
 * kilobyte), then the fp32 factor 1/f0. */
MSK_DEV void row_quant8(const Ctx& c, const float4* v, int d, float r, const float* gain, uint8_t* xq) {
  const int cw = (threadIdx.x >> 5) - CONS_WARP0, lane = threadIdx.x & 31;
  const int sl = d / NCW, base = cw * sl + lane * 4;
  float x[ROWV][4];
  float mx = 0.f;
#pragma unroll
  for (int u = 0; u < ROWV; ++u) {
    const int i = base + u * 128;
    x[u][0] = x[u][1] = x[u][2] = x[u][3] = 0.f;
    if (i < (cw + 1) * sl) {
      const float4 gg = gain ? *reinterpret_cast<const float4*>(gain + i) : make_float4(1.f, 1.f, 1.f, 1.f);
      x[u][0] = v[u].x * r * gg.x;
      x[u][1] = v[u].y * r * gg.y;
      x[u][2] = v[u].z * r * gg.z;
      x[u][3] = v[u].w * r * gg.w;
      mx = fmaxf(mx, fmaxf(fmaxf(fabsf(x[u][0]), fabsf(x[u][1])), fmaxf(fabsf(x[u][2]), fabsf(x[u][3]))));
    }
  }
  mx = cta_max(c, mx);
  int pe = 0;
  if (mx > 0.f) pe = max(-100, min(100, (int)floorf(log2f(6.0f / mx))));
  float fj = __int_as_float((127 + pe) << 23); /* f0 */
  const float finv = __int_as_float((127 - pe) << 23);
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const float inv = 1.0f / fj; /* powers of two: exact */
#pragma unroll
    for (int u = 0; u < ROWV; ++u) {
      const int i = base + u * 128;
      const uint32_t c01 = f32x2_to_e2m1x2(x[u][0] * fj, x[u][1] * fj), c23 = f32x2_to_e2m1x2(x[u][2] * fj, x[u][3] * fj);
      const uint32_t h01 = e2m1x2_to_f16x2(c01), h23 = e2m1x2_to_f16x2(c23);
      x[u][0] -= f16lo_f32(h01) * inv;
      x[u][1] -= f16hi_f32(h01) * inv;
      x[u][2] -= f16lo_f32(h23) * inv;
      x[u][3] -= f16hi_f32(h23) * inv;
      if (i < (cw + 1) * sl)
        *reinterpret_cast<uint16_t*>(xq + (size_t)(i / 32) * 128 + t * 16 + (i % 32) / 2) = (uint16_t)(c01 | (c23 << 8));
    }
    fj *= 4.0f;
  }
  if (cw == 0 && lane == 0) *reinterpret_cast<float*>(xq + (size_t)4 * d) = finv;
}

/* The SwiGLU rows of the step's (token, expert) pairs as eight e2m1 terms
 * for the block-scaled down projection: the encoding of row_quant8 with
 * unit gains (the same terms, bit for bit), one warp per pair (pair p by
 * warp p mod (ncta NCW)); lane l codes the 32-value core columns l, l + 32,
 * ... of the row, one 16-byte row per term.  Each pair's ready word is
 * released once its row and factor are written. */
MSK_DEV void phase_ut(const Ctx& c, int layer) {
  const MskParams* P = c.P;
  const int cw = (threadIdx.x >> 5) - CONS_WARP0, lane = threadIdx.x & 31;
  const int f = P->f, nkk = f / 32, npairs = c.st.T * P->k;
  const size_t utb = MSK_XQ_BYTES(f);
  for (int pr = c.cta * NCW + cw; pr < npairs; pr += c.ncta * NCW) {
    const uint16_t* ur = P->u + (size_t)pr * f;
    uint8_t* xq = P->ut + (size_t)pr * utb;
    float mx = 0.f;
    for (int kk = lane; kk < nkk; kk += 32) {
      const uint4* s4 = reinterpret_cast<const uint4*>(ur + kk * 32);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 w = s4[q];
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) mx = fmaxf(mx, fmaxf(fabsf(f16lo_f32(ws[e])), fabsf(f16hi_f32(ws[e]))));
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    int pe = 0;
    if (mx > 0.f) pe = max(-100, min(100, (int)floorf(log2f(6.0f / mx))));
    const float f0 = __int_as_float((127 + pe) << 23), finv = __int_as_float((127 - pe) << 23);
    for (int kk = lane; kk < nkk; kk += 32) {
      float x[32];
      const uint4* s4 = reinterpret_cast<const uint4*>(ur + kk * 32);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 w = s4[q];
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          x[8 * q + 2 * e] = f16lo_f32(ws[e]);
          x[8 * q + 2 * e + 1] = f16hi_f32(ws[e]);
        }
      }
      float fj = f0;
#pragma unroll 1
      for (int t = 0; t < 8; ++t) {
        const float inv = 1.0f / fj; /* powers of two: exact */
        uint32_t wd[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t word = 0;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = 8 * q + 2 * e;
            const uint32_t cb = f32x2_to_e2m1x2(x[i] * fj, x[i + 1] * fj), h = e2m1x2_to_f16x2(cb);
            x[i] -= f16lo_f32(h) * inv;
            x[i + 1] -= f16hi_f32(h) * inv;
            word |= cb << (8 * e);
          }
          wd[q] = word;
        }
        *reinterpret_cast<uint4*>(xq + (size_t)kk * 128 + t * 16) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        fj *= 4.0f;
      }
    }
    if (lane == 0) *reinterpret_cast<float*>(xq + (size_t)4 * f) = finv;
    __threadfence();
    __syncwarp();
    if (lane == 0) st_release_u32(&P->ctrl[CTRL_UT0 + pr], (uint32_t)(layer + 1));
  }
}

MSK_DEV void phase_in(const Ctx& c) {
  const MskParams* P = c.P;
  const int cw = (threadIdx.x >> 5) - CONS_WARP0, lane = threadIdx.x & 31;
  const int d = P->d, sl = d / NCW, base = cw * sl + lane * 4;
  for (int t = c.cta; t < c.st.T; t += c.ncta) {
    float4 v[ROWV];
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < ROWV; ++u) {
      const int i = base + u * 128;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < (cw + 1) * sl) {
        const uint2 hb = *reinterpret_cast<const uint2*>(c.st.hidden_in + (size_t)t * d + i);
        v[u] = make_float4(bf16_to_f32(hb.x & 0xFFFF), bf16_to_f32(hb.x >> 16), bf16_to_f32(hb.y & 0xFFFF),
                           bf16_to_f32(hb.y >> 16));
        *reinterpret_cast<float4*>(P->h + (size_t)t * d + i) = v[u];
        ss += v[u].x * v[u].x + v[u].y * v[u].y + v[u].z * v[u].z + v[u].w * v[u].w;
      }
    }
    const float r = 1.0f / sqrtf(cta_sum(c, ss) / d + P->eps);
    row_norm_store(v, d, r, P->layers[0].g_attn, P->x + (size_t)t * d, nullptr);
  }
}

/* QK-norm of q and k heads, fp8 quantisation of k and v into the cache */
MSK_DEV void phase_qknorm(const Ctx& c, int layer) {
  const MskParams* P = c.P;
  const MskLayer& Ly = P->layers[layer];
  const int lane = threadIdx.x & 31;
  const int hd = P->hd, nh = P->hq + 2 * P->hkv, per = hd / 32;
  for (int item = gwarp(c); item < c.st.T * nh; item += nwarps(c)) {
    const int t = item / nh, hh = item % nh;
    float v[4];
    qkv_head(c, Ly, t, hh, v);
    if (hh < P->hq) {
      uint16_t* dst = P->qs + (size_t)t * P->qd + hh * hd + lane * per;
      for (int i = 0; i < per; ++i) dst[i] = f32_to_f16(v[i]);
    } else {
      const int isv = hh >= P->hq + P->hkv;
      kv_store(c, layer, t, hh - P->hq - (isv ? P->hkv : 0), isv, v);
    }
  }
  fence_proxy_async_global();
}

/* o = sum of partials / sum of l over the pair's segments */
MSK_DEV void phase_attc(const Ctx& c, int layer) {
  const MskParams* P = c.P;
  const int lane = threadIdx.x & 31, hd = P->hd, per = hd / 32;
  const AttGeo& g = c.S->ag; /* set by this layer's attention phase */
  (void)layer;
  for (int item = gwarp(c); item < c.st.T * P->hq; item += nwarps(c)) {
    const int t = item / P->hq, h = item % P->hq;
    const int b = t / c.st.Tq, ti = t % c.st.Tq;
    const int pair = b * P->hkv + h / P->G;
    const int rho = ti * P->G + h % P->G;
    const int cf = att_owner(g, g.off[pair]), cl = att_owner(g, g.off[pair + 1] - 1);
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, l = 0.f;
#pragma unroll 4
    for (int cc = cf; cc <= cl; ++cc) {
      const float* row = P->part + (size_t)(cc + pair) * P->part_stride + (size_t)rho * (hd + 4);
      if (per == 4) {
        const float4 q = *reinterpret_cast<const float4*>(row + lane * 4);
        acc[0] += q.x; acc[1] += q.y; acc[2] += q.z; acc[3] += q.w;
      } else {
        for (int i = 0; i < per; ++i) acc[i] += row[lane * per + i];
      }
      l += row[hd];
    }
    const float inv = 1.0f / l;
    uint16_t* dst = P->o + (size_t)t * P->qd + h * hd + lane * per;
    for (int i = 0; i < per; ++i) dst[i] = f32_to_f16(acc[i] * inv);
    if (P->dbg_attn) {
      float* dbg = P->dbg_attn + ((size_t)layer * c.st.T + t) * P->qd + h * hd + lane * per;
      for (int i = 0; i < per; ++i) dbg[i] = acc[i] * inv;
    }
  }
}

MSK_DEV void phase_moenorm(const Ctx& c, int layer) {
  const MskParams* P = c.P;
  const int cw = (threadIdx.x >> 5) - CONS_WARP0, lane = threadIdx.x & 31;
  const int d = P->d, sl = d / NCW, base = cw * sl + lane * 4;
  const int So = P->qd <= DKS_MAX ? 1 : P->qd / DKS_MAX;
  for (int t = c.cta; t < c.st.T; t += c.ncta) {
    float4 v[ROWV];
    float ss = 0.f;
    /* residual + W_o o, the projection's K slices added in order; all loads
     * issued before the first store */
#pragma unroll
    for (int u = 0; u < ROWV; ++u) {
      const int i = base + u * 128;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < (cw + 1) * sl) v[u] = *reinterpret_cast<const float4*>(P->h + (size_t)t * d + i);
    }
#pragma unroll
    for (int s = 0; s < MAX_KS; ++s) {
      if (s < So) {
        float4 q[ROWV];
#pragma unroll
        for (int u = 0; u < ROWV; ++u) {
          const int i = base + u * 128;
          q[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (i < (cw + 1) * sl) q[u] = *reinterpret_cast<const float4*>(P->qkv + ((size_t)s * c.st.T + t) * d + i);
        }
#pragma unroll
        for (int u = 0; u < ROWV; ++u) { v[u].x += q[u].x; v[u].y += q[u].y; v[u].z += q[u].z; v[u].w += q[u].w; }
      }
    }
#pragma unroll
    for (int u = 0; u < ROWV; ++u) {
      const int i = base + u * 128;
      if (i < (cw + 1) * sl) {
        *reinterpret_cast<float4*>(P->h + (size_t)t * d + i) = v[u];
        ss += v[u].x * v[u].x + v[u].y * v[u].y + v[u].z * v[u].z + v[u].w * v[u].w;
      }
    }
    const float r = 1.0f / sqrtf(cta_sum(c, ss) / d + P->eps);
    row_norm_store(v, d, r, P->layers[layer].g_moe, P->x2h + (size_t)t * d, P->x2f + (size_t)t * d);
    if (tc_experts(P)) row_quant8(c, v, d, r, P->layers[layer].g_moe, P->xq + (size_t)t * MSK_XQ_BYTES(d));
  }
}

/* router logits in fp32: CTA items of 8 tokens x 16 experts.  The 8
 * tokens' normed rows are staged in the ring (idle between the W_o products
 * and the expert phases), read once from L2 per item; warp w takes experts
 * 2w, 2w+1 of the item, its lanes 4 consecutive elements of every 128. */
MSK_DEV void phase_router(const Ctx& c, int layer) {
  const MskParams* P = c.P;
  const float* Wr = P->layers[layer].router;
  const int cw = (threadIdx.x >> 5) - CONS_WARP0, lane = threadIdx.x & 31, ctid = threadIdx.x - CONS0, d = P->d;
  const int ntg = (c.st.T + 7) / 8, neg = (P->E + 15) / 16;
  float* xs = reinterpret_cast<float*>(c.ring);
  int staged = -1;
  for (int item = c.cta; item < ntg * neg; item += c.ncta) {
    const int tg = item / neg, e0 = (item % neg) * 16 + 2 * cw;
    const int nt = min(8, c.st.T - tg * 8);
    if (tg != staged) {
      named_sync(BAR_CONS, NCT); /* every warp done with the previous rows */
      const float4* src = reinterpret_cast<const float4*>(P->x2f + (size_t)tg * 8 * d);
      float4* dst = reinterpret_cast<float4*>(xs);
      const int n4 = nt * d / 4;
#pragma unroll 8
      for (int q = ctid; q < n4; q += NCT) dst[q] = src[q];
      named_sync(BAR_CONS, NCT);
      staged = tg;
    }
    if (e0 >= P->E) continue;
    float a0[8], a1[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) a0[j] = a1[j] = 0.f;
    const float* w0p = Wr + (size_t)e0 * d;
    const float* w1p = w0p + d;
#pragma unroll 4
    for (int i = lane * 4; i < d; i += 128) {
      const float4 w0 = *reinterpret_cast<const float4*>(w0p + i), w1 = *reinterpret_cast<const float4*>(w1p + i);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < nt) {
          const float4 x = *reinterpret_cast<const float4*>(xs + (size_t)j * d + i);
          a0[j] += w0.x * x.x + w0.y * x.y + w0.z * x.z + w0.w * x.w;
          a1[j] += w1.x * x.x + w1.y * x.y + w1.z * x.z + w1.w * x.w;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float s0 = warp_sum(a0[j]), s1 = warp_sum(a1[j]);
      if (lane == 0 && j < nt) {
        P->logits[(size_t)(tg * 8 + j) * P->E + e0] = s0;
        P->logits[(size_t)(tg * 8 + j) * P->E + e0 + 1] = s1;
      }
    }
  }
}
static_assert(8 * 4096 * 4 <= MSK_NST * MSK_STAGE, "the router stages 8 rows of d <= 4096 floats in the ring");

static_assert(MSK_MAX_TOKENS * 256 * 4 <= MSK_NST * MSK_STAGE, "top-k copies every logit into the stage ring");
/* the counting sort's per-chunk counts [chunk][E] (int16) in the ring after the logits */
constexpr uint32_t TOPK_CNT_OFF = MSK_MAX_TOKENS * 256 * 4;
static_assert(TOPK_CNT_OFF + (MSK_MAX_TOKENS * 8 / 32) * 256 * 2 <= MSK_NST * MSK_STAGE, "top-k scratch fits the ring");

/* order-preserving map of a non-NaN float to u32, -0 taken as +0 */
MSK_DEV uint32_t ord_key(float x) {
  const uint32_t b = x == 0.f ? 0u : __float_as_uint(x);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
MSK_DEV float ord_val(uint32_t k) { return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k); }

/* top-k of every token (value desc, index asc), softmax weights, and the
 * expert work list grouped by expert; every CTA computes the same lists */
MSK_DEV bool phase_topk(Ctx& c, int layer, uint32_t& dpar) {
  const MskParams* P = c.P;
  Route& R = c.S->route;
  const int lane = threadIdx.x & 31, cw = (threadIdx.x >> 5) - CONS_WARP0;
  const int E = P->E, k = P->k, per = E / 32, ctid = threadIdx.x - CONS0;
  /* every token's logits into the (idle) stage ring by one bulk copy */
  const float* lg = reinterpret_cast<const float*>(c.ring);
  {
    const uint32_t par = (dpar >> 9) & 1u, bytes = (uint32_t)(c.st.T * E * 4);
    dpar ^= 1u << 9;
    fence_proxy_async_shared();
    if (ctid == 0) mbar_arrive_tx(&c.S->rfull, bytes);
    named_sync(BAR_CONS, NCT);
    if (ctid == 0) {
      fence_proxy_async_global();
      bulk_g2s(c.ring, P->logits, bytes, &c.S->rfull);
    }
    if (!wait_bar(c, &c.S->rfull, par, layer, PH_TOPK)) {
      if (ctid == 0) { /* the copy must land before the CTA may exit */
        const uint64_t t0 = gtimer();
        while (!mbar_try(&c.S->rfull, par) && gtimer() - t0 < 2 * (uint64_t)P->timeout_ns) {
        }
      }
      c.S->abort = 1;
    }
    if (named_sync_or(BAR_CONS, NCT, c.S->abort != 0)) return false;
  }
  /* four tokens per warp at a time (t = t0 + 8 q), their picks interleaved */
  constexpr int TQ = 4;
  for (int t0 = cw; t0 < c.st.T; t0 += TQ * NCW) {
    uint32_t key[TQ][8], taken[TQ];
#pragma unroll
    for (int q = 0; q < TQ; ++q) {
      const int t = t0 + q * NCW;
      taken[q] = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        key[q][i] = 0u; /* below every real key: never picked while k <= E */
        if (t < c.st.T && i < per) { /* lane holds experts lane + 32 i (conflict-free loads) */
          const float x = lg[(size_t)t * E + lane + 32 * i];
          key[q][i] = ord_key(x == x ? x : -INFINITY); /* a NaN logit ranks last */
        }
      }
    }
#pragma unroll 1
    for (int s = 0; s < k; ++s) {
      /* per token: this lane's best untaken logit (equal keys: lower index),
       * then the warp's largest key and, among lanes holding it, the lowest
       * index */
      uint32_t bk[TQ], wk[TQ], cand[TQ];
      int bi[TQ];
#pragma unroll
      for (int q = 0; q < TQ; ++q) {
        bk[q] = 0;
        bi[q] = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (!((taken[q] >> i) & 1u) && key[q][i] > bk[q]) { bk[q] = key[q][i]; bi[q] = i; }
      }
#pragma unroll
      for (int q = 0; q < TQ; ++q) wk[q] = __reduce_max_sync(0xffffffffu, bk[q]);
#pragma unroll
      for (int q = 0; q < TQ; ++q) cand[q] = bk[q] == wk[q] ? (uint32_t)(lane + 32 * bi[q]) : 0xFFFFFFFFu;
#pragma unroll
      for (int q = 0; q < TQ; ++q) {
        const uint32_t wi = __reduce_min_sync(0xffffffffu, cand[q]);
        if (cand[q] == wi) taken[q] |= 1u << bi[q];
        const int t = t0 + q * NCW;
        if (lane == 0 && t < c.st.T) {
          R.ids[t * k + s] = (int16_t)wi;
          R.w[t * k + s] = ord_val(wk[q]);
        }
      }
    }
  }
  named_sync(BAR_CONS, NCT);
  /* softmax of each token's k picks (the first is the largest): eight lanes
   * per token, lane s one pick, the sum by a fixed shuffle tree */
  for (int base = cw * 32; base < c.st.T * 8; base += NCT) { /* whole warps: the shuffles take every lane */
    const int i = base + lane, t = i >> 3, sl = i & 7;
    const bool act = i < c.st.T * 8 && sl < k;
    float* w = R.w + t * k;
    const float e = act ? expf(w[sl] - w[0]) : 0.f;
    float sum = e;
#pragma unroll
    for (int o = 4; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o, 8);
    if (act) w[sl] = e / sum;
  }
  named_sync(BAR_CONS, NCT);
  /* Counting sort of the pairs (token * k + slot) by expert, stable in pair
   * order.  Warp w takes the 32-pair chunks w, w + 8: per chunk, each pair's
   * rank among the chunk's pairs of its expert (match_any) and the chunk's
   * count per expert; then per expert the counts' prefix over chunks, the
   * experts' starts, and every pair's place. */
  {
    const int np = c.st.T * k, nchunk = (np + 31) / 32;
    int16_t* ccnt = reinterpret_cast<int16_t*>(c.ring + TOPK_CNT_OFF); /* [chunk][E] */
    for (int i = ctid; i < nchunk * E; i += NCT) ccnt[i] = 0;
    named_sync(BAR_CONS, NCT);
    int myrank[2] = {0, 0};
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int ch = cw + q * NCW;
      if (ch < nchunk) {
        const int pi = 32 * ch + lane;
        const bool valid = pi < np;
        const int e = valid ? R.ids[pi] : -1 - lane;
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        myrank[q] = __popc(peers & ((1u << lane) - 1));
        if (valid && myrank[q] == 0) ccnt[ch * E + e] = (int16_t)__popc(peers);
      }
    }
    named_sync(BAR_CONS, NCT);
    for (int e = ctid; e < E; e += NCT) { /* per expert: exclusive prefix over the chunks */
      int run = 0;
      for (int ch = 0; ch < nchunk; ++ch) {
        const int v = ccnt[ch * E + e];
        ccnt[ch * E + e] = (int16_t)run;
        run += v;
      }
      R.cnt[e] = (int16_t)run;
    }
    named_sync(BAR_CONS, NCT);
    if (cw == 0) { /* exclusive scan of the counts -> start */
      int run = 0;
      for (int base = 0; base < E; base += 32) {
        int v = R.cnt[base + lane], x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          int y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        R.start[base + lane] = (int16_t)(run + x - v);
        run += __shfl_sync(0xffffffffu, x, 31);
      }
      if (lane == 0) R.start[E] = (int16_t)run;
    }
    named_sync(BAR_CONS, NCT);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int ch = cw + q * NCW, pi = 32 * ch + lane;
      if (ch < nchunk && pi < np) {
        const int e = R.ids[pi];
        R.pairs[R.start[e] + ccnt[ch * E + e] + myrank[q]] = (int16_t)pi;
      }
    }
    named_sync(BAR_CONS, NCT);
  }
  if (cw == 0) {
    /* units: experts with tokens, split into groups of <= MSK_UNIT_TOK;
     * the units with at least tau tokens (block-scaled gate/up) first, in
     * expert order, then the others */
    const int tau = P->tau;
    auto tc_units = [tau](int n) {
      const int full = n / MSK_UNIT_TOK, rem = n % MSK_UNIT_TOK;
      return (MSK_UNIT_TOK >= tau ? full : 0) + (rem > 0 && rem >= tau ? 1 : 0);
    };
    int ntc = 0;
    for (int base = 0; base < E; base += 32) {
      int v = tc_units(R.cnt[base + lane]);
#pragma unroll
      for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      ntc += v;
    }
    int nu = 0, nt = 0, nd = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane, n = R.cnt[e];
      const int mine = (n + MSK_UNIT_TOK - 1) / MSK_UNIT_TOK, mt = tc_units(n), mc = mine - mt;
      int xt = mt, xc = mc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int yt = __shfl_up_sync(0xffffffffu, xt, o), yc = __shfl_up_sync(0xffffffffu, xc, o);
        if (lane >= o) { xt += yt; xc += yc; }
      }
      int pt = nt + xt - mt, pc = ntc + (nu - nt) + xc - mc;
      for (int u = 0; u < mine; ++u) {
        const int un = min(MSK_UNIT_TOK, n - u * MSK_UNIT_TOK);
        const int at = un >= tau ? pt++ : pc++;
        R.unit_e[at] = (int16_t)e;
        R.unit_start[at] = (int16_t)(R.start[e] + u * MSK_UNIT_TOK);
        R.unit_n[at] = (int16_t)un;
      }
      nt += __shfl_sync(0xffffffffu, xt, 31);
      nu += __shfl_sync(0xffffffffu, xt + xc, 31);
      nd += __popc(__ballot_sync(0xffffffffu, n > 0));
    }
    if (lane == 0) { R.n_units = nu; R.n_units_tc = nt; R.n_distinct = nd; }
  }
  named_sync(BAR_CONS, NCT);
  if (c.cta == 0) {
    const int ctid = threadIdx.x - CONS0;
    if (ctid == 0) P->n_distinct[layer] = R.n_distinct;
    const int np = c.st.T * k;
    for (int i = ctid; i < np; i += NCT) {
      if (P->dbg_ids) P->dbg_ids[(size_t)layer * np + i] = R.ids[i];
      if (P->dbg_w) P->dbg_w[(size_t)layer * np + i] = R.w[i];
    }
    if (P->dbg_logits)
      for (int i = ctid; i < c.st.T * E; i += NCT) P->dbg_logits[(size_t)layer * c.st.T * E + i] = P->logits[i];
  }
  /* the ring's next writer is the copy engine (the expert tiles) */
  fence_proxy_async_shared();
  named_sync(BAR_CONS, NCT);
  if (threadIdx.x == CONS0) {
    __threadfence_block();
    c.S->route_ready = layer + 1;
    /* trace: CTA 0 has its routing (top-k has no grid barrier of its own) */
    if (c.P->dbg_trace && c.cta == 0) c.P->dbg_trace[layer * 16 + PH_TOPK] = gtimer();
  }
  return true;
}

/* h += sum_slot w * y (slot order); then the next layer's attention norm, or
 * the bf16 output after the last layer.  One CTA per token. */
MSK_DEV void phase_comb(const Ctx& c, int layer) {
  const MskParams* P = c.P;
  const Route& R = c.S->route;
  const int cw = (threadIdx.x >> 5) - CONS_WARP0, lane = threadIdx.x & 31, k = P->k;
  const int d = P->d, sl = d / NCW, base = cw * sl + lane * 4;
  const bool last = layer == P->L - 1;
  for (int t = c.cta; t < c.st.T; t += c.ncta) {
    float4 v[ROWV];
    float ss = 0.f;
#pragma unroll
    /* all loads issued before the first store; slots added in order */
#pragma unroll
    for (int u = 0; u < ROWV; ++u) {
      const int i = base + u * 128;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < (cw + 1) * sl) v[u] = *reinterpret_cast<const float4*>(P->h + (size_t)t * d + i);
    }
#pragma unroll
    for (int s = 0; s < TOPK_MAX; ++s) {
      if (s < k) {
        const float w = R.w[t * k + s];
        float4 y[ROWV];
#pragma unroll
        for (int u = 0; u < ROWV; ++u) {
          const int i = base + u * 128;
          y[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (i < (cw + 1) * sl) y[u] = *reinterpret_cast<const float4*>(P->y + (size_t)(t * k + s) * d + i);
        }
#pragma unroll
        for (int u = 0; u < ROWV; ++u) { v[u].x += w * y[u].x; v[u].y += w * y[u].y; v[u].z += w * y[u].z; v[u].w += w * y[u].w; }
      }
    }
#pragma unroll
    for (int u = 0; u < ROWV; ++u) {
      const int i = base + u * 128;
      if (i < (cw + 1) * sl) {
        const float4 acc = v[u];
        *reinterpret_cast<float4*>(P->h + (size_t)t * d + i) = acc;
        ss += acc.x * acc.x + acc.y * acc.y + acc.z * acc.z + acc.w * acc.w;
        if (last) {
          uint16_t* out = c.st.hidden_out + (size_t)t * d + i;
          *reinterpret_cast<uint2*>(out) =
              make_uint2((uint32_t)f32_to_bf16(acc.x) | ((uint32_t)f32_to_bf16(acc.y) << 16),
                         (uint32_t)f32_to_bf16(acc.z) | ((uint32_t)f32_to_bf16(acc.w) << 16));
        }
      }
    }
    if (!last) {
      const float r = 1.0f / sqrtf(cta_sum(c, ss) / d + P->eps);
      row_norm_store(v, d, r, P->layers[layer + 1].g_attn, P->x + (size_t)t * d, nullptr);
    }
  }
}

/* ---- consumer: expert tiles from the producer's ring --------------------------------- */
/*
 * One warp's 16 rows of NM NVFP4 matrices (gate and up, or down) times the
 * unit's 8 activation columns over one K chunk, all operands in shared
 * memory.  Lane (g, cq) owns the NVFP4 blocks 4 qb + cq of the chunk (16 k
 * each, so one scale per block and lane): per block its 16 codes of rows g
 * and g+8 (8 bytes each), the two scales, and 16 activations of column g.
 * Each block is 4 m16n8k16 steps whose k slots map onto the block's 16 k in
 * the same order on both operands.  Decoding is exact: e2m1 and e4m3 are
 * exact in f16 and so is their product.
 */
template <int NM>
MSK_DEV void xgemm(uint32_t codes, uint32_t scales, uint32_t mstride, uint32_t cpitch, uint32_t spitch, uint32_t bsm,
                   uint32_t bpitch, int KC, float (*acc)[4], float (*acc2)[4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, cq = lane & 3;
  /* bytes [s(g), s(g), s(g+8), s(g+8)] of the two rows' scale words */
  const uint32_t sel = (uint32_t)(cq | (cq << 4) | ((cq + 4) << 8) | ((cq + 4) << 12));
  const uint32_t a0 = codes + g * cpitch + 8 * cq, a1 = a0 + 8 * cpitch;
  const uint32_t s0 = scales + g * spitch, s1 = s0 + 8 * spitch;
  const uint32_t b = bsm + g * bpitch + 32 * cq;
  const int nq = KC / 64;
#pragma unroll 2
  for (int qb = 0; qb < nq; ++qb) {
    const uint4 b0 = lds128(b + 128 * qb), b1 = lds128(b + 128 * qb + 16);
#pragma unroll
    for (int m = 0; m < NM; ++m) {
      const uint32_t mo = m * mstride;
      const uint2 c0 = lds64(a0 + mo + 32 * qb), c1 = lds64(a1 + mo + 32 * qb);
      const uint32_t w0 = lds32(s0 + mo + 4 * qb), w1 = lds32(s1 + mo + 4 * qb);
      uint32_t sc[2];
      e4m3x4_to_f16x2x2(__byte_perm(w0, w1, sel), sc);
      uint32_t r0[8], r1[8];
      e2m1x8_to_f16x2x4(c0.x, r0);
      e2m1x8_to_f16x2x4(c0.y, r0 + 4);
      e2m1x8_to_f16x2x4(c1.x, r1);
      e2m1x8_to_f16x2x4(c1.y, r1 + 4);
#pragma unroll
      for (int st = 0; st < 4; ++st) {
        uint32_t a[4];
        a[0] = hmul2(r0[2 * st], sc[0]);
        a[1] = hmul2(r1[2 * st], sc[1]);
        a[2] = hmul2(r0[2 * st + 1], sc[0]);
        a[3] = hmul2(r1[2 * st + 1], sc[1]);
        const uint4& bb = (st >> 1) ? b1 : b0;
        /* alternate two accumulators: two independent mma chains */
        mma_f16((st & 1) ? acc2[m] : acc[m], a, (st & 1) ? bb.z : bb.x, (st & 1) ? bb.w : bb.y);
      }
    }
  }
}

/* Gate/up of the selected experts on the block-scaled tensor cores
 * (tcgen05.mma kind::mxf4nvf4, M = 128 weight rows, N = 8 tokens x 8 term
 * rows, K = 64 per instruction, fp32 accumulators in TMEM).  The producer
 * lands each chunk's codes, its scale-factor atoms (repacked once by
 * msk_create into the layout the scale copies read) and the unit's
 * activation terms; the issuing warp copies the scales into TMEM, issues
 * the MMAs, commits the slot back to the producer and, after an item's last
 * chunk, to that item's accumulator buffer (two buffers, so an item's
 * epilogue overlaps the next item's MMAs).  The consumer warps only run the
 * epilogue: read the accumulators (TMEM lane = weight row), sum each token's
 * eight term columns, undo the token's power-of-two factor, apply the global
 * scales and SwiGLU.
 * xpar: bits 0-3 weight-slot fill parities (the issuer waits for the fills;
 * the consumers count them, for the down projection's waits); 12-13
 * accumulator-buffer parities. */
MSK_DEV bool expert_gu_tc(Ctx& c, int layer, uint32_t& xpar) {
  const MskParams* P = c.P;
  const MskLayer& Ly = P->layers[layer];
  const Route& R = c.S->route;
  const int cw = (threadIdx.x >> 5) - CONS_WARP0, lane = threadIdx.x & 31;
  XGeo x;
  xgeo(c, XP_TC, x);
  const int f = P->f;
  const float gs0 = Ly.wg.gs, gs1 = Ly.wu.gs;
  const size_t xqb = MSK_XQ_BYTES(P->d);
  const uint32_t tb = c.S->tmem_base;
  const int q = (threadIdx.x >> 5) & 3, th = cw >> 2; /* TMEM lane quadrant, token half of the epilogue */
  bool ok = true;
  for (int item = x.a; item < x.b; ++item) {
    const int unit = x.u0 + item / x.ngroups, grp = item % x.ngroups, db = (item - x.a) & 1;
    const int n = R.unit_n[unit], st0 = R.unit_start[unit];
    xpar ^= fill_parity_run(x, item - x.a);
    const uint32_t dp = (xpar >> (12 + db)) & 1u;
    xpar ^= 1u << (12 + db);
    if (ok && !wait_bar(c, &c.S->dfull2[db], dp, layer, PH_GU)) ok = false;
    ok = __all_sync(0xffffffffu, ok) != 0; /* warp-uniform: the TMEM loads below are warp-collective */
    if (!ok) continue;
    tc_fence_after();
    uint32_t gr[32], ur[32];
    const uint32_t dcol = tb + TM_D + db * 128 + ((uint32_t)(q * 32) << 16) + th * 32;
    tc_ld32(dcol, gr);
    tc_ld32(dcol + TM_DU, ur);
    tc_wait_ld();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&c.S->dempty2[db]); /* the buffer may take the item after next */
    const int row = grp * XROWS + q * 32 + lane;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int tt = th * 4 + t;
      if (tt < n) {
        const int pair = R.pairs[st0 + tt];
        const float fi = *reinterpret_cast<const float*>(P->xq + (size_t)(pair / P->k) * xqb + xqb - 16);
        float gsum = 0.f, usum = 0.f;
#pragma unroll
        for (int jt = 7; jt >= 0; --jt) { /* term jt weighs 4^-jt; smallest first */
          gsum = gsum * 0.25f + __uint_as_float(gr[8 * t + jt]);
          usum = usum * 0.25f + __uint_as_float(ur[8 * t + jt]);
        }
        const float gv = gsum * fi * gs0, uv = usum * fi * gs1;
        P->u[(size_t)pair * f + row] = f32_to_f16(gv / (1.0f + expf(-gv)) * uv);
      }
    }
  }
  if (!ok) c.S->abort = 1;
  /* one answer for every warp, even if the abort word changes meanwhile */
  return !named_sync_or(BAR_CONS, NCT, c.S->abort != 0);
}

/* Down projection of the block-scaled units on the block-scaled tensor
 * cores (tcgen05.mma kind::mxf4nvf4, M = 128 weight rows, N = 8 pairs x 8
 * term rows, K = 64 per instruction): the issuing warps walk the items (see
 * issuer); the consumer warps run the epilogue, as for gate/up: read the
 * item's accumulators (TMEM lane = output row), sum each pair's eight term
 * columns, undo the pair's power-of-two factor and apply the global scale. */
MSK_DEV bool expert_dt_tc(Ctx& c, int layer, uint32_t& xpar) {
  const MskParams* P = c.P;
  const MskLayer& Ly = P->layers[layer];
  const Route& R = c.S->route;
  const int cw = (threadIdx.x >> 5) - CONS_WARP0, lane = threadIdx.x & 31;
  XGeo x;
  xgeo(c, XP_DT, x);
  const int d = P->d;
  const float gs = Ly.wd.gs;
  const size_t utb = MSK_XQ_BYTES(P->f);
  const uint32_t tb = c.S->tmem_base;
  const int q = (threadIdx.x >> 5) & 3, th = cw >> 2; /* TMEM lane quadrant, pair half of the epilogue */
  bool ok = true;
  int funit = -1;  /* the unit whose pair factors fiv holds */
  float fiv[4] = {0.f, 0.f, 0.f, 0.f};
  for (int item = x.a; item < x.b; ++item) {
    const int unit = x.u0 + item / x.ngroups, grp = item % x.ngroups, db = (item - x.a) & 1;
    const int n = R.unit_n[unit], st0 = R.unit_start[unit];
    if (unit != funit) { /* the factors of this warp's four pairs (their words are set: the terms went into the products) */
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int tt = th * 4 + t;
        if (tt < n) {
          const int pair = R.pairs[st0 + tt];
          if (!wait_gword(c, &P->ctrl[CTRL_UT0 + pair], (uint32_t)(layer + 1), layer, PH_DN)) ok = false;
          fiv[t] = *reinterpret_cast<const float*>(P->ut + (size_t)pair * utb + utb - 16);
        }
      }
      funit = unit;
    }
    xpar ^= fill_parity_run(x, item - x.a);
    const uint32_t dp = (xpar >> (12 + db)) & 1u;
    xpar ^= 1u << (12 + db);
    if (ok && !wait_bar(c, &c.S->dfull2[db], dp, layer, PH_DN)) ok = false;
    ok = __all_sync(0xffffffffu, ok) != 0; /* warp-uniform: the TMEM loads below are warp-collective */
    if (!ok) continue;
    tc_fence_after();
    uint32_t yr[32];
    tc_ld32(tb + TM_D + db * 128 + ((uint32_t)(q * 32) << 16) + th * 32, yr);
    tc_wait_ld();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&c.S->dempty2[db]); /* the buffer may take the item after next */
    const int row = grp * XROWS + q * 32 + lane;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int tt = th * 4 + t;
      if (tt < n) {
        const int pair = R.pairs[st0 + tt];
        float ysum = 0.f;
#pragma unroll
        for (int jt = 7; jt >= 0; --jt) ysum = ysum * 0.25f + __uint_as_float(yr[8 * t + jt]); /* smallest first */
        P->y[(size_t)pair * d + row] = ysum * fiv[t] * gs;
      }
    }
  }
  if (!ok) c.S->abort = 1;
  return !named_sync_or(BAR_CONS, NCT, c.S->abort != 0);
}

/* Gate/up (GU) or down projection of the selected experts on the CUDA-core
 * tensor path (mma.sync, weights decoded in registers): this CTA's items,
 * 16 rows per warp, weight chunks and the unit's activation rows from the
 * producer's ring.  After a chunk every warp meets at a CTA barrier and
 * one thread releases the slot.  xpar bit s is the parity of weight slot
 * s's uses. */
template <bool GU>
MSK_DEV bool expert_mma(Ctx& c, int layer, uint32_t& xpar) {
  const MskParams* P = c.P;
  const MskLayer& Ly = P->layers[layer];
  const Route& R = c.S->route;
  const int cw = (threadIdx.x >> 5) - CONS_WARP0, lane = threadIdx.x & 31, g = lane >> 2, cq = lane & 3;
  const int phase = GU ? PH_GU : PH_DN;
  XGeo x;
  xgeo(c, GU ? XP_CC : XP_DN, x);
  const int d = P->d, f = P->f;
  const float gs0 = GU ? Ly.wg.gs : Ly.wd.gs, gs1 = Ly.wu.gs;
  const uint32_t ring = smem_u32(c.ring);
  float acc[2][4], acc2[2][4];
  int j = 0;
  bool ok = true;
  for (int item = x.a; item < x.b; ++item) {
    const int unit = x.u0 + item / x.ngroups, grp = item % x.ngroups;
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[0][e] = acc[1][e] = acc2[0][e] = acc2[1][e] = 0.f;
    for (int kc = 0; kc < x.nkc; ++kc, ++j) {
      const int s = j % x.ns;
      if (ok && !wait_bar(c, &c.S->xfull[s], (xpar >> s) & 1u, layer, phase)) ok = false;
      xpar ^= 1u << s;
      const uint32_t slot = ring + (uint32_t)s * x.slot_bytes;
      if (ok)
        xgemm<GU ? 2 : 1>(slot + cw * 16 * x.cpitch, slot + XROWS * x.cpitch + cw * 16 * x.spitch, x.mat_bytes,
                          x.cpitch, x.spitch, slot + x.b_off, x.bpitch, x.KC, acc, acc2);
      /* each warp releases the slot when it is done with it: no CTA barrier
       * per chunk; the producer refills once all eight have arrived */
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.S->xempty_cc[s]);
    }
    if (!ok) continue;
    const int n = R.unit_n[unit], st0 = R.unit_start[unit];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int col = 2 * cq + (e & 1), row = grp * XROWS + cw * 16 + g + 8 * (e >> 1);
      if (col < n) {
        const int pair = R.pairs[st0 + col];
        if (GU) {
          const float gv = (acc[0][e] + acc2[0][e]) * gs0, uv = (acc[1][e] + acc2[1][e]) * gs1;
          P->u[(size_t)pair * f + row] = f32_to_f16(gv / (1.0f + expf(-gv)) * uv);
        } else {
          P->y[(size_t)pair * d + row] = (acc[0][e] + acc2[0][e]) * gs0;
        }
      }
    }
  }
  if (!ok) c.S->abort = 1;
  /* one answer for every warp, even if the abort word changes meanwhile */
  return !named_sync_or(BAR_CONS, NCT, c.S->abort != 0);
}

/* ---- consumer main loop ---------------------------------------------------------------- */
template <int HD>
MSK_DEV void consumer(Ctx& c) {
  const MskParams* P = c.P;
  Cons q;
  q.c = &c;
  q.it = 0;
  uint32_t xpar = 0; /* this warp's expert-slot parities */
  uint32_t dpar = 0; /* this warp's dense-slot and activation-slice parities */
  uint32_t ait = 0, aseg = 0; /* tensor-core attention stages and segments consumed */
  phase_in(c);
  if (!grid_sync(c, 0, PH_IN)) return;
  for (int l = 0; l < P->L; ++l) {
    if (!dense_phase<true>(c, l, dpar)) return;
    if (!grid_sync(c, l, PH_QKV)) return;
    phase_qknorm(c, l);
    if (!grid_sync(c, l, PH_QKNORM)) return;
    if (threadIdx.x == CONS0) c.S->kv_ready = l + 1;
    bool ok;
    if constexpr (HD == 128) {
      const int RP = atc_rp(c.st.Tq * P->G);
      ok = RP == 16 ? attention_phase_tc<16>(c, l, ait, aseg)
                    : (RP == 32 ? attention_phase_tc<32>(c, l, ait, aseg) : attention_phase_tc<64>(c, l, ait, aseg));
    } else {
      ok = attention_phase<HD>(q, l);
    }
    if (!ok) return;
    if (!grid_sync(c, l, PH_ATT)) return;
    if constexpr (HD != 128) { /* head dim 128 combines inside its attention phase */
      phase_attc(c, l);
      if (!grid_sync(c, l, PH_ATTC)) return;
    }
    if (!dense_phase<false>(c, l, dpar)) return;
    if (!grid_sync(c, l, PH_WO)) return;
    phase_moenorm(c, l);
    if (!grid_sync(c, l, PH_MOENORM)) return;
    phase_router(c, l);
    if (!grid_sync(c, l, PH_ROUTER)) return;
    if (!phase_topk(c, l, dpar)) return;
    if (tc_experts(P) && !expert_gu_tc(c, l, xpar)) return;
    if (!expert_mma<true>(c, l, xpar)) return;
    if (!grid_sync(c, l, PH_GU)) return;
    if (threadIdx.x == CONS0) c.S->dn_ready = l + 1;
    if (tc_down(P) && c.S->route.n_units_tc > 0) {
      phase_ut(c, l);
      if (!expert_dt_tc(c, l, xpar)) return;
    }
    if (!expert_mma<false>(c, l, xpar)) return;
    named_sync(BAR_CONS, NCT);
    if (threadIdx.x == CONS0) c.S->ring_free = l + 1;
    if (!grid_sync(c, l, PH_DN)) return;
    phase_comb(c, l);
    if (l + 1 < P->L && !grid_sync(c, l, PH_COMB)) return;
  }
}

}  // namespace

template <int HD>
__global__ void __launch_bounds__(MSK_NTHREADS, 1)
    msk_step_kernel(const MskParams* __restrict__ P, const MskStep st, const __grid_constant__ CUtensorMap kvmap) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctx c;
  c.P = P;
  c.st = st;
  c.kvmap = &kvmap;
  c.ring = base;
  c.scr = reinterpret_cast<float*>(base + (size_t)MSK_NST * MSK_STAGE);
  c.S = reinterpret_cast<Smem*>(base + (size_t)MSK_NST * MSK_STAGE + MSK_SCR);
  c.cta = blockIdx.x;
  c.ncta = gridDim.x;
  c.nbar = 0;
  if (threadIdx.x == 0) {
    for (int i = 0; i < MSK_NST; ++i) {
      mbar_init(&c.S->full[i], 1);
      mbar_init(&c.S->empty[i], NCW);
    }
    c.S->kv_ready = 0;
    c.S->route_ready = 0;
    c.S->ring_free = 0;
    c.S->abort = 0;
    c.S->dn_ready = 0;
    c.S->dense_done = 0;
    for (int w = 0; w < MSK_NCW; ++w)
      for (int i = 0; i < DNS; ++i) {
        mbar_init(&c.S->dfull[w][i], 1);
        mbar_init(&c.S->dempty[w][i], 1);
      }
    mbar_init(&c.S->bfull, 1);
    mbar_init(&c.S->rfull, 1);
    for (int i = 0; i < XNS_MAX; ++i) {
      mbar_init(&c.S->xfull[i], 1);
      mbar_init(&c.S->xempty[i], 2);  /* two tensor-core commits */
      mbar_init(&c.S->xempty_cc[i], NCW);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c.S->dfull2[i], 2); /* both issuing roles commit */
      mbar_init(&c.S->dempty2[i], NCW);
    }
    mbar_init(&c.S->tfin, 2);
    for (int i = 0; i < 6; ++i) {
      mbar_init(&c.S->kfull[i], 1);
      mbar_init(&c.S->kempty[i], 1);
      mbar_init(&c.S->vfull[i], 1);
      mbar_init(&c.S->vempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c.S->s_ready[i], 1);
      mbar_init(&c.S->s_free[i], NCW);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&c.S->p_ready[i], NCW);
      mbar_init(&c.S->pv_done[i], 1);
    }
    mbar_init(&c.S->q_ready, 1);
    mbar_init(&c.S->o_free, 1);
    c.S->ag_ready = 0;
    c.S->issuer_done = 0;
    mbar_fence_init();
  }
  /* positions: contiguous per sequence, inside the cache */
  __shared__ int s_bad;
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < st.T; i += blockDim.x) {
    const int b = i / st.Tq, t = i % st.Tq;
    const int p = st.positions[i], p0 = st.positions[b * st.Tq];
    if (p != p0 + t || p0 < 0 || (int64_t)p0 + st.Tq > st.kv_cap) s_bad = 1;
    if (t == 0) c.S->pos0[b] = p0;
  }
  __syncthreads();
  if (s_bad) {
    if (threadIdx.x == 0 && blockIdx.x == 0) atomicCAS(&P->status[ST_CODE], 0u, (uint32_t)MSK_ERR_KV_RANGE);
    return;
  }
  if (blockIdx.x == 0 && threadIdx.x < st.S) {
    if (threadIdx.x == 0) { P->last_shape[0] = st.S; P->last_shape[1] = st.Tq; }
    P->last_shape[2 + threadIdx.x] = c.S->pos0[threadIdx.x];
  }
  if (threadIdx.x < CONS0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_PRODUCER));
    if (threadIdx.x < 32) producer(c);
    else if (threadIdx.x < 96) issuer(c, (threadIdx.x >> 5) - 1);
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_CONSUMER));
    const bool w0 = (threadIdx.x >> 5) == CONS_WARP0;
    /* the whole TMEM of the SM (one CTA per SM): gate/up accumulators and
     * scale factors of the block-scaled expert MMAs */
    if (w0) tmem_alloc(&c.S->tmem_base, TM_COLS);
    tc_fence_before();
    named_sync(BAR_CONS, NCT);
    tc_fence_after();
    consumer<HD>(c);
    /* every consumer warp leaves the step at the same barrier; wait for the
     * tensor-core work issued so far (bounded), then free the TMEM */
    named_sync(BAR_CONS, NCT);
    if (threadIdx.x == CONS0) {
      const uint64_t t0 = gtimer();
      while (c.S->issuer_done < 2 && gtimer() - t0 < 2 * (uint64_t)P->timeout_ns) __nanosleep(64);
      while (!mbar_try(&c.S->tfin, 0) && gtimer() - t0 < 4 * (uint64_t)P->timeout_ns) {
      }
    }
    tc_fence_before();
    named_sync(BAR_CONS, NCT);
    tc_fence_after();
    if (w0) tmem_dealloc(c.S->tmem_base, TM_COLS);
  }
}

/* fp32 -> fp8 e4m3 codes with the KV write's conversion (RNE, satfinite),
 * four values per thread */
__global__ void msk_kv_encode_kernel(const float4* __restrict__ in, uint32_t* __restrict__ out, int64_t n4) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
    const float4 v = in[i];
    out[i] = f32x2_to_e4m3x2(v.x, v.y) | (f32x2_to_e4m3x2(v.z, v.w) << 16);
  }
}
__global__ void msk_kv_encode_tail(const float* __restrict__ in, uint8_t* __restrict__ out, int64_t i0, int64_t n) {
  const int64_t i = i0 + threadIdx.x;
  if (i < n) out[i] = (uint8_t)f32x2_to_e4m3x2(in[i], 0.f);
}

/* Expert weight tiles for whole-slot bulk copies (one contiguous copy per
 * K chunk instead of a 2-D box per row: 2-D boxes of 128-byte rows stream at
 * about 5.0 TB/s on this part, contiguous 32-48 KB bulk copies at 7.2-7.4).
 * Gate/up for the block-scaled path, per (expert, 128-row group, 256-wide K
 * chunk), 36 KB laid out as the slot: gate codes [128][128 B] and up codes,
 * each as the 128-byte-swizzled image the tensor copy would have written
 * (16-byte chunk c of row r at (c xor r mod 8)), then the gate and up
 * scale-factor atoms of the chunk's four 64-wide K steps. */
__global__ void msk_xtile_gu_kernel(const uint8_t* __restrict__ gc, const uint8_t* __restrict__ uc,
                                    const uint8_t* __restrict__ gsc, const uint8_t* __restrict__ usc,
                                    uint4* __restrict__ out, int64_t ntiles, int f, int d) {
  const int nkc = d / 256, ng = f / 128, k16 = d / 16;
  const int64_t nch = ntiles * (GU_SLOT - 8192) / 16; /* 2304 chunks of 16 bytes per tile */
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < nch; q += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = q / 2304;
    const int qi = (int)(q - t * 2304);
    const int kc = (int)(t % nkc), g = (int)((t / nkc) % ng);
    const int64_t e = t / ((int64_t)nkc * ng);
    const int64_t row0 = e * f + (int64_t)g * 128;
    uint4 v;
    if (qi < 2048) { /* codes: matrix m, row r, physical chunk p */
      const int m = qi >> 10, r = (qi >> 3) & 127, pch = qi & 7, lch = pch ^ (r & 7);
      v = *reinterpret_cast<const uint4*>((m ? uc : gc) + (row0 + r) * (d / 2) + kc * 128 + lch * 16);
    } else { /* scale atoms: matrix m, step st, atom row r: rows r + 32 m1, four blocks */
      const int ai = qi - 2048, m = ai >> 7, st = (ai >> 5) & 3, r = ai & 31;
      const uint8_t* sc = m ? usc : gsc;
      uint32_t w[4];
#pragma unroll
      for (int m1 = 0; m1 < 4; ++m1)
        w[m1] = *reinterpret_cast<const uint32_t*>(sc + (row0 + r + 32 * m1) * k16 + (kc * 4 + st) * 4);
      v = make_uint4(w[0], w[1], w[2], w[3]);
    }
    out[q] = v;
  }
}

/* Down projection tiles for the block-scaled path, per (expert, 128-row
 * group, 512-wide K chunk): the gate/up tile layout with the chunk's two
 * 256-wide halves in place of the two matrices (swizzled codes of half 0,
 * of half 1, then each half's four scale-factor atoms). */
__global__ void msk_xtile_dt_kernel(const uint8_t* __restrict__ dc, const uint8_t* __restrict__ dsc,
                                    uint4* __restrict__ out, int64_t ntiles, int rows_per_expert, int K) {
  const int nkc = K / 512, ng = rows_per_expert / 128, k16 = K / 16;
  const int64_t nch = ntiles * 2304;
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < nch; q += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = q / 2304;
    const int qi = (int)(q - t * 2304);
    const int kc = (int)(t % nkc), g = (int)((t / nkc) % ng);
    const int64_t e = t / ((int64_t)nkc * ng);
    const int64_t row0 = e * rows_per_expert + (int64_t)g * 128;
    uint4 v;
    if (qi < 2048) { /* codes: half h, row r, physical chunk p */
      const int h = qi >> 10, r = (qi >> 3) & 127, pch = qi & 7, lch = pch ^ (r & 7);
      v = *reinterpret_cast<const uint4*>(dc + (row0 + r) * (K / 2) + (2 * kc + h) * 128 + lch * 16);
    } else { /* scale atoms: half h, step st, atom row r: rows r + 32 m1, four blocks */
      const int ai = qi - 2048, h = ai >> 7, st = (ai >> 5) & 3, r = ai & 31;
      uint32_t w[4];
#pragma unroll
      for (int m1 = 0; m1 < 4; ++m1)
        w[m1] = *reinterpret_cast<const uint32_t*>(dsc + (row0 + r + 32 * m1) * k16 + ((2 * kc + h) * 4 + st) * 4);
      v = make_uint4(w[0], w[1], w[2], w[3]);
    }
    out[q] = v;
  }
}

/* Down projection tiles for the CUDA-core path, per (expert, 128-row group,
 * K chunk of KC = min(K, 512)), laid out as its slot: codes [128][KC/2 + 32]
 * (the 32 padding bytes zero) then scales [128][KC/16]. */
__global__ void msk_xtile_dn_kernel(const uint8_t* __restrict__ dc, const uint8_t* __restrict__ dsc,
                                    uint4* __restrict__ out, int64_t ntiles, int rows_per_expert, int K) {
  const int KC = K < 512 ? K : 512, nkc = K / KC, ng = rows_per_expert / 128;
  const int cp = KC / 2 + 32, sp = KC / 16;
  const int tile16 = 128 * (cp + sp) / 16;
  const int64_t nch = ntiles * tile16;
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < nch; q += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = q / tile16;
    const int qi = (int)(q - t * tile16);
    const int kc = (int)(t % nkc), g = (int)((t / nkc) % ng);
    const int64_t e = t / ((int64_t)nkc * ng);
    const int64_t row0 = e * rows_per_expert + (int64_t)g * 128;
    uint4 v = make_uint4(0, 0, 0, 0);
    const int off = qi * 16;
    if (off < 128 * cp) {
      const int r = off / cp, c = off - r * cp;
      if (c < KC / 2) v = *reinterpret_cast<const uint4*>(dc + (row0 + r) * (K / 2) + kc * (KC / 2) + c);
    } else {
      const int so = off - 128 * cp, r = so / sp, c = so - r * sp;
      v = *reinterpret_cast<const uint4*>(dsc + (row0 + r) * (K / 16) + kc * sp + c);
    }
    out[q] = v;
  }
}

/* ---- launch ---------------------------------------------------------------------------- */
extern "C" size_t msk_kernel_smem_bytes() { return SMEM_BYTES; }

extern "C" size_t msk_kernel_xtile_gu_bytes(int E, int f, int d) { return (size_t)E * (f / 128) * (d / 256) * (GU_SLOT - 8192); }
extern "C" size_t msk_kernel_xtile_dn_bytes(int E, int rows_per_expert, int K) {
  const int KC = K < 512 ? K : 512;
  return (size_t)E * (rows_per_expert / 128) * (K / KC) * 128 * (KC / 2 + 32 + KC / 16);
}
extern "C" size_t msk_kernel_xtile_dt_bytes(int E, int rows_per_expert, int K) {
  return (size_t)E * (rows_per_expert / 128) * (K / 512) * 36864;
}
extern "C" cudaError_t msk_kernel_xtile(int kind, const uint8_t* c0, const uint8_t* c1, const uint8_t* s0, const uint8_t* s1,
                                        uint8_t* out, int E, int rows_per_expert, int K, cudaStream_t st) {
  if (kind == 0) {
    const int64_t ntiles = (int64_t)E * (rows_per_expert / 128) * (K / 256);
    const int64_t n = ntiles * 2304;
    msk_xtile_gu_kernel<<<(unsigned)((n + 255) / 256 < 148 * 64 ? (n + 255) / 256 : 148 * 64), 256, 0, st>>>(
        c0, c1, s0, s1, reinterpret_cast<uint4*>(out), ntiles, rows_per_expert, K);
  } else if (kind == 2) {
    const int64_t ntiles = (int64_t)E * (rows_per_expert / 128) * (K / 512);
    const int64_t n = ntiles * 2304;
    msk_xtile_dt_kernel<<<(unsigned)((n + 255) / 256 < 148 * 64 ? (n + 255) / 256 : 148 * 64), 256, 0, st>>>(
        c0, s0, reinterpret_cast<uint4*>(out), ntiles, rows_per_expert, K);
  } else {
    const int KC = K < 512 ? K : 512;
    const int64_t ntiles = (int64_t)E * (rows_per_expert / 128) * (K / KC);
    const int64_t n = ntiles * 128 * (KC / 2 + 32 + KC / 16) / 16;
    msk_xtile_dn_kernel<<<(unsigned)((n + 255) / 256 < 148 * 64 ? (n + 255) / 256 : 148 * 64), 256, 0, st>>>(
        c0, s0, reinterpret_cast<uint4*>(out), ntiles, rows_per_expert, K);
  }
  return cudaGetLastError();
}

extern "C" cudaError_t msk_kernel_kv_encode(const float* in, uint8_t* out, int64_t n, cudaStream_t stream) {
  const int64_t n4 = n / 4;
  if (n4 > 0) {
    const int64_t blocks = (n4 + 255) / 256;
    msk_kv_encode_kernel<<<(unsigned)(blocks < 148 * 16 ? blocks : 148 * 16), 256, 0, stream>>>(
        reinterpret_cast<const float4*>(in), reinterpret_cast<uint32_t*>(out), n4);
  }
  if (n % 4) msk_kv_encode_tail<<<1, 32, 0, stream>>>(in, out, n4 * 4, n);
  return cudaGetLastError();
}

static const void* kernel_for(int hd) {
  return hd == 128 ? (const void*)msk_step_kernel<128> : (const void*)msk_step_kernel<64>;
}

extern "C" cudaError_t msk_kernel_setup(int hd, int* ctas_per_sm) {
  const void* k = kernel_for(hd);
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  /* the register split must fit the pool the block is launched with */
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, k);
  if (e != cudaSuccess) return e;
  if (128 * REGS_PRODUCER + 2 * 128 * REGS_CONSUMER > MSK_NTHREADS * fa.numRegs) {
    *ctas_per_sm = 0;
    return cudaSuccess;
  }
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, k, MSK_NTHREADS, SMEM_BYTES);
}

extern "C" cudaError_t msk_kernel_launch(int hd, const MskParams* P_dev, const MskStep* st, const CUtensorMap* map,
                                         int ncta, cudaStream_t stream) {
  void* args[3] = {(void*)&P_dev, (void*)st, (void*)map};
  return cudaLaunchCooperativeKernel(kernel_for(hd), dim3(ncta), dim3(MSK_NTHREADS), args, SMEM_BYTES, stream);
}
