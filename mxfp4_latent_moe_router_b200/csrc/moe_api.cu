// moe_api.cu -- the C ABI declared in include/moe.h.
//
// A plan owns: packed weights, the per-forward workspace (activations, routing
// tables, split-K partial sums, scheduling counters and flags).  moe_forward
// only enqueues work on the caller's stream; all memory exists from
// moe_plan_create on.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/moe.h"
#include "engine.cuh"
#include "layout.cuh"

using namespace moe;

namespace {

constexpr int kScratchOff = 1024;
constexpr int kScratchBytes = 20480;
constexpr int kStageOff = kScratchOff + kScratchBytes;
// The tensor-core expert kernels at up to two token tiles use at most 8.5 KB
// of the consumers' scratch (the accumulator staging, 128 rows x 17 floats;
// the split-K sums, 16 columns x 128 rows): the rest goes to the ring.
constexpr int kScratchBytesUmmaSmall = 9216;
constexpr int kHdr = 128;
// per-kind slots (scheduling state, profile, trace), one for the fused
// single launch, and two for the side lane's kernels (the shared expert's
// gate/up rows and its down projection, on the side stream)
constexpr int kSlots = KIND_COUNT + 3;
constexpr int kFused = KIND_COUNT;
constexpr int kSideFront = KIND_COUNT + 1;
constexpr int kSideTail = KIND_COUNT + 2;
// largest batch that runs the shared expert as a side lane (a second stream
// whose CTAs share the SMs with the routed chain's): every kernel of either
// lane then fits in half an SM's shared memory
constexpr int kSideMaxTokens = 4;
// largest batch whose routing CTA sums the router pieces' partials itself
constexpr int kDirectRouteMaxTokens = 4;
// kernels moe_debug_geometry describes: the routed chain's four, then the
// side lane's two
constexpr int kGeometryKinds = KIND_COUNT + 2;
// largest batch the fused single launch takes (one 8-column token tile)
constexpr int kFusedMaxTokens = 8;
// tokens a tail pass takes: 64 (eight token tiles) with formed records; the
// fused single launch stages the k slots' y rows per token and takes at most
// 8 tokens
constexpr int kTailTg = 64;
// Tokens per virtual expert (an expert's slots are cut into groups of at most
// this many).  Groups of 8 keep the expert kernels at one token tile, where
// two CTAs share an SM.  That wins even for 128 Zipf-skewed tokens (675 vs
// 772 us per step), although a popular expert's weights are then read once
// per 8 tokens: its groups are adjacent in the piece order and tend to run
// at about the same time, so most re-reads can hit L2.  Groups of 32 (four
// tiles, one CTA per SM) remain for batches above the environment variable
// MOE_EXPERT_SMALL_MAX_B.
constexpr int kExpertTgSmall = 8, kExpertTgLarge = 32, kExpertTgUmmaLarge = 16;
constexpr int kBigSmem = 227 * 1024;
// two CTAs of the one-tile expert kernels share an SM (228 KB, 1 KB reserved
// per CTA): twice the warps to hide the MXFP4 loop's latencies
constexpr int kHalfSmem = 113 * 1024;

struct KindGeom {
  int RB = 0, C = 0, KL = 0;
  size_t tile_bytes = 0;
  size_t weight_bytes = 0;  // packed (per expert for EGU/EDN)
};

struct DevBuf {
  void* p = nullptr;
  size_t n = 0;
};

}  // namespace

struct moe_plan_s {
  moe_config cfg{};
  int device = 0;
  int num_sms = 0;
  bool loaded = false;
  int last_B = 0;

  KindGeom g[KIND_COUNT];
  int RB_router = 0, RB_lat = 0, C_lat = 0, tail_tg = kTailTg, ve_max = 0;

  std::vector<void*> allocs;
  size_t packed_bytes = 0, workspace_bytes = 0;

  // cross-layer prefetch (moe_set_next_layer): the plan whose front weights
  // each forward pulls into L2, and how many of their bytes
  moe_plan_s* next_layer = nullptr;
  long long next_bytes = 0;

  uint8_t* w_front = nullptr;
  uint8_t* w_egu = nullptr;
  uint8_t* w_edn = nullptr;
  uint8_t* w_tail = nullptr;
  uint8_t* w_tail_um = nullptr;   // the tail's tiles in the tensor-core order (umma_tail)
  uint8_t* w_front_um = nullptr;  // the front's tiles in the tensor-core order (umma_front)
  float* bias = nullptr;

  float* logits = nullptr;
  uint8_t* z_mx = nullptr;
  float* h_s = nullptr;
  uint8_t* h_mx = nullptr;
  float* y = nullptr;
  int* ids = nullptr;
  float* wts = nullptr;
  int* slots_sorted = nullptr;
  VExpert* ve = nullptr;
  int* nve = nullptr;
  Ctl* ctl = nullptr;  // [kSlots]
  int* done = nullptr;  // [4] phase completion counts of the fused launch
  int* counters[KIND_COUNT] = {};
  size_t counter_n[KIND_COUNT] = {};  // tickets per kind
  int* router_done = nullptr;
  int* route_ready = nullptr;
  float* partials[KIND_COUNT] = {};
  size_t partial_cap[KIND_COUNT] = {};  // floats
  float* side_partials = nullptr;       // the side lane's front (shared gate/up rows)
  float* rpart = nullptr;               // router pieces' partials, read by the routing CTA
  uint8_t* t_rec = nullptr;             // the tail's formed activation records
  int* t_ready = nullptr;
  int* route_cnt = nullptr;
  size_t rpart_floats = 0;
  size_t side_partial_cap = 0;
  cudaStream_t side = nullptr;          // the side lane's stream
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr, ev_egu = nullptr;
  bool side_env_off = false;            // environment MOE_SIDE_LANE=0
  // L2 prefetch of the chosen experts' tiles by the routing CTA, at most this
  // many bytes (environment MOE_PREFETCH_MB; 0 turns it off)
  long long prefetch_bytes = 0;
  // the routing CTA sums the router partials itself for few tokens
  // (environment MOE_DIRECT_ROUTE=0 turns it off)
  bool direct_route = true;
  // tokens a routing CTA selects (one a warp), and the most routing CTAs
  // (environment MOE_ROUTE_TPC, MOE_ROUTE_MAX_CTAS).  Measured per step:
  // b64 452.2 us with 8 tokens a CTA against 458.2 with 16; b8 and b128 the
  // same within noise (b128 351.7 vs 351.5)
  int route_tpc = 8, route_max_ctas = 16;
  // few tokens: the selection and table build of route_few (environment
  // MOE_ROUTE_FEW=0: the general path)
  bool route_few = true;
  // expert kernels on the 5th-generation tensor cores (block-scaled MMA of
  // e2m1 weights and e4m3 activation terms; environment MOE_UMMA=0 keeps
  // the warp-level MMA): decides the expert tiles' packed order and the
  // activation records' form, so it is fixed when the plan is made
  bool umma = true;
  int act_rec = kActRecBytesU;
  // the tail on the tensor cores (bf16 MMA of the formed records' hi and lo
  // parts) whenever its activation is staged from formed records; needs a
  // second copy of the tail's tiles (environment MOE_UMMA_TAIL=0 turns it off)
  bool umma_tail = true;
  // the front on the tensor cores (bf16 MMA with x) from two token tiles on;
  // a second copy of the front's tiles (environment MOE_UMMA_FRONT=0 turns it off)
  bool umma_front = true;
  bool w_front_um_ok = false;  // umma_front, and the plan takes more than 8 tokens
  int* err = nullptr;
  uint16_t* x_stage = nullptr;
  uint16_t* out_stage = nullptr;


  // tuning knobs read once at plan creation (environment): the price of a
  // split-K piece end in the split choice, whether kernels chain with
  // programmatic dependent launch, and whether small batches run fused
  int split_cost = 2;  // split-K piece-end price in stages (environment MOE_SPLIT_COST)
  // fixed split-K factors of the front and tail kernels (environment
  // MOE_FRONT_PPR, MOE_TAIL_PPR; 0: the makespan model's)
  int front_ppr_fixed = 0, tail_ppr_fixed = 0;
  int max_stages = 5;  // ring depth cap (environment MOE_MAX_STAGES)
  int expert_per_sm_max = 2;     // environment MOE_EXPERT_CTAS_PER_SM
  int expert_small_max_b = 128;  // environment MOE_EXPERT_SMALL_MAX_B
  int expert_tg_fixed = 0;       // environment MOE_EXPERT_TG (8, 16 or 32; 0: by batch size)
  // the expert kernels' split-K factor (environment MOE_EXPERT_PPR; 0: the
  // makespan model).  One piece a row block measured fastest: b1 75.2 - 75.6
  // us per step against 78.7 - 79.0 with the model, b8 152.2 - 152.6 against
  // 156.5 - 156.9 (paired runs on two boxes)
  int expert_ppr_fixed = 1;
  bool use_pdl = true;
  int fail_alloc_after = -1;     // environment MOE_FAIL_ALLOC_AFTER (tests only)
  int prod_sleep = 200, cons_sleep = 32;  // environment MOE_PROD_SLEEP / MOE_CONS_SLEEP (ns)
  // the tail streams its shared-expert part first, without waiting for the
  // routed experts (environment MOE_TAIL_SPLIT=0 turns it off)
  bool tail_split = true;
  // expert gate/up waits for the latent row blocks' count, not the whole
  // front grid (environment MOE_Z_FLAG=0 turns it off)
  bool z_flag = true;
  // the expert down kernel starts a virtual expert once the gate/up kernel's
  // row blocks of it are done, not after the whole gate/up grid
  // (environment MOE_H_FLAG=0 turns it off)
  bool h_flag = true;
  int* z_done = nullptr;
  int* h_done = nullptr;  // per virtual expert (ve_max)
  // one launch per forward for B <= kFusedMaxTokens (environment MOE_FUSED=1);
  // off by default: measured slower than the four-launch chain at B = 1
  bool use_fused = false;

  unsigned long long* trace = nullptr;  // [KIND_COUNT][max grid][8] when MOE_TRACE is set

  bool profiling = false;
  cudaEvent_t ev_prof[kSlots][2] = {};
  double prof_ms[kSlots] = {};
  int prof_count = 0;
};

// Live plans, so that destroying one clears every other plan's
// cross-layer prefetch of it.
std::mutex g_plans_mu;
std::vector<moe_plan_s*> g_plans;

// tokens per virtual expert for a forward of B tokens
int expert_tg(const moe_plan_s* p, int B) {
  if (p->expert_tg_fixed) return p->expert_tg_fixed;
  // the tensor-core kernels take 16-token groups above 64 tokens: two token
  // tiles cost their MMAs little, and a popular expert's weights are read
  // half as often (128 Zipf-skewed tokens: 578 vs 603 us per step; at 64
  // near-uniform tokens, where few experts see more than 8, 536 vs 515)
  if (p->umma && B > 64 && B <= p->expert_small_max_b) return kExpertTgUmmaLarge;
  return B <= p->expert_small_max_b ? kExpertTgSmall : kExpertTgLarge;
}

// Most virtual experts a forward with `slots` = B * k expert slots can have:
// an expert per slot (at most E) plus one group boundary per 8 slots.
int ve_bound(const moe_plan_s* p, int slots) {
  return std::min(p->ve_max, std::min(p->cfg.num_experts, slots) + ceil_div(slots, kExpertTgSmall) + 1);
}

// Whether a forward of B tokens runs the shared expert as a side lane.
// (shared_sms 0 is the measured choice: no side lane -- at B = 1 it took
// 95-100 us per step against 82-85 us with the shared expert's rows in the
// front pass and its down projection leading the tail)
bool side_lane(const moe_plan_s* p, int B) {
  return p->cfg.shared_inter > 0 && p->cfg.shared_sms > 0 && !p->side_env_off &&
         B <= kSideMaxTokens;
}

namespace {

struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

int pow2_at_least(int v) {
  int r = 1;
  while (r < v) r <<= 1;
  return r;
}

moe_status alloc(moe_plan p, void** out, size_t bytes, bool packed) {
  void* d = nullptr;
  if (bytes == 0) bytes = 16;
  // injected failure for tests of the OOM path (host side only): the plan's
  // countdown comes from MOE_FAIL_ALLOC_AFTER at plan creation
  if (p->fail_alloc_after >= 0 && p->fail_alloc_after-- == 0) return MOE_ERR_OOM;
  cudaError_t e = cudaMalloc(&d, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return e == cudaErrorMemoryAllocation ? MOE_ERR_OOM : MOE_ERR_CUDA;
  }
  p->allocs.push_back(d);
  (packed ? p->packed_bytes : p->workspace_bytes) += bytes;
  *out = d;
  return MOE_OK;
}

bool aligned16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; }

// Whether the front runs on the tensor cores: two token tiles or more (its
// MMA needs N >= 16), the whole SM (no side lane).
bool front_umma_for(const moe_plan_s* p, int nt, int budget) {
  return p->w_front_um_ok && nt >= 2 && budget > kHalfSmem;
}

int scratch_bytes(const moe_plan_s* p, int kind, int nt) {
  return ((kind == KIND_EGU || kind == KIND_EDN) && p->umma && nt <= 2) ? kScratchBytesUmmaSmall
                                                                          : kScratchBytes;
}

struct SmemGeom {
  int stage_bytes, nstages, act_off, act_stride, table_bytes, stage_off, res_bytes;
  int table_off;  // after the consumers' scratch
  size_t total;
};

// bytes of the tail's resident activation for B tokens (0: too large, use per-stage staging)
constexpr int kResidentMax = 72 * 1024;
int resident_stride(int res_k) { return res_k * 4 + 64; }

SmemGeom smem_geom(const moe_plan_s* p, int kind, int nt, int tail_tg_eff, int slots,
                   int res_bytes = 0, int budget = kBigSmem, bool formed = false) {
  const int topk = p->cfg.top_k, ve_max = ve_bound(p, slots);
  SmemGeom s;
  // routing tables (virtual experts + expert-sorted slots) for the expert kernels
  s.table_bytes = 0;
  if (kind == KIND_EGU || kind == KIND_EDN)
    s.table_bytes = ((ve_max * (int)sizeof(VExpert) + slots * 4) + 127) / 128 * 128;
  s.res_bytes = res_bytes;
  s.table_off = kScratchOff + scratch_bytes(p, kind, nt);
  const int stage_off = s.table_off + s.table_bytes + res_bytes;
  int act = 0;
  s.act_stride = 0;
  if (kind == KIND_FRONT) {
    s.act_stride = 192;
    // (the tensor-core front: 128 bytes a token, in core matrices)
    act = front_umma_for(p, nt, budget) ? 8 * nt * 128 : 8 * nt * s.act_stride;
  } else if ((kind == KIND_EGU || kind == KIND_EDN) && p->umma) {
    // tensor-core stage: unpacked codes, scales, the token-term rows
    s.act_stride = 0;
    s.act_off = kUBOff;
    s.stage_bytes = umma_stage_bytes(nt);
  } else if (kind == KIND_EGU || kind == KIND_EDN) {
    s.act_stride = 576;
    act = 8 * nt * s.act_stride;
  } else {
    // resident: none; formed records: 256 bytes a token (the tensor-core
    // tail: its 8 NT token rows, two 128-byte parts each); else the k slots'
    // y rows a token (the fused single launch)
    act = res_bytes ? 0
          : formed  ? (p->umma_tail ? 8 * nt * 256 : tail_tg_eff * 256)
                    : tail_tg_eff * std::max(1, topk) * 256;
  }
  const int tile = (kind == KIND_EGU || kind == KIND_EDN) ? kMxTileBytes : kDenseTileBytes;
  if (!((kind == KIND_EGU || kind == KIND_EDN) && p->umma)) {
    s.act_off = kHdr + tile;
    s.stage_bytes = ((kHdr + tile + act) + 127) / 128 * 128;
  }
  // one CTA per SM (the whole shared memory for the ring): a running kernel
  // and the next one, launched early by programmatic dependent launch, never
  // share an SM; with the half budget, two CTAs of one expert kernel do
  // enough bytes in flight to saturate HBM (about 6 x 16 KB per SM); more only
  // lengthens the queues every other memory request waits behind
  s.nstages = std::max(2, std::min(p->max_stages, (budget - stage_off) / s.stage_bytes));
  s.stage_off = stage_off;
  s.total = (size_t)stage_off + (size_t)s.nstages * s.stage_bytes;
  // more than half of the SM's shared memory: never two CTAs on one SM
  // (unless the budget is the half that two CTAs share)
  if (budget > kHalfSmem) s.total = std::max(s.total, (size_t)(116 * 1024));
  return s;
}

// token geometry of one forward
struct FwdGeom {
  int nt_front, nt_e, nt_tail, tail_tg;
  int front_grid, front_workers, tail_grid, expert_grid;
  int expert_per_sm;  // CTAs of each expert kernel per SM (1 or 2)
  int route_ctas;     // the front's routing CTAs (its last ones)
  bool side;          // the shared expert runs as a side lane
  int side_grid;      // CTAs of each side-lane kernel
  int budget;         // shared memory one CTA of the front and tail kernels may take
};

FwdGeom fwd_geom(const moe_plan_s* p, int B) {
  FwdGeom f;
  f.nt_front = pow2_at_least((B + 7) / 8);
  f.nt_e = pow2_at_least((std::min(B, expert_tg(p, B)) + 7) / 8);
  f.tail_tg = p->tail_tg;
  f.nt_tail = pow2_at_least((std::min(B, p->tail_tg) + 7) / 8);
  // every kernel takes every SM (one CTA each; the one-tile expert kernels
  // two, when half the shared memory still holds a ring of 3 stages); the
  // front kernel's last CTA is the routing CTA and streams nothing
  // one routing CTA selects up to route_tpc tokens (8: one a warp); more
  // tokens share the selection over more CTAs, the last of which builds the
  // tables
  f.route_ctas = std::max(1, std::min(p->route_max_ctas, (B + p->route_tpc - 1) / p->route_tpc));
  f.front_grid = p->num_sms;
  f.front_workers = p->num_sms - f.route_ctas;
  f.tail_grid = p->num_sms;
  f.expert_per_sm = 1;
  // (the tensor-core kernels: up to two token tiles, each CTA then holding
  // half the SM's tensor memory)
  if (f.nt_e <= (p->umma ? 2 : 1) && p->expert_per_sm_max >= 2) {
    const int slots = B * p->cfg.top_k;
    const SmemGeom h = smem_geom(p, KIND_EGU, f.nt_e, 1, slots, 0, kHalfSmem);
    if (h.nstages >= 3 && h.total <= (size_t)kHalfSmem) f.expert_per_sm = 2;
  }
  f.expert_grid = p->num_sms * f.expert_per_sm;
  f.side = side_lane(p, B);
  f.side_grid = f.side ? std::min(p->cfg.shared_sms, p->num_sms) : 0;
  f.budget = f.side ? kHalfSmem : kBigSmem;
  return f;
}

// Row blocks of the routed lane's front (router + latent rows) and the side
// lane's (the shared expert's gate/up rows).
int rb_routed(const moe_plan_s* p) { return p->RB_router + p->RB_lat; }
int rb_shared(const moe_plan_s* p) { return p->g[KIND_FRONT].RB - rb_routed(p); }

// Front split-K factor: over every row block, or over one lane's.  Its
// piece-end price in the makespan model is twice the base (a little more at
// 16 token tiles), as measured by sweeping the factor at the full-size
// dimensions (us per step): B = 1 pieces of 8 chunks 83.0 against 14 85.5
// (6: 84.6, 4: 89.1), B = 8 158.4 against 159.6, B = 128 7 pieces a row
// block 347.5 against 4 350.6 (10: 374.4); B = 64 keeps 7.
int front_ppr(const moe_plan_s* p, const FwdGeom& f, bool side_part) {
  const KindGeom& g = p->g[KIND_FRONT];
  if (p->front_ppr_fixed > 0) return std::min(p->front_ppr_fixed, g.C);
  const int cost = 2 * p->split_cost + f.nt_front / 16;
  if (!f.side) return best_ppr(g.RB, g.C, f.front_workers, cost);
  const int mats = side_part ? rb_shared(p) : rb_routed(p);
  const int ctas = side_part ? f.side_grid : f.front_workers;
  return best_ppr(mats, g.C, ctas, cost);
}

Params base_params(const moe_plan_s* p, int B) {
  Params q;
  std::memset(&q, 0, sizeof(q));
  const moe_config& c = p->cfg;
  q.H = c.hidden;
  q.L = c.latent;
  q.E = c.num_experts;
  q.topk = c.top_k;
  q.I = c.expert_inter;
  q.Is = c.shared_inter;
  q.B = B;
  q.score_fn = c.score_fn;
  q.renorm = c.renormalize;
  q.routed_scale = c.routed_scale;
  q.bias = p->bias;
  q.logits = p->logits;
  q.z_mx = p->z_mx;
  q.h_s = p->h_s;
  q.h_mx = p->h_mx;
  q.y = p->y;
  q.ld_slots = B * c.top_k;
  q.ids = p->ids;
  q.wts = p->wts;
  q.slots_sorted = p->slots_sorted;
  q.ve = p->ve;
  q.nve = p->nve;
  q.ve_max = ve_bound(p, B * c.top_k);
  q.router_done = p->router_done;
  q.route_ready = p->route_ready;
  q.err = p->err;
  q.z_done = p->z_flag ? p->z_done : nullptr;
  q.h_done = p->h_flag ? p->h_done : nullptr;
  q.RB_egu = p->g[KIND_EGU].RB;
  q.t_ready = p->t_ready;
  q.route_cnt = p->route_cnt;
  q.RB_lat = p->RB_lat;
  q.prod_sleep = p->prod_sleep;
  q.cons_sleep = p->cons_sleep;
  q.C_lat = p->C_lat;
  q.KS = c.shared_inter;
  q.scratch_off = kScratchOff;
  q.umma = p->umma ? 1 : 0;
  q.act_rec = p->act_rec;
  return q;
}

void set_kind(Params& q, const moe_plan_s* p, int kind, const SmemGeom& s) {
  q.RB = p->g[kind].RB;
  q.C = p->g[kind].C;
  q.KL = p->g[kind].KL;
  q.ctl = p->ctl + kind;
  q.trace = p->trace ? p->trace + (size_t)kind * 2 * p->num_sms * 24 : nullptr;
  q.counters = p->counters[kind];
  q.partials = p->partials[kind];
  q.nstages = s.nstages;
  q.stage_bytes = s.stage_bytes;
  q.act_off = s.act_off;
  q.act_stride = s.act_stride;
  q.table_off = s.table_off;
  q.stage_off = s.stage_off;
  q.matrix_bytes = (long long)p->g[kind].weight_bytes;
  switch (kind) {
    case KIND_FRONT: {  // its routing CTA groups expert tokens by tg
      q.wt = p->w_front;
      q.rb_lo = 0;
      q.rb_hi = p->g[KIND_FRONT].RB;
      q.pf_egu = p->w_egu;
      q.pf_edn = p->w_edn;
      q.pf_egu_bytes = (long long)p->g[KIND_EGU].weight_bytes;
      q.pf_edn_bytes = (long long)p->g[KIND_EDN].weight_bytes;
      const long long per = q.pf_egu_bytes + q.pf_edn_bytes;
      q.pf_ves = per > 0 ? (int)std::min<long long>(p->ve_max, p->prefetch_bytes / per) : 0;
      q.tg = expert_tg(p, q.B);
      q.RB_router = p->RB_router;
      q.RB_lat = p->RB_lat;
      q.route_cta = 1;
      break;
    }
    case KIND_EGU: q.wt = p->w_egu; q.tg = expert_tg(p, q.B); q.PPR = p->expert_ppr_fixed; break;
    case KIND_EDN: q.wt = p->w_edn; q.tg = expert_tg(p, q.B); q.PPR = p->expert_ppr_fixed; break;
    default: q.wt = p->w_tail; q.tg = p->tail_tg; break;
  }
}

// Price of a split-K piece end in stages: partial sums out and the
// finalising sums back in grow with the piece's token tiles, but more slowly
// than a stage's own work does (a stage of 16 tiles costs about 2x one of 1).
int split_cost_for(const moe_plan_s* p, int nt) { return p->split_cost * (1 + std::max(1, nt) / 4); }

// split-K factor of a kind whose row-block count the host knows
int ppr_for(const moe_plan_s* p, int mats, int C, int ctas, int nt) {
  return best_ppr(mats, C, ctas, split_cost_for(p, nt));
}

// The expert kernels' split-K factor for `mats` row blocks (the device
// computes the same from the routing's count of virtual experts), or the
// fixed one of MOE_EXPERT_PPR (at most the chunk count).
int expert_ppr(const moe_plan_s* p, int mats, int C, int ctas, int nt) {
  if (p->expert_ppr_fixed > 0) return std::min(p->expert_ppr_fixed, C);
  return ppr_for(p, mats, C, ctas, nt);
}

// Router row blocks are the first pieces handed out and the routing waits
// for all of them: they get pieces of at most ~C/12 chunks.
// (Dealing them over every CTA instead -- each CTA's first piece a router
// piece -- brought the logits no earlier at B = 1 and cost 30 us at B = 128,
// where every router piece writes 64 KB of partial sums.)
int router_ppr(int ppr, int C) { return std::max(1, std::min(C, std::max(ppr, 12))); }

// The tail's pieces per row block with its shared part first: ppr pieces
// split between the latent chunks and the shared-expert chunks in proportion
// (at least one each, at most one chunk a piece); without a shared expert,
// or with the split off, one split over all chunks (ppr_sh = 0).
struct TailSplit {
  int ppr_lat, ppr_sh;
};
// The split pays where the tail keeps its activation resident (at most 4
// tokens: b1 92 -> 84 us per step); with staged activations it cost about
// 10% of the tail (b64 109 -> 119 us), so larger batches keep one split.
TailSplit tail_split_for(const moe_plan_s* p, int ppr, int B) {
  const int C = p->g[KIND_TAIL].C, C_lat = p->C_lat, C_sh = C - p->C_lat;
  if (!p->tail_split || C_sh <= 0 || B > kSideMaxTokens) return {ppr, 0};
  int lat = (int)std::lround((double)ppr * C_lat / C);
  lat = std::max(1, std::min(C_lat, lat));
  const int sh = std::max(1, std::min(C_sh, ppr - lat));
  return {lat, sh};
}
// The tail's split-K factor over `mats` row blocks (before the lane split).
// Its piece-end price depends on how the activation reaches the stages, as
// measured by sweeping the factor at the full-size dimensions (us per step):
//   resident activation (few tokens): three times the base, B = 1 pieces of
//     13 chunks (5 a row block) 81.8 against 8 85.5;
//   formed records, one or two token tiles: half the base, B = 8 13 pieces
//     a row block 156.9 against 8 159.6;
//   formed records, more tiles: the token-tile scaled price plus one, 4
//     pieces a row block at B = 64 (444.2 against 5 451.8; 3: 453.4) and
//     at B = 128 (350.6; 3: 353.4).
int tail_base_ppr(const moe_plan_s* p, int B, int mats, int ctas, int nt) {
  const int C = p->g[KIND_TAIL].C;
  if (p->tail_ppr_fixed > 0) return std::min(p->tail_ppr_fixed, C);
  const bool resident = B * resident_stride(C * kDenseChunkK) <= kResidentMax;
  const int cost = resident ? 3 * p->split_cost
                   : nt <= 2 ? p->split_cost / 2
                             : p->split_cost * (1 + nt / 4) + 1;
  if (!resident) return best_ppr(mats, C, ctas, cost);
  // resident: of equal makespans the finer split (the 4 row blocks of 8
  // chunks at the tiny dimensions: 8 pieces 26.0 us per step against 1 27.1)
  int best = 1;
  long long best_t = -1;
  for (int ppr = 1; ppr <= C; ++ppr) {
    const long long piece = ceil_div(C, ppr) + (ppr > 1 ? cost : 0);
    const long long t = ((long long)mats * ppr * piece + ctas - 1) / ctas + piece;
    if (best_t < 0 || t <= best_t) {
      best_t = t;
      best = ppr;
    }
  }
  return best;
}
int tail_ppr(const moe_plan_s* p, int ppr, int B) {
  const TailSplit t = tail_split_for(p, ppr, B);
  return t.ppr_lat + t.ppr_sh;
}

// largest number of partial-sum floats the side lane's front can need
size_t side_partial_floats(const moe_plan_s* p) {
  size_t best = 0;
  for (int B = 1; B <= p->cfg.max_tokens; ++B) {
    const FwdGeom f = fwd_geom(p, B);
    if (!f.side) continue;
    best = std::max(best, (size_t)rb_shared(p) * front_ppr(p, f, true) * f.nt_front * 1024);
  }
  return best;
}

// largest number of partial-sum floats a kind can need for B <= maxB
size_t partial_floats(const moe_plan_s* p, int kind) {
  size_t best = 0;
  for (int B = 1; B <= p->cfg.max_tokens; ++B) {
    FwdGeom f = fwd_geom(p, B);
    size_t pieces = 0;
    int nt = 1;
    const KindGeom& g = p->g[kind];
    if (kind == KIND_FRONT) {
      nt = f.nt_front;
      const int ppr = front_ppr(p, f, false);
      const int rb_hi = f.side ? rb_routed(p) : g.RB;
      pieces = (size_t)p->RB_router * router_ppr(ppr, g.C) + (size_t)(rb_hi - p->RB_router) * ppr;
      if (p->use_fused && B <= kFusedMaxTokens) {
        // the single launch: every row block, never a side lane
        FwdGeom fg = f;
        fg.side = false;
        const int pf = front_ppr(p, fg, false);
        pieces = std::max(pieces, (size_t)p->RB_router * router_ppr(pf, g.C) + (size_t)(g.RB - p->RB_router) * pf);
      }
    } else if (kind == KIND_TAIL) {
      nt = f.nt_tail;
      const int passes = (B + p->tail_tg - 1) / p->tail_tg;
      pieces = (size_t)passes * g.RB * tail_ppr(p, tail_base_ppr(p, B, g.RB * passes, f.tail_grid, nt), B);
    } else {
      nt = f.nt_e;
      // the split depends on the routing: take the largest over every
      // possible count of virtual experts
      for (int V = 1; V <= p->ve_max; ++V)
        pieces = std::max(pieces, (size_t)V * g.RB * expert_ppr(p, V * g.RB, g.C, f.expert_grid, nt));
    }
    best = std::max(best, pieces * (size_t)nt * 1024);
  }
  return best;
}

#define TRY(x)                          \
  do {                                  \
    moe_status _s = (x);                \
    if (_s != MOE_OK) return _s;        \
  } while (0)
#define CUDA_TRY(x)                      \
  do {                                   \
    if ((x) != cudaSuccess) {            \
      cudaGetLastError();                \
      return MOE_ERR_CUDA;               \
    }                                    \
  } while (0)

moe_status check_cfg(const moe_config* c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->hidden <= 0 || c->latent <= 0 || c->num_experts <= 0 || c->expert_inter <= 0 ||
      c->shared_inter < 0 || c->top_k <= 0 || c->max_tokens <= 0)
    return MOE_ERR_INVALID_ARG;
  if (c->hidden % 32 || c->latent % 32 || c->expert_inter % 32 || c->shared_inter % 32)
    return MOE_ERR_INVALID_ARG;
  if (c->top_k > c->num_experts) return MOE_ERR_INVALID_ARG;
  if (c->score_fn != MOE_SCORE_SOFTMAX && c->score_fn != MOE_SCORE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (!(c->routed_scale == c->routed_scale)) return MOE_ERR_INVALID_ARG;
  if (c->shared_sms < -1) return MOE_ERR_INVALID_ARG;
  if (c->num_experts > 1024 || c->top_k > 16 || c->max_tokens > 128) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// Row blocks, chunks and packed sizes of every kind, the tail's token group
// and the routing-table bound: everything about a plan that follows from its
// shape alone (no device involved).
void plan_shape(moe_plan_s* p) {
  const moe_config& c = p->cfg;
  const int H = c.hidden, L = c.latent, E = c.num_experts, I = c.expert_inter, Is = c.shared_inter;
  // the front kernel's row blocks: router (first, so the routing starts
  // early), latent projection, shared expert gate/up (64 + 64 rows a block)
  p->RB_router = ceil_div(E, kRowsPerBlock);
  p->RB_lat = ceil_div(L, kRowsPerBlock);
  KindGeom& fr = p->g[KIND_FRONT];
  fr.RB = p->RB_router + p->RB_lat + ceil_div(Is, 64);
  fr.C = ceil_div(H, kDenseChunkK);
  fr.KL = H;
  fr.weight_bytes = (size_t)fr.RB * fr.C * kDenseTileBytes;
  KindGeom& eg = p->g[KIND_EGU];
  eg.RB = ceil_div(I, 64);
  eg.C = ceil_div(L, kMxChunkK);
  eg.KL = L;
  eg.weight_bytes = (size_t)eg.RB * eg.C * kMxTileBytes;
  KindGeom& ed = p->g[KIND_EDN];
  ed.RB = ceil_div(L, kRowsPerBlock);
  ed.C = ceil_div(I, kMxChunkK);
  ed.KL = I;
  ed.weight_bytes = (size_t)ed.RB * ed.C * kMxTileBytes;
  KindGeom& tl = p->g[KIND_TAIL];
  p->C_lat = ceil_div(L, kDenseChunkK);
  tl.RB = ceil_div(H, kRowsPerBlock);
  tl.C = p->C_lat + ceil_div(Is, kDenseChunkK);
  tl.KL = L;
  tl.weight_bytes = (size_t)tl.RB * tl.C * kDenseTileBytes;
  p->tail_tg = kTailTg;

  const int maxB = c.max_tokens, K = c.top_k;
  const int slots = maxB * K;
  p->ve_max = std::min(E, slots) + ceil_div(slots, kExpertTgSmall) + 1;  // any group size
}

// Tuning knobs and switches from the environment, read when a plan is made
// (and by moe_debug_geometry, which reports what such a plan would launch).
void read_env(moe_plan_s* p) {
  if (const char* e = getenv("MOE_SPLIT_COST")) p->split_cost = std::max(0, atoi(e));
  if (const char* e = getenv("MOE_FRONT_PPR")) p->front_ppr_fixed = std::max(0, std::min(64, atoi(e)));
  if (const char* e = getenv("MOE_TAIL_PPR")) p->tail_ppr_fixed = std::max(0, std::min(64, atoi(e)));
  if (const char* e = getenv("MOE_EXPERT_CTAS_PER_SM")) p->expert_per_sm_max = std::max(1, std::min(2, atoi(e)));
  if (const char* e = getenv("MOE_EXPERT_SMALL_MAX_B")) p->expert_small_max_b = std::max(0, atoi(e));
  if (const char* e = getenv("MOE_EXPERT_PPR")) p->expert_ppr_fixed = std::max(0, std::min(8, atoi(e)));
  if (const char* e = getenv("MOE_EXPERT_TG")) {
    const int v = atoi(e);
    p->expert_tg_fixed = (v == 8 || v == 16 || v == 32) ? v : 0;
  }
  if (const char* e = getenv("MOE_NO_PDL")) p->use_pdl = atoi(e) == 0;
  if (const char* e = getenv("MOE_FUSED")) p->use_fused = atoi(e) != 0;
  if (const char* e = getenv("MOE_MAX_STAGES")) p->max_stages = std::max(2, std::min(8, atoi(e)));
  if (const char* e = getenv("MOE_FAIL_ALLOC_AFTER")) p->fail_alloc_after = std::max(0, atoi(e));
  if (const char* e = getenv("MOE_PROD_SLEEP")) p->prod_sleep = std::max(0, std::min(2000, atoi(e)));
  if (const char* e = getenv("MOE_TAIL_SPLIT")) p->tail_split = atoi(e) != 0;
  if (const char* e = getenv("MOE_Z_FLAG")) p->z_flag = atoi(e) != 0;
  if (const char* e = getenv("MOE_H_FLAG")) p->h_flag = atoi(e) != 0;
  if (const char* e = getenv("MOE_SIDE_LANE")) p->side_env_off = atoi(e) == 0;
  if (const char* e = getenv("MOE_PREFETCH_MB")) p->prefetch_bytes = std::max(0LL, (long long)atoi(e)) << 20;
  if (const char* e = getenv("MOE_DIRECT_ROUTE")) p->direct_route = atoi(e) != 0;
  if (const char* e = getenv("MOE_ROUTE_FEW")) p->route_few = atoi(e) != 0;
  if (const char* e = getenv("MOE_ROUTE_TPC")) p->route_tpc = std::max(1, std::min(128, atoi(e)));
  if (const char* e = getenv("MOE_ROUTE_MAX_CTAS")) p->route_max_ctas = std::max(1, std::min(32, atoi(e)));
  if (const char* e = getenv("MOE_CONS_SLEEP")) p->cons_sleep = std::max(0, std::min(2000, atoi(e)));
  if (const char* e = getenv("MOE_UMMA")) p->umma = atoi(e) != 0;
  if (const char* e = getenv("MOE_UMMA_TAIL")) p->umma_tail = atoi(e) != 0;
  p->umma_tail = p->umma_tail && p->umma;
  if (const char* e = getenv("MOE_UMMA_FRONT")) p->umma_front = atoi(e) != 0;
  p->umma_front = p->umma_front && p->umma;
  p->w_front_um_ok = p->umma_front && p->cfg.max_tokens > 8;
  p->act_rec = p->umma ? kActRecBytesU : kActRecBytes;
  if (p->umma) p->use_fused = false;  // the single launch keeps the warp-level MMA
}

// The control block (routing count, router-row count, error word, routing
// flag, phase counts, per-kind piece cursors) and every kind's split-K
// tickets back to zero, as a fresh plan has them.  Synchronous.
constexpr size_t kControlBytes = 1024 + sizeof(Ctl) * kSlots;
moe_status reset_control(moe_plan p) {
  CUDA_TRY(cudaMemset(p->nve, 0, kControlBytes));
  CUDA_TRY(cudaMemset(p->rpart, 0xFF, sizeof(float) * p->rpart_floats));  // "not yet written"
  for (int k = 0; k < KIND_COUNT; ++k) CUDA_TRY(cudaMemset(p->counters[k], 0, sizeof(int) * p->counter_n[k]));
  CUDA_TRY(cudaDeviceSynchronize());
  return MOE_OK;
}

moe_status create_impl(const moe_config* cfg, int device, moe_plan p) {
  p->cfg = *cfg;
  p->device = device;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
    cudaGetLastError();
    return MOE_ERR_UNSUPPORTED;
  }
  cudaDeviceProp prop;
  CUDA_TRY(cudaGetDeviceProperties(&prop, device));
  if (prop.major != 10) return MOE_ERR_UNSUPPORTED;  // built for sm_100a only
  p->num_sms = prop.multiProcessorCount;
  read_env(p);
  if (set_smem_limits(kBigSmem) != 0) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }

  const moe_config& c = *cfg;
  const int H = c.hidden, L = c.latent, E = c.num_experts, I = c.expert_inter, Is = c.shared_inter;
  plan_shape(p);
  KindGeom& fr = p->g[KIND_FRONT];
  KindGeom& eg = p->g[KIND_EGU];
  KindGeom& ed = p->g[KIND_EDN];
  KindGeom& tl = p->g[KIND_TAIL];
  const int maxB = c.max_tokens, K = c.top_k;
  const int slots = maxB * K;

  void* v;
  TRY(alloc(p, &v, fr.weight_bytes, true));
  p->w_front = (uint8_t*)v;
  if (p->w_front_um_ok) {  // (the tensor-core front takes more than 8 tokens)
    TRY(alloc(p, &v, fr.weight_bytes, true));
    p->w_front_um = (uint8_t*)v;
  }
  TRY(alloc(p, &v, (size_t)E * eg.weight_bytes, true));
  p->w_egu = (uint8_t*)v;
  TRY(alloc(p, &v, (size_t)E * ed.weight_bytes, true));
  p->w_edn = (uint8_t*)v;
  TRY(alloc(p, &v, tl.weight_bytes, true));
  p->w_tail = (uint8_t*)v;
  if (p->umma_tail) {
    TRY(alloc(p, &v, tl.weight_bytes, true));
    p->w_tail_um = (uint8_t*)v;
  }
  TRY(alloc(p, &v, sizeof(float) * E, true));
  p->bias = (float*)v;

  TRY(alloc(p, &v, sizeof(float) * maxB * E, false));
  p->logits = (float*)v;
  // (zeroed: the entries past L and I are never written and must read as 0)
  TRY(alloc(p, &v, (size_t)maxB * ceil_div(L, kMxChunkK) * p->act_rec, false));
  p->z_mx = (uint8_t*)v;
  CUDA_TRY(cudaMemset(v, 0, (size_t)maxB * ceil_div(L, kMxChunkK) * p->act_rec));
  TRY(alloc(p, &v, sizeof(float) * (size_t)ceil_div(std::max(Is, 1), 64) * maxB * 64, false));
  p->h_s = (float*)v;
  TRY(alloc(p, &v, (size_t)ceil_div(I, kMxChunkK) * slots * p->act_rec, false));
  p->h_mx = (uint8_t*)v;
  CUDA_TRY(cudaMemset(v, 0, (size_t)ceil_div(I, kMxChunkK) * slots * p->act_rec));
  TRY(alloc(p, &v, sizeof(float) * (size_t)ceil_div(L, 64) * slots * 64, false));
  p->y = (float*)v;
  TRY(alloc(p, &v, sizeof(int) * slots, false));
  p->ids = (int*)v;
  TRY(alloc(p, &v, sizeof(float) * slots, false));
  p->wts = (float*)v;
  TRY(alloc(p, &v, sizeof(int) * slots, false));
  p->slots_sorted = (int*)v;
  TRY(alloc(p, &v, sizeof(VExpert) * p->ve_max, false));
  p->ve = (VExpert*)v;
  TRY(alloc(p, &v, sizeof(int) * p->ve_max, false));
  p->h_done = (int*)v;
  CUDA_TRY(cudaMemset(v, 0, sizeof(int) * p->ve_max));
  // small control block: nve, router_done, err, Ctl[KIND_COUNT]
  TRY(alloc(p, &v, kControlBytes, false));
  p->nve = (int*)v;
  p->router_done = p->nve + 1;
  p->err = p->nve + 2;
  p->done = p->nve + 8;
  p->route_ready = p->nve + 3;
  p->z_done = p->nve + 5;  // (nve + 4: a flag nothing sets, for the expiring-wait test)
  p->t_ready = p->nve + 6;
  p->route_cnt = p->nve + 7;
  p->ctl = reinterpret_cast<Ctl*>((uint8_t*)v + 1024);
  CUDA_TRY(cudaMemset(v, 0, kControlBytes));
  const int cnt_n[KIND_COUNT] = {fr.RB, p->ve_max * eg.RB, p->ve_max * ed.RB, maxB * tl.RB};
  for (int k = 0; k < KIND_COUNT; ++k) {
    p->counter_n[k] = cnt_n[k];
    TRY(alloc(p, &v, sizeof(int) * cnt_n[k], false));
    p->counters[k] = (int*)v;
    CUDA_TRY(cudaMemset(v, 0, sizeof(int) * cnt_n[k]));
    p->partial_cap[k] = partial_floats(p, k);
    TRY(alloc(p, &v, sizeof(float) * std::max<size_t>(p->partial_cap[k], 4), false));
    p->partials[k] = (float*)v;
  }
  // router pieces' partial sums for the routing CTA (few tokens: one token
  // tile, at most one piece per chunk), every element "not yet written"
  p->rpart_floats = (size_t)p->RB_router * fr.C * 8 * kRowsPerBlock;
  TRY(alloc(p, &v, sizeof(float) * p->rpart_floats, false));
  p->rpart = (float*)v;
  CUDA_TRY(cudaMemset(v, 0xFF, sizeof(float) * p->rpart_floats));
  // the tail's formed activation records, [C chunks][max_tokens][256 bytes]
  TRY(alloc(p, &v, (size_t)tl.C * maxB * 256, false));
  p->t_rec = (uint8_t*)v;
  p->side_partial_cap = side_partial_floats(p);
  TRY(alloc(p, &v, sizeof(float) * std::max<size_t>(p->side_partial_cap, 4), false));
  p->side_partials = (float*)v;
  CUDA_TRY(cudaStreamCreateWithFlags(&p->side, cudaStreamNonBlocking));
  CUDA_TRY(cudaEventCreateWithFlags(&p->ev_fork, cudaEventDisableTiming));
  CUDA_TRY(cudaEventCreateWithFlags(&p->ev_join, cudaEventDisableTiming));
  CUDA_TRY(cudaEventCreateWithFlags(&p->ev_egu, cudaEventDisableTiming));
  if (getenv("MOE_TRACE")) {
    // rows for up to two CTAs per SM in every slot
    TRY(alloc(p, &v, sizeof(unsigned long long) * kSlots * 2 * p->num_sms * 24, false));
    p->trace = (unsigned long long*)v;
    CUDA_TRY(cudaMemset(v, 0, sizeof(unsigned long long) * kSlots * 2 * p->num_sms * 24));
  }
  TRY(alloc(p, &v, sizeof(uint16_t) * (size_t)maxB * H, false));
  p->x_stage = (uint16_t*)v;
  TRY(alloc(p, &v, sizeof(uint16_t) * (size_t)maxB * H, false));
  p->out_stage = (uint16_t*)v;

  for (int k = 0; k < kSlots; ++k)
    for (int j = 0; j < 2; ++j) CUDA_TRY(cudaEventCreate(&p->ev_prof[k][j]));
  CUDA_TRY(cudaDeviceSynchronize());
  if (getenv("MOE_LOG")) {
    fprintf(stderr,
            "[moe] plan dev=%d sms=%d H=%d L=%d E=%d k=%d I=%d Is=%d maxB=%d packed=%.1fMB "
            "workspace=%.1fMB\n",
            device, p->num_sms, H, L, E, K, I, Is, maxB, p->packed_bytes / 1e6,
            p->workspace_bytes / 1e6);
  }
  return MOE_OK;
}

void destroy_impl(moe_plan p) {
  if (!p) return;
  {
    std::lock_guard<std::mutex> lk(g_plans_mu);
    g_plans.erase(std::remove(g_plans.begin(), g_plans.end(), p), g_plans.end());
    for (moe_plan_s* o : g_plans)
      if (o->next_layer == p) {
        o->next_layer = nullptr;
        o->next_bytes = 0;
      }
  }
  DeviceGuard g(p->device);
  cudaDeviceSynchronize();
  for (void* a : p->allocs) cudaFree(a);
  for (int k = 0; k < kSlots; ++k)
    for (int j = 0; j < 2; ++j)
      if (p->ev_prof[k][j]) cudaEventDestroy(p->ev_prof[k][j]);
  if (p->ev_fork) cudaEventDestroy(p->ev_fork);
  if (p->ev_join) cudaEventDestroy(p->ev_join);
  if (p->ev_egu) cudaEventDestroy(p->ev_egu);
  if (p->side) cudaStreamDestroy(p->side);
  cudaGetLastError();
  delete p;
}

// The whole block as one launch (B <= kFusedMaxTokens): every phase's
// Params share one shared-memory layout -- routing tables, the tail's resident
// activation, and a ring of the largest stage any phase needs.
moe_status enqueue_fused(moe_plan p, const Params& base, const FwdGeom& f, int B, cudaStream_t s) {
  const moe_config& c = p->cfg;
  const int tail_tg_eff = std::min(B, p->tail_tg);
  const int res_k = p->g[KIND_TAIL].C * kDenseChunkK;
  const int res_bytes = (B * resident_stride(res_k) <= kResidentMax) ? B * resident_stride(res_k) : 0;
  SmemGeom g[KIND_COUNT];
  int stage_bytes = 0;
  for (int k = 0; k < KIND_COUNT; ++k) {
    g[k] = smem_geom(p, k, 1, tail_tg_eff, B * c.top_k, k == KIND_TAIL ? res_bytes : 0);
    stage_bytes = std::max(stage_bytes, g[k].stage_bytes);
  }
  const int table_bytes = g[KIND_EGU].table_bytes;
  const int stage_off = kStageOff + table_bytes + res_bytes;
  const int nstages = std::max(2, std::min(p->max_stages, (kBigSmem - stage_off) / stage_bytes));
  const size_t total = std::max((size_t)stage_off + (size_t)nstages * stage_bytes, (size_t)(116 * 1024));
  MegaParams mp;
  std::memset(&mp, 0, sizeof(mp));
  for (int k = 0; k < KIND_COUNT; ++k) {
    Params q = base;
    set_kind(q, p, k, g[k]);
    q.nstages = nstages;
    q.stage_bytes = stage_bytes;
    q.stage_off = stage_off;
    q.table_off = kStageOff;
    q.ctl = p->ctl + kFused;
    q.z_done = nullptr;  // the single launch counts phases in `done`
    q.h_done = nullptr;
    q.trace = p->trace ? p->trace + (size_t)kFused * 2 * p->num_sms * 24 : nullptr;
    q.done = p->done;
    q.need_rb_edn = p->g[KIND_EDN].RB;
    q.need_rb_sh = p->g[KIND_FRONT].RB - p->RB_router - p->RB_lat;
    // (split factors from the functions that size the partial-sum buffers)
    if (k == KIND_FRONT) {
      FwdGeom fg = f;
      fg.side = false;
      q.PPR = front_ppr(p, fg, false);
      q.PPR_r = router_ppr(q.PPR, q.C);
      mp.n_front = p->RB_router * q.PPR_r + (q.RB - p->RB_router) * q.PPR;
    } else if (k == KIND_EGU || k == KIND_EDN) {
      q.piece_ctas = f.expert_grid;
      q.split_cost = split_cost_for(p, 1);
    } else {
      if (res_bytes) {
        q.res_off = kStageOff + table_bytes;
        q.res_stride = resident_stride(res_k);
        q.res_k = res_k;
      }
      const int passes = (B + p->tail_tg - 1) / p->tail_tg;
      q.PPR = tail_base_ppr(p, B, q.RB * passes, f.tail_grid, 1);
    }
    mp.k[k] = q;
  }
  if (p->profiling) CUDA_TRY(cudaEventRecord(p->ev_prof[kFused][0], s));
  CUDA_TRY((cudaError_t)launch_mega(mp, p->num_sms, total, s, p->use_pdl));
  if (p->profiling) {
    CUDA_TRY(cudaEventRecord(p->ev_prof[kFused][1], s));
    CUDA_TRY(cudaEventSynchronize(p->ev_prof[kFused][1]));
    float ms = 0.f;
    CUDA_TRY(cudaEventElapsedTime(&ms, p->ev_prof[kFused][0], p->ev_prof[kFused][1]));
    p->prof_ms[kFused] += ms;
    ++p->prof_count;
  }
  p->last_B = B;
  return MOE_OK;
}

// Front launch of one forward: every row block (part 0), the routed lane's
// router + latent rows with the routing CTA (part 1), or the side lane's
// shared-expert gate/up rows (part 2).
struct FrontLaunch {
  SmemGeom sm;
  int grid, ppr, ppr_r, rb_lo, rb_hi, route_cta;
};
FrontLaunch front_launch(const moe_plan_s* p, const FwdGeom& f, int B, int part) {
  FrontLaunch l;
  const int tail_tg_eff = std::min(B, p->tail_tg);
  l.sm = smem_geom(p, KIND_FRONT, f.nt_front, tail_tg_eff, B * p->cfg.top_k, 0, f.budget);
  const KindGeom& g = p->g[KIND_FRONT];
  l.ppr = front_ppr(p, f, part == 2);
  l.ppr_r = router_ppr(l.ppr, g.C);
  l.rb_lo = part == 2 ? rb_routed(p) : 0;
  l.rb_hi = part == 1 ? rb_routed(p) : g.RB;
  l.route_cta = part == 2 ? 0 : f.route_ctas;
  l.grid = part == 2 ? f.side_grid : f.front_grid;
  return l;
}

// Tail launch: every piece (part 0, shared part first), the latent pieces
// (part 1, the routed lane) or the shared-expert pieces (part 2, the side
// lane).  A lane keeps only its own part of the resident activation.
struct TailLaunch {
  SmemGeom sm;
  int grid, ppr, ppr_lat, ppr_sh, split, res_bytes, res_k0, res_k;
  bool formed;  // staged activations from formed records (not resident)
};
TailLaunch tail_launch(const moe_plan_s* p, const FwdGeom& f, int B, int part) {
  TailLaunch l;
  const int tail_tg_eff = std::min(B, p->tail_tg);
  const KindGeom& g = p->g[KIND_TAIL];
  const int klat = p->C_lat * kDenseChunkK, kall = g.C * kDenseChunkK;
  l.res_k0 = part == 2 ? klat : 0;
  l.res_k = part == 1 ? klat : (part == 2 ? kall - klat : kall);
  l.res_bytes = (B * resident_stride(l.res_k) <= kResidentMax) ? B * resident_stride(l.res_k) : 0;
  l.formed = l.res_bytes == 0;
  l.sm = smem_geom(p, KIND_TAIL, f.nt_tail, tail_tg_eff, B * p->cfg.top_k, l.res_bytes, f.budget,
                   l.formed);
  const int passes = (B + p->tail_tg - 1) / p->tail_tg;
  const int grid = part == 2 ? f.side_grid : f.tail_grid;
  // one split for both lanes: they share every row block's partial-sum slots
  // and its ticket count
  const TailSplit ts = tail_split_for(p, tail_base_ppr(p, B, g.RB * passes, f.tail_grid, f.nt_tail), B);
  l.ppr_lat = ts.ppr_lat;
  l.ppr_sh = ts.ppr_sh;
  l.ppr = ts.ppr_lat + ts.ppr_sh;
  l.split = ts.ppr_sh > 0;
  l.grid = grid;
  return l;
}

moe_status launch_timed(moe_plan p, int slot, int kind, int nt, const Params& q, int grid, size_t smem,
                        cudaStream_t s) {
  if (p->profiling) CUDA_TRY(cudaEventRecord(p->ev_prof[slot][0], s));
  CUDA_TRY((cudaError_t)launch_kind(kind, nt, q, grid, smem, s, p->use_pdl));
  if (p->profiling) CUDA_TRY(cudaEventRecord(p->ev_prof[slot][1], s));
  return MOE_OK;
}

moe_status enqueue_forward(moe_plan p, const void* x, int B, void* out, cudaStream_t s) {
  const moe_config& c = p->cfg;
  const FwdGeom f = fwd_geom(p, B);
  const int tail_tg_eff = std::min(B, p->tail_tg);
  Params base = base_params(p, B);
  base.x = (const uint16_t*)x;
  base.out = (uint16_t*)out;
  if (p->use_fused && B <= kFusedMaxTokens) return enqueue_fused(p, base, f, B, s);

  // Routed chain on `s`, each kernel a programmatic dependent of the one
  // before: front (router, latent [, shared gate/up]) -> expert gate/up ->
  // expert down -> tail.  With the side lane, the shared expert's gate/up
  // rows and its down projection run as two kernels of their own on the
  // plan's side stream (forked from and joined back to `s`), their CTAs
  // sharing the SMs with the routed chain's: the shared expert overlaps the
  // routing and the routed experts ("Hyper Optimizing Kimi K3 in vLLM",
  // section 从算子之间找时间), and it streams while the routed chain waits at
  // its kernel boundaries.  The two lanes meet in the tail's row blocks.
  if (f.side) {
    CUDA_TRY(cudaEventRecord(p->ev_fork, s));
    CUDA_TRY(cudaStreamWaitEvent(p->side, p->ev_fork, 0));
    {
      Params q = base;
      const FrontLaunch l = front_launch(p, f, B, 2);
      set_kind(q, p, KIND_FRONT, l.sm);
      q.ctl = p->ctl + kSideFront;
      q.trace = p->trace ? p->trace + (size_t)kSideFront * 2 * p->num_sms * 24 : nullptr;
      q.partials = p->side_partials;
      q.PPR = l.ppr;
      q.PPR_r = l.ppr_r;
      q.rb_lo = l.rb_lo;
      q.rb_hi = l.rb_hi;
      q.route_cta = 0;
      q.half_sm = 1;
      TRY(launch_timed(p, kSideFront, KIND_FRONT, f.nt_front, q, l.grid, l.sm.total, p->side));
    }
  }
  {
    Params q = base;
    const FrontLaunch l = front_launch(p, f, B, f.side ? 1 : 0);
    set_kind(q, p, KIND_FRONT, l.sm);
    q.PPR = l.ppr;
    q.PPR_r = l.ppr_r;
    q.rb_lo = l.rb_lo;
    q.rb_hi = l.rb_hi;
    q.route_cta = l.route_cta;
    q.half_sm = f.side ? 1 : 0;
    if (B <= kDirectRouteMaxTokens && f.nt_front == 1 && p->direct_route) {
      // at most 16 router pieces a row block: the routing CTA's poll keeps
      // every load of a round in flight
      q.rpart = p->rpart;
      q.PPR_r = std::min(q.C, 16);
    }
    q.route_few = p->route_few ? 1 : 0;
    if (front_umma_for(p, f.nt_front, f.budget) && !f.side && !q.rpart) {
      q.front_umma = 1;
      q.wt = p->w_front_um;
    }
    TRY(launch_timed(p, KIND_FRONT, KIND_FRONT, f.nt_front, q, l.grid, l.sm.total, s));
  }
  {
    Params q = base;
    const SmemGeom sm = smem_geom(p, KIND_EGU, f.nt_e, tail_tg_eff, B * c.top_k, 0,
                                  f.expert_per_sm == 2 ? kHalfSmem : kBigSmem);
    set_kind(q, p, KIND_EGU, sm);
    q.half_sm = f.expert_per_sm == 2 ? 1 : 0;
    q.piece_ctas = f.expert_grid;
    q.split_cost = split_cost_for(p, f.nt_e);
    TRY(launch_timed(p, KIND_EGU, KIND_EGU, f.nt_e, q, f.expert_grid, sm.total, s));
  }
  if (f.side) {
    // The side lane's down projection starts after expert gate/up: until
    // then the SMs that the front kernels free go to the routed chain, whose
    // latency is the step's critical path.
    CUDA_TRY(cudaEventRecord(p->ev_egu, s));
    CUDA_TRY(cudaStreamWaitEvent(p->side, p->ev_egu, 0));
    {
      Params q = base;
      const TailLaunch l = tail_launch(p, f, B, 2);
      set_kind(q, p, KIND_TAIL, l.sm);
      q.ctl = p->ctl + kSideTail;
      q.trace = p->trace ? p->trace + (size_t)kSideTail * 2 * p->num_sms * 24 : nullptr;
      if (l.res_bytes) {
        q.res_off = kStageOff + l.sm.table_bytes;
        q.res_stride = resident_stride(l.res_k);
        q.res_k = l.res_k;
        q.res_k0 = l.res_k0;
      }
      q.PPR = l.ppr;
      q.ppr_lat = l.ppr_lat;
      q.ppr_sh = l.ppr_sh;
      q.tail_split = l.split;
      q.tail_part = 2;
      q.half_sm = 1;
      q.umma = 0;  // (the side lane's tail keeps the warp-level MMA)
      TRY(launch_timed(p, kSideTail, KIND_TAIL, f.nt_tail, q, l.grid, l.sm.total, p->side));
    }
    CUDA_TRY(cudaEventRecord(p->ev_join, p->side));
  }
  {
    Params q = base;
    const SmemGeom sm = smem_geom(p, KIND_EDN, f.nt_e, tail_tg_eff, B * c.top_k, 0,
                                  f.expert_per_sm == 2 ? kHalfSmem : kBigSmem);
    set_kind(q, p, KIND_EDN, sm);
    q.half_sm = f.expert_per_sm == 2 ? 1 : 0;
    q.piece_ctas = f.expert_grid;
    q.split_cost = split_cost_for(p, f.nt_e);
    {
      // the next layer's front weights (router rows first) into L2 while
      // this layer's expert and tail phases leave HBM idle
      std::lock_guard<std::mutex> lk(g_plans_mu);
      if (p->next_layer && p->next_bytes > 0) {
        // (the copy its front kernel streams at this batch size)
        const moe_plan_s* n = p->next_layer;
        const FwdGeom fn = fwd_geom(n, std::min(B, n->cfg.max_tokens));
        q.pf_src = (front_umma_for(n, fn.nt_front, fn.budget) && !fn.side) ? n->w_front_um : n->w_front;
        q.pf_bytes = p->next_bytes;
      }
    }
    TRY(launch_timed(p, KIND_EDN, KIND_EDN, f.nt_e, q, f.expert_grid, sm.total, s));
  }
  {
    Params q = base;
    const TailLaunch l = tail_launch(p, f, B, f.side ? 1 : 0);
    set_kind(q, p, KIND_TAIL, l.sm);
    if (l.res_bytes) {
      q.res_off = kStageOff + l.sm.table_bytes;
      q.res_stride = resident_stride(l.res_k);
      q.res_k = l.res_k;
      q.res_k0 = l.res_k0;
    }
    q.PPR = l.ppr;
    q.tail_split = l.split;
    q.ppr_lat = l.ppr_lat;
    q.ppr_sh = l.ppr_sh;
    q.tail_part = f.side ? 1 : 0;
    q.half_sm = f.side ? 1 : 0;
    if (l.formed) q.t_rec = p->t_rec;
    // the tensor-core tail: formed records, the whole K range, no side lane
    q.umma = (p->umma_tail && l.formed && !l.split && !f.side) ? 1 : 0;
    if (q.umma) q.wt = p->w_tail_um;
    TRY(launch_timed(p, KIND_TAIL, KIND_TAIL, f.nt_tail, q, f.tail_grid, l.sm.total, s));
  }
  if (f.side) CUDA_TRY(cudaStreamWaitEvent(s, p->ev_join, 0));
  p->last_B = B;
  if (p->profiling) {
    for (int k = 0; k < kSlots; ++k) {
      if (k == kFused || ((k == kSideFront || k == kSideTail) && !f.side)) continue;
      CUDA_TRY(cudaEventSynchronize(p->ev_prof[k][1]));
      float ms = 0.f;
      CUDA_TRY(cudaEventElapsedTime(&ms, p->ev_prof[k][0], p->ev_prof[k][1]));
      p->prof_ms[k] += ms;
    }
    ++p->prof_count;
  }
  return MOE_OK;
}

float half_to_float(uint16_t h) {
  const uint32_t sign = (h >> 15) & 1, ex = (h >> 10) & 0x1F, man = h & 0x3FF;
  float v;
  if (ex == 0)
    v = std::ldexp((float)man, -24);
  else if (ex == 31)
    v = man ? NAN : INFINITY;
  else
    v = std::ldexp((float)(man | 0x400), (int)ex - 25);
  return sign ? -v : v;
}

}  // namespace

extern "C" {

const char* moe_status_str(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or device";
    case MOE_ERR_NOT_LOADED: return "weights not loaded";
    case MOE_ERR_OOM: return "out of memory";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_RANGE: return "weights hold a rejected encoding (e8m0 NaN)";
  }
  return "unknown status";
}

moe_status moe_plan_create(const moe_config* cfg, int device, moe_plan* out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  moe_plan p = new (std::nothrow) moe_plan_s();
  if (!p) return MOE_ERR_OOM;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
    cudaGetLastError();
    delete p;
    return MOE_ERR_UNSUPPORTED;
  }
  if (device < 0 || device >= ndev) {
    delete p;
    return MOE_ERR_INVALID_ARG;
  }
  {
    DeviceGuard g(device);
    st = create_impl(cfg, device, p);
  }
  if (st != MOE_OK) {
    destroy_impl(p);
    return st;
  }
  {
    std::lock_guard<std::mutex> lk(g_plans_mu);
    g_plans.push_back(p);
  }
  *out = p;
  return MOE_OK;
}

void moe_plan_destroy(moe_plan p) { destroy_impl(p); }

moe_status moe_set_next_layer(moe_plan p, moe_plan next, int64_t bytes) {
  if (!p || bytes < 0) return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_plans_mu);
  if (std::find(g_plans.begin(), g_plans.end(), p) == g_plans.end()) return MOE_ERR_INVALID_ARG;
  if (!next || bytes == 0) {
    p->next_layer = nullptr;
    p->next_bytes = 0;
    return MOE_OK;
  }
  if (std::find(g_plans.begin(), g_plans.end(), next) == g_plans.end() || next->device != p->device)
    return MOE_ERR_INVALID_ARG;
  const long long have = (long long)next->g[KIND_FRONT].weight_bytes;
  p->next_layer = next;
  p->next_bytes = std::min<long long>(bytes, have) & ~15LL;
  return MOE_OK;
}

moe_status moe_load_weights(moe_plan p, const moe_weights* w, void* stream) {
  if (!p || !w) return MOE_ERR_INVALID_ARG;
  const moe_config& c = p->cfg;
  const void* need[] = {w->router_w, w->w_in, w->w_out, w->gu_codes, w->gu_scales, w->dn_codes,
                        w->dn_scales};
  for (const void* q : need)
    if (!q || !aligned16(q)) return MOE_ERR_INVALID_ARG;
  if (c.shared_inter > 0) {
    const void* sh[] = {w->sh_gate, w->sh_up, w->sh_down};
    for (const void* q : sh)
      if (!q || !aligned16(q)) return MOE_ERR_INVALID_ARG;
  }
  // the selection bias is copied as floats: 4-byte alignment is all it needs
  const bool use_bias = w->router_bias && c.score_fn == MOE_SCORE_SIGMOID;
  if (use_bias && (reinterpret_cast<uintptr_t>(w->router_bias) & 3)) return MOE_ERR_INVALID_ARG;
  DeviceGuard g(p->device);
  cudaStream_t s = (cudaStream_t)stream;
  p->loaded = false;
  const int H = c.hidden, L = c.latent, E = c.num_experts, I = c.expert_inter, Is = c.shared_inter;
  CUDA_TRY(cudaMemsetAsync(p->err, 0, sizeof(int), s));
  // front tiles: router row blocks, then latent, then shared gate/up, all
  // from [H][N] tensors
  const KindGeom& fr = p->g[KIND_FRONT];
  const size_t rb_bytes = (size_t)fr.C * kDenseTileBytes;
  // the front's tiles, and their tensor-core copy when the plan has one
  for (int um = 0; um < (p->w_front_um ? 2 : 1); ++um) {
    uint8_t* wf = um ? p->w_front_um : p->w_front;
    CUDA_TRY((cudaError_t)launch_pack_dense(w->router_w, H, E, 0, p->RB_router, fr.C, E, wf, s,
                                            nullptr, 0, 0, um));
    CUDA_TRY((cudaError_t)launch_pack_dense(w->w_in, H, L, 0, p->RB_lat, fr.C, L,
                                            wf + p->RB_router * rb_bytes, s, nullptr, 0, 0, um));
    if (Is > 0)
      CUDA_TRY((cudaError_t)launch_pack_dense(w->sh_gate, H, Is, 1, fr.RB - p->RB_router - p->RB_lat,
                                              fr.C, Is, wf + (p->RB_router + p->RB_lat) * rb_bytes, s,
                                              w->sh_up, 0, 0, um));
  }
  const KindGeom& tl = p->g[KIND_TAIL];
  CUDA_TRY((cudaError_t)launch_pack_dense(w->w_out, L, H, 2, tl.RB, tl.C, H, p->w_tail, s,
                                          Is > 0 ? w->sh_down : w->w_out, Is, p->C_lat));
  if (p->w_tail_um)
    CUDA_TRY((cudaError_t)launch_pack_dense(w->w_out, L, H, 2, tl.RB, tl.C, H, p->w_tail_um, s,
                                            Is > 0 ? w->sh_down : w->w_out, Is, p->C_lat, 1));
  const KindGeom& eg = p->g[KIND_EGU];
  CUDA_TRY((cudaError_t)launch_pack_mx(w->gu_codes, w->gu_scales, E, 2 * I, L, 1, eg.RB, eg.C,
                                       p->w_egu, p->err, s, p->umma ? 1 : 0));
  const KindGeom& ed = p->g[KIND_EDN];
  CUDA_TRY((cudaError_t)launch_pack_mx(w->dn_codes, w->dn_scales, E, L, I, 0, ed.RB, ed.C,
                                       p->w_edn, p->err, s, p->umma ? 1 : 0));
  if (use_bias) {
    CUDA_TRY(cudaMemcpyAsync(p->bias, w->router_bias, sizeof(float) * E, cudaMemcpyDeviceToDevice, s));
  } else {
    CUDA_TRY(cudaMemsetAsync(p->bias, 0, sizeof(float) * E, s));
  }
  int err = 0;
  CUDA_TRY(cudaMemcpyAsync(&err, p->err, sizeof(int), cudaMemcpyDeviceToHost, s));
  CUDA_TRY(cudaStreamSynchronize(s));
  if (err & (1 << ERR_NAN_SCALE)) {
    CUDA_TRY(cudaMemset(p->err, 0, sizeof(int)));
    return MOE_ERR_RANGE;
  }
  p->loaded = true;
  return MOE_OK;
}

moe_status moe_forward(moe_plan p, const void* x, int32_t num_tokens, void* out, void* stream) {
  if (!p || !x || !out) return MOE_ERR_INVALID_ARG;
  if (num_tokens < 1 || num_tokens > p->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  const size_t bytes = (size_t)num_tokens * p->cfg.hidden * 2;
  const uint8_t* xa = (const uint8_t*)x;
  const uint8_t* oa = (const uint8_t*)out;
  if (xa < oa + bytes && oa < xa + bytes) return MOE_ERR_INVALID_ARG;
  if (!p->loaded) return MOE_ERR_NOT_LOADED;
  DeviceGuard g(p->device);
  return enqueue_forward(p, x, num_tokens, out, (cudaStream_t)stream);
}

moe_status moe_forward_host(moe_plan p, const void* x_host, int32_t num_tokens, void* out_host,
                            void* stream) {
  if (!p || !x_host || !out_host) return MOE_ERR_INVALID_ARG;
  if (num_tokens < 1 || num_tokens > p->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
  if (!p->loaded) return MOE_ERR_NOT_LOADED;
  DeviceGuard g(p->device);
  cudaStream_t s = (cudaStream_t)stream;
  const size_t bytes = (size_t)num_tokens * p->cfg.hidden * 2;
  CUDA_TRY(cudaMemcpyAsync(p->x_stage, x_host, bytes, cudaMemcpyHostToDevice, s));
  TRY(enqueue_forward(p, p->x_stage, num_tokens, p->out_stage, s));
  CUDA_TRY(cudaMemcpyAsync(out_host, p->out_stage, bytes, cudaMemcpyDeviceToHost, s));
  return MOE_OK;
}

moe_status moe_sync_status(moe_plan p) {
  if (!p) return MOE_ERR_INVALID_ARG;
  DeviceGuard g(p->device);
  CUDA_TRY(cudaDeviceSynchronize());
  int err = 0;
  CUDA_TRY(cudaMemcpy(&err, p->err, sizeof(int), cudaMemcpyDeviceToHost));
  if (err) {
    CUDA_TRY(cudaMemset(p->err, 0, sizeof(int)));
    if (err & ((1 << ERR_WAIT_FULL) | (1 << ERR_WAIT_EMPTY) | (1 << ERR_WAIT_DEP))) {
      // A forward whose wait gave up may have left partial counts behind
      // (router row blocks, split-K tickets, piece cursors, the routing flag,
      // the fused launch's phase counts).  Nothing runs after the
      // synchronisation above, so they are cleared here and the next forward
      // starts from the state a fresh plan has.
      TRY(reset_control(p));
      return MOE_ERR_TIMEOUT;
    }
    return MOE_ERR_RANGE;
  }
  return MOE_OK;
}

moe_status moe_debug_expire_wait(moe_plan p, int32_t limit_polls, void* stream) {
  if (!p || limit_polls < 1 || limit_polls > (1 << 22)) return MOE_ERR_INVALID_ARG;
  DeviceGuard g(p->device);
  CUDA_TRY((cudaError_t)launch_expire_wait(p->nve + 4, p->err, p->router_done, p->counters[KIND_FRONT],
                                           p->ctl + KIND_FRONT, p->route_ready,
                                           (unsigned)limit_polls, stream));
  return MOE_OK;
}

moe_status moe_last_routing(moe_plan p, int32_t* ids_host, float* w_host, int32_t num_tokens) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (num_tokens < 1 || num_tokens > p->last_B) return MOE_ERR_INVALID_ARG;
  DeviceGuard g(p->device);
  CUDA_TRY(cudaDeviceSynchronize());
  const size_t n = (size_t)num_tokens * p->cfg.top_k;
  if (ids_host) CUDA_TRY(cudaMemcpy(ids_host, p->ids, n * sizeof(int), cudaMemcpyDeviceToHost));
  if (w_host) CUDA_TRY(cudaMemcpy(w_host, p->wts, n * sizeof(float), cudaMemcpyDeviceToHost));
  return MOE_OK;
}

// e2m1 code -> float: sign, 2 exponent bits (bias 1), 1 mantissa bit;
// exponent 0 is subnormal (0 or 0.5)
float e2m1_value(int code) {
  const int e = (code >> 1) & 3, m = code & 1;
  const float v = e == 0 ? 0.5f * m : std::ldexp(1.0f + 0.5f * m, e - 1);
  return (code & 8) ? -v : v;
}

// element i (0..255) of one activation record, in either form (layout.cuh)
float record_value(const moe_plan_s* p, const uint8_t* rec, int i) {
  if (p->umma) {
    float v = 0.f;
    for (int t = 0; t < kUTerms; ++t) {
      const uint8_t sb = rec[kUTerms * kUTermBytes + t * 8 + i / 32];
      if (sb == 0xFF) return NAN;
      const int code = (rec[t * kUTermBytes + i / 2] >> (4 * (i & 1))) & 15;
      v += e2m1_value(code) * std::ldexp(1.0f, (int)sb - 127);
    }
    return v;
  }
  uint16_t hv;
  float sc;
  std::memcpy(&hv, rec + i * 2, 2);
  std::memcpy(&sc, rec + 512 + 4 * (i / 32), 4);
  return half_to_float(hv) * sc;
}

moe_status moe_debug_fetch(moe_plan p, int32_t what, int32_t num_tokens, float* host,
                           int64_t count) {
  if (!p || !host) return MOE_ERR_INVALID_ARG;
  const int B = p->last_B;
  if (B < 1 || num_tokens != B) return MOE_ERR_INVALID_ARG;
  const moe_config& c = p->cfg;
  const int L = c.latent, E = c.num_experts, K = c.top_k, I = c.expert_inter, Is = c.shared_inter;
  DeviceGuard g(p->device);
  CUDA_TRY(cudaDeviceSynchronize());
  const int slots = B * K;
  switch (what) {
    case MOE_DBG_LOGITS: {
      if (count != (int64_t)B * E) return MOE_ERR_INVALID_ARG;
      CUDA_TRY(cudaMemcpy(host, p->logits, sizeof(float) * B * E, cudaMemcpyDeviceToHost));
      return MOE_OK;
    }
    case MOE_DBG_Z: {
      if (count != (int64_t)B * L) return MOE_ERR_INVALID_ARG;
      const int cz = ceil_div(L, kMxChunkK);
      std::vector<uint8_t> raw((size_t)B * cz * p->act_rec);
      CUDA_TRY(cudaMemcpy(raw.data(), p->z_mx, raw.size(), cudaMemcpyDeviceToHost));
      for (int b = 0; b < B; ++b)
        for (int l = 0; l < L; ++l) {
          const uint8_t* rec = raw.data() + ((size_t)b * cz + l / kMxChunkK) * p->act_rec;
          host[(size_t)b * L + l] = record_value(p, rec, l % kMxChunkK);
        }
      return MOE_OK;
    }
    case MOE_DBG_H: {
      if (count != (int64_t)slots * I) return MOE_ERR_INVALID_ARG;
      const int ci = ceil_div(I, kMxChunkK);
      std::vector<uint8_t> raw((size_t)ci * slots * p->act_rec);
      std::vector<int> sorted(slots);
      CUDA_TRY(cudaMemcpy(raw.data(), p->h_mx, raw.size(), cudaMemcpyDeviceToHost));
      CUDA_TRY(cudaMemcpy(sorted.data(), p->slots_sorted, sizeof(int) * slots, cudaMemcpyDeviceToHost));
      for (int pos = 0; pos < slots; ++pos) {
        const int slot = sorted[pos];
        if (slot < 0 || slot >= slots) return MOE_ERR_RANGE;
        for (int i = 0; i < I; ++i) {
          const uint8_t* rec = raw.data() + ((size_t)(i / kMxChunkK) * slots + pos) * p->act_rec;
          host[(size_t)slot * I + i] = record_value(p, rec, i % kMxChunkK);
        }
      }
      return MOE_OK;
    }
    case MOE_DBG_Y: {
      if (count != (int64_t)slots * L) return MOE_ERR_INVALID_ARG;
      const int cy = ceil_div(L, 64);
      std::vector<float> raw((size_t)cy * slots * 64);
      CUDA_TRY(cudaMemcpy(raw.data(), p->y, raw.size() * sizeof(float), cudaMemcpyDeviceToHost));
      for (int s = 0; s < slots; ++s)
        for (int l = 0; l < L; ++l) host[(size_t)s * L + l] = raw[((size_t)(l / 64) * slots + s) * 64 + l % 64];
      return MOE_OK;
    }
    case MOE_DBG_HS: {
      if (Is == 0 || count != (int64_t)B * Is) return MOE_ERR_INVALID_ARG;
      const int cs = ceil_div(Is, 64);
      std::vector<float> raw((size_t)cs * B * 64);
      CUDA_TRY(cudaMemcpy(raw.data(), p->h_s, raw.size() * sizeof(float), cudaMemcpyDeviceToHost));
      for (int b = 0; b < B; ++b)
        for (int i = 0; i < Is; ++i) host[(size_t)b * Is + i] = raw[((size_t)(i / 64) * B + b) * 64 + i % 64];
      return MOE_OK;
    }
    default: return MOE_ERR_INVALID_ARG;
  }
}

moe_status moe_get_plan_info(moe_plan p, moe_plan_info* info) {
  if (!p || !info) return MOE_ERR_INVALID_ARG;
  const FwdGeom f = fwd_geom(p, p->cfg.max_tokens);
  info->device = p->device;
  info->num_sms = p->num_sms;
  info->front_ctas = f.front_workers;
  info->expert_ctas = f.expert_grid;
  info->packed_bytes = (int64_t)p->packed_bytes;
  info->workspace_bytes = (int64_t)p->workspace_bytes;
  const moe_config& c = p->cfg;
  info->dense_weight_bytes =
      2LL * c.hidden * (c.num_experts + c.latent) + 2LL * c.latent * c.hidden +
      6LL * c.hidden * c.shared_inter;
  info->expert_weight_bytes =
      (3LL * c.expert_inter * c.latent) / 2 + (3LL * c.expert_inter * c.latent) / 32;
  info->kernels_per_forward = (p->use_fused && p->cfg.max_tokens <= kFusedMaxTokens)
                                 ? 1
                                 : KIND_COUNT + (side_lane(p, p->cfg.max_tokens) ? 2 : 0);
  return MOE_OK;
}

moe_status moe_debug_trace(moe_plan p, uint64_t* host, int64_t count) {
  if (!p || !host) return MOE_ERR_INVALID_ARG;
  if (!p->trace) return MOE_ERR_UNSUPPORTED;
  const int64_t n = (int64_t)kSlots * p->num_sms * 24;
  if (count != n) return MOE_ERR_INVALID_ARG;
  DeviceGuard g(p->device);
  CUDA_TRY(cudaDeviceSynchronize());
  // the first num_sms CTAs of each slot (a grid of two CTAs per SM traces
  // its second half into rows that are not returned)
  const size_t row = (size_t)p->num_sms * 24;
  for (int k = 0; k < kSlots; ++k)
    CUDA_TRY(cudaMemcpy(host + k * row, p->trace + (size_t)k * 2 * row, sizeof(uint64_t) * row,
                        cudaMemcpyDeviceToHost));
  return MOE_OK;
}

moe_status moe_set_profiling(moe_plan p, int32_t enable) {
  if (!p) return MOE_ERR_INVALID_ARG;
  p->profiling = enable != 0;
  return MOE_OK;
}

moe_status moe_get_profile(moe_plan p, float* ms, int32_t* count) {
  if (!p || !ms || !count) return MOE_ERR_INVALID_ARG;
  for (int k = 0; k < kSlots; ++k) {
    ms[k] = (float)p->prof_ms[k];
    p->prof_ms[k] = 0.0;
  }
  *count = p->prof_count;
  p->prof_count = 0;
  return MOE_OK;
}

moe_status moe_debug_geometry(const moe_config* cfg, int32_t num_sms, int32_t num_tokens,
                              moe_geometry* out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  const moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (num_sms < 2 || num_tokens < 1 || num_tokens > cfg->max_tokens) return MOE_ERR_INVALID_ARG;
  moe_plan_s* p = new (std::nothrow) moe_plan_s();
  if (!p) return MOE_ERR_OOM;
  p->cfg = *cfg;
  p->num_sms = num_sms;
  read_env(p);
  plan_shape(p);
  const moe_config& c = p->cfg;
  const int B = num_tokens, K = c.top_k;
  const FwdGeom f = fwd_geom(p, B);
  const int tail_tg_eff = std::min(B, p->tail_tg);
  // out[0..3]: the routed chain's kernels; out[4], out[5]: the side lane's
  // front and tail (grid 0 when this forward has no side lane)
  for (int k = 0; k < kGeometryKinds; ++k) {
    moe_geometry& o = out[k];
    std::memset(&o, 0, sizeof(o));
    o.kind = k;
    const int kk = k == 4 ? KIND_FRONT : k == 5 ? KIND_TAIL : k;
    o.partial_floats_capacity = (int64_t)(k == 4 ? p->side_partial_cap = side_partial_floats(p)
                                                 : partial_floats(p, kk));
    const KindGeom& g = p->g[kk];
    SmemGeom sm;
    if (k >= 4 && !f.side) continue;
    if (kk == KIND_FRONT) {
      const FrontLaunch l = front_launch(p, f, B, k == 4 ? 2 : (f.side ? 1 : 0));
      sm = l.sm;
      const int pieces = (l.rb_lo == 0 ? p->RB_router * l.ppr_r : 0) +
                         (l.rb_hi - (l.rb_lo == 0 ? p->RB_router : l.rb_lo)) * l.ppr;
      o.grid = l.grid;
      o.ctas_per_sm = 1;  // (with the side lane: one CTA of either lane per half SM)
      o.token_tiles = f.nt_front;
      o.max_piece_tokens = B;
      o.pieces_per_row_block = l.ppr;
      o.partial_floats_needed = (int64_t)pieces * f.nt_front * 1024;
      if (l.route_cta)
        o.route_logit_floats = sm.nstages * sm.stage_bytes / 4 - ((c.num_experts + 31) & ~31);
    } else if (kk == KIND_EGU || kk == KIND_EDN) {
      sm = smem_geom(p, kk, f.nt_e, tail_tg_eff, B * K, 0, f.expert_per_sm == 2 ? kHalfSmem : kBigSmem);
      o.grid = f.expert_grid;
      o.ctas_per_sm = f.expert_per_sm;
      o.token_tiles = f.nt_e;
      o.max_piece_tokens = std::min(B, expert_tg(p, B));
      o.pieces_per_row_block = expert_ppr(p, ve_bound(p, B * K) * g.RB, g.C, f.expert_grid, f.nt_e);
      int64_t most = 0;
      for (int V = 1; V <= p->ve_max; ++V)
        most = std::max(most, (int64_t)V * g.RB * expert_ppr(p, V * g.RB, g.C, f.expert_grid, f.nt_e));
      o.partial_floats_needed = most * f.nt_e * 1024;
    } else {
      const TailLaunch l = tail_launch(p, f, B, k == 5 ? 2 : (f.side ? 1 : 0));
      sm = l.sm;
      const int passes = (B + p->tail_tg - 1) / p->tail_tg;
      o.grid = l.grid;
      o.ctas_per_sm = 1;
      o.token_tiles = f.nt_tail;
      o.max_piece_tokens = tail_tg_eff;
      o.pieces_per_row_block = l.ppr;
      o.partial_floats_needed = (int64_t)passes * g.RB * l.ppr * f.nt_tail * 1024;
      o.resident_tail_bytes = l.res_bytes;
    }
    o.stages = sm.nstages;
    o.stage_bytes = sm.stage_bytes;
    o.smem_bytes = (int64_t)sm.total;
  }
  delete p;
  return MOE_OK;
}

}  // extern "C"
