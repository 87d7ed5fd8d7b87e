// engine.cuh -- kernel parameters shared by the launchers and the kernels.
#pragma once
#include <cstdint>

#include "layout.cuh"

namespace moe {

enum Kind : int {
  KIND_FRONT = 0,  // x . [W_r | W_in | W_sg,W_su]: router logits, latent z, shared h_s
  KIND_EGU = 1,    // routed experts gate/up + SwiGLU, MXFP4
  KIND_EDN = 2,    // routed experts down projection, MXFP4
  KIND_TAIL = 3,   // weighted combine + W_out, plus shared down projection -> out
  KIND_COUNT = 4
};

// Per-kernel scheduling state in device memory, zero between launches: the
// piece cursor is reset by the last CTA to leave.
struct Ctl {
  int cursor;
  int exits;
  int pad[30];
};

// error word bits
enum : int {
  ERR_WAIT_FULL = 0,
  ERR_WAIT_EMPTY = 1,
  ERR_NAN_SCALE = 2,
  ERR_WAIT_DEP = 3,  // a routing flag or a phase-completion count never arrived
};

struct VExpert {  // one token group of one routed expert
  int expert, start, count, pad;
};

struct Params {
  int H, L, E, topk, I, Is;
  int B;  // tokens of this forward
  int score_fn, renorm;
  float routed_scale;

  // iteration space: virtual matrices x row blocks x pieces
  int RB;             // row blocks per virtual matrix
  int C;              // K chunks per row block
  int PPR;            // pieces per row block (0: computed on the device, EGU/EDN)
  int PPR_r;          // FRONT: pieces per router row block
  int piece_ctas;     // EGU/EDN: CTAs taking pieces (for the split-K choice)
  int split_cost;     // EGU/EDN: price of a split-K piece end, in stages
  int C_lat;          // TAIL: chunks covering L; chunks >= C_lat cover I_s
  // TAIL, shared part first (0: one split over all C chunks): pieces over
  // the I_s chunks come first in the schedule and need nothing from the
  // routed experts (h_s is complete before this kernel starts), so CTAs that
  // land while the expert kernels finish stream them at once; the latent
  // pieces follow.  ppr_sh + ppr_lat == PPR pieces per row block.
  int tail_split, ppr_lat, ppr_sh;
  // TAIL, one lane of two (the shared expert on a side stream): 0 every
  // piece, 1 the latent pieces only (the routed lane), 2 the shared-expert
  // pieces only (the side lane).  Both lanes share the row blocks' tickets and
  // partial-sum slots, so whichever finishes a row block last writes it.
  int tail_part;
  // FRONT: the row blocks this launch streams, [rb_lo, rb_hi): everything
  // (0, RB), or one lane -- router + latent rows (the routed lane, with the
  // routing CTA) or the shared expert's gate/up rows (the side lane)
  int rb_lo, rb_hi;
  // TAIL: first k of the resident activation (its record holds k in
  // [res_k0, res_k0 + res_k)); a lane keeps only its own part
  int res_k0;
  // host side: launch the instantiation compiled for two CTAs per SM (at most
  // 112 registers a thread), so that a CTA of the other lane fits beside it
  int half_sm;
  // FRONT, routing CTA: once the experts are chosen it asks L2 for their
  // packed gate/up and down tiles (the kernels that stream them start a few
  // round trips later), for the chosen experts whose first virtual expert
  // index is below pf_ves; 0 = none
  const uint8_t* pf_egu;
  const uint8_t* pf_edn;
  long long pf_egu_bytes, pf_edn_bytes;  // per expert
  int pf_ves;
  // FRONT, few tokens: the router pieces write their partial sums here (no
  // tickets, no finalisation) and the routing CTA sums them itself, polling
  // on the data: every element starts as the 0xFFFFFFFF pattern, which no
  // sum takes, and the routing CTA restores it after reading.  That is one
  // round trip from the last router piece to the selection instead of four
  // (ticket, partial sums, count, logits).  Null: the usual split-K finish.
  float* rpart;
  // TAIL with staged activations (more than the resident size): the tail's
  // CTAs first form every token's activation once -- the combine c = sum_j
  // w_j y_j for the latent chunks, h_s for the shared ones -- as records of
  // 64 bf16 hi then 64 bf16 lo values, t_rec[chunk][B][256 bytes], and count
  // themselves done in t_ready (release); the producers stream activation
  // rows from those records once the count reaches the grid.  Null: the
  // combine is formed per stage (the fused single launch).
  uint8_t* t_rec;
  int* t_ready;
  // EGU/EDN on the 5th-generation tensor cores (block-scaled tcgen05 MMA,
  // e2m1 weights x e4m3 activation terms): the packed tiles and the z / h
  // records take the layouts of layout.cuh; FRONT and EGU write their
  // records in that form.  0: the warp-level MMA; else nonzero, and at an
  // expert kernel's launch the token tiles of its stages (its NT)
  int umma;
  // FRONT on the tensor cores (bf16 MMA of the weight rows with x): 0, or its
  // token tiles (set at launch)
  int front_umma;
  int act_rec;  // bytes of one activation record (kActRecBytes or kActRecBytesU)
  // EGU: the latent row blocks' finalisations count up here (release); the
  // expert gate/up kernel reads z once it reaches RB_lat instead of waiting
  // for the whole front grid (whose last CTAs stream shared-expert rows)
  int* z_done;
  // per virtual expert: EGU's row-block finalisations of its h count up
  // here (release); the expert down kernel streams a virtual expert's
  // activations once its count reaches RB_egu instead of waiting for the
  // whole gate/up grid.  Zeroed by the routing with the tables.
  int* h_done;
  int RB_egu;
  int RB_router;      // FRONT: leading row blocks holding router rows
  int RB_lat;         // FRONT: row blocks of the latent projection (after the router's);
                      // the shared expert's gate/up row blocks follow
  int route_cta;      // FRONT: routing CTAs, the grid's last ones (no pieces); 0: none
  int route_few;      // FRONT, B * k <= 32 with direct logits: the one-warp table build
  int tg;             // tokens per group (EGU/EDN/TAIL)
  int KL;             // K extent of the chunked dimension (for ragged last chunk)
  int KS;             // TAIL: K extent of the shared part (I_s)
  // EDN: the next layer's front weights, pulled into L2 once this CTA's own
  // stages are issued (cross-layer prefetch); pf_bytes a multiple of 16, 0:
  // none
  const uint8_t* pf_src;
  long long pf_bytes;

  // shared memory geometry (bytes)
  int nstages, stage_bytes, act_off, act_stride, scratch_off, stage_off;
  int table_off;  // EGU/EDN: shared-memory copy of the routing tables
  // TAIL with few tokens: the whole activation [c ; h_s] of every token is
  // formed once per CTA in shared memory (bf16 hi + lo per value); 0 = off
  int res_off, res_stride, res_k;

  const uint8_t* wt;       // packed tiles
  long long matrix_bytes;  // EGU/EDN: bytes of one expert's tiles

  const uint16_t* x;   // [B][H] bf16
  const float* bias;   // [E] or null
  float* logits;       // [maxB][E]
  uint8_t* z_mx;       // [B][ceil(L/256)][544]
  float* h_s;          // [ceil(Is/64)][B][64]
  uint8_t* h_mx;       // [ceil(I/256)][B*k][544] in expert-sorted slot order
  float* y;            // [ceil(L/64)][B*k][64]
  uint16_t* out;       // [B][H] bf16
  int ld_slots;        // B*k (row count of h_mx / y chunk planes)

  int* ids;            // [B][k]
  float* wts;          // [B][k]
  int* slots_sorted;   // [B*k]
  VExpert* ve;         // virtual experts
  int* nve;
  int ve_max;

  Ctl* ctl;
  // optional trace: per CTA 8 x u64 {start ns, end ns, pieces, finalizes,
  // route start ns, route end ns, first stage ready ns, 0}; null when off
  unsigned long long* trace;
  int* counters;   // finalize tickets per (virtual matrix, row block)
  int* router_done;
  int* route_cnt;  // FRONT, several routing CTAs: tickets of those done selecting
  // 1 once this forward's routing tables are published (release by the
  // routing CTA); the expert kernels stream their experts' tiles as soon as
  // it is set, before their own dependency resolves.  Cleared by the tail,
  // which no reader of it can still be running beside.
  int* route_ready;
  // fused single-launch path only (null otherwise): completion counts that
  // later phases wait on, each raised with release semantics once a row
  // block's outputs are stored: [0] latent row blocks (z), [1] shared-expert
  // row blocks (h_s), [2] expert gate/up matrices (h), [3] expert down
  // matrices (y)
  int* done;
  // fused launch, tail phase: the counts it waits for (expert-down row
  // blocks per virtual expert; shared-expert row blocks)
  int need_rb_edn, need_rb_sh;
  float* partials;
  int* err;
  // ns a producer (consumer) warp sleeps after a failed poll of a ring
  // barrier before polling again
  int prod_sleep, cons_sleep;
};

// The single-launch path (few tokens): one Params per phase, all with the
// same shared-memory layout and ring, and the size of the front phase (the
// first part of the ordered piece list).
struct MegaParams {
  Params k[KIND_COUNT];
  int n_front;
};

// Host-side launchers (defined in moe_kernels.cu and moe_k_mega.cu).
int launch_kind(int kind, int nt, const Params& p, int grid, size_t smem, void* stream, bool pdl);
int launch_mega(const MegaParams& mp, int grid, size_t smem, void* stream, bool pdl);
int max_smem_optin();
int launch_expire_wait(int* never, int* err, int* router_done, int* ticket, Ctl* ctl,
                       int* route_ready, unsigned limit, void* stream);
int set_smem_limits(size_t bytes);

int launch_pack_dense(const void* src, int K, int N, int layout, int RB, int C, int rows_valid,
                      uint8_t* dst, void* stream, const void* src2, int K2, int C_first, int umma = 0);
int launch_pack_mx(const uint8_t* codes, const uint8_t* scales, int E, int rows, int K,
                   int layout, int RB, int C, uint8_t* dst, int* err, void* stream, int umma);

}  // namespace moe
