/*
 * moe.h -- C ABI of the B200 latent-MoE decode block (libmoe_b200.so).
 *
 * The block, per token b of a decode batch (B = 1..128 tokens):
 *
 *   logits = x . W_r                 router scores          } one weight-streaming pass
 *   z      = x . W_in                latent input projection} over the same x
 *   ids, w = top-k of the scores     softmax, or sigmoid + per-expert selection bias;
 *                                    weights renormalised over the k chosen experts
 *   y_j    = SwiGLU expert ids[j] on z, MXFP4 weights (e2m1 elements, e8m0 scale per 32)
 *   out    = (sum_j w_j y_j) . W_out + SwiGLU_shared(x) . W_sd
 *
 * Sources of the operation:
 *   - router scoring and the latent input projection computed together as one
 *     matmul; the shared expert on its own stream, overlapping routing and the
 *     selected experts: page "Hyper Optimizing Kimi K3 in vLLM: Moving Fast and
 *     Responsibly", section 从算子之间找时间 ("finding time between operators");
 *   - the MXFP4 top-k finalize (weighted combine) fused into the latent-tail
 *     kernel, saving one launch and one intermediate write + re-read: page
 *     "Kimi K3 在 vLLM 中的性能优化", section 延迟 MXFP4 最终化 ("deferred MXFP4
 *     finalize");
 *   - decode batch 1-64 and the 16 x 8 speculative-verify shape: page
 *     "Hyper Optimizing Kimi K3 in vLLM: Moving Fast and Responsibly",
 *     introduction, and page "Kimi K3 vLLM 优化：NVIDIA 解码速度提升 1.68×",
 *     section 上游测试实际展示了什么.
 *   MXFP4 encodings follow the OCP Microscaling (MX) v1.0 specification.
 *
 * Conventions for every call:
 *   - Status codes are returned; nothing throws across the ABI.  Invalid
 *     arguments are detected on the host before anything is launched.
 *   - "device pointer" means memory of the plan's device; "host pointer" means
 *     ordinary or pinned host memory.
 *   - Streams are passed as void* and are cudaStream_t values (NULL = legacy
 *     default stream).
 *   - A plan is used by one host thread and one stream at a time.
 *   - There is no CPU fallback: without a usable sm_100 device every call that
 *     needs the GPU returns MOE_ERR_UNSUPPORTED or MOE_ERR_CUDA.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer, B out of range */
  MOE_ERR_UNSUPPORTED = 2, /* shape or device this library does not implement */
  MOE_ERR_NOT_LOADED = 3,  /* moe_forward before moe_load_weights succeeded */
  MOE_ERR_OOM = 4,         /* a device or host allocation failed (plan create / load only) */
  MOE_ERR_CUDA = 5,        /* a CUDA runtime call failed; the plan should be destroyed */
  MOE_ERR_TIMEOUT = 6,     /* a device-side bounded wait gave up (reported by moe_sync_status) */
  MOE_ERR_RANGE = 7        /* weights hold an encoding the block rejects (e8m0 NaN byte 0xFF) */
} moe_status;

enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 };

/* Layer shape and routing rule, fixed at plan creation. */
typedef struct moe_config {
  int32_t hidden;       /* H: multiple of 32 */
  int32_t latent;       /* L: multiple of 32 */
  int32_t num_experts;  /* E: 1..1024 */
  int32_t top_k;        /* k: 1..min(E, 16) */
  int32_t expert_inter; /* I: multiple of 32 */
  int32_t shared_inter; /* I_s: multiple of 32, or 0 for no shared expert */
  int32_t max_tokens;   /* largest B a forward may pass: 1..128 */
  int32_t score_fn;     /* MOE_SCORE_SOFTMAX or MOE_SCORE_SIGMOID */
  int32_t renormalize;  /* 1: combine weights divided by their sum over the k chosen */
  float routed_scale;   /* factor applied to every combine weight (1.0 = none) */
  int32_t shared_sms;   /* the shared expert as a side lane for forwards of at
                           most 4 tokens: n > 0 = its gate/up rows and its down
                           projection run as two kernels of n CTAs each on a
                           side stream, sharing the SMs with the routed
                           experts' chain; 0 (the measured best) or -1 = no
                           side lane: its gate/up rows ride the front pass and
                           its down projection leads the tail.  Ignored when
                           shared_inter == 0. */
} moe_config;

/*
 * Weights in canonical layout, all DEVICE pointers, row-major, 16-byte aligned
 * (router_bias: 4-byte aligned).
 * bf16 tensors are in "x . W" orientation [in][out]; MXFP4 tensors are
 * output-row-major with K (the reduction index) contiguous:
 *   router_w   bf16 [H][E]
 *   router_bias f32 [E]       selection bias (sigmoid scoring only); may be NULL
 *   w_in       bf16 [H][L]
 *   w_out      bf16 [L][H]
 *   gu_codes   u8   [E][2I][L/2]   rows 0..I-1 gate, rows I..2I-1 up;
 *                                  element 2t in the low nibble of byte t
 *   gu_scales  u8   [E][2I][L/32]  e8m0, value 2^(s-127); 0xFF (NaN) rejected;
 *                                  0 (2^-127) is applied as 0 (every weight of
 *                                  such a block is below fp32's normal range)
 *   dn_codes   u8   [E][L][I/2]
 *   dn_scales  u8   [E][L][I/32]
 *   sh_gate    bf16 [H][I_s]   (ignored when I_s == 0)
 *   sh_up      bf16 [H][I_s]
 *   sh_down    bf16 [I_s][H]
 * The caller keeps ownership and may free them once moe_load_weights returns.
 */
typedef struct moe_weights {
  const void *router_w;
  const float *router_bias;
  const void *w_in;
  const void *w_out;
  const uint8_t *gu_codes;
  const uint8_t *gu_scales;
  const uint8_t *dn_codes;
  const uint8_t *dn_scales;
  const void *sh_gate;
  const void *sh_up;
  const void *sh_down;
} moe_weights;

typedef struct moe_plan_s *moe_plan;

/* What a plan chose, for logging and for checking that the fast path runs. */
typedef struct moe_plan_info {
  int32_t device;
  int32_t num_sms;
  int32_t front_ctas;       /* CTAs streaming the router / latent / shared gate-up rows */
  int32_t expert_ctas;      /* CTAs of each routed-expert kernel for max_tokens tokens
                               (two per SM when a piece holds one token tile) */
  int64_t packed_bytes;     /* library-owned packed weights */
  int64_t workspace_bytes;  /* library-owned activations, routing metadata, partial sums */
  int64_t dense_weight_bytes;      /* bf16 bytes one forward streams regardless of routing */
  int64_t expert_weight_bytes;     /* MXFP4 bytes of one expert (gate/up + down, codes + scales) */
  int32_t kernels_per_forward;     /* launches one moe_forward of max_tokens tokens makes
                                      (six with the side lane's two) */
} moe_plan_info;

/*
 * Create a plan on `device`: checks the shape, allocates packed-weight storage
 * and workspace.  *out receives the plan.
 * Errors: INVALID_ARG (null, bad shape), UNSUPPORTED (no sm_100 device, shape
 * beyond the limits above), OOM, CUDA.
 *
 * Environment variables read here (measurement and tuning; every default is
 * the measured best, and none changes a result beyond rounding order):
 *   MOE_TRACE               keep the per-CTA timeline (moe_debug_trace)
 *   MOE_LOG                 print the plan's geometry to stderr
 *   MOE_FUSED=1             one launch per forward for B <= 8 (slower)
 *   MOE_NO_PDL=1            no programmatic dependent launch between kernels
 *   MOE_MAX_STAGES=n        ring depth cap, 2..8 (default 5)
 *   MOE_SPLIT_COST=n        split-K piece-end price in stages (default 2)
 *   MOE_UMMA=0              expert kernels on the warp-level MMA (e2m1 decoded
 *                           to f16, f16 activations with a power-of-two scale
 *                           per 32) instead of the 5th-generation tensor cores
 *                           (block-scaled e2m1 x e2m1 MMA, activations as four
 *                           e2m1 terms); fixes the packed weight order, so it
 *                           holds for the plan's life.  MOE_UMMA=0 also allows
 *                           MOE_FUSED, which keeps the warp-level MMA, and
 *                           keeps the front and tail on the warp-level MMA
 *   MOE_UMMA_TAIL=0         the tail keeps the warp-level MMA (default: bf16
 *                           tensor-core MMA when its activation comes from
 *                           formed records; a second copy of its tiles)
 *   MOE_UMMA_FRONT=0        the front keeps the warp-level MMA (default: bf16
 *                           tensor-core MMA above 8 tokens, for plans of more
 *                           than 8 tokens; a second copy of its tiles)
 *   MOE_EXPERT_CTAS_PER_SM=1  one CTA per SM for the expert kernels (default
 *                           2 at one token tile, and at two on the tensor cores)
 *   MOE_EXPERT_SMALL_MAX_B=n  largest B with 8-token virtual experts (16-token
 *                           ones on the tensor cores above B = 64; default
 *                           128; above it, 32-token groups)
 *   MOE_EXPERT_TG=8|16|32   tokens per virtual expert for every B
 *   MOE_EXPERT_PPR=n        the expert kernels' split-K factor (default 1, one
 *                           piece a row block, measured fastest; 0: the
 *                           makespan model, chosen on the device)
 *   MOE_FRONT_PPR=n, MOE_TAIL_PPR=n  fixed split-K factors (pieces a row block)
 *                           of the front and tail kernels (default: the
 *                           makespan model with the piece-end prices measured
 *                           for each kernel and activation form)
 *   MOE_ROUTE_TPC=n, MOE_ROUTE_MAX_CTAS=n  tokens per routing CTA and the
 *                           most routing CTAs (defaults 8 and 16)
 *   MOE_ROUTE_FEW=0         no one-warp selection and table build for B <= 8
 *                           with B * k <= 64 (the general path instead)
 *   MOE_SIDE_LANE=0         no side lane, whatever shared_sms says
 *   MOE_TAIL_SPLIT=0        the tail's shared-expert part is not scheduled first
 *   MOE_Z_FLAG=0            expert gate/up waits for the whole front kernel
 *   MOE_H_FLAG=0            expert down waits for the whole gate/up kernel (default:
 *                           per virtual expert, for its gate/up row blocks)
 *   MOE_PREFETCH_MB=n       L2 prefetch of the chosen experts' tiles by the
 *                           routing CTA once they are known, at most n MB
 *                           (default 0 = off: one SM issues them too slowly)
 *   MOE_DIRECT_ROUTE=0      the routing CTA waits for summed logits also at
 *                           B <= 4 (default: it sums the router partials itself)
 *   MOE_PROD_SLEEP, MOE_CONS_SLEEP  ns a ring warp sleeps between barrier polls
 *   MOE_FAIL_ALLOC_AFTER=n  fail this plan's (n+1)-th device allocation with
 *                           MOE_ERR_OOM (tests of the error path; everything
 *                           allocated before it is released)
 */
MOE_API moe_status moe_plan_create(const moe_config *cfg, int device, moe_plan *out);

/*
 * Pack canonical weights (device pointers, see moe_weights) into the plan's
 * kernel layouts.  Runs kernels on `stream` and synchronises it before
 * returning.  Rejects e8m0 byte 0xFF with MOE_ERR_RANGE (plan stays unloaded).
 */
MOE_API moe_status moe_load_weights(moe_plan p, const moe_weights *w, void *stream);

/*
 * out[B][H] (bf16, device) = block(x[B][H] bf16, device).  B = num_tokens,
 * 1..max_tokens.  x and out must be 16-byte aligned and must not overlap.
 * Asynchronous on `stream`: allocates nothing, does no host synchronisation,
 * may be captured into a CUDA graph.  Every kernel runs on `stream`, each a
 * programmatic dependent launch of the one before.  Errors: INVALID_ARG,
 * NOT_LOADED, CUDA (launch failure).
 */
MOE_API moe_status moe_forward(moe_plan p, const void *x, int32_t num_tokens, void *out, void *stream);

/*
 * Same block with HOST buffers: copies x_host to a plan-owned device buffer,
 * runs moe_forward and copies the result to out_host, all enqueued on
 * `stream`.  With pinned host memory the call is asynchronous; the caller
 * synchronises `stream` before reading out_host.
 */
MOE_API moe_status moe_forward_host(moe_plan p, const void *x_host, int32_t num_tokens, void *out_host,
                            void *stream);

/*
 * Copy the routing of the most recent forward to host memory (synchronises
 * the device): ids_host[B][k] int32 in key-descending order, w_host[B][k]
 * float combine weights.  Either pointer may be NULL.
 */
MOE_API moe_status moe_last_routing(moe_plan p, int32_t *ids_host, float *w_host, int32_t num_tokens);

/* Intermediates of the most recent forward, decoded to float32 (synchronises). */
enum {
  MOE_DBG_LOGITS = 0, /* [B][E] router logits */
  MOE_DBG_Z = 1,      /* [B][L] latent activations as stored for the experts (f16 with a
                         power-of-two scale per 32, or the sum of four e2m1 terms) */
  MOE_DBG_H = 2,      /* [B][k][I] expert SwiGLU outputs as stored for the down projection */
  MOE_DBG_Y = 3,      /* [B][k][L] expert outputs (before the weighted combine) */
  MOE_DBG_HS = 4      /* [B][I_s] shared-expert SwiGLU output */
};
MOE_API moe_status moe_debug_fetch(moe_plan p, int32_t what, int32_t num_tokens, float *host, int64_t count);

/* Synchronise the device and report the plan's device-side error word
 * (MOE_ERR_TIMEOUT if a bounded wait gave up), then clear it.  After a
 * timeout the plan's scheduling state (split-K tickets, piece cursors, the
 * routing flag and counts) is also cleared, so the next forward starts as on
 * a fresh plan; the output of the forward that timed out is undefined. */
MOE_API moe_status moe_sync_status(moe_plan p);

/*
 * Test of the timeout path, for tests only.  Enqueues on `stream` one thread
 * that leaves the plan's scheduling state as a forward cut short by an
 * expired wait could (a router row block counted, a split-K ticket taken, a
 * piece cursor advanced, the routing flag raised), then runs the kernels'
 * bounded flag wait on a flag that nothing sets, giving up after
 * limit_polls polls (1..2^22; 1000 polls take well under a millisecond).
 * The next moe_sync_status returns MOE_ERR_TIMEOUT and clears that state.
 * Errors: INVALID_ARG, CUDA.
 */
MOE_API moe_status moe_debug_expire_wait(moe_plan p, int32_t limit_polls, void* stream);

MOE_API moe_status moe_get_plan_info(moe_plan p, moe_plan_info *info);

/*
 * Per-kernel timing, for measurement only.  While enabled, moe_forward brackets
 * each of its kernels with CUDA events on the stream that kernel runs on and
 * waits for them before returning (so profiled forwards are synchronous and
 * must not be captured into a graph).  moe_get_profile writes the accumulated
 * milliseconds per kernel to ms[0..6] -- {dense front (router, latent
 * [, shared gate/up], top-k), expert gate/up, expert down, latent tail, fused
 * single launch, side-lane front (shared gate/up), side-lane tail (shared
 * down)}; the fused launch (MOE_FUSED=1, at most 8 tokens) replaces the
 * first four, the side lane (at most 4 tokens, shared_sms > 0) adds the
 * last two -- and the number of profiled forwards to *count, then clears
 * both.
 */
MOE_API moe_status moe_set_profiling(moe_plan p, int32_t enable);

/*
 * Per-CTA timeline of the most recent forward, for measurement only; exists
 * when the plan was created with the environment variable MOE_TRACE set
 * (else MOE_ERR_UNSUPPORTED).  host receives count = 7 * num_sms * 24 uint64:
 * for launch slot k (as in moe_get_profile) and CTA c, the 24 values at
 * (k * num_sms + c) * 24 are (ns from globaltimer, cycles from clock64):
 *   0 start ns, 1 end ns, 2 pieces, 3 finalizes, 4/5 top-k start/end ns (the
 *   routing CTA), 6 first stage ready ns, 7 ns spent finalising, 8..10
 *   consumer cycles waiting for data / computing / closing pieces (8..11 in
 *   the fused slot: ns the producer took its first piece of each phase),
 *   11..13 producer cycles waiting for a free stage / issuing / stages issued,
 *   14 the SM the CTA ran on, 15..18 fused slot: ns of the consumers' first
 *   stage of each phase (the routing CTA: top-k phase stamps in 16..18),
 *   19 ns the router logits of a row block were published, 21..22 routing
 *   CTA: slice selection end, merge end (8 or more tokens: logits staged,
 *   first token selected; 20: the first warp's tokens of the first staged
 *   group selected); in the expert kernels' slots 20/21 producer cycles
 *   setting stages up (header, weight tile) / copying activations, 22/23 the
 *   tensor-core MMA warp's cycles waiting for stages / issuing.
 * Synchronises the device.
 */
MOE_API moe_status moe_debug_trace(moe_plan p, uint64_t *host, int64_t count);
MOE_API moe_status moe_get_profile(moe_plan p, float *ms, int32_t *count);

/* Launch geometry of one kernel kind, as moe_forward would choose it. */
typedef struct moe_geometry {
  int32_t kind;               /* 0 dense front, 1 expert gate/up, 2 expert down, 3 latent tail,
                                 4 side-lane front (shared gate/up), 5 side-lane tail
                                 (shared down) */
  int32_t grid;               /* CTAs launched */
  int32_t ctas_per_sm;        /* 1, or 2 for the one-tile expert kernels */
  int32_t token_tiles;        /* 8-column token tiles the kernel is instantiated for */
  int32_t max_piece_tokens;   /* most tokens one piece can hold */
  int32_t stages;             /* ring depth */
  int32_t stage_bytes;        /* bytes of one ring stage */
  int32_t pieces_per_row_block; /* split-K factor (expert kinds: at the most virtual experts) */
  int64_t smem_bytes;         /* dynamic shared memory per CTA */
  int64_t partial_floats_needed;   /* split-K partial sums this forward can write */
  int64_t partial_floats_capacity; /* what a plan allocates (largest over every B) */
  int32_t route_logit_floats; /* front: logits the routing CTA can stage at once (else 0) */
  int32_t resident_tail_bytes; /* tail: shared-memory bytes of the resident activation (0: staged) */
} moe_geometry;

/*
 * The geometry moe_forward(num_tokens) would use on a device with num_sms
 * SMs, for the 6 kinds (out[0..5]; the side lane's two have grid 0 when the
 * forward has no side lane), with the default settings (environment
 * variables are not read).  Host only: needs no device and allocates no
 * device memory, so the planner can be checked anywhere.
 * Errors: INVALID_ARG (null, bad shape, num_sms < 2, num_tokens outside
 * 1..max_tokens), UNSUPPORTED (shape beyond the limits above), OOM.
 */
MOE_API moe_status moe_debug_geometry(const moe_config *cfg, int32_t num_sms, int32_t num_tokens,
                                      moe_geometry *out);

/*
 * Router scores and top-k for callers that cannot allocate device memory.
 * The source pages have no counterpart to this call; it exists for code that
 * runs where no allocation may happen (a fixed up-front memory budget, a
 * custom allocator that must account for every byte, a thread that may not
 * call cudaMalloc) and therefore cannot create a plan.
 *
 * Computes the routing step of moe_forward for B = num_tokens tokens on the
 * CURRENT device: logits = x . router_w, scores (softmax, or sigmoid plus the
 * selection bias), top-k with ties to the lower index, combine weights
 * renormalised when `renormalize`, times routed_scale.
 *   x         device bf16 [B][hidden]
 *   router_w  device bf16 [hidden][num_experts] (canonical, unpacked)
 *   router_bias device f32 [num_experts] or NULL (used for sigmoid scoring only)
 *   ids       device int32 [B][top_k] out, key-descending
 *   weights   device f32   [B][top_k] out
 * Allocates nothing: its only scratch is a 512 KB array in the library's
 * device memory (statically sized, present on every GPU that loads the
 * library until the process exits).  The first call on a device looks up that
 * array's device address; make that first call before any stream capture.
 * Every call shares the array, so calls whose kernels overlap on the GPU
 * (different streams, or different host threads) race; serialise them.
 * Limits: B <= 128, num_experts <= 1024, top_k <= 16, else MOE_ERR_UNSUPPORTED.
 * Asynchronous on `stream`.
 */
MOE_API moe_status moe_route_noalloc(const void *x, const void *router_w, const float *router_bias,
                                     int32_t num_tokens, int32_t hidden, int32_t num_experts,
                                     int32_t top_k, int32_t score_fn, int32_t renormalize,
                                     float routed_scale, int32_t *ids, float *weights, void *stream);

/*
 * Cross-layer weight prefetch ("Hyper Optimizing Kimi K3 in vLLM", section
 * 从算子之间找时间: fetch the next step's weights while HBM is under-used).
 * From now on every forward of `p` also pulls the first `bytes` bytes of
 * `next`'s front weights into L2: the router rows first, then the latent
 * projection's, then the shared expert's gate/up rows (the order in which
 * next's front kernel streams them).  The requests are issued by p's expert
 * down kernel once each of its CTAs has issued its own stages, so they fill
 * the HBM idle time of p's expert and tail phases; a forward of `next` that
 * follows on the same GPU then reads those rows from L2.
 *   next   a live plan on the same device (it may be p itself), or NULL
 *   bytes  clamped to next's front weight size and rounded down to 16;
 *          0 or next == NULL turns the prefetch off
 * Results are unchanged: only where next's front kernel finds its weights.
 * Destroying `next` turns the prefetch off on every plan that names it.  A
 * captured CUDA graph keeps the pointer it was captured with: keep `next`
 * alive while such a graph may run.
 * Errors: MOE_ERR_INVALID_ARG for a p or next that is not a live plan,
 * bytes < 0, or plans on different devices (p is then unchanged).
 * Host-side only; thread-safe with respect to plan creation and destruction.
 */
MOE_API moe_status moe_set_next_layer(moe_plan p, moe_plan next, int64_t bytes);

/* Release everything the plan owns.  NULL is ignored. */
MOE_API void moe_plan_destroy(moe_plan p);

/* Static string for a status code. */
MOE_API const char *moe_status_str(moe_status s);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
