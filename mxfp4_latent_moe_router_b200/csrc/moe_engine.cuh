// moe_engine.cuh -- the four kernels of one latent-MoE decode step on sm_100a
// (device code; each kind is instantiated in its own moe_k_<kind>.cu).
//
// One engine serves all four: a CTA of 8 consumer warps and 1 producer warp.
// The producer grabs "pieces" (a row block of 128 output rows x a run of K
// chunks) from a global cursor and streams each chunk's weight tile plus the
// activation rows it multiplies into a ring of shared-memory stages with bulk
// copies (TMA engine) that complete on mbarriers.  Each consumer warp owns 16
// of the 128 rows and multiplies them with m16n8k16 warp MMAs, weights as the
// 16-row A operand and up to 8*NT tokens as the 8-column B operand ("swap
// AB"), fp32 accumulators in registers.  When a piece ends, its fp32 partial
// sums go to global memory; the CTA that completes the last piece of a row
// block sums all of them in piece order (deterministic split-K) and runs the
// kernel's epilogue.  Dynamic piece grabbing balances the work across SMs and
// lets a CTA that does extra epilogue work fall behind without stalling the
// others.
//
//   KIND_FRONT x . [W_r | W_in | W_sg,W_su] in one weight-streaming pass over
//             every SM: router logits (fp32), latent z (f16 MX) and the shared
//             expert's h_s = silu(g) * u (fp32).  The router row blocks come
//             first; the grid's last CTA takes no pieces and runs top-k and
//             the per-expert token lists as soon as they are summed, while
//             the other CTAs still stream the rest.
//             (page "Hyper Optimizing Kimi K3 in vLLM: Moving Fast and
//              Responsibly", section 从算子之间找时间: the router scores and the
//              latent input projection as one matmul, and the shared expert
//              overlapping the routing.  One GPU has no ranks to split the
//              matmul over, and a second stream would only contend for the
//              same HBM, so the shared expert's rows join the same pass.)
//   KIND_EGU  per routed expert, z . [Wg | Wu] (MXFP4) -> h = silu(g) * u (f16 MX)
//   KIND_EDN  per routed expert, h . Wd (MXFP4) -> y (fp32, per token slot)
//   KIND_TAIL c = sum_j w_j y_j formed from y while staging the activation
//             tile (never written to memory), then [c ; h_s] . [W_out ; W_sd]
//             -> out (bf16).
//             (page "Kimi K3 在 vLLM 中的性能优化", section 延迟 MXFP4 最终化:
//              the MXFP4 top-k finalize fused into the latent-tail kernel.)
//
// Only static weights are fetched before griddepcontrol.wait; activations are
// fetched after it (page "Hyper Optimizing Kimi K3 in vLLM: Moving Fast and
// Responsibly", section 更快的代码需要更有针对性的验证: an activation load
// hoisted above a synchronisation wait was a real bug).  The expert kernels
// may also read the routing tables before it, but only after acquiring the
// flag that publishes them.
#pragma once
#include <cuda_runtime.h>

#include "engine.cuh"
#include "layout.cuh"
#include "ptx.cuh"
#include "topk.cuh"
#include "umma.cuh"

namespace moe {

constexpr int kHdrBytes = 128;
static_assert(kHdrBytes == kUHdrBytes, "tensor-core stages share the header size");
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kMaxStages = 8;
constexpr int kTraceStride = 24;  // u64 per CTA in the optional trace

enum : int { HDR_FIRST = 1, HDR_LAST = 2, HDR_END = 4 };

struct Hdr {
  int flags;
  int piece, v, rb;
  int chunk, nb, ntok, tok0;
  int expert, ppr, act_bytes;
  int p0;  // first partial slot of this row block (its partial sums are p0 .. p0 + ppr - 1)
  int c_first, c_last;  // chunks of this piece
  int dep;              // 1: its activations need the kernel's dependency resolved
  // fused single-launch path: this piece's kind, and on its last stage the
  // kind of the piece the producer streams next (-1: none)
  int kind, next_kind;
};

template <int KIND>
struct KindTraits {
  static constexpr bool kMx = (KIND == KIND_EGU || KIND == KIND_EDN);
  static constexpr int kTileBytes = kMx ? kMxTileBytes : kDenseTileBytes;
  static constexpr int kChunkK = kMx ? kMxChunkK : kDenseChunkK;
  static constexpr bool kDynamicSpace = (KIND == KIND_EGU || KIND == KIND_EDN);
};

__device__ __forceinline__ uint4 lds128(const uint8_t* p) {
  return *reinterpret_cast<const uint4*>(p);
}

__device__ __forceinline__ float silu(float t) { return __fdividef(t, 1.0f + __expf(-t)); }

// ---------------------------------------------------------------------------
// iteration space

struct Space {
  int total;  // pieces
  int ppr;
};

// V: virtual experts (the routing's nve), read by the caller together with
// the routing tables so that sizing the space costs no extra round trip
template <int KIND>
__device__ __forceinline__ Space make_space(const Params& p, int V = 0) {
  Space s;
  if (KIND == KIND_EGU || KIND == KIND_EDN) {
    const int mats = V * p.RB;
    const int ppr = p.PPR > 0 ? min(p.PPR, p.C) : best_ppr(mats, p.C, p.piece_ctas, p.split_cost);
    s.ppr = ppr;
    s.total = mats * ppr;
  } else if (KIND == KIND_TAIL) {
    const int passes = (p.B + p.tg - 1) / p.tg;
    s.ppr = p.PPR;
    const int per = p.tail_part == 1 ? p.ppr_lat : p.tail_part == 2 ? p.ppr_sh : p.PPR;
    s.total = passes * p.RB * per;  // (split or not: ppr_sh + ppr_lat == PPR)
  } else {
    // FRONT: the router row blocks come first, in pieces of their own size
    // (when this launch holds them), then the rest of [rb_lo, rb_hi)
    s.ppr = p.PPR;
    const bool router = p.rb_lo == 0;
    const int rb0 = router ? p.RB_router : p.rb_lo;
    s.total = (router ? p.RB_router * p.PPR_r : 0) + (p.rb_hi - rb0) * p.PPR;
  }
  return s;
}

// number of 32-wide K blocks in chunk c
template <int KIND>
__device__ __forceinline__ int chunk_blocks(const Params& p, int c) {
  constexpr int kMaxB = KindTraits<KIND>::kChunkK / 32;
  int k0, kext;
  if (KIND == KIND_TAIL) {
    if (c < p.C_lat) {
      k0 = c * kDenseChunkK;
      kext = p.L;
    } else {
      k0 = (c - p.C_lat) * kDenseChunkK;
      kext = p.KS;
    }
  } else {
    k0 = c * KindTraits<KIND>::kChunkK;
    kext = p.KL;
  }
  int nb = (kext - k0) / 32;
  return nb > kMaxB ? kMaxB : nb;
}

// ---------------------------------------------------------------------------
// producer warp

// Per piece: everything except the chunk-dependent fields.
template <int KIND>
__device__ __forceinline__ void piece_header(const Params& p, const Space& sp, int piece, Hdr& h,
                                             const VExpert* ve_tab) {
  h.piece = piece;
  h.expert = 0;
  h.dep = 1;
  if (KIND == KIND_TAIL && (p.tail_split || p.tail_part)) {
    // shared-expert pieces of every (pass, row block) first, then the latent
    // ones; a row block's partial slots stay contiguous (latent j, then
    // shared ppr_lat + j) so the finalising sum keeps one fixed order.  A
    // lane (tail_part 1 or 2) holds only one of the two kinds, and waits for
    // its own predecessor before reading any activation.
    const int n_sh = p.tail_part == 1 ? 0 : p.tail_part == 2 ? sp.total : sp.total / p.PPR * p.ppr_sh;
    int q, pp, cb, cn, slot0;
    if (piece < n_sh) {
      q = piece / p.ppr_sh;
      pp = piece % p.ppr_sh;
      cb = p.C_lat;
      cn = p.C - p.C_lat;
      slot0 = p.ppr_lat;
      h.dep = 0;
    } else {
      q = (piece - n_sh) / p.ppr_lat;
      pp = (piece - n_sh) % p.ppr_lat;
      cb = 0;
      cn = p.C_lat;
      slot0 = 0;
    }
    const int pieces_here = h.dep ? p.ppr_lat : p.ppr_sh;
    if (p.tail_part) h.dep = 1;
    h.v = q / p.RB;
    h.rb = q % p.RB;
    h.ppr = p.PPR;
    h.p0 = q * p.PPR;
    h.piece = h.p0 + slot0 + pp;
    h.c_first = cb + (pp * cn) / pieces_here;
    h.c_last = cb + ((pp + 1) * cn) / pieces_here;
    h.tok0 = h.v * p.tg;
    h.ntok = min(p.tg, p.B - h.tok0);
    return;
  }
  const int nr = (KIND == KIND_FRONT && p.rb_lo == 0) ? p.RB_router * p.PPR_r : 0;
  if (piece < nr) {  // router row blocks (smaller pieces, so the logits are summed early)
    h.v = 0;
    h.rb = piece / p.PPR_r;
    h.ppr = p.PPR_r;
    h.p0 = h.rb * p.PPR_r;
  } else {
    const int q = piece - nr;
    const int rb0 = KIND == KIND_FRONT ? (p.rb_lo == 0 ? p.RB_router : p.rb_lo) : 0;
    const int rb1 = KIND == KIND_FRONT ? p.rb_hi : p.RB;
    const int per_v = (rb1 - rb0) * sp.ppr;
    const int v = q / per_v;
    const int rem = q - v * per_v;
    h.v = v;
    h.rb = rb0 + rem / sp.ppr;
    h.ppr = sp.ppr;
    h.p0 = piece - rem % sp.ppr;
  }
  if (KIND == KIND_FRONT) {
    h.ntok = p.B;
    h.tok0 = 0;
  } else if (KIND == KIND_TAIL) {
    h.tok0 = h.v * p.tg;
    h.ntok = min(p.tg, p.B - h.tok0);
  } else {
    const VExpert ve = ve_tab[h.v];
    h.expert = ve.expert;
    h.tok0 = ve.start;
    h.ntok = ve.count;
  }
  const int pr = h.piece - h.p0;
  h.c_first = (pr * p.C) / h.ppr;
  h.c_last = ((pr + 1) * p.C) / h.ppr;
}

// Per chunk: flags, block count and activation bytes.
template <int KIND>
__device__ __forceinline__ void chunk_header(const Params& p, int c, int c_first, int c_last, Hdr& h) {
  h.flags = (c == c_first ? HDR_FIRST : 0) | (c == c_last - 1 ? HDR_LAST : 0);
  h.chunk = c;
  h.nb = chunk_blocks<KIND>(p, c);
  int ab;
  if (KIND == KIND_FRONT)
    ab = h.ntok * h.nb * 64;
  else if (KIND == KIND_EGU || KIND == KIND_EDN)
    ab = h.ntok * p.act_rec;
  else
    ab = p.res_off ? 0 : p.t_rec ? h.ntok * 256 : ((c < p.C_lat) ? h.ntok * p.topk * 256 : h.ntok * 256);
  h.act_bytes = ab;
}

template <int KIND>
__device__ __forceinline__ const uint8_t* weight_src(const Params& p, const Hdr& h) {
  const long long tile = (long long)h.rb * p.C + h.chunk;
  if (KindTraits<KIND>::kMx)
    return p.wt + (long long)h.expert * p.matrix_bytes + tile * kMxTileBytes;
  return p.wt + tile * kDenseTileBytes;
}

// A stage's activation rows are one bulk copy each, but the copy engine takes
// bulk copies one at a time: past 8 rows (64 rows of 128 bytes at B = 64)
// issuing them outlasts the stage's own weight tile.  Such stages copy their
// rows in 16-byte pieces from all producer lanes instead; their full barrier
// then expects only the weight tile's bytes and completes once the lanes'
// copies have landed and lane 0 has arrived.
constexpr int kBulkRowsMax = 8;
template <int KIND>
__device__ __forceinline__ bool rows_async(const Params& p, const Hdr& h) {
  if ((KIND == KIND_EGU || KIND == KIND_EDN || KIND == KIND_TAIL) && p.umma)
    return true;  // scattered into the MMA's B layout
  if (KIND == KIND_FRONT && p.front_umma) return true;
  return (KIND == KIND_FRONT || KIND == KIND_EGU || KIND == KIND_EDN) && h.ntok > kBulkRowsMax;
}

// Lane 0: a stage's header, its barrier expectation and its weight tile.
template <int KIND>
__device__ __forceinline__ void stage_begin(const Params& p, const Hdr& h, uint8_t* sb, uint64_t* bar) {
  constexpr int kTile = KindTraits<KIND>::kTileBytes;
  *reinterpret_cast<Hdr*>(sb) = h;
  // A slot's activation rows come in 16-byte copies for stages of more than
  // kBulkRowsMax rows and in bulk copies otherwise.  Only the warp-level
  // expert kernels with token groups above that size can mix the two in one
  // launch: there a slot's earlier copies are ordered before the next bulk
  // copy into it.  (The front kernel's stages all hold the same B rows; the
  // tensor-core stages fill each region one way.)
  if ((KIND == KIND_EGU || KIND == KIND_EDN) && !p.umma && p.tg > kBulkRowsMax)
    fence_proxy_async_smem();
  if (rows_async<KIND>(p, h))
    mbar_expect_tx(bar, kTile);  // lane 0 arrives once the rows are issued
  else
    mbar_arrive_expect_tx(bar, kTile + h.act_bytes);
  if (KindTraits<KIND>::kMx && p.umma) {
    // the packed codes as the A operand, the scales behind them
    const uint8_t* src = weight_src<KIND>(p, h);
    bulk_g2s(sb + kUAOff, src, kMxCodeBytes, bar);
    bulk_g2s(sb + kUSfaOff, src + kMxCodeBytes, kMxScaleBytes, bar);
    return;
  }
  bulk_g2s(sb + kHdrBytes, weight_src<KIND>(p, h), kTile, bar);
}

// The lanes' 16-byte copies are issued: the barrier now tracks their
// completion, and lane 0 adds its arrival once every lane has registered.
__device__ __forceinline__ void rows_async_done(uint64_t* bar, int lane) {
  cp_async_mbar_arrive(bar);
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

// Front: token rows of x, 2^lg_per 16-byte pieces each, rows ld bytes apart.
__device__ __forceinline__ void copy_x_rows_async(uint8_t* act, int stride, int nrows, int lg_per,
                                                  const uint8_t* src, long long ld, uint64_t* bar,
                                                  int lane) {
  for (int i = lane; i < (nrows << lg_per); i += 32) {
    const int r = i >> lg_per, q = i & ((1 << lg_per) - 1);
    cp_async16(act + r * stride + q * 16, src + r * ld + q * 16);
  }
  rows_async_done(bar, lane);
}

// Expert kernels: nrows activation records (kActRecBytes each).  Gathered
// rows (nrows <= 32) come from lane r's row pointer; otherwise the records
// are consecutive from src.
__device__ __forceinline__ void copy_records_async(uint8_t* act, int stride, int nrows,
                                                   const uint8_t* src, bool gathered,
                                                   uint64_t* bar, int lane) {
  constexpr int kPer = kActRecBytes / 16;
  const int n = nrows * kPer;
  for (int i0 = 0; i0 < n; i0 += 32) {  // the whole warp in every round (shuffles)
    const int i = i0 + lane;
    const int r = min(i / kPer, nrows - 1), q = i - r * kPer;
    const uint8_t* row =
        gathered ? reinterpret_cast<const uint8_t*>(
                       __shfl_sync(0xffffffffu, reinterpret_cast<uintptr_t>(src), r))
                 : src + (long long)r * kActRecBytes;
    if (i < n) cp_async16(act + r * stride + q * 16, row + q * 16);
  }
  rows_async_done(bar, lane);
}

// Tensor-core stage: every token's kUTerms term rows into the B operand's
// core-matrix layout (row n = term * 8 NT + token; K block kb of row n at
// (kb * ng + n / 8) * 128 + (n % 8) * 16, ng = rows / 8) and their scales into
// the two 512-byte units; 16- and 4-byte copies spread over the producer
// lanes.  nt: the kernel's token tiles.
template <int KIND>
__device__ __forceinline__ void copy_records_umma(const Params& p, const Hdr& h, uint8_t* sb,
                                                  uint64_t* bar, int lane, const int* slot_tab,
                                                  int nt) {
  const int rows = umma_rows(nt), ng = rows / 8, per_tok = 8 * nt;
  uint8_t* B = sb + kUBOff;
  uint8_t* sfb = B + rows * kUTermBytes;
  const int cz = (p.L + kMxChunkK - 1) / kMxChunkK;
  // lane -> (token, term) rows, the token fastest: one record pointer a row,
  // then its 8 K blocks of 16 bytes and 2 scale words
  for (int it = lane; it < per_tok * kUTerms; it += 32) {
    const int tok = it & (per_tok - 1), t = it / per_tok;
    if (tok >= h.ntok) continue;
    const uint8_t* rec;
    if (KIND == KIND_EGU)
      rec = p.z_mx + ((long long)(slot_tab[h.tok0 + tok] / p.topk) * cz + h.chunk) * p.act_rec;
    else
      rec = p.h_mx + ((long long)h.chunk * p.ld_slots + h.tok0 + tok) * p.act_rec;
    const int n = t * per_tok + tok;
    uint8_t* dst = B + (n >> 3) * 128 + (n & 7) * 16;
    const uint8_t* src = rec + t * kUTermBytes;
#pragma unroll
    for (int q = 0; q < kMxChunkK / 32; ++q) cp_async16(dst + q * ng * 128, src + q * 16);
    const uint8_t* ssrc = rec + kUTerms * kUTermBytes + t * 8;
    uint8_t* sdst = sfb + (n & 31) * 16 + (n >> 5) * 4;
    cp_async4(sdst, ssrc);
    cp_async4(sdst + 512, ssrc + 4);
  }
  rows_async_done(bar, lane);
}

// Tensor-core tail stage: every token's formed record (bf16 hi and lo parts
// of one 64-wide chunk) as two rows of the B operand (row n = part * 8 NT +
// token; K block kb of row n at (kb * ng + n / 8) * 128 + (n % 8) * 16).
__device__ __forceinline__ void copy_tail_records_umma(const Params& p, const Hdr& h, uint8_t* B,
                                                       uint64_t* bar, int lane, int nt) {
  const int per_tok = 8 * nt, ng = 2 * per_tok / 8;
  for (int it = lane; it < 2 * per_tok; it += 32) {
    const int tok = it & (per_tok - 1), part = it / per_tok;
    if (tok >= h.ntok) continue;
    const uint8_t* src = p.t_rec + ((long long)h.chunk * p.B + h.tok0 + tok) * 256 + part * 128;
    const int n = part * per_tok + tok;
    uint8_t* dst = B + (n >> 3) * 128 + (n & 7) * 16;
#pragma unroll
    for (int q = 0; q < kDenseChunkK / 8; ++q) cp_async16(dst + q * ng * 128, src + q * 16);
  }
  rows_async_done(bar, lane);
}

// Tensor-core front stage: the tokens' x rows of this 64-wide chunk into the
// B operand's core-matrix layout (token n's K block kb at (kb * NT + n / 8) *
// 128 + (n % 8) * 16); K blocks past the chunk's valid blocks (a ragged last
// chunk) are zero-filled, reading nothing.
__device__ __forceinline__ void copy_x_rows_umma(const Params& p, const Hdr& h, uint8_t* B,
                                                 uint64_t* bar, int lane, int nt) {
  const uint8_t* x = reinterpret_cast<const uint8_t*>(p.x + h.chunk * kDenseChunkK);
  const int kb_valid = h.nb * 4;  // 16-byte K blocks holding real columns
  for (int tok = lane; tok < h.ntok; tok += 32) {
    const uint8_t* src = x + (long long)tok * p.H * 2;
    uint8_t* dst = B + (tok >> 3) * 128 + (tok & 7) * 16;
#pragma unroll
    for (int q = 0; q < kDenseChunkK / 8; ++q)
      cp_async16_zfill(dst + q * nt * 128, q < kb_valid ? src + q * 16 : src, q < kb_valid ? 16u : 0u);
  }
  rows_async_done(bar, lane);
}

// Issue this stage's activation copies (all 32 producer lanes).
template <int KIND>
__device__ __forceinline__ void issue_act(const Params& p, const Hdr& h, uint8_t* act, uint64_t* bar,
                                          int lane, const int* slot_tab) {
  if ((KIND == KIND_EGU || KIND == KIND_EDN) && p.umma) {
    copy_records_umma<KIND>(p, h, act - p.act_off, bar, lane, slot_tab, p.umma);  // (umma = NT)
    return;
  }
  if (KIND == KIND_TAIL && p.umma) {
    copy_tail_records_umma(p, h, act, bar, lane, p.umma);  // (umma = NT)
    return;
  }
  if (KIND == KIND_FRONT && p.front_umma) {
    copy_x_rows_umma(p, h, act, bar, lane, p.front_umma);  // (front_umma = NT)
    return;
  }
  if (rows_async<KIND>(p, h)) {
    if (KIND == KIND_FRONT) {
      const uint8_t* x = reinterpret_cast<const uint8_t*>(p.x + h.chunk * kDenseChunkK);
      copy_x_rows_async(act, p.act_stride, h.ntok, h.nb == 2 ? 3 : 2, x, (long long)p.H * 2, bar, lane);
    } else if (KIND == KIND_EGU) {
      // lane r: token row of slot r (a virtual expert holds at most 32 slots)
      const int cz = (p.L + kMxChunkK - 1) / kMxChunkK;
      const uint8_t* mine = p.z_mx + (long long)h.chunk * p.act_rec;
      if (lane < h.ntok) mine += (long long)(slot_tab[h.tok0 + lane] / p.topk) * cz * p.act_rec;
      copy_records_async(act, p.act_stride, h.ntok, mine, true, bar, lane);
    } else {
      copy_records_async(act, p.act_stride, h.ntok,
                         p.h_mx + ((long long)h.chunk * p.ld_slots + h.tok0) * p.act_rec, false,
                         bar, lane);
    }
    return;
  }
  if (KIND == KIND_FRONT) {
    const int bytes = h.nb * 64;
    for (int r = lane; r < h.ntok; r += 32)
      bulk_g2s(act + r * p.act_stride, p.x + (long long)r * p.H + h.chunk * kDenseChunkK, bytes, bar);
  } else if (KIND == KIND_EGU) {
    const int cz = (p.L + kMxChunkK - 1) / kMxChunkK;
    for (int r = lane; r < h.ntok; r += 32) {
      const int slot = slot_tab[h.tok0 + r];
      const int tok = slot / p.topk;
      bulk_g2s(act + r * p.act_stride, p.z_mx + ((long long)tok * cz + h.chunk) * kActRecBytes,
               kActRecBytes, bar);
    }
  } else if (KIND == KIND_EDN) {
    for (int r = lane; r < h.ntok; r += 32)
      bulk_g2s(act + r * p.act_stride,
               p.h_mx + ((long long)h.chunk * p.ld_slots + h.tok0 + r) * kActRecBytes, kActRecBytes,
               bar);
  } else {
    if (lane == 0 && !p.res_off && p.t_rec) {
      bulk_g2s(act, p.t_rec + ((long long)h.chunk * p.B + h.tok0) * 256, h.act_bytes, bar);
    } else if (lane == 0 && !p.res_off) {
      if (h.chunk < p.C_lat)
        bulk_g2s(act, p.y + ((long long)h.chunk * p.ld_slots + (long long)h.tok0 * p.topk) * 64,
                 h.act_bytes, bar);
      else
        bulk_g2s(act, p.h_s + ((long long)(h.chunk - p.C_lat) * p.B + h.tok0) * 64, h.act_bytes,
                 bar);
    }
  }
}

// Bounded wait (about a second at the default limit of 2^22 polls) until
// *flag != 0, with acquire semantics for the calling thread; false (and an
// error bit) if it never is.
__device__ __forceinline__ bool wait_flag(const int* flag, int* err, int err_bit, int lane,
                                          uint32_t limit = 1u << 22) {
  for (uint32_t i = 0; i < limit; ++i) {
    if (ld_acquire(flag) != 0) return true;
    __nanosleep(256);
  }
  if (lane == 0) atomicOr(err, 1 << err_bit);
  return false;
}

// Bounded wait until *counter >= target (acquire); false and an error bit on
// expiry.
__device__ __forceinline__ bool wait_count(const int* counter, int target, int* err, int lane) {
  for (uint32_t i = 0; i < (1u << 22); ++i) {
    if (ld_acquire(counter) >= target) return true;
    __nanosleep(128);
  }
  if (lane == 0) atomicOr(err, 1 << ERR_WAIT_DEP);
  return false;
}

// The producer's dependency: what its activation copies must wait for.
//   FRONT, EDN, TAIL: the previous kernel of the stream, complete
//                     (griddepcontrol.wait);
//   EGU with z_done:  only the latent row blocks of the front kernel (z), by
//                     their release count -- the front's last CTAs stream
//                     shared-expert rows this kernel never reads.  Its
//                     dependents may launch at once; each CTA still waits for
//                     the front grid before it exits, so that this grid's
//                     completion implies the front's (the tail reads h_s and
//                     the combine weights after waiting only for its own
//                     predecessor).
//   EDN with h_done:  per piece, its virtual expert's h rows (the gate/up
//                     kernel's row-block count of that expert; see the
//                     producer), likewise with the exit wait.
template <int KIND>
__device__ __forceinline__ bool producer_dep_wait(const Params& p, int lane) {
  if (KIND == KIND_TAIL && p.t_rec) {
    // the records the grid's consumers form after the expert kernels
    pdl_trigger();
    const bool ok = wait_count(p.t_ready, (int)gridDim.x, p.err, lane);
    fence_proxy_async_global();  // the records are read by bulk copies
    return ok;
  }
  if (KIND == KIND_EGU && p.z_done) {
    const bool ok = wait_count(p.z_done, p.RB_lat, p.err, lane);
    fence_proxy_async_global();  // the z records are read by bulk copies
    return ok;
  }
  pdl_wait();
  pdl_trigger();
  return true;
}

template <int KIND>
__device__ void producer(const Params& p, Ctl* ctl, uint8_t* stage_base, uint8_t* tables,
                         uint64_t* full, uint64_t* empty, int lane) {
  int stage = 0;
  uint32_t ephase = 1;  // empty barriers start "released"
  Space sp;
  // every kind streams up to one ring of weight tiles before its dependency
  // resolves (stages filled with weights only, their activations pending:
  // always the last `prefetched` stages issued, from ring slot pend_first on)
  int prefetched = 0, pend_first = 0;
  bool waited = false;
  // The tail with its shared part first: those pieces need no dependency, so
  // CTAs take pieces (and keep a grab in flight) from the start; the first
  // latent piece they hold waits for it.
  const bool free_start = KIND == KIND_TAIL && p.tail_split && !p.tail_part;
  // The expert down kernel with per-expert counts: a piece's activations are
  // issued at once when its virtual expert's h is complete, else after its
  // weight tiles, once the count is reached (pending stages stay contiguous
  // in the ring: after one is deferred, the rest of the piece is too).
  const bool ve_dep = KIND == KIND_EDN && p.h_done != nullptr;
  if ((KIND == KIND_EGU && p.z_done) || ve_dep) pdl_trigger();
  // routing tables in shared memory: the per-stage lookups then cost no
  // global round trip (they are visible to the consumers through the first
  // full-barrier completion).  The whole capacity is copied so that these
  // loads and the count load below are independent and overlap.
  VExpert* ve_tab = reinterpret_cast<VExpert*>(tables);
  int* slot_tab = reinterpret_cast<int*>(tables + (size_t)p.ve_max * sizeof(VExpert));
  // The routing is published by the front kernel's routing CTA while the
  // front kernel may still run (every CTA of it is resident before this
  // kernel can launch, so the wait ends): wait for its flag, then read the
  // tables and start streaming the chosen experts' tiles before this kernel's
  // own dependency resolves.
  const bool route_ok = KindTraits<KIND>::kDynamicSpace ? wait_flag(p.route_ready, p.err, ERR_WAIT_DEP, lane) : true;
  int V = 0;
  if (KindTraits<KIND>::kDynamicSpace && route_ok) {
    // L2 reads, all in one round trip: the tables and the count were written
    // by another kernel that may still run
    V = __ldcg(p.nve);
    for (int i = lane; i < p.ve_max; i += 32) {
      const int4 v = __ldcg(reinterpret_cast<const int4*>(p.ve + i));
      ve_tab[i] = VExpert{v.x, v.y, v.z, v.w};
    }
    for (int i = lane; i < p.ld_slots; i += 32) slot_tab[i] = __ldcg(p.slots_sorted + i);
  }
  sp = make_space<KIND>(p, V);
  if (!route_ok) sp.total = 0;  // no pieces: straight to the end marker
  __syncwarp();

  // Resolve the dependency and issue the pending stages' activations.
  auto resolve = [&]() {
    if (ve_dep) {
      int v_ok = -1;
      for (int j = 0; j < prefetched; ++j) {
        const int s = (pend_first + j) % p.nstages;
        uint8_t* sb = stage_base + (size_t)s * p.stage_bytes;
        const Hdr& hs = *reinterpret_cast<const Hdr*>(sb);
        if (hs.v != v_ok) {
          if (!wait_count(p.h_done + hs.v, p.RB_egu, p.err, lane)) sp.total = 0;
          fence_proxy_async_global();  // (bulk copies read the records)
          v_ok = hs.v;
        }
        issue_act<KIND>(p, hs, sb + p.act_off, &full[s], lane, slot_tab);
      }
      prefetched = 0;
      return;
    }
    if (!producer_dep_wait<KIND>(p, lane)) sp.total = 0;  // gave up: no further pieces
    waited = true;
    for (int j = 0; j < prefetched; ++j) {
      const int s = (pend_first + j) % p.nstages;
      uint8_t* sb = stage_base + (size_t)s * p.stage_bytes;
      const Hdr& hs = *reinterpret_cast<const Hdr*>(sb);
      issue_act<KIND>(p, hs, sb + p.act_off, &full[s], lane, slot_tab);
    }
    prefetched = 0;
  };

  // every CTA starts on piece blockIdx.x (no round trip before the first
  // tile); later pieces come from the cursor, offset by the number of
  // piece-taking CTAs.  Lane 0 keeps one grab in flight and reads its result
  // one piece later -- but only once the dependency has resolved (or from the
  // start where the first pieces need none): CTAs that land early (while the
  // previous kernel's last CTAs still run) would otherwise take several
  // pieces each before the late ones can start, and finish last.
  long long pw = 0, pi = 0, nst = 0, pb = 0, pa = 0;
  int grabbed = 0;
  bool in_flight = false;
  const int workers = (int)gridDim.x - (KIND == KIND_FRONT ? p.route_cta : 0);
  int piece = blockIdx.x;
  if ((waited || free_start || ve_dep) && piece < sp.total) {
    if (lane == 0) grabbed = atomicAdd(&ctl->cursor, 1) + workers;
    in_flight = true;
  }
  while (true) {
    if (piece >= sp.total) break;
    Hdr ph;
    piece_header<KIND>(p, sp, piece, ph, ve_tab);
    const int c_first = ph.c_first, c_last = ph.c_last;
    if (ve_dep) {
      // its virtual expert's h complete already?
      int cnt = 0;
      if (lane == 0) cnt = ld_acquire(p.h_done + ph.v);
      ph.dep = __shfl_sync(0xffffffffu, cnt, 0) < p.RB_egu ? 1 : 0;
      if (!ph.dep) fence_proxy_async_global();
    }
    for (int c = c_first; c < c_last; ++c) {
      // before the dependency resolves, fill at most one ring of weight-only
      // stages: the slot to reuse next would otherwise be a pending one
      if (!waited && prefetched == p.nstages) resolve();
      const long long tw0 = clock64();
      if (!mbar_wait_bounded(&empty[stage], ephase, p.err, ERR_WAIT_EMPTY, p.prod_sleep)) return;
      const long long tw1 = clock64();
      pw += tw1 - tw0;
      uint8_t* sb = stage_base + (size_t)stage * p.stage_bytes;
      Hdr h = ph;
      chunk_header<KIND>(p, c, c_first, c_last, h);
      if (lane == 0) stage_begin<KIND>(p, h, sb, &full[stage]);
      __syncwarp();
      const long long tb = clock64();
      pb += tb - tw1;
      if ((waited || !h.dep) && !(ve_dep && prefetched > 0)) {
        issue_act<KIND>(p, h, sb + p.act_off, &full[stage], lane, slot_tab);
        pa += clock64() - tb;
      } else {
        if (prefetched == 0) pend_first = stage;
        ++prefetched;
      }
      if (++stage == p.nstages) {
        stage = 0;
        ephase ^= 1;
      }
      pi += clock64() - tw1;
      ++nst;
    }
    // a piece issued with pending activations: stop prefetching here
    if (!waited && (prefetched > 0 || (!free_start && !ve_dep))) resolve();
    if (!in_flight && lane == 0) grabbed = atomicAdd(&ctl->cursor, 1) + workers;
    piece = __shfl_sync(0xffffffffu, grabbed, 0);
    in_flight = piece < sp.total;
    if (lane == 0 && in_flight) grabbed = atomicAdd(&ctl->cursor, 1) + workers;
  }
  if (!waited && (prefetched > 0 || (!free_start && !ve_dep))) resolve();
  // cross-layer prefetch: this CTA's share of the next layer's front weights
  // into L2, 16 KB a request (no data lands in this CTA; the copies only warm
  // L2 for the next forward's front kernel)
  if (KIND == KIND_EDN && p.pf_bytes > 0) {
    const long long per = (p.pf_bytes / gridDim.x + 16383) & ~16383LL;
    const long long lo = (long long)blockIdx.x * per, hi = min(p.pf_bytes, lo + per);
    for (long long o = lo + (long long)lane * 16384; o < hi; o += 32LL * 16384)
      prefetch_l2(p.pf_src + o, (uint32_t)min(16384LL, hi - o));
  }
  if (p.trace && lane == 0) {
    unsigned long long* tr = p.trace + (size_t)blockIdx.x * kTraceStride;
    tr[11] = (unsigned long long)pw;
    tr[12] = (unsigned long long)pi;
    tr[13] = (unsigned long long)nst;
    if (KIND == KIND_EGU || KIND == KIND_EDN) {  // (slots the routing uses in the front kernel)
      tr[20] = (unsigned long long)pb;
      tr[21] = (unsigned long long)pa;
    }
  }
  // end marker
  if (!mbar_wait_bounded(&empty[stage], ephase, p.err, ERR_WAIT_EMPTY, p.prod_sleep)) return;
  if (lane == 0) {
    uint8_t* sb = stage_base + (size_t)stage * p.stage_bytes;
    reinterpret_cast<Hdr*>(sb)->flags = HDR_END;
    mbar_arrive(&full[stage]);
  }
}

// ---------------------------------------------------------------------------
// consumer math

template <int NT>
__device__ __forceinline__ void zero_acc(float (&acc)[NT][4]) {
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[t][q] = 0.f;
}

// bf16 weights x bf16 token rows (x): RL, SGU
template <int NT>
__device__ __forceinline__ void mma_dense_x(const Params& p, const Hdr& h, const uint8_t* tile,
                                            const uint8_t* act, float (&acc)[NT][4],
                                            float (&acc2)[NT][4], int warp, int lane) {
  const int g = lane >> 2, tig = lane & 3;
  // loads first and unconditionally, then the MMAs.  Token columns past ntok
  // read token 0's row again: their sums are finite duplicates that no
  // epilogue, partial or store ever reads.
  uint4 a[2][2];
#pragma unroll
  for (int b = 0; b < 2; ++b)
#pragma unroll
    for (int s = 0; s < 2; ++s) a[b][s] = lds128(tile + ((warp * 2 + b) * 2 + s) * 512 + lane * 16);
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int tok = 8 * t + g;
    const bool tv = tok < h.ntok;
    const uint8_t* row = act + (tv ? tok : 0) * p.act_stride + 8 * tig * 2;
    uint4 bv[2] = {lds128(row), lds128(row + 64)};
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      if (b < h.nb) {
        const uint32_t A0[4] = {a[b][0].x, a[b][0].y, a[b][0].z, a[b][0].w};
        const uint32_t A1[4] = {a[b][1].x, a[b][1].y, a[b][1].z, a[b][1].w};
        mma_bf16(acc[t], A0, bv[b].x, bv[b].y);
        // four or more tiles give the tensor pipe independent MMAs already:
        // one accumulator set, half the registers
        if constexpr (NT >= 4)
          mma_bf16(acc[t], A1, bv[b].z, bv[b].w);
        else
          mma_bf16(acc2[t], A1, bv[b].z, bv[b].w);
      }
    }
  }
}

// MXFP4 weights x f16-MX activation records: EGU, EDN.  Every shared-memory
// load of the stage is issued first and unconditionally; token columns past
// ntok read token 0's record (finite duplicates that nothing downstream
// reads), so the inner loop carries no per-element selects.  The loop is bound
// by the integer pipe (two warp instructions per clock per SM): per 32-wide
// block a lane spends 8 e2m1 conversions and 2 scale extractions there, the
// scale shifts go to the multiply-add pipe as integer multiplies.
//
// e8m0 scale byte s -> fp32 2^(s-127) by placing s in the exponent field.
// s = 0 (2^-127, below fp32's normal range) becomes 0.0: every weight of such
// a block has magnitude at most 6 * 2^-127.  0xFF (NaN) is rejected at load.
// (j is a constant after unrolling, so the branch folds away)
__device__ __forceinline__ float e8m0_byte_to_float(uint32_t word, int j) {
  const uint32_t t = (j == 3) ? __umulhi(word, 0x80000000u) : word * (1u << (23 - 8 * j));
  return __uint_as_float(t & 0x7F800000u);
}

// Several token tiles (a virtual expert of up to 8*NT tokens): the 32-wide
// blocks are decoded four at a time (codes and scales into registers) and
// each decoded half serves every tile that holds tokens of this piece; tiles
// past ceil(ntok/8) are skipped (the test is uniform over the CTA), so an
// expert chosen by 2 tokens costs one tile.  A tile's shared-memory loads are
// issued together before its MMAs, as in the one-tile loop below.  (Halves,
// not all eight blocks at once: 288 threads leave 168 registers a thread.)
template <int NT>
__device__ __forceinline__ void mma_mx_tiles(const Params& p, const Hdr& h, const uint8_t* tile,
                                             const uint8_t* act, float (&acc)[NT][4], int warp,
                                             int lane) {
  const int g = lane >> 2, tig = lane & 3;
  const int nact = (h.ntok + 7) >> 3;
  const uint4 sc = lds128(tile + kMxCodeBytes + (warp * 8 + g) * 16);
  const uint32_t scw[4] = {sc.x, sc.y, sc.z, sc.w};
  const bool full = h.nb == 8;
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    if (!full && 4 * hf >= h.nb) break;
    uint32_t A[4][2][4];
    float sw[4][2];
    const uint4 c0 = lds128(tile + (warp * 4 + 2 * hf) * 512 + lane * 16);
    const uint4 c1 = lds128(tile + (warp * 4 + 2 * hf + 1) * 512 + lane * 16);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 w4 = (i >> 1) ? c1 : c0;
      e2m1x8_to_f16x2x4((i & 1) ? w4.z : w4.x, A[i][0]);
      e2m1x8_to_f16x2x4((i & 1) ? w4.w : w4.y, A[i][1]);
      sw[i][0] = e8m0_byte_to_float(scw[hf], i);
      sw[i][1] = e8m0_byte_to_float(scw[2 + hf], i);
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      if (t >= nact) break;
      const int tok = 8 * t + g;
      const int cc = 8 * t + 2 * tig;
      const uint8_t* arow = act + (tok < h.ntok ? tok : 0) * p.act_stride + tig * 16 + hf * 256;
      const float* s0 = reinterpret_cast<const float*>(act + (cc < h.ntok ? cc : 0) * p.act_stride + 512) + 4 * hf;
      const float* s1 =
          reinterpret_cast<const float*>(act + (cc + 1 < h.ntok ? cc + 1 : 0) * p.act_stride + 512) + 4 * hf;
      uint4 bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) bv[i] = lds128(arow + i * 64);
      const float4 s0v = *reinterpret_cast<const float4*>(s0);
      const float4 s1v = *reinterpret_cast<const float4*>(s1);
      const float sa0[4] = {s0v.x, s0v.y, s0v.z, s0v.w};
      const float sa1[4] = {s1v.x, s1v.y, s1v.z, s1v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (full || 4 * hf + i < h.nb) {
          float tmp[4];
          mma_f16_zc(tmp, A[i][0], bv[i].x, bv[i].y);
          mma_f16(tmp, A[i][1], bv[i].z, bv[i].w);
          acc[t][0] = fmaf(sw[i][0] * sa0[i], tmp[0], acc[t][0]);
          acc[t][1] = fmaf(sw[i][0] * sa1[i], tmp[1], acc[t][1]);
          acc[t][2] = fmaf(sw[i][1] * sa0[i], tmp[2], acc[t][2]);
          acc[t][3] = fmaf(sw[i][1] * sa1[i], tmp[3], acc[t][3]);
        }
      }
    }
  }
}

template <int NT>
__device__ __forceinline__ void mma_mx(const Params& p, const Hdr& h, const uint8_t* tile,
                                       const uint8_t* act, float (&acc)[NT][4], int warp, int lane) {
  if constexpr (NT > 1) {
    mma_mx_tiles<NT>(p, h, tile, act, acc, warp, lane);
    return;
  }
  const int g = lane >> 2, tig = lane & 3;
  const uint4 sc = lds128(tile + kMxCodeBytes + (warp * 8 + g) * 16);
  const uint32_t scw[4] = {sc.x, sc.y, sc.z, sc.w};
  uint4 cw[4];
#pragma unroll
  for (int bp = 0; bp < 4; ++bp) cw[bp] = lds128(tile + (warp * 4 + bp) * 512 + lane * 16);
  const bool full = h.nb == 8;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int tok = 8 * t + g;
    const int c0 = 8 * t + 2 * tig;
    const uint8_t* arow = act + (tok < h.ntok ? tok : 0) * p.act_stride + tig * 16;
    const float* s0 = reinterpret_cast<const float*>(act + (c0 < h.ntok ? c0 : 0) * p.act_stride + 512);
    const float* s1 = reinterpret_cast<const float*>(act + (c0 + 1 < h.ntok ? c0 + 1 : 0) * p.act_stride + 512);
    uint4 bv[8];
#pragma unroll
    for (int b = 0; b < 8; ++b) bv[b] = lds128(arow + b * 64);
    const float4 s0a = *reinterpret_cast<const float4*>(s0);
    const float4 s0b = *reinterpret_cast<const float4*>(s0 + 4);
    const float4 s1a = *reinterpret_cast<const float4*>(s1);
    const float4 s1b = *reinterpret_cast<const float4*>(s1 + 4);
    const float sa0[8] = {s0a.x, s0a.y, s0a.z, s0a.w, s0b.x, s0b.y, s0b.z, s0b.w};
    const float sa1[8] = {s1a.x, s1a.y, s1a.z, s1a.w, s1b.x, s1b.y, s1b.z, s1b.w};
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      if (full || b < h.nb) {
        uint32_t A0[4], A1[4];
        const uint4 w4 = cw[b >> 1];
        e2m1x8_to_f16x2x4((b & 1) ? w4.z : w4.x, A0);
        e2m1x8_to_f16x2x4((b & 1) ? w4.w : w4.y, A1);
        const float sw0 = e8m0_byte_to_float(scw[b >> 2], b & 3);
        const float sw1 = e8m0_byte_to_float(scw[2 + (b >> 2)], b & 3);
        float tmp[4];
        mma_f16_zc(tmp, A0, bv[b].x, bv[b].y);
        mma_f16(tmp, A1, bv[b].z, bv[b].w);
        acc[t][0] = fmaf(sw0 * sa0[b], tmp[0], acc[t][0]);
        acc[t][1] = fmaf(sw0 * sa1[b], tmp[1], acc[t][1]);
        acc[t][2] = fmaf(sw1 * sa0[b], tmp[2], acc[t][2]);
        acc[t][3] = fmaf(sw1 * sa1[b], tmp[3], acc[t][3]);
      }
    }
  }
}

// TAIL, few tokens: form every token's whole activation once per CTA.  Token
// b's record holds bf16 hi values for k in [0, res_k), then the lo parts.
// k < C_lat*64 is the combine c = sum_j w_j y_j (zero past L); the rest is h_s.
// Only the groups of eight k in [kbeg, kend) are formed (multiples of 8): the
// h_s part can be built before the routed experts finish, the combine after.
// The record holds k in [res_k0, res_k0 + res_k) (one lane's part, or all).
__device__ __forceinline__ void build_resident(const Params& p, uint8_t* res, int tid, int kbeg,
                                               int kend) {
  const int K = p.topk, KR = p.res_k, klat = p.C_lat * 64;
  const int n8 = (kend - kbeg) / 8;
  const int groups = p.B * n8;
  for (int gi = tid; gi < groups; gi += kConsumerThreads) {
    const int b = gi / n8, k0 = kbeg + (gi % n8) * 8;
    float v[8];
    if (k0 < klat) {
      // K <= 16: compile-time slots keep everything in registers, loads first
      float4 ya[16], yb[16];
      float wj[16];
      const float* ybase = p.y + ((long long)(k0 >> 6) * p.ld_slots + (long long)b * K) * 64 + (k0 & 63);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (j < K) {
          wj[j] = __ldcg(p.wts + b * K + j);
          ya[j] = __ldcg(reinterpret_cast<const float4*>(ybase + j * 64));
          yb[j] = __ldcg(reinterpret_cast<const float4*>(ybase + j * 64 + 4));
        } else {
          wj[j] = 0.f;
          ya[j] = yb[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        v[0] = fmaf(wj[j], ya[j].x, v[0]);
        v[1] = fmaf(wj[j], ya[j].y, v[1]);
        v[2] = fmaf(wj[j], ya[j].z, v[2]);
        v[3] = fmaf(wj[j], ya[j].w, v[3]);
        v[4] = fmaf(wj[j], yb[j].x, v[4]);
        v[5] = fmaf(wj[j], yb[j].y, v[5]);
        v[6] = fmaf(wj[j], yb[j].z, v[6]);
        v[7] = fmaf(wj[j], yb[j].w, v[7]);
      }
      if (k0 >= p.L) {
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = 0.f;
      }
    } else {
      const int ks = k0 - klat;
      if (ks < p.KS) {
        const float* hb = p.h_s + ((long long)(ks >> 6) * p.B + b) * 64 + (ks & 63);
        const float4 a = __ldcg(reinterpret_cast<const float4*>(hb));
        const float4 c = __ldcg(reinterpret_cast<const float4*>(hb + 4));
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = c.x; v[5] = c.y; v[6] = c.z; v[7] = c.w;
      } else {
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = 0.f;
      }
    }
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      hi[u] = pack_bf16x2(v[2 * u], v[2 * u + 1]);
      lo[u] = pack_bf16x2(v[2 * u] - bf16_lo_to_float(hi[u]), v[2 * u + 1] - bf16_hi_to_float(hi[u]));
    }
    uint8_t* rec = res + (size_t)b * p.res_stride;
    const int kr = k0 - p.res_k0;
    *reinterpret_cast<uint4*>(rec + kr * 2) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(rec + KR * 2 + kr * 2) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

template <int NT>
__device__ __forceinline__ void mma_tail_resident(const Params& p, const Hdr& h, const uint8_t* tile,
                                                  const uint8_t* res, float (&acc)[NT][4],
                                                  float (&acc2)[NT][4], int warp, int lane) {
  const int g = lane >> 2, tig = lane & 3;
  const int kbase = h.chunk * kDenseChunkK - p.res_k0;
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    if (b < h.nb) {
      const uint4 a0 = lds128(tile + ((warp * 2 + b) * 2 + 0) * 512 + lane * 16);
      const uint4 a1 = lds128(tile + ((warp * 2 + b) * 2 + 1) * 512 + lane * 16);
      const uint32_t A0[4] = {a0.x, a0.y, a0.z, a0.w};
      const uint32_t A1[4] = {a1.x, a1.y, a1.z, a1.w};
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const int tok = 8 * t + g;
        const bool tv = tok < h.ntok;
        const uint8_t* rec = res + (size_t)(h.tok0 + (tv ? tok : 0)) * p.res_stride +
                             (kbase + 32 * b + 8 * tig) * 2;
        const uint4 bh = lds128(rec), bl = lds128(rec + p.res_k * 2);
        mma_bf16(acc[t], A0, bh.x, bh.y);
        mma_bf16(acc2[t], A1, bh.z, bh.w);
        mma_bf16(acc[t], A0, bl.x, bl.y);
        mma_bf16(acc2[t], A1, bl.z, bl.w);
      }
    }
  }
}

// TAIL with formed records: token b's row in the stage is 64 bf16 hi values
// then 64 bf16 lo values (256 bytes); two MMAs per k16 step.
template <int NT>
__device__ __forceinline__ void mma_tail_formed(const Hdr& h, const uint8_t* tile, const uint8_t* act,
                                                float (&acc)[NT][4], float (&acc2)[NT][4], int warp,
                                                int lane) {
  const int g = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    if (b < h.nb) {
      const uint4 a0 = lds128(tile + ((warp * 2 + b) * 2 + 0) * 512 + lane * 16);
      const uint4 a1 = lds128(tile + ((warp * 2 + b) * 2 + 1) * 512 + lane * 16);
      const uint32_t A0[4] = {a0.x, a0.y, a0.z, a0.w};
      const uint32_t A1[4] = {a1.x, a1.y, a1.z, a1.w};
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        if (8 * t >= h.ntok) break;  // (uniform over the CTA)
        const int tok = 8 * t + g < h.ntok ? 8 * t + g : 0;
        const uint8_t* rec = act + tok * 256 + (32 * b + 8 * tig) * 2;
        const uint4 bh = lds128(rec), bl = lds128(rec + 128);
        mma_bf16(acc[t], A0, bh.x, bh.y);
        mma_bf16(acc2[t], A1, bh.z, bh.w);
        mma_bf16(acc[t], A0, bl.x, bl.y);
        mma_bf16(acc2[t], A1, bl.z, bl.w);
      }
    }
  }
}

// TAIL, staged activations: form the records (see Params::t_rec) for every
// (chunk, token) -- this CTA's share of the grid-wide work, 8 values an item.
__device__ __forceinline__ void form_tail_records(const Params& p, int tid) {
  const int K = p.topk, klat = p.C_lat * 64;
  const long long items = (long long)p.C * p.B * 8;
  for (long long it = (long long)blockIdx.x * kConsumerThreads + tid; it < items;
       it += (long long)gridDim.x * kConsumerThreads) {
    const int c = (int)(it / (p.B * 8)), rem = (int)(it % (p.B * 8));
    const int b = rem >> 3, q = rem & 7;
    const int k0 = c * 64 + q * 8;  // K index of the chunk space ([L chunks ; I_s chunks])
    float v[8];
    if (c < p.C_lat) {
      float4 ya[16], yb[16];
      float wj[16];
      const float* ybase = p.y + ((long long)c * p.ld_slots + (long long)b * K) * 64 + q * 8;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (j < K) {
          wj[j] = __ldcg(p.wts + b * K + j);
          ya[j] = __ldcg(reinterpret_cast<const float4*>(ybase + j * 64));
          yb[j] = __ldcg(reinterpret_cast<const float4*>(ybase + j * 64 + 4));
        } else {
          wj[j] = 0.f;
          ya[j] = yb[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        v[0] = fmaf(wj[j], ya[j].x, v[0]);
        v[1] = fmaf(wj[j], ya[j].y, v[1]);
        v[2] = fmaf(wj[j], ya[j].z, v[2]);
        v[3] = fmaf(wj[j], ya[j].w, v[3]);
        v[4] = fmaf(wj[j], yb[j].x, v[4]);
        v[5] = fmaf(wj[j], yb[j].y, v[5]);
        v[6] = fmaf(wj[j], yb[j].z, v[6]);
        v[7] = fmaf(wj[j], yb[j].w, v[7]);
      }
      if (k0 >= p.L) {
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = 0.f;
      }
    } else {
      const int ks = k0 - klat;
      if (ks < p.KS) {
        const float* hb = p.h_s + ((long long)(ks >> 6) * p.B + b) * 64 + (ks & 63);
        const float4 a = __ldcg(reinterpret_cast<const float4*>(hb));
        const float4 d = __ldcg(reinterpret_cast<const float4*>(hb + 4));
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = d.x; v[5] = d.y; v[6] = d.z; v[7] = d.w;
      } else {
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = 0.f;
      }
    }
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      hi[u] = pack_bf16x2(v[2 * u], v[2 * u + 1]);
      lo[u] = pack_bf16x2(v[2 * u] - bf16_lo_to_float(hi[u]), v[2 * u + 1] - bf16_hi_to_float(hi[u]));
    }
    uint8_t* rec = p.t_rec + ((long long)c * p.B + b) * 256 + q * 16;
    *reinterpret_cast<uint4*>(rec) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(rec + 128) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

// TAIL: build the activation tile (combine of y, or h_s) as bf16 hi + lo in a
// transform buffer, then bf16 MMAs against W_out / W_sd.
template <int NT>
__device__ __forceinline__ void mma_tail(const Params& p, const Hdr& h, const uint8_t* tile,
                                         const uint8_t* act, uint8_t* tbuf, float (&acc)[NT][4],
                                         float (&acc2)[NT][4], int warp, int lane, int tid) {
  constexpr int kTStride = 320;  // bytes per token row: 64 bf16 hi, 64 bf16 lo, padding
  const int K = p.topk;
  const bool lat = h.chunk < p.C_lat;
  for (int idx = tid; idx < h.ntok * 16; idx += kConsumerThreads) {
    const int tk = idx >> 4, q = idx & 15;
    float4 v;
    if (lat) {
      const float* yrow = reinterpret_cast<const float*>(act) + (tk * K) * 64 + q * 4;
      const float* wrow = p.wts + (long long)(h.tok0 + tk) * K;
      v = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int j = 0; j < K; ++j) {
        const float wj = wrow[j];
        const float4 yv = *reinterpret_cast<const float4*>(yrow + j * 64);
        v.x = fmaf(wj, yv.x, v.x);
        v.y = fmaf(wj, yv.y, v.y);
        v.z = fmaf(wj, yv.z, v.z);
        v.w = fmaf(wj, yv.w, v.w);
      }
    } else {
      v = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(act) + tk * 64 + q * 4);
    }
    const uint32_t h01 = pack_bf16x2(v.x, v.y), h23 = pack_bf16x2(v.z, v.w);
    const uint32_t l01 = pack_bf16x2(v.x - bf16_lo_to_float(h01), v.y - bf16_hi_to_float(h01));
    const uint32_t l23 = pack_bf16x2(v.z - bf16_lo_to_float(h23), v.w - bf16_hi_to_float(h23));
    *reinterpret_cast<uint2*>(tbuf + tk * kTStride + q * 8) = make_uint2(h01, h23);
    *reinterpret_cast<uint2*>(tbuf + tk * kTStride + 128 + q * 8) = make_uint2(l01, l23);
  }
  named_sync(1, kConsumerThreads);
  const int g = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    if (b < h.nb) {
      const uint4 a0 = lds128(tile + ((warp * 2 + b) * 2 + 0) * 512 + lane * 16);
      const uint4 a1 = lds128(tile + ((warp * 2 + b) * 2 + 1) * 512 + lane * 16);
      const uint32_t A0[4] = {a0.x, a0.y, a0.z, a0.w};
      const uint32_t A1[4] = {a1.x, a1.y, a1.z, a1.w};
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const int tok = 8 * t + g < h.ntok ? 8 * t + g : 0;
        const uint4 bh = lds128(tbuf + tok * kTStride + (32 * b + 8 * tig) * 2);
        const uint4 bl = lds128(tbuf + tok * kTStride + 128 + (32 * b + 8 * tig) * 2);
        mma_bf16(acc[t], A0, bh.x, bh.y);
        mma_bf16(acc2[t], A1, bh.z, bh.w);
        mma_bf16(acc[t], A0, bl.x, bl.y);
        mma_bf16(acc2[t], A1, bl.z, bl.w);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// epilogues

// f16 "MX" store: values of a 32-wide block of the activation index share one
// power-of-two scale per token, chosen so the block's largest magnitude lands
// in [2^14, 2^15).  `wpb` warps own one 32-wide block.  Each thread provides
// up to two rows (r0 = g, r1 = g + 8) per token column.
__device__ __forceinline__ void mx_scale_of(float amax, float& s, float& inv) {
  if (!(amax > 0.f)) {
    s = 1.f;
    inv = 1.f;
    if (amax != amax) s = amax;  // NaN propagates through the scale
    return;
  }
  int ex = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;
  int se = ex - 14;
  se = se < -100 ? -100 : (se > 127 ? 127 : se);
  s = __uint_as_float((uint32_t)(se + 127) << 23);
  inv = __uint_as_float((uint32_t)(127 - se) << 23);
}

template <int NT, int ROWS>
__device__ __forceinline__ void store_f16mx(const float (&val)[NT][2][2], int warp, int lane,
                                            int wpb, int ntok, float* amax_s,
                                            uint8_t* const (&rec)[NT][2], const int (&idx)[2],
                                            bool row_valid0, bool row_valid1) {
  // val[t][c][r]: token column 8t + 2tig + c, row r (r < ROWS)
  const int g = lane >> 2, tig = lane & 3;
  float m[NT][2];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      float a = row_valid0 ? fabsf(val[t][c][0]) : 0.f;
      if (ROWS > 1 && row_valid1) a = fmaxf(a, fabsf(val[t][c][1]));
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 8));
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 16));
      m[t][c] = a;
    }
  if (g == 0) {
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int c = 0; c < 2; ++c) amax_s[warp * (NT * 8) + 8 * t + 2 * tig + c] = m[t][c];
  }
  named_sync(1, kConsumerThreads);
  const int w0 = (warp / wpb) * wpb;
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int col = 8 * t + 2 * tig + c;
      if (col >= ntok) continue;
      float a = 0.f;
      for (int ww = w0; ww < w0 + wpb; ++ww) a = fmaxf(a, amax_s[ww * (NT * 8) + col]);
      float s, inv;
      mx_scale_of(a, s, inv);
      uint8_t* r = rec[t][c];
#pragma unroll
      for (int rr = 0; rr < ROWS; ++rr) {
        const bool ok = rr == 0 ? row_valid0 : row_valid1;
        if (!ok) continue;
        const int i = idx[rr] & (kMxChunkK - 1);
        *reinterpret_cast<uint16_t*>(r + i * 2) =
            (uint16_t)(pack_f16x2(val[t][c][rr] * inv, 0.f) & 0xFFFF);
      }
      if (g == 0 && warp == w0 && row_valid0) {
        const int i = idx[0] & (kMxChunkK - 1);
        *reinterpret_cast<float*>(r + 512 + 4 * (i >> 5)) = s;
      }
    }
  named_sync(1, kConsumerThreads);
}

// The tensor-core record (layout.cuh): per 32-block of a token, kUTerms e2m1
// terms.  The block maximum a sets term 1's exponent e1, the least with
// a <= 4 * 2^e1; term t + 1 takes 2^(e1 - 3 t).  Every element's term code is
// its remaining value over the term's scale rounded to e2m1, and that code's
// value comes off the remainder (which stays within 4 times the next scale).
//
// The tile's values go through shared memory, two token tiles at a time
// ([token][row], row stride padded to 4 mod 32 floats: conflict-free on both
// sides); then four adjacent threads take one (token, 32-row block), eight
// rows each, and store each term's eight codes as one word.
__device__ __forceinline__ float pow2f(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }

// SWIGLU: the tile has 64 rows, row 8 warp + g of token column col holding
// silu(acc[t][c]) * acc[t][2 + c] (the expert gate/up kernel); otherwise 128
// rows, rows 16 warp + g and + 8 holding acc[t][c] and acc[t][2 + c].  Token
// column col's record is rec0 + col * col_stride; the tile's row r sits at
// position pos0 + r of the record (pos0 a multiple of 32), and rows from
// nrows on lie beyond K (not stored).
template <int NT, bool SWIGLU>
__device__ __forceinline__ void store_e2m1_terms(const float (&acc)[NT][4], int warp, int lane, int tid,
                                                 int ntok, float* sv, uint8_t* rec0,
                                                 long long col_stride, int pos0, int nrows) {
  constexpr int kRows = SWIGLU ? 64 : 128;
  constexpr int kLd = kRows + 4;
  constexpr int kChunk = NT < 2 ? NT : 2;  // token tiles staged at a time
  constexpr int kBlocks = kRows / 32;
  const int g = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int t0 = 0; t0 < NT; t0 += kChunk) {
    // this chunk's values into shared memory
#pragma unroll
    for (int tt = 0; tt < kChunk; ++tt)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int tok = 8 * tt + 2 * tig + c;
        const int t = t0 + tt;
        if (SWIGLU) {
          sv[tok * kLd + 8 * warp + g] = silu(acc[t][c]) * acc[t][2 + c];
        } else {
          sv[tok * kLd + 16 * warp + g] = acc[t][c];
          sv[tok * kLd + 16 * warp + g + 8] = acc[t][2 + c];
        }
      }
    named_sync(1, kConsumerThreads);
    // four threads a (token, block): quarter q holds rows 8 q .. 8 q + 7
    const int q = tid & 3, grp = tid >> 2;
    const int blk = grp % kBlocks, tokl = grp / kBlocks;
    const bool active = tokl < 8 * kChunk;
    const int tok = 8 * t0 + (active ? tokl : 0);
    const int r0 = 32 * blk + 8 * q;
    float v[8];
    float a = 0.f;
    {
      const float4* src = reinterpret_cast<const float4*>(sv + (active ? tokl : 0) * kLd + r0);
      const float4 x0 = src[0], x1 = src[1];
      v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w;
      v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (r0 + i >= nrows) v[i] = 0.f;
        a = fmaxf(a, fabsf(v[i]));
      }
    }
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
    // e1: the least e with a <= 4 * 2^e (kept where every term's scale and
    // its inverse are normal floats); a NaN or infinite maximum makes every
    // scale NaN
    const bool nan = (__float_as_uint(a) & 0x7F800000u) == 0x7F800000u;
    int e1 = -118;
    if (a > 0.f && !nan) {
      const uint32_t bits = __float_as_uint(a * 0.25f);
      e1 = (int)((bits >> 23) & 0xFF) - 127 + ((bits & 0x7FFFFFu) ? 1 : 0);
      e1 = e1 < -118 ? -118 : (e1 > 126 ? 126 : e1);
    }
    const bool store = active && tok < ntok && 32 * blk < nrows;
    uint8_t* r = rec0 + (long long)tok * col_stride;
    const int pos = pos0 + r0;
#pragma unroll
    for (int term = 0; term < kUTerms; ++term) {
      const int e = e1 - 3 * term;
      const float inv = pow2f(-e), sc = pow2f(e);
      uint32_t w = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t code = f32_to_e2m1(v[i] * inv);
        v[i] -= e2m1_to_f32(code) * sc;
        w |= code << (4 * i);
      }
      if (store) *reinterpret_cast<uint32_t*>(r + term * kUTermBytes + (pos >> 1)) = w;
    }
    if (store && q == 0) {
#pragma unroll
      for (int term = 0; term < kUTerms; ++term)
        r[kUTerms * kUTermBytes + term * 8 + (pos >> 5)] = nan ? (uint8_t)0xFF : (uint8_t)(e1 - 3 * term + 127);
    }
    named_sync(1, kConsumerThreads);  // (the staging is reused)
  }
}

__device__ __forceinline__ bool route_tokens(const Params& p, const float* bias, uint8_t* scratch,
                                          float* lg_s, int lg_cap, int* wtot, int tid, int warp,
                                          int lane, const float* lg_sm = nullptr, int b_lo = 0,
                                          int b_hi = -1);

template <int KIND, int NT>
__device__ __forceinline__ void epilogue(const Params& p, const Hdr& h, float (&acc)[NT][4], uint8_t* scratch,
                         int* sm_flag, const int* slot_tab, int tid, int warp, int lane) {
  const int g = lane >> 2, tig = lane & 3;
  if (KIND == KIND_FRONT && h.rb < p.RB_router) {
    // router rows: publish the logits; the routing CTA waits for all of them
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int row = 16 * warp + ((q & 2) ? g + 8 : g);
        const int col = 8 * t + 2 * tig + (q & 1);
        const int e = h.rb * kRowsPerBlock + row;
        if (e < p.E && col < p.B) p.logits[(long long)col * p.E + e] = acc[t][q];
      }
    // every thread's logits precede thread 0's release (barrier cumulativity)
    named_sync(1, kConsumerThreads);
    if (p.trace && tid == 0) p.trace[(size_t)blockIdx.x * kTraceStride + 19] = global_ns();
    if (tid == 0) atom_add_acqrel(p.router_done, 1);
  } else if (KIND == KIND_FRONT && h.rb < p.RB_router + p.RB_lat) {
    // latent rows -> z records
    const int cz = (p.L + kMxChunkK - 1) / kMxChunkK;
    const int l0 = (h.rb - p.RB_router) * kRowsPerBlock + 16 * warp + g;
    if (p.umma) {
      const int lb = (h.rb - p.RB_router) * kRowsPerBlock;  // the tile's first latent row
      store_e2m1_terms<NT, false>(acc, warp, lane, tid, p.B, reinterpret_cast<float*>(scratch),
                                  p.z_mx + (long long)(lb >> 8) * p.act_rec, (long long)cz * p.act_rec,
                                  lb & (kMxChunkK - 1), p.L - lb);  // ends with a barrier
    } else {
      const int idx[2] = {l0, l0 + 8};
      float val[NT][2][2];
      uint8_t* rec[NT][2];
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          val[t][c][0] = acc[t][c];
          val[t][c][1] = acc[t][2 + c];
          const int col = 8 * t + 2 * tig + c;
          rec[t][c] = p.z_mx + ((long long)(col < p.B ? col : 0) * cz + (l0 >> 8)) * p.act_rec;
        }
      store_f16mx<NT, 2>(val, warp, lane, 2, p.B, reinterpret_cast<float*>(scratch), rec, idx,
                         l0 < p.L, l0 + 8 < p.L);  // ends with a barrier
    }
    if (p.done && tid == 0) red_release_add(p.done + 0, 1);
    // every thread's records precede the release (barrier cumulativity)
    if (p.z_done && tid == 0) red_release_add(p.z_done, 1);
  } else if (KIND == KIND_FRONT) {
    // shared expert gate/up rows (64 gate + 64 up per block) -> h_s
    const int i = 64 * (h.rb - p.RB_router - p.RB_lat) + 8 * warp + g;
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int col = 8 * t + 2 * tig + c;
        if (col < p.B && i < p.Is)
          p.h_s[((long long)(i >> 6) * p.B + col) * 64 + (i & 63)] = silu(acc[t][c]) * acc[t][2 + c];
      }
    if (p.done) {
      named_sync(1, kConsumerThreads);  // every thread's h_s precede the release
      if (tid == 0) red_release_add(p.done + 1, 1);
    }
  } else if (KIND == KIND_EGU) {
    const int i = 64 * h.rb + 8 * warp + g;
    if (p.umma) {
      const int ib = 64 * h.rb;  // the tile's first h row
      store_e2m1_terms<NT, true>(acc, warp, lane, tid, h.ntok, reinterpret_cast<float*>(scratch),
                                 p.h_mx + ((long long)(ib >> 8) * p.ld_slots + h.tok0) * p.act_rec,
                                 (long long)p.act_rec, ib & (kMxChunkK - 1), p.I - ib);  // ends with a barrier
    } else {
      const int idx[2] = {i, i};
      float val[NT][2][2];
      uint8_t* rec[NT][2];
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          val[t][c][0] = silu(acc[t][c]) * acc[t][2 + c];
          val[t][c][1] = 0.f;
          const int col = 8 * t + 2 * tig + c;
          const int pos = h.tok0 + (col < h.ntok ? col : 0);
          rec[t][c] = p.h_mx + ((long long)(i >> 8) * p.ld_slots + pos) * p.act_rec;
        }
      store_f16mx<NT, 1>(val, warp, lane, 4, h.ntok, reinterpret_cast<float*>(scratch), rec, idx,
                         i < p.I, false);  // ends with a barrier
    }
    if (p.done && tid == 0) red_release_add(p.done + 2, 1);
    // every thread's records precede the release (barrier cumulativity)
    if (p.h_done && tid == 0) red_release_add(p.h_done + h.v, 1);
  } else if (KIND == KIND_EDN) {
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int l = h.rb * kRowsPerBlock + 16 * warp + ((q & 2) ? g + 8 : g);
        const int col = 8 * t + 2 * tig + (q & 1);
        if (col < h.ntok && l < p.L) {
          const int slot = slot_tab[h.tok0 + col];
          p.y[((long long)(l >> 6) * p.ld_slots + slot) * 64 + (l & 63)] = acc[t][q];
        }
      }
    if (p.done) {
      named_sync(1, kConsumerThreads);  // every thread's y precede the release
      if (tid == 0) red_release_add(p.done + 3, 1);
    }
  } else {  // TAIL
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int n = h.rb * kRowsPerBlock + 16 * warp + ((q & 2) ? g + 8 : g);
        const int col = 8 * t + 2 * tig + (q & 1);
        if (col < h.ntok && n < p.H)
          p.out[(long long)(h.tok0 + col) * p.H + n] =
              (uint16_t)(pack_bf16x2(acc[t][q], 0.f) & 0xFFFF);
      }
  }
}

// ---------------------------------------------------------------------------
// top-k routing and per-expert token lists (one CTA, 256 threads); the
// per-token selection is warp_topk (topk.cuh).

// Copy n floats that other CTAs wrote (read past L1) into shared memory, with
// eight 16-byte loads (or sixteen 4-byte ones) in flight per thread.
__device__ __forceinline__ void stage_floats(const float* src, int n, float* dst, int tid) {
  if ((reinterpret_cast<uintptr_t>(src) & 15) == 0 && (n & 3) == 0) {
    const float4* s4 = reinterpret_cast<const float4*>(src);
    float4* d4 = reinterpret_cast<float4*>(dst);
    const int n4 = n >> 2;
    for (int i0 = tid; i0 < n4; i0 += kConsumerThreads * 8) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * kConsumerThreads;
        v[u] = i < n4 ? __ldcg(s4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * kConsumerThreads;
        if (i < n4) d4[i] = v[u];
      }
    }
  } else {
    for (int i0 = tid; i0 < n; i0 += kConsumerThreads * 16) {
      float v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int i = i0 + u * kConsumerThreads;
        v[u] = i < n ? __ldcg(src + i) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int i = i0 + u * kConsumerThreads;
        if (i < n) dst[i] = v[u];
      }
    }
  }
}

// lg_s: shared memory for lg_cap floats of logits (at least E).
// lg_sm: the logits [B][E] already in shared memory (few tokens, summed by
// the routing CTA itself), else they are read from p.logits.
// [b_lo, b_hi): the tokens this CTA selects for (b_hi < 0: all).  With
// several routing CTAs (p.route_cta > 1) each selects its share; the last to
// finish (a ticket) gathers every token's choice and builds the tables, and
// only it returns true (the caller then publishes them).
__device__ __forceinline__ bool route_tokens(const Params& p, const float* bias, uint8_t* scratch,
                                          float* lg_s, int lg_cap, int* wtot, int tid, int warp,
                                          int lane, const float* lg_sm, int b_lo, int b_hi) {
  const int E = p.E, K = p.topk, B = p.B;
  if (b_hi < 0) b_hi = B;
  const int tg = p.tg > 0 ? p.tg : 1;
  int* cnt = reinterpret_cast<int*>(scratch);  // [E] slots per expert
  int* fill = cnt + E;                          // [E] placement cursor
  int* off = fill + E;                          // [E] first sorted position
  int* ids_s = off + E;                         // [B*K]
  unsigned long long* tr = (p.trace && tid == 0) ? p.trace + (size_t)blockIdx.x * kTraceStride : nullptr;
  for (int i = tid; i < E; i += kConsumerThreads) {
    cnt[i] = 0;
    fill[i] = 0;
  }
  named_sync(1, kConsumerThreads);
  if (tr) tr[16] = global_ns();
  // Few tokens: P warps share a token (each selects within a slice of the
  // experts, one warp merges); 8 or more tokens: one warp per token, the
  // logits of as many tokens as lg_s holds first copied there together (one
  // round trip for all of them instead of one per token and warp).
  const int P = B >= kConsumerWarps ? 1 : kConsumerWarps / B;  // B * P <= 8 warps
  if (P == 1) {
    const bool staged = lg_cap >= E;  // (the ring always holds a token's logits)
    const int chunk = staged ? min(b_hi - b_lo, lg_cap / E) : b_hi - b_lo;
    for (int b0 = b_lo; b0 < b_hi; b0 += chunk) {
      const int nb = min(chunk, b_hi - b0);
      if (staged) {
        stage_floats(p.logits + (long long)b0 * E, nb * E, lg_s, tid);
        named_sync(1, kConsumerThreads);
      }
      if (tr && b0 == b_lo) tr[21] = global_ns();
      for (int bl = warp; bl < nb; bl += kConsumerWarps) {
        const int b = b0 + bl;
        int sel_id;
        float sel_w;
        if (staged)
          warp_topk<true>(lg_s + bl * E, E, K, p.score_fn, bias, p.renorm, p.routed_scale, lane,
                          sel_id, sel_w);
        else
          warp_topk<false>(p.logits + (long long)b * E, E, K, p.score_fn, bias, p.renorm,
                           p.routed_scale, lane, sel_id, sel_w);
        if (lane < K) {
          p.ids[b * K + lane] = sel_id;
          p.wts[b * K + lane] = sel_w;
          ids_s[b * K + lane] = sel_id;
          atomicAdd(&cnt[sel_id], 1);
        }
        if (tr && b0 == b_lo && bl == 0) tr[22] = global_ns();
      }
      if (tr && b0 == b_lo) tr[20] = global_ns();
      named_sync(1, kConsumerThreads);  // every warp is done with lg_s
    }
  } else {
    // candidates after the token table: [B][P][K] TopkCand, then [B][P] partials
    TopkCand* cand = reinterpret_cast<TopkCand*>(
        reinterpret_cast<uint8_t*>(ids_s) + ((B * K * 4 + 15) & ~15));
    float2* part = reinterpret_cast<float2*>(cand + B * P * K);
    if (warp < B * P) {
      const int b = warp / P, q = warp % P;
      const int e0 = (int)((long long)q * E / P), e1 = (int)((long long)(q + 1) * E / P);
      TopkCand c;
      float smax, ssum;
      if (lg_sm)
        warp_topk_slice_any<true>(lg_sm + (long long)b * E, bias, e0, e1, K, p.score_fn, lane, c,
                                  smax, ssum);
      else
        warp_topk_slice_any(p.logits + (long long)b * E, bias, e0, e1, K, p.score_fn, lane, c,
                            smax, ssum);
      if (lane < K) cand[(b * P + q) * K + lane] = c;
      if (lane == 0) part[b * P + q] = make_float2(smax, ssum);
    }
    if (tr) tr[21] = global_ns();
    named_sync(1, kConsumerThreads);
    if (warp < B) {
      const int b = warp;
      int sel_id;
      float sel_w;
      warp_topk_merge(cand + b * P * K, part + b * P, P, K, E, p.score_fn, p.renorm,
                      p.routed_scale, lane, sel_id, sel_w);
      if (tr) tr[22] = global_ns();
      if (lane < K) {
        p.ids[b * K + lane] = sel_id;
        p.wts[b * K + lane] = sel_w;
        ids_s[b * K + lane] = sel_id;
        atomicAdd(&cnt[sel_id], 1);
      }
    }
  }
  named_sync(1, kConsumerThreads);
  if (tr) tr[17] = global_ns();
  if (p.route_cta > 1) {
    // every CTA's ids precede its ticket (barrier cumulativity); the last
    // one gathers all of them
    int* flag = wtot + 16;
    if (tid == 0) flag[0] = atom_add_acqrel(p.route_cnt, 1) == p.route_cta - 1;
    named_sync(1, kConsumerThreads);
    if (!flag[0]) return false;
    for (int i = tid; i < E; i += kConsumerThreads) cnt[i] = 0;
    named_sync(1, kConsumerThreads);
    for (int sl = tid; sl < B * K; sl += kConsumerThreads) {
      const int e = ld_cg(p.ids + sl);
      ids_s[sl] = e;
      atomicAdd(&cnt[e], 1);
    }
    if (tid == 0) {
      *p.route_cnt = 0;    // every routing CTA has taken its ticket
      *p.router_done = 0;  // ... so each has seen the router rows complete
    }
    named_sync(1, kConsumerThreads);
  }
  // block-wide exclusive scan of (slots, token groups) per expert; thread t
  // owns experts 4t .. 4t+3 (E <= 1024)
  int c[4], gsz[4], sc = 0, sg = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = 4 * tid + i;
    c[i] = e < E ? cnt[e] : 0;
    gsz[i] = (c[i] + tg - 1) / tg;
    sc += c[i];
    sg += gsz[i];
  }
  int ic = sc, ig = sg;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int uc = __shfl_up_sync(0xffffffffu, ic, o);
    const int ug = __shfl_up_sync(0xffffffffu, ig, o);
    if (lane >= o) {
      ic += uc;
      ig += ug;
    }
  }
  if (lane == 31) {
    wtot[warp] = ic;
    wtot[8 + warp] = ig;
  }
  named_sync(1, kConsumerThreads);
  int bc = ic - sc, bg = ig - sg;  // exclusive within the warp
  for (int w = 0; w < warp; ++w) {
    bc += wtot[w];
    bg += wtot[8 + w];
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = 4 * tid + i;
    if (e < E) {
      off[e] = bc;
      for (int gi = 0; gi < gsz[i]; ++gi) {
        VExpert ve;
        ve.expert = e;
        ve.start = bc + gi * tg;
        ve.count = min(tg, c[i] - gi * tg);
        ve.pad = 0;
        if (bg + gi < p.ve_max) {
          p.ve[bg + gi] = ve;
          if (p.h_done) p.h_done[bg + gi] = 0;
        }
      }
    }
    bc += c[i];
    bg += gsz[i];
  }
  if (tid == kConsumerThreads - 1) *p.nve = bg < p.ve_max ? bg : p.ve_max;
  // the chosen experts' weights into L2, gate/up before down, in the order
  // the expert kernels take them (virtual expert index), 64 KB a request
  if (p.pf_ves > 0) {
    for (int pass = 0; pass < 2; ++pass) {
      const uint8_t* base = pass == 0 ? p.pf_egu : p.pf_edn;
      const long long per = pass == 0 ? p.pf_egu_bytes : p.pf_edn_bytes;
      int v = bg - sg;  // this thread's first virtual expert index
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int e = 4 * tid + i;
        if (e < E && gsz[i] > 0 && v < p.pf_ves) {
          const uint8_t* src = base + (long long)e * per;
          for (long long o = 0; o < per; o += 65536)
            prefetch_l2(src + o, (uint32_t)min(65536LL, per - o));
        }
        v += gsz[i];
      }
    }
  }
  named_sync(1, kConsumerThreads);
  if (tr) tr[18] = global_ns();
  for (int s = tid; s < B * K; s += kConsumerThreads) {
    const int e = ids_s[s];
    const int pos = off[e] + atomicAdd(&fill[e], 1);
    p.slots_sorted[pos] = s;
  }
  named_sync(1, kConsumerThreads);
  return true;
}

// ---------------------------------------------------------------------------
// the front kernel's routing CTA

// The front grid's last CTA takes no pieces.  Its consumer warps wait until
// every router row block has been summed, select the experts, build the
// per-expert token lists and publish them; the other CTAs keep streaming the
// latent and shared-expert rows meanwhile.
// Few tokens (p.rpart): the router logits are the sums of the router pieces'
// partials, read straight from where the pieces wrote them, polling on the
// data (see Params::rpart).  pstride: floats between two pieces' partials.
// Writes the logits to lgs [B][E] (shared memory) and to p.logits; false if
// they never all arrived (the wait is bounded).
__device__ __forceinline__ bool route_poll_logits(const Params& p, float* lgs, int pstride, int tid) {
  constexpr int kMaxPieces = 16;  // router pieces per row block in this mode (host: at most 16)
  constexpr int kOut = 2;         // outputs a thread sums per round: 32 loads in flight
  const int E = p.E, B = p.B, ppr = p.PPR_r, n = B * E;
  const unsigned long long t0 = global_ns();
  for (uint32_t it = 0; it < (1u << 20); ++it) {
    bool missing = false;
    for (int o0 = tid; o0 < n; o0 += kOut * kConsumerThreads) {
      float v[kOut][kMaxPieces];
      // every load of the round first (one round trip), then the sums, each
      // in piece order (the same sum every run)
#pragma unroll
      for (int u = 0; u < kOut; ++u) {
        const int o = o0 + u * kConsumerThreads;
        const int b = o / E, e = o - b * E;
        const float* src =
            p.rpart + (long long)(e >> 7) * ppr * pstride + b * kRowsPerBlock + (e & 127);
#pragma unroll
        for (int j = 0; j < kMaxPieces; ++j)
          v[u][j] = (o < n && j < ppr) ? __ldcg(src + (long long)j * pstride) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kOut; ++u) {
        const int o = o0 + u * kConsumerThreads;
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxPieces; ++j) {
          missing |= __float_as_uint(v[u][j]) == 0xFFFFFFFFu;
          acc += v[u][j];
        }
        if (o < n) lgs[o] = acc;
      }
    }
    if (!named_sync_or(1, kConsumerThreads, missing)) {
      // every piece's partials arrived: publish the logits, restore the marks
      for (int o = tid; o < n; o += kConsumerThreads) {
        p.logits[o] = lgs[o];
        const int b = o / E, e = o - b * E;
        float* dst = p.rpart + (long long)(e >> 7) * ppr * pstride + b * kRowsPerBlock + (e & 127);
        for (int j = 0; j < ppr; ++j) dst[(long long)j * pstride] = __uint_as_float(0xFFFFFFFFu);
      }
      return true;
    }
    __nanosleep(64);
    if ((it & 15) == 15 && global_ns() - t0 > 1000000000ull) break;
  }
  if (tid == 0) atomicOr(p.err, 1 << ERR_WAIT_DEP);
  return false;
}

// Few tokens (B <= 8, B * k <= 64, logits in shared memory): one warp a
// token selects its experts over all of them, then warp 0 sorts the B * k
// (expert, slot) pairs (bitonic, two a lane: positions 2 lane and 2 lane + 1)
// and writes the tables itself: a virtual expert per run of equal experts
// (at most B <= tg tokens), its positions in slot order.  Two barriers
// instead of the general path's slices, merge and CTA-wide scan, each of
// which costs several µs while the weights stream.  es: 64 ints of shared
// memory (the sorted experts, for the run lengths).
constexpr int kRouteFewSlots = 64;
__device__ __forceinline__ void route_few(const Params& p, const float* bias, const float* lg_sm,
                                          int* ids_s, int* es, int warp, int lane) {
  const int K = p.topk, B = p.B, E = p.E;
  if (warp < B) {
    int sel_id;
    float sel_w;
    warp_topk<true>(lg_sm + (long long)warp * E, E, K, p.score_fn, bias, p.renorm, p.routed_scale,
                    lane, sel_id, sel_w);
    if (lane < K) {
      p.ids[warp * K + lane] = sel_id;
      p.wts[warp * K + lane] = sel_w;
      ids_s[warp * K + lane] = sel_id;
    }
  }
  named_sync(1, kConsumerThreads);
  if (warp == 0) {
    const int n = B * K;
    // expert in the high bits, slot in the low 6; positions past n sort last
    uint32_t key[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int pos = 2 * lane + h;
      key[h] = pos < n ? ((uint32_t)ids_s[pos] << 6) | (uint32_t)pos : 0xFFFFFFFFu;
    }
#pragma unroll
    for (int k = 2; k <= kRouteFewSlots; k <<= 1) {
      const bool ascending = ((2 * lane) & k) == 0;  // (bit k >= 2 is the lane's for both)
#pragma unroll
      for (int j = k >> 1; j > 0; j >>= 1) {
        if (j == 1) {  // the lane's two positions
          const uint32_t lo = min(key[0], key[1]), hi = max(key[0], key[1]);
          key[0] = ascending ? lo : hi;
          key[1] = ascending ? hi : lo;
        } else {
          const bool lower = (lane & (j >> 1)) == 0;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t other = __shfl_xor_sync(0xffffffffu, key[h], j >> 1);
            key[h] = (lower == ascending) ? min(key[h], other) : max(key[h], other);
          }
        }
      }
    }
    const int e0 = (int)(key[0] >> 6), e1 = (int)(key[1] >> 6);
    es[2 * lane] = e0;
    es[2 * lane + 1] = e1;
    const int prev1 = __shfl_up_sync(0xffffffffu, e1, 1);  // position 2 lane - 1
    const bool st0 = 2 * lane < n && (lane == 0 || prev1 != e0);
    const bool st1 = 2 * lane + 1 < n && e1 != e0;
    // virtual expert index: run starts up to each position (warp prefix sum)
    const int c = (int)st0 + (int)st1;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    const int excl = incl - c;
    __syncwarp();  // es complete
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int pos = 2 * lane + h;
      if (pos < n) p.slots_sorted[pos] = (int)(key[h] & 63u);
      const bool st = h == 0 ? st0 : st1;
      if (st) {
        const int v = excl + (h == 0 ? 0 : (int)st0);
        const int e = h == 0 ? e0 : e1;
        int len = 1;
        while (pos + len < n && es[pos + len] == e) ++len;  // (a run holds at most B tokens)
        VExpert ve;
        ve.expert = e;
        ve.start = pos;
        ve.count = len;
        ve.pad = 0;
        p.ve[v] = ve;
        if (p.h_done) p.h_done[v] = 0;
      }
    }
    if (lane == 31) *p.nve = incl;
  }
  named_sync(1, kConsumerThreads);  // (every table write precedes the release)
}

__device__ __forceinline__ void route_cta(const Params& p, uint8_t* scratch, float* bias_s,
                                          int* sm_flag, int tid, int warp, int lane, int pstride) {
  unsigned long long* tr = p.trace ? p.trace + (size_t)blockIdx.x * kTraceStride : nullptr;
  // the previous forward's tail is complete (this CTA waited for it): its
  // record count starts again from zero
  if (p.t_ready && tid == 0 && blockIdx.x == gridDim.x - 1) *p.t_ready = 0;
  // the selection bias is static: stage it in shared memory before the
  // logits exist, so the selection waits on one round trip, not two
  const float* bias = nullptr;
  if (p.bias) {
    for (int i = tid; i < p.E; i += kConsumerThreads) bias_s[i] = __ldg(p.bias + i);
    bias = bias_s;
  }
  named_sync(1, kConsumerThreads);
  // the rest of the idle ring holds staged logits
  const int bias_floats = (p.E + 31) & ~31;
  const int ring_floats = p.nstages * p.stage_bytes / 4;
  float* lgs = bias_s + bias_floats;
  if (p.rpart) {
    // the logits straight from the router pieces' partial sums
    const bool ok = route_poll_logits(p, lgs, pstride, tid);
    named_sync(1, kConsumerThreads);
    if (!ok) return;
    if (tr && tid == 0) tr[4] = global_ns();
    if (p.B * p.topk <= kRouteFewSlots && p.route_few)
      route_few(p, bias, lgs, reinterpret_cast<int*>(scratch),
                reinterpret_cast<int*>(scratch) + kRouteFewSlots, warp, lane);  // ends with a barrier
    else
      route_tokens(p, bias, scratch, lgs + p.B * p.E, ring_floats - bias_floats - p.B * p.E,
                   sm_flag + 16, tid, warp, lane, lgs);  // ends with a barrier
    if (tid == 0) {
      if (tr) tr[5] = global_ns();
      st_release(p.route_ready, 1);
    }
    return;
  }
  if (tid == 0) {
    bool ok = false;
    for (uint32_t i = 0; i < (1u << 22); ++i) {
      if (ld_acquire(p.router_done) >= p.RB_router) {
        ok = true;
        break;
      }
      __nanosleep(64);
    }
    if (!ok) atomicOr(p.err, 1 << ERR_WAIT_DEP);
    sm_flag[0] = ok ? 1 : 0;
  }
  named_sync(1, kConsumerThreads);  // thread 0's acquire covers the others' logit reads
  if (!sm_flag[0]) return;
  if (tr && tid == 0) tr[4] = global_ns();
  if (p.route_cta == 1 && p.B <= kConsumerWarps && p.B * p.topk <= kRouteFewSlots && p.route_few) {
    // few tokens: their logits into the idle ring with every load in flight,
    // then the one-warp table build
    float* lgs = bias_s + bias_floats;
    stage_floats(p.logits, p.B * p.E, lgs, tid);
    named_sync(1, kConsumerThreads);
    route_few(p, bias, lgs, reinterpret_cast<int*>(scratch), reinterpret_cast<int*>(scratch) + kRouteFewSlots,
              warp, lane);  // ends with a barrier
    if (tid == 0) {
      if (tr) tr[5] = global_ns();
      *p.router_done = 0;
      st_release(p.route_ready, 1);
    }
    return;
  }
  // this routing CTA's share of the tokens
  const int R = p.route_cta;
  const int r = (int)blockIdx.x - ((int)gridDim.x - R);
  const int per = (p.B + R - 1) / R;
  const int b_lo = min(p.B, r * per), b_hi = min(p.B, b_lo + per);
  const bool last = route_tokens(p, bias, scratch, bias_s + bias_floats, ring_floats - bias_floats,
                                 sm_flag + 16, tid, warp, lane, nullptr, b_lo, b_hi);
  if (last && tid == 0) {
    if (tr) tr[5] = global_ns();
    if (R == 1) *p.router_done = 0;
    // every thread's table writes precede this release (barrier cumulativity)
    st_release(p.route_ready, 1);
  }
}

// ---------------------------------------------------------------------------
// consumer warps

// Split-K partial sums: [piece][token column][128 rows] floats, only the
// columns that hold tokens are written.
template <int NT>
__device__ __forceinline__ void write_partial(const Params& p, int piece, int ntok,
                                              const float (&acc)[NT][4], int warp, int lane) {
  const int g = lane >> 2, tig = lane & 3;
  float* base = p.partials + (long long)piece * (NT * 8 * kRowsPerBlock);
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int col = 8 * t + 2 * tig + (q & 1);
      const int row = 16 * warp + ((q & 2) ? g + 8 : g);
      if (col < ntok) base[col * kRowsPerBlock + row] = acc[t][q];
    }
}

// Sum of ppr pieces' partials for n4 groups of four consecutive floats:
// thread tid owns groups tid + 256 j (j < JG) and keeps JG * PB 16-byte loads
// in flight.  Pieces are added in piece order.
template <int JG, int PB>
__device__ __forceinline__ void sum_groups(const float* base, long long stride, int ppr, int n4,
                                           float* rs, int tid) {
  float4 s[JG];
#pragma unroll
  for (int j = 0; j < JG; ++j) s[j] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int pr = 0; pr < ppr; pr += PB) {
    float4 v[JG][PB];
#pragma unroll
    for (int j = 0; j < JG; ++j)
#pragma unroll
      for (int u = 0; u < PB; ++u) {
        const int i = tid + j * kConsumerThreads;
        v[j][u] = (i < n4 && pr + u < ppr)
                      ? __ldcg(reinterpret_cast<const float4*>(base + (pr + u) * stride) + i)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
    for (int j = 0; j < JG; ++j)
#pragma unroll
      for (int u = 0; u < PB; ++u) {
        s[j].x += v[j][u].x;
        s[j].y += v[j][u].y;
        s[j].z += v[j][u].z;
        s[j].w += v[j][u].w;
      }
  }
#pragma unroll
  for (int j = 0; j < JG; ++j) {
    const int i = tid + j * kConsumerThreads;
    if (i < n4) reinterpret_cast<float4*>(rs)[i] = s[j];
  }
}

// Sum the row block's pieces in piece order (the same order whatever CTA ran
// them, so the result is deterministic).  All consumer threads share the
// loads and hand the sums back through shared memory, 32 token columns
// (16 KB of scratch) at a time: up to 8 columns one group of four rows a
// thread with 16 pieces in flight, more columns four groups a thread with 4
// pieces in flight.
template <int NT>
__device__ __forceinline__ void sum_partials(const Params& p, const Hdr& h, float (&acc)[NT][4],
                                             float* rs, int tid, int warp, int lane) {
  const long long stride = NT * 8 * kRowsPerBlock;
  const float* base = p.partials + (long long)h.p0 * stride;
  const int g = lane >> 2, tig = lane & 3;
  for (int c0 = 0; c0 < h.ntok; c0 += 32) {
    const int ncol = min(32, h.ntok - c0);
    const int n4 = ncol * (kRowsPerBlock / 4);
    if (ncol <= 8)
      sum_groups<1, 16>(base + c0 * kRowsPerBlock, stride, h.ppr, n4, rs, tid);
    else
      sum_groups<4, 4>(base + c0 * kRowsPerBlock, stride, h.ppr, n4, rs, tid);
    named_sync(1, kConsumerThreads);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      if (8 * t < c0 || 8 * t >= c0 + 32) continue;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int col = 8 * t + 2 * tig + (q & 1);
        const int row = 16 * warp + ((q & 2) ? g + 8 : g);
        acc[t][q] = col < h.ntok ? rs[(col - c0) * kRowsPerBlock + row] : 0.f;
      }
    }
    named_sync(1, kConsumerThreads);
  }
}

template <int KIND, int NT>
__device__ __forceinline__ void finalize(const Params& p, const Hdr& h, float (&acc)[NT][4], uint8_t* scratch,
                         int* sm_flag, const int* slot_tab, int tid, int warp, int lane) {
  sum_partials<NT>(p, h, acc, reinterpret_cast<float*>(scratch), tid, warp, lane);
  if (tid == 0) p.counters[h.v * p.RB + h.rb] = 0;  // ready for the next launch
  epilogue<KIND, NT>(p, h, acc, scratch, sm_flag, slot_tab, tid, warp, lane);
}

// ---------------------------------------------------------------------------
// expert kernels on the 5th-generation tensor cores (p.umma = token tiles)
//
// Warp roles: the producer streams stages as for the warp-level MMA; one MMA
// warp (its lane 0) issues each stage's four K = 64 block-scaled MMAs
// (e2m1 weights x the activation's e2m1 terms) and releases the stage when
// they complete; the eight consumer warps take each finished piece's sums
// out of tensor memory and run the split-K and epilogue logic.  Two
// accumulator buffers let the MMAs of the next piece run meanwhile.
//
// Tensor memory of a CTA: accumulator buffer b at columns N b, 128 rows x
// (N = kUTerms x 8 NT token terms); then per ring slot s 16 columns of
// scales at 2 N + 16 s: the weights' at +0, the activations' at +8, each two
// 4-column units (K blocks 0-3, 4-7).  A slot's scales are rewritten only
// after the MMAs that read them have completed (they release the slot).
// Up to two token tiles the CTA takes 256 columns (two CTAs can share an
// SM), at four 512.
// The tail's bf16 MMA (its activation as hi and lo parts, two rows a token)
// needs no scale columns: 2 x 16 NT accumulator columns.
// (the front's bf16 MMA: x once, one row a token)
template <int KIND>
__host__ __device__ constexpr int umma_terms() {
  return KIND == KIND_TAIL ? 2 : KIND == KIND_FRONT ? 1 : kUTerms;
}
template <int KIND, int NT>
__host__ __device__ constexpr uint32_t tmem_dcols() { return (uint32_t)(umma_terms<KIND>() * 8 * NT); }
template <int KIND, int NT>
__host__ __device__ constexpr uint32_t tmem_sf() { return 2 * tmem_dcols<KIND, NT>(); }
template <int KIND, int NT>
__host__ __device__ constexpr uint32_t tmem_cols() {
  // (a power of two, at least 32: two accumulator buffers, and the expert
  // kernels' scale columns)
  return KIND == KIND_FRONT ? (NT <= 2 ? 32u : NT == 4 ? 64u : NT == 8 ? 128u : 256u)
         : KIND == KIND_TAIL ? (NT <= 4 ? 128u : 256u)
                             : (NT <= 2 ? 256u : 512u);
}
static_assert(tmem_sf<KIND_FRONT, 16>() <= tmem_cols<KIND_FRONT, 16>(), "two accumulator buffers");
static_assert(tmem_sf<KIND_FRONT, 2>() <= tmem_cols<KIND_FRONT, 2>(), "two accumulator buffers");
static_assert(tmem_sf<KIND_EGU, 1>() + 16 * kMaxStages <= tmem_cols<KIND_EGU, 1>(), "scale columns");
static_assert(tmem_sf<KIND_EGU, 2>() + 16 * kMaxStages <= tmem_cols<KIND_EGU, 2>(), "scale columns");
static_assert(tmem_sf<KIND_EGU, 4>() + 16 * kMaxStages <= tmem_cols<KIND_EGU, 4>(), "scale columns");
static_assert(tmem_sf<KIND_TAIL, 8>() <= tmem_cols<KIND_TAIL, 8>(), "two accumulator buffers");
static_assert(tmem_sf<KIND_TAIL, 4>() <= tmem_cols<KIND_TAIL, 4>(), "two accumulator buffers");
// shared-memory handover: tensor-memory base at flag word kUTmemWord,
// accumulator-full barriers (MMA completion + the header's release) at words
// kUDfullWord + 2 b, accumulator-free barriers at kUDfreeWord + 2 b, the MMA
// warp's drain barrier at kUDrainWord; the finished pieces' headers at byte
// kUPqByte of shared memory (between the flags and the scratch)
constexpr int kUTmemWord = 48, kUDfullWord = 50, kUDfreeWord = 54, kUDrainWord = 58;
constexpr int kUPqByte = 512;
static_assert(kUPqByte + 2 * sizeof(Hdr) <= 1024, "two piece headers before the consumers' scratch");
constexpr int kThreadsU = kThreads + 32;  // + the MMA warp
constexpr int kMmaWarp = kConsumerWarps + 1;

template <int KIND, int NT>
__device__ void mma_issuer(const Params& p, uint8_t* stage_base, uint64_t* full, uint64_t* empty,
                           uint64_t* dfull, uint64_t* dfree, uint64_t* drain, Hdr* pq, uint32_t tmem) {
  constexpr int kRows = umma_terms<KIND>() * 8 * NT, kNg = kRows / 8;
  int stage = 0, buf = 0;
  uint32_t phase = 0, uses[2] = {0u, 0u};
  long long mw = 0, mi = 0, t0 = clock64();
  while (true) {
    if (!mbar_wait_bounded(&full[stage], phase, p.err, ERR_WAIT_FULL, p.cons_sleep)) break;
    const long long t1 = clock64();
    mw += t1 - t0;
    const uint8_t* sb = stage_base + (size_t)stage * p.stage_bytes;
    const Hdr h = *reinterpret_cast<const Hdr*>(sb);
    const bool first = (h.flags & HDR_FIRST) != 0;
    // a piece's first stage overwrites its accumulator buffer (and the end
    // mark its header): the consumers must have read the piece before last
    // out of it
    if ((first || (h.flags & HDR_END)) &&
        !mbar_wait_bounded(&dfree[buf], (uses[buf] & 1u) ^ 1u, p.err, ERR_WAIT_FULL, p.cons_sleep))
      break;
    if (h.flags & HDR_END) {
      pq[buf] = h;
      mbar_arrive(&dfull[buf]);
      mbar_arrive(&dfull[buf]);
      break;
    }
    fence_proxy_async_smem();  // the activation rows came in by cp.async
    umma::fence_after_sync();
    const uint32_t d = tmem + (uint32_t)buf * tmem_dcols<KIND, NT>();
    if constexpr (KIND == KIND_TAIL || KIND == KIND_FRONT) {
      // bf16 weights (128 x 64 K) x the records' hi and lo rows (tail) or the
      // x rows (front): four K = 16
      const uint8_t* A = sb + kHdrBytes;
      const uint8_t* B = sb + p.act_off;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint64_t ad = umma::smem_desc(A + j * 4096, 2048, 128);
        const uint64_t bd = umma::smem_desc(B + j * 2 * kNg * 128, kNg * 128, 128);
        umma::mma_bf16(d, ad, bd, umma::idesc_bf16(128, kRows), !(first && j == 0));
      }
    } else {
      const uint8_t* A = sb + kUAOff;
      const uint8_t* B = sb + kUBOff;
      const uint32_t sfa_t = tmem + tmem_sf<KIND, NT>() + 16u * (uint32_t)stage, sfb_t = sfa_t + 8;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        umma::cp_scales(sfa_t + 4 * u, umma::smem_desc(sb + kUSfaOff + 512 * u, 128, 128));
        umma::cp_scales(sfb_t + 4 * u, umma::smem_desc(B + kRows * kUTermBytes + 512 * u, 128, 128));
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint64_t ad = umma::smem_desc(A + j * 4096, 2048, 128);
        const uint64_t bd = umma::smem_desc(B + j * 2 * kNg * 128, kNg * 128, 128);
        umma::mma_mxf4(d, ad, bd, umma::idesc_mxf4(128, kRows, 2 * (j & 1), 2 * (j & 1)),
                       sfa_t + 4 * (j >> 1), sfb_t + 4 * (j >> 1), !(first && j == 0));
      }
    }
    umma::commit(&empty[stage]);  // the slot is free once these MMAs have read it
    if (h.flags & HDR_LAST) {
      pq[buf] = h;
      umma::commit(&dfull[buf]);  // the sums are complete ...
      mbar_arrive(&dfull[buf]);   // ... and the header is written
      ++uses[buf];
      buf ^= 1;
    }
    if (++stage == p.nstages) {
      stage = 0;
      phase ^= 1;
    }
    t0 = clock64();
    mi += t0 - t1;
  }
  if (p.trace) {
    unsigned long long* tr = p.trace + (size_t)blockIdx.x * kTraceStride;
    tr[22] = (unsigned long long)mw;
    tr[23] = (unsigned long long)mi;
  }
  // MMAs cut short by an error may still run: drain them before the tensor
  // memory is given back
  umma::commit(drain);
  mbar_wait_bounded(drain, 0, p.err, ERR_WAIT_FULL, p.cons_sleep);
}

// A finished piece's sums out of tensor memory into the MMA-fragment
// registers the epilogues take: warps 0-3 read their 32 rows (lane quarter
// = warp), add the TERMS terms of each token and stage the sums in shared
// memory (128 rows x up to 32 tokens at a time); the buffer is released to
// the MMA warp once read, and every warp picks its fragments.
template <int NT, int TERMS>
__device__ __forceinline__ void umma_read_acc(uint32_t d, float* stage_s, float (&acc)[NT][4], int warp,
                                             int lane, int tid, uint64_t* dfree_bar) {
  umma::fence_after_sync();
  constexpr int kTok = 8 * NT;                 // columns of one term
  constexpr int kGrp = NT < 4 ? NT : 4;        // token tiles staged at a time
  constexpr int kLd = 8 * kGrp + 1;            // (row stride padded: no bank conflicts)
  const int g = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int t0 = 0; t0 < NT; t0 += kGrp) {
    if (warp < 4) {
      const int row = 32 * warp + lane;
      const uint32_t lane_addr = d + ((uint32_t)(32 * warp) << 16);
#pragma unroll
      for (int c = 0; c < kGrp; ++c) {
        float sum[8], t[8];
        umma::ld_32x32b_x8(lane_addr + 8 * (t0 + c), sum);
        umma::wait_ld();
#pragma unroll
        for (int term = 1; term < TERMS; ++term) {
          umma::ld_32x32b_x8(lane_addr + term * kTok + 8 * (t0 + c), t);
          umma::wait_ld();
#pragma unroll
          for (int i = 0; i < 8; ++i) sum[i] += t[i];
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) stage_s[row * kLd + 8 * c + i] = sum[i];
      }
    }
    if (t0 + kGrp >= NT) umma::fence_before_sync();
    named_sync(1, kConsumerThreads);
    if (t0 + kGrp >= NT && tid == 0) mbar_arrive(dfree_bar);
#pragma unroll
    for (int c = 0; c < kGrp; ++c)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int col = 8 * c + 2 * tig + (q & 1);
        const int row = 16 * warp + ((q & 2) ? g + 8 : g);
        acc[t0 + c][q] = stage_s[row * kLd + col];
      }
    named_sync(1, kConsumerThreads);
  }
}

template <int KIND, int NT, bool UM>
__device__ void consumer(const Params& p, uint8_t* stage_base, uint64_t* full, uint64_t* empty,
                         uint8_t* scratch, int* sm_flag, const int* slot_tab, int warp, int lane) {
  const int tid = warp * 32 + lane;
  int stage = 0;
  uint32_t phase = 0;
  int nbuf = 0;
  // two accumulator sets (k16 steps 0 and 1) so consecutive MMAs do not wait
  // on each other; folded together when a piece ends
  float acc[NT][4], acc2[NT][4];
  zero_acc(acc);
  zero_acc(acc2);
  // A piece whose ticket (finalize counter) is still in flight: thread 0
  // issues the atomic after the piece's partials are written and reads its
  // result only at the next piece end, so nobody waits on the round trip.
  bool pend = false;
  Hdr pend_h{};
  int ticket = 0;
  int* tflag = sm_flag + 4;  // two alternating slots
  int tslot = 0;
  // Activations, routing tables and partial sums of the previous kernel are
  // read only after the dependency has resolved; the next kernel may then be
  // scheduled (it cannot overtake this one's own predecessor).  Two kinds
  // wait elsewhere:
  //   - the tail with its shared part first waits when its first latent
  //     stage arrives (the shared part reads h_s, complete before this
  //     kernel starts, and the stages the producer filled);
  //   - the expert gate/up kernel with a z count reads nothing of the front
  //     kernel but what its producer copies after that count; it waits for
  //     the front grid only before exiting.
  const bool lazy = KIND == KIND_TAIL && p.tail_split && !p.tail_part;
  const bool late = (KIND == KIND_EGU && p.z_done) || (KIND == KIND_EDN && p.h_done);
  uint8_t* res = stage_base - p.stage_off + p.res_off;  // shared-memory base + offset
  const int klat = p.C_lat * 64;
  // Past the wait every earlier kernel of the forward has finished, so no
  // reader of the routing flag or of the z count is left: clear both for the
  // next forward.
  auto tail_dep = [&](int kbeg, int kend) {
    pdl_wait();
    pdl_trigger();
    // (the side lane's tail waits only for the shared expert's gate/up, so
    // it leaves them alone)
    if (KIND == KIND_TAIL && tid == 0 && p.tail_part != 2) {
      *p.route_ready = 0;
      if (p.z_done) *p.z_done = 0;
    }
    if (KIND == KIND_TAIL && p.res_off) {
      build_resident(p, res, tid, kbeg, kend);
      named_sync(1, kConsumerThreads);
    }
    if (KIND == KIND_TAIL && p.t_rec) {
      form_tail_records(p, tid);
      named_sync(1, kConsumerThreads);  // every thread's records precede the release
      if (tid == 0) red_release_add(p.t_ready, 1);
    }
  };
  bool dep_done = !lazy;
  if (lazy) {
    if (p.res_off) {
      build_resident(p, res, tid, klat, p.res_k);
      named_sync(1, kConsumerThreads);
    }
  } else if (!late) {
    // everything the record holds: both parts, or one lane's
    tail_dep(p.res_k0, p.res_k0 + p.res_k);
  }
  unsigned long long* tr = p.trace ? p.trace + (size_t)blockIdx.x * kTraceStride : nullptr;
  int n_pieces = 0, n_fin = 0;
  long long c_wait = 0, c_comp = 0, c_end = 0, t_a = clock64();
  // tensor-core expert kernels: tensor memory base, the handover barriers
  // and the finished pieces' headers
  const uint32_t tmem = UM ? *reinterpret_cast<volatile uint32_t*>(sm_flag + kUTmemWord) : 0u;
  uint64_t* dfull = reinterpret_cast<uint64_t*>(sm_flag + kUDfullWord);
  uint64_t* dfree = reinterpret_cast<uint64_t*>(sm_flag + kUDfreeWord);
  const Hdr* pq = reinterpret_cast<const Hdr*>(stage_base - p.stage_off + kUPqByte);
  // a piece's sums are in acc (+ acc2): split-K partials, tickets,
  // finalisation, epilogue
  auto piece_done = [&](const Hdr& h) {
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[t][q] += acc2[t][q];

    if (KIND == KIND_FRONT && p.rpart && h.rb < p.RB_router) {
      // router piece, few tokens: its partial sums go where the routing CTA
      // polls for them; no ticket, no finalisation
      Params q = p;
      q.partials = p.rpart;
      write_partial<NT>(q, h.piece, h.ntok, acc, warp, lane);
      const long long t_c = clock64();
      c_end += t_c - t_a;
      t_a = t_c;
      return;
    }
    if (h.ppr == 1) {
      ++n_fin;
      epilogue<KIND, NT>(p, h, acc, scratch, sm_flag, slot_tab, tid, warp, lane);
      return;
    }
    write_partial<NT>(p, h.piece, h.ntok, acc, warp, lane);
    if ((KIND == KIND_FRONT) && h.rb < p.RB_router) {
      // Router row blocks take their ticket at once: the routing waits on
      // all of them, and the latent rows behind it hide the round trip.
      if (tid == 0) {
        if (pend) tflag[tslot] = (ticket == pend_h.ppr - 1);
        sm_flag[6] = (atom_add_acqrel(p.counters + h.v * p.RB + h.rb, 1) == h.ppr - 1);
      }
      named_sync(1, kConsumerThreads);
      const bool fin_prev = pend && tflag[tslot] != 0;
      const bool fin_now = sm_flag[6] != 0;
      const Hdr prev = pend_h;
      pend = false;
      named_sync(1, kConsumerThreads);  // flags read before they are reused
      if (fin_prev) {
        ++n_fin;
        finalize<KIND, NT>(p, prev, acc, scratch, sm_flag, slot_tab, tid, warp, lane);
      }
      if (fin_now) {
        ++n_fin;
        const unsigned long long t0 = tr ? global_ns() : 0ull;
        finalize<KIND, NT>(p, h, acc, scratch, sm_flag, slot_tab, tid, warp, lane);
        if (tr && tid == 0) tr[7] += global_ns() - t0;
      }
      const long long t_c = clock64();
      c_end += t_c - t_a;
      t_a = t_c;
      return;
    }
    if (tid == 0 && pend) tflag[tslot] = (ticket == pend_h.ppr - 1);
    named_sync(1, kConsumerThreads);  // every warp's partials precede thread 0's release
    const bool fin = pend && tflag[tslot] != 0;
    if (tid == 0) ticket = atom_add_acqrel(p.counters + h.v * p.RB + h.rb, 1);
    const Hdr prev = pend_h;
    pend_h = h;
    pend = true;
    tslot ^= 1;
    if (fin) {
      ++n_fin;
      const unsigned long long t0 = tr ? global_ns() : 0ull;
      finalize<KIND, NT>(p, prev, acc, scratch, sm_flag, slot_tab, tid, warp, lane);
      if (tr && tid == 0) tr[7] += global_ns() - t0;
    }
    const long long t_c = clock64();
    c_end += t_c - t_a;
    t_a = t_c;
  };
  if constexpr (UM) {
    // tensor-core expert kernels: the MMA warp hands over each finished
    // piece (its header in pq, its sums in accumulator buffer buf)
    int buf = 0;
    uint32_t uses[2] = {0u, 0u};
    while (true) {
      if (!mbar_wait_bounded(&dfull[buf], uses[buf] & 1u, p.err, ERR_WAIT_FULL, p.cons_sleep)) break;
      long long t_b = clock64();
      c_wait += t_b - t_a;
      const Hdr h = pq[buf];
      if (h.flags & HDR_END) break;
      if (tr && tid == 0 && n_pieces == 0) tr[6] = global_ns();
      zero_acc(acc2);
      umma_read_acc<NT, umma_terms<KIND>()>(tmem + (uint32_t)buf * tmem_dcols<KIND, NT>(),
                                            reinterpret_cast<float*>(scratch), acc, warp,
                        lane, tid, &dfree[buf]);
      ++uses[buf];
      buf ^= 1;
      t_a = clock64();
      c_comp += t_a - t_b;
      ++n_pieces;
      piece_done(h);
    }
  } else {
    while (true) {
      if (!mbar_wait_bounded(&full[stage], phase, p.err, ERR_WAIT_FULL, p.cons_sleep)) break;
      long long t_b = clock64();
      c_wait += t_b - t_a;
      uint8_t* sb = stage_base + (size_t)stage * p.stage_bytes;
      const Hdr h = *reinterpret_cast<const Hdr*>(sb);
      if (tr && tid == 0 && n_pieces == 0 && (h.flags & HDR_FIRST)) tr[6] = global_ns();
      if (h.flags & HDR_END) break;
      if (lazy && !dep_done && h.dep) {
        tail_dep(0, klat);  // the first latent stage: y, and the combine, need the expert phases
        dep_done = true;
      }
      if (h.flags & HDR_FIRST) {
        zero_acc(acc);
        zero_acc(acc2);
      }
      const uint8_t* tile = sb + kHdrBytes;
      const uint8_t* act = sb + p.act_off;
      if (KIND == KIND_FRONT) {
        mma_dense_x<NT>(p, h, tile, act, acc, acc2, warp, lane);
      } else if (KIND == KIND_EGU || KIND == KIND_EDN) {
        mma_mx<NT>(p, h, tile, act, acc, warp, lane);
      } else if (p.res_off) {
        mma_tail_resident<NT>(p, h, tile, res, acc, acc2, warp, lane);
      } else if (p.t_rec) {
        mma_tail_formed<NT>(h, tile, act, acc, acc2, warp, lane);
      } else {
        uint8_t* tbuf = scratch + 4096 + (nbuf & 1) * (16 * 320);
        ++nbuf;
        mma_tail<NT>(p, h, tile, act, tbuf, acc, acc2, warp, lane, tid);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      if (++stage == p.nstages) {
        stage = 0;
        phase ^= 1;
      }
      t_a = clock64();
      c_comp += t_a - t_b;
      if (!(h.flags & HDR_LAST)) continue;
      ++n_pieces;
      piece_done(h);
    }
  }
  if (pend) {
    if (tid == 0) tflag[tslot] = (ticket == pend_h.ppr - 1);
    named_sync(1, kConsumerThreads);
    if (tflag[tslot] != 0) {
      ++n_fin;
      finalize<KIND, NT>(p, pend_h, acc, scratch, sm_flag, slot_tab, tid, warp, lane);
    }
  }
  if (late) pdl_wait();  // this grid completes only after the front grid
  if (tr && tid == 0) {
    tr[2] = (unsigned long long)n_pieces;
    tr[3] = (unsigned long long)n_fin;
    tr[8] = (unsigned long long)c_wait;
    tr[9] = (unsigned long long)c_comp;
    tr[10] = (unsigned long long)c_end;
  }
}

// ---------------------------------------------------------------------------

// MINB: CTAs per SM the instantiation is compiled for.  Two for the expert
// kernels at one token tile, and for the one-tile front and tail variants the
// side lane uses (a CTA of each lane on one SM); one otherwise.
// UM: the expert kernels' tensor-core instantiation (its own kernel, so that
// neither variant's registers are sized for the other's code).
template <int KIND, int NT, int MINB, bool UM>
__global__ void __launch_bounds__(UM ? kThreadsU : kThreads, MINB)
    moe_kernel(const __grid_constant__ Params p) {
  // shared memory: [0,128) full barriers, [128,256) empty barriers,
  // [256,512) flags, [512,1024) the tensor-core kernels' piece headers,
  // [scratch_off, ...) scratch, [table_off, ...) routing
  // tables (expert kernels), [stage_off, ...) ring
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kMaxStages;
  int* sm_flag = reinterpret_cast<int*>(smem + 256);
  uint8_t* scratch = smem + p.scratch_off;
  uint8_t* stages = smem + p.stage_off;
  uint8_t* tables = smem + p.table_off;
  const int* slot_tab = reinterpret_cast<const int*>(tables + (size_t)p.ve_max * sizeof(VExpert));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Ctl* ctl = p.ctl;
  if (p.trace && threadIdx.x == 0) {
    unsigned long long* tr = p.trace + (size_t)blockIdx.x * kTraceStride;
    tr[0] = global_ns();
    for (int i = 2; i < kTraceStride; ++i) tr[i] = 0;
    tr[14] = smid();
  }
  // tensor-core expert kernels: a stage is released by the commit of its
  // MMAs (one arrival); an accumulator buffer is full once its MMAs have
  // completed and the MMA warp has written the piece's header (two
  // arrivals), free once the consumers have read it (one); tensor memory for
  // the accumulators and the scales
  static_assert(!UM || MINB == 1 || KIND == KIND_EGU || KIND == KIND_EDN,
                "two tensor-core CTAs an SM: expert kernels only");
  constexpr bool um = UM;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm_flag + kUTmemWord);
  uint64_t* dfull = reinterpret_cast<uint64_t*>(sm_flag + kUDfullWord);
  uint64_t* dfree = reinterpret_cast<uint64_t*>(sm_flag + kUDfreeWord);
  uint64_t* drain = reinterpret_cast<uint64_t*>(sm_flag + kUDrainWord);
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nstages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], um ? 1 : kConsumerWarps);
    }
    if (um) {
      for (int b = 0; b < 2; ++b) {
        mbar_init(&dfull[b], 2);
        mbar_init(&dfree[b], 1);
      }
      mbar_init(drain, 1);
    }
    fence_mbar_init();
  }
  if (um && warp == 0) umma::tmem_alloc(tmem_slot, tmem_cols<KIND, NT>());
  if (um) umma::fence_before_sync();
  __syncthreads();
  if (um) umma::fence_after_sync();
  if (KIND == KIND_FRONT && p.route_cta && (int)blockIdx.x >= (int)gridDim.x - p.route_cta) {
    // it writes the routing tables the previous forward's tail reads
    pdl_wait();
    pdl_trigger();
    if (warp < kConsumerWarps)
      route_cta(p, scratch, reinterpret_cast<float*>(stages), sm_flag, threadIdx.x, warp, lane,
                NT * 8 * kRowsPerBlock);
  } else if (warp == kConsumerWarps) {
    producer<KIND>(p, ctl, stages, tables, full, empty, lane);
  } else if (UM && warp == kMmaWarp) {
    if (lane == 0)
      mma_issuer<KIND, NT>(p, stages, full, empty, dfull, dfree, drain,
                     reinterpret_cast<Hdr*>(smem + kUPqByte), *tmem_slot);
  } else {
    consumer<KIND, NT, UM>(p, stages, full, empty, scratch, sm_flag, slot_tab, warp, lane);
  }
  if (um) umma::fence_before_sync();
  __syncthreads();
  if (um && warp == 0) {
    umma::fence_after_sync();
    umma::tmem_dealloc(*tmem_slot, tmem_cols<KIND, NT>());
  }
  if (p.trace && threadIdx.x == 0) p.trace[(size_t)blockIdx.x * kTraceStride + 1] = global_ns();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&ctl->exits, 1) == (int)gridDim.x - 1) {
      ctl->cursor = 0;
      ctl->exits = 0;
      __threadfence();
    }
  }
}

// ---------------------------------------------------------------------------
// host-side launch of one instantiation

template <int KIND, int NT>
constexpr int default_minb() {
  return (KIND == KIND_EGU || KIND == KIND_EDN) && NT == 1 ? 2 : 1;
}

template <int KIND, int NT, int MINB = default_minb<KIND, NT>(), bool UM = false>
static int launch_one(const Params& p, int grid, size_t smem, cudaStream_t s, bool pdl) {
  auto kfn = moe_kernel<KIND, NT, MINB, UM>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(UM ? kThreadsU : kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return (int)cudaLaunchKernelEx(&cfg, kfn, p);
}

template <int KIND, int NT, int MINB = default_minb<KIND, NT>(), bool UM = false>
static int set_attr(size_t bytes) {
  return (int)cudaFuncSetAttribute(moe_kernel<KIND, NT, MINB, UM>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// Token tiles (NT) each kind is built for: the front up to 16 (128 tokens),
// expert kinds up to 4 (groups of 32), the tail up to 8 (passes of 64); the
// front and tail also at one tile for two CTAs per SM (p.half_sm).
template <int KIND>
static int launch_kind_nt(int nt, const Params& p0, int grid, size_t smem, cudaStream_t s, bool pdl) {
  constexpr bool kDense = (KIND == KIND_FRONT);
  // the tensor-core expert stages are laid out for the instantiation's tiles
  Params p = p0;
  if constexpr (KIND == KIND_EGU || KIND == KIND_EDN) {
    if (p.umma) {
      // half_sm: two CTAs an SM (up to two token tiles)
      p.umma = nt;
      switch (nt) {
        case 1: return p.half_sm ? launch_one<KIND, 1, 2, true>(p, grid, smem, s, pdl)
                                 : launch_one<KIND, 1, 1, true>(p, grid, smem, s, pdl);
        case 2: return p.half_sm ? launch_one<KIND, 2, 2, true>(p, grid, smem, s, pdl)
                                 : launch_one<KIND, 2, 1, true>(p, grid, smem, s, pdl);
        case 4: return p.half_sm ? (int)cudaErrorInvalidValue : launch_one<KIND, 4, 1, true>(p, grid, smem, s, pdl);
        default: return (int)cudaErrorInvalidValue;
      }
    }
  }
  constexpr bool kHalf = (KIND == KIND_FRONT || KIND == KIND_TAIL);
  if constexpr (KIND == KIND_FRONT) {
    if (p.front_umma) {  // the tensor-core front (two token tiles or more)
      p.front_umma = nt;
      switch (nt) {
        case 2: return launch_one<KIND, 2, 1, true>(p, grid, smem, s, pdl);
        case 4: return launch_one<KIND, 4, 1, true>(p, grid, smem, s, pdl);
        case 8: return launch_one<KIND, 8, 1, true>(p, grid, smem, s, pdl);
        case 16: return launch_one<KIND, 16, 1, true>(p, grid, smem, s, pdl);
        default: return (int)cudaErrorInvalidValue;
      }
    }
  }
  if constexpr (KIND == KIND_TAIL) {
    if (p.umma) {  // the tensor-core tail (formed records)
      p.umma = nt;
      switch (nt) {
        case 1: return launch_one<KIND, 1, 1, true>(p, grid, smem, s, pdl);
        case 2: return launch_one<KIND, 2, 1, true>(p, grid, smem, s, pdl);
        case 4: return launch_one<KIND, 4, 1, true>(p, grid, smem, s, pdl);
        case 8: return launch_one<KIND, 8, 1, true>(p, grid, smem, s, pdl);
        default: return (int)cudaErrorInvalidValue;
      }
    }
  }
  if constexpr (kHalf) {
    if (p.half_sm) return nt == 1 ? launch_one<KIND, 1, 2>(p, grid, smem, s, pdl) : (int)cudaErrorInvalidValue;
  }
  switch (nt) {
    case 1: return launch_one<KIND, 1>(p, grid, smem, s, pdl);
    case 2: return launch_one<KIND, 2>(p, grid, smem, s, pdl);
    case 4: return launch_one<KIND, 4>(p, grid, smem, s, pdl);
    case 8:
      if constexpr (kDense || KIND == KIND_TAIL) return launch_one<KIND, 8>(p, grid, smem, s, pdl);
      break;
    case 16:
      if constexpr (kDense) return launch_one<KIND, 16>(p, grid, smem, s, pdl);
      break;
    default: break;
  }
  return (int)cudaErrorInvalidValue;
}

template <int KIND>
static int set_attr_kind(size_t bytes) {
  int e = set_attr<KIND, 1>(bytes) | set_attr<KIND, 2>(bytes) | set_attr<KIND, 4>(bytes);
  if constexpr (KIND == KIND_FRONT || KIND == KIND_TAIL) e |= set_attr<KIND, 8>(bytes);
  if constexpr (KIND == KIND_FRONT) e |= set_attr<KIND, 16>(bytes);
  if constexpr (KIND == KIND_FRONT || KIND == KIND_TAIL) e |= set_attr<KIND, 1, 2>(bytes);
  if constexpr (KIND == KIND_EGU || KIND == KIND_EDN)
    e |= set_attr<KIND, 1, 1, true>(bytes) | set_attr<KIND, 2, 1, true>(bytes) |
         set_attr<KIND, 4, 1, true>(bytes) | set_attr<KIND, 1, 2, true>(bytes) |
         set_attr<KIND, 2, 2, true>(bytes);
  if constexpr (KIND == KIND_TAIL)
    e |= set_attr<KIND, 1, 1, true>(bytes) | set_attr<KIND, 2, 1, true>(bytes) |
         set_attr<KIND, 4, 1, true>(bytes) | set_attr<KIND, 8, 1, true>(bytes);
  if constexpr (KIND == KIND_FRONT)
    e |= set_attr<KIND, 2, 1, true>(bytes) | set_attr<KIND, 4, 1, true>(bytes) |
         set_attr<KIND, 8, 1, true>(bytes) | set_attr<KIND, 16, 1, true>(bytes);
  return e;
}

}  // namespace moe
