// moe_kernels.cu -- the five kernels of one latent-MoE decode step on sm_100a.
//
// One engine serves all five: a CTA of 8 consumer warps and 1 producer warp.
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
//   KIND_RL   x . [W_r | W_in] -> router logits (fp32) and latent z (f16 MX);
//             the CTA that finalises the last router row block runs top-k and
//             builds the per-expert token lists while the rest of the grid is
//             still streaming W_in.
//             (page "Hyper Optimizing Kimi K3 in vLLM: Moving Fast and
//              Responsibly", section 从算子之间找时间: router scores and the
//              latent input projection as one matmul.)
//   KIND_SGU  x . [W_sg | W_su] -> h_s = silu(g) * u (fp32), side stream.
//             (same section: the shared expert on its own stream.)
//   KIND_EGU  per routed expert, z . [Wg | Wu] (MXFP4) -> h = silu(g) * u (f16 MX)
//   KIND_EDN  per routed expert, h . Wd (MXFP4) -> y (fp32, per token slot)
//   KIND_TAIL c = sum_j w_j y_j formed from y while staging the activation
//             tile (never written to memory), then [c ; h_s] . [W_out ; W_sd]
//             -> out (bf16).
//             (page "Kimi K3 在 vLLM 中的性能优化", section 延迟 MXFP4 最终化:
//              the MXFP4 top-k finalize fused into the latent-tail kernel.)
//
// Only static weights are fetched before griddepcontrol.wait; activations are
// fetched after it (page 1, section 更快的代码需要更有针对性的验证: an
// activation load hoisted above a synchronisation wait was a real bug).
#include <cuda_runtime.h>

#include <cstdio>

#include "engine.cuh"
#include "layout.cuh"
#include "ptx.cuh"
#include "topk.cuh"

namespace moe {

constexpr int kHdrBytes = 128;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kMaxStages = 8;

enum : int { HDR_FIRST = 1, HDR_LAST = 2, HDR_END = 4 };

struct Hdr {
  int flags;
  int piece, v, rb;
  int chunk, nb, ntok, tok0;
  int expert, ppr, act_bytes, pad;
};

template <int KIND>
struct KindTraits {
  static constexpr bool kMx = (KIND == KIND_EGU || KIND == KIND_EDN);
  static constexpr int kTileBytes = kMx ? kMxTileBytes : kDenseTileBytes;
  static constexpr int kChunkK = kMx ? kMxChunkK : kDenseChunkK;
  // weights may be fetched before the previous kernel finishes
  static constexpr bool kPrefetchWeights = (KIND == KIND_RL || KIND == KIND_TAIL);
  static constexpr bool kDynamicSpace = (KIND == KIND_EGU || KIND == KIND_EDN);
};

__device__ __forceinline__ uint4 lds128(const uint8_t* p) {
  return *reinterpret_cast<const uint4*>(p);
}

__device__ __forceinline__ float silu(float t) { return t / (1.0f + expf(-t)); }

// ---------------------------------------------------------------------------
// iteration space

struct Space {
  int total;  // pieces
  int ppr;
};

template <int KIND>
__device__ __forceinline__ Space make_space(const Params& p) {
  Space s;
  if (KIND == KIND_EGU || KIND == KIND_EDN) {
    const int V = *reinterpret_cast<volatile int*>(p.nve);
    const int mats = V * p.RB;
    int ppr = mats > 0 ? (p.target_pieces + mats - 1) / mats : 1;
    ppr = ppr < 1 ? 1 : (ppr > p.C ? p.C : ppr);
    s.ppr = ppr;
    s.total = mats * ppr;
  } else if (KIND == KIND_TAIL) {
    const int passes = (p.B + p.tg - 1) / p.tg;
    s.ppr = p.PPR;
    s.total = passes * p.RB * p.PPR;
  } else {
    s.ppr = p.PPR;
    s.total = p.RB * p.PPR;
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

template <int KIND>
__device__ __forceinline__ void fill_header(const Params& p, const Space& sp, int piece, int c,
                                            int c_first, int c_last, Hdr& h,
                                            const VExpert* ve_tab) {
  const int per_v = p.RB * sp.ppr;
  const int v = piece / per_v;
  const int rem = piece - v * per_v;
  const int rb = rem / sp.ppr;
  h.flags = (c == c_first ? HDR_FIRST : 0) | (c == c_last - 1 ? HDR_LAST : 0);
  h.piece = piece;
  h.v = v;
  h.rb = rb;
  h.chunk = c;
  h.nb = chunk_blocks<KIND>(p, c);
  h.ppr = sp.ppr;
  h.expert = 0;
  if (KIND == KIND_RL || KIND == KIND_SGU) {
    h.ntok = p.B;
    h.tok0 = 0;
  } else if (KIND == KIND_TAIL) {
    h.tok0 = v * p.tg;
    h.ntok = min(p.tg, p.B - h.tok0);
  } else {
    const VExpert ve = ve_tab[v];
    h.expert = ve.expert;
    h.tok0 = ve.start;
    h.ntok = ve.count;
  }
  // activation bytes of this stage
  int ab = 0;
  if (KIND == KIND_RL || KIND == KIND_SGU) {
    ab = h.ntok * h.nb * 64;
  } else if (KIND == KIND_EGU || KIND == KIND_EDN) {
    ab = h.ntok * kActRecBytes;
  } else {
    ab = (c < p.C_lat) ? h.ntok * p.topk * 256 : h.ntok * 256;
  }
  h.act_bytes = ab;
}

template <int KIND>
__device__ __forceinline__ const uint8_t* weight_src(const Params& p, const Hdr& h) {
  const long long tile = (long long)h.rb * p.C + h.chunk;
  if (KindTraits<KIND>::kMx)
    return p.wt + (long long)h.expert * p.matrix_bytes + tile * kMxTileBytes;
  return p.wt + tile * kDenseTileBytes;
}

// Issue this stage's activation copies (all 32 producer lanes).
template <int KIND>
__device__ __forceinline__ void issue_act(const Params& p, const Hdr& h, uint8_t* act, uint64_t* bar,
                                          int lane, const int* slot_tab) {
  if (KIND == KIND_RL || KIND == KIND_SGU) {
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
    if (lane == 0) {
      if (h.chunk < p.C_lat)
        bulk_g2s(act, p.y + ((long long)h.chunk * p.ld_slots + (long long)h.tok0 * p.topk) * 64,
                 h.act_bytes, bar);
      else
        bulk_g2s(act, p.h_s + ((long long)(h.chunk - p.C_lat) * p.B + h.tok0) * 64, h.act_bytes,
                 bar);
    }
  }
}

template <int KIND>
__device__ void producer(const Params& p, Ctl* ctl, uint8_t* stage_base, uint8_t* tables,
                         uint64_t* full, uint64_t* empty, int lane) {
  int stage = 0;
  uint32_t ephase = 1;  // empty barriers start "released"
  Space sp;
  int prefetched = 0;  // stages filled with weights only, waiting for pdl_wait
  bool waited = false;
  if (!KindTraits<KIND>::kPrefetchWeights) {
    pdl_wait();
    pdl_trigger();
    waited = true;
  }
  sp = make_space<KIND>(p);
  // routing tables in shared memory: the per-stage lookups then cost no
  // global round trip (they are visible to the consumers through the first
  // full-barrier completion)
  VExpert* ve_tab = reinterpret_cast<VExpert*>(tables);
  int* slot_tab = reinterpret_cast<int*>(tables + (size_t)p.ve_max * sizeof(VExpert));
  if (KindTraits<KIND>::kDynamicSpace) {
    const int nve = *reinterpret_cast<volatile int*>(p.nve);
    for (int i = lane; i < nve; i += 32) ve_tab[i] = p.ve[i];
    for (int i = lane; i < p.ld_slots; i += 32) slot_tab[i] = p.slots_sorted[i];
    __syncwarp();
  }

  // lane 0 keeps one cursor grab in flight; its result is read one piece later
  int grabbed = 0;
  if (lane == 0) grabbed = atomicAdd(&ctl->cursor, 1);
  int piece = __shfl_sync(0xffffffffu, grabbed, 0);
  if (lane == 0) grabbed = atomicAdd(&ctl->cursor, 1);
  while (true) {
    if (piece >= sp.total) break;
    const int per_v = p.RB * sp.ppr;
    const int pr = (piece % per_v) % sp.ppr;
    const int c_first = (int)((long long)pr * p.C / sp.ppr);
    const int c_last = (int)((long long)(pr + 1) * p.C / sp.ppr);
    for (int c = c_first; c < c_last; ++c) {
      // before the dependency resolves, fill at most one ring of weight-only stages
      if (!waited && prefetched == p.nstages) {
        pdl_wait();
        pdl_trigger();
        waited = true;
        for (int s = 0; s < prefetched; ++s) {
          uint8_t* sb = stage_base + (size_t)s * p.stage_bytes;
          const Hdr& hs = *reinterpret_cast<const Hdr*>(sb);
          issue_act<KIND>(p, hs, sb + p.act_off, &full[s], lane, slot_tab);
        }
      }
      if (!mbar_wait_bounded(&empty[stage], ephase, p.err, ERR_WAIT_EMPTY)) return;
      uint8_t* sb = stage_base + (size_t)stage * p.stage_bytes;
      Hdr h;
      fill_header<KIND>(p, sp, piece, c, c_first, c_last, h, ve_tab);
      if (lane == 0) {
        *reinterpret_cast<Hdr*>(sb) = h;
        mbar_arrive_expect_tx(&full[stage], KindTraits<KIND>::kTileBytes + h.act_bytes);
        bulk_g2s(sb + kHdrBytes, weight_src<KIND>(p, h), KindTraits<KIND>::kTileBytes, &full[stage]);
      }
      __syncwarp();
      if (waited)
        issue_act<KIND>(p, h, sb + p.act_off, &full[stage], lane, slot_tab);
      else
        ++prefetched;
      if (++stage == p.nstages) {
        stage = 0;
        ephase ^= 1;
      }
    }
    piece = __shfl_sync(0xffffffffu, grabbed, 0);
    if (lane == 0 && piece < sp.total) grabbed = atomicAdd(&ctl->cursor, 1);
  }
  if (!waited) {
    pdl_wait();
    pdl_trigger();
    for (int s = 0; s < prefetched; ++s) {
      uint8_t* sb = stage_base + (size_t)s * p.stage_bytes;
      const Hdr& hs = *reinterpret_cast<const Hdr*>(sb);
      issue_act<KIND>(p, hs, sb + p.act_off, &full[s], lane, slot_tab);
    }
  }
  // end marker
  if (!mbar_wait_bounded(&empty[stage], ephase, p.err, ERR_WAIT_EMPTY)) return;
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
                                            const uint8_t* act, float (&acc)[NT][4], int warp,
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
        const int tok = 8 * t + g;
        uint4 bv = make_uint4(0, 0, 0, 0);
        if (tok < h.ntok) bv = lds128(act + tok * p.act_stride + (32 * b + 8 * tig) * 2);
        mma_bf16(acc[t], A0, bv.x, bv.y);
        mma_bf16(acc[t], A1, bv.z, bv.w);
      }
    }
  }
}

// MXFP4 weights x f16-MX activation records: EGU, EDN
template <int NT>
__device__ __forceinline__ void mma_mx(const Params& p, const Hdr& h, const uint8_t* tile,
                                       const uint8_t* act, float (&acc)[NT][4], int warp, int lane) {
  const int g = lane >> 2, tig = lane & 3;
  const uint4 sc = lds128(tile + kMxCodeBytes + (warp * 8 + g) * 16);
  const uint32_t scw[4] = {sc.x, sc.y, sc.z, sc.w};
#pragma unroll
  for (int bp = 0; bp < 4; ++bp) {
    if (2 * bp < h.nb) {
      const uint4 cw = lds128(tile + (warp * 4 + bp) * 512 + lane * 16);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int b = 2 * bp + half;
        if (b < h.nb) {
          uint32_t A0[4], A1[4];
          e2m1x8_to_f16x2x4(half ? cw.z : cw.x, A0);
          e2m1x8_to_f16x2x4(half ? cw.w : cw.y, A1);
          // row g scales are bytes 0..7 (words 0,1), row g+8 bytes 8..15 (words 2,3)
          const float sw0 = e8m0_to_float((scw[b >> 2] >> (8 * (b & 3))) & 0xFF);
          const float sw1 = e8m0_to_float((scw[2 + (b >> 2)] >> (8 * (b & 3))) & 0xFF);
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const int tok = 8 * t + g;
            uint4 bv = make_uint4(0, 0, 0, 0);
            if (tok < h.ntok) bv = lds128(act + tok * p.act_stride + b * 64 + tig * 16);
            const int c0 = 8 * t + 2 * tig;
            float sa0 = 0.f, sa1 = 0.f;
            if (c0 < h.ntok)
              sa0 = *reinterpret_cast<const float*>(act + c0 * p.act_stride + 512 + 4 * b);
            if (c0 + 1 < h.ntok)
              sa1 = *reinterpret_cast<const float*>(act + (c0 + 1) * p.act_stride + 512 + 4 * b);
            float tmp[4] = {0.f, 0.f, 0.f, 0.f};
            mma_f16(tmp, A0, bv.x, bv.y);
            mma_f16(tmp, A1, bv.z, bv.w);
            acc[t][0] = fmaf(sw0 * sa0, tmp[0], acc[t][0]);
            acc[t][1] = fmaf(sw0 * sa1, tmp[1], acc[t][1]);
            acc[t][2] = fmaf(sw1 * sa0, tmp[2], acc[t][2]);
            acc[t][3] = fmaf(sw1 * sa1, tmp[3], acc[t][3]);
          }
        }
      }
    }
  }
}

// TAIL: build the activation tile (combine of y, or h_s) as bf16 hi + lo in a
// transform buffer, then bf16 MMAs against W_out / W_sd.
template <int NT>
__device__ __forceinline__ void mma_tail(const Params& p, const Hdr& h, const uint8_t* tile,
                                         const uint8_t* act, uint8_t* tbuf, float (&acc)[NT][4],
                                         int warp, int lane, int tid) {
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
        const int tok = 8 * t + g;
        uint4 bh = make_uint4(0, 0, 0, 0), bl = make_uint4(0, 0, 0, 0);
        if (tok < h.ntok) {
          bh = lds128(tbuf + tok * kTStride + (32 * b + 8 * tig) * 2);
          bl = lds128(tbuf + tok * kTStride + 128 + (32 * b + 8 * tig) * 2);
        }
        mma_bf16(acc[t], A0, bh.x, bh.y);
        mma_bf16(acc[t], A1, bh.z, bh.w);
        mma_bf16(acc[t], A0, bl.x, bl.y);
        mma_bf16(acc[t], A1, bl.z, bl.w);
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

__device__ void route_tokens(const Params& p, uint8_t* scratch, int tid, int warp, int lane);

template <int KIND, int NT>
__device__ void epilogue(const Params& p, const Hdr& h, float (&acc)[NT][4], uint8_t* scratch,
                         int* sm_flag, const int* slot_tab, int tid, int warp, int lane) {
  const int g = lane >> 2, tig = lane & 3;
  if (KIND == KIND_RL) {
    if (h.rb < p.RB_router) {
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int row = 16 * warp + ((q & 2) ? g + 8 : g);
          const int col = 8 * t + 2 * tig + (q & 1);
          const int e = h.rb * kRowsPerBlock + row;
          if (e < p.E && col < p.B) p.logits[(long long)col * p.E + e] = acc[t][q];
        }
      __threadfence();
      named_sync(1, kConsumerThreads);
      if (tid == 0) *sm_flag = (atomicAdd(p.router_done, 1) == p.RB_router - 1);
      named_sync(1, kConsumerThreads);
      if (*sm_flag) {
        __threadfence();
        route_tokens(p, scratch, tid, warp, lane);
        if (tid == 0) *p.router_done = 0;
      }
      named_sync(1, kConsumerThreads);
    } else {
      const int cz = (p.L + kMxChunkK - 1) / kMxChunkK;
      const int l0 = (h.rb - p.RB_router) * kRowsPerBlock + 16 * warp + g;
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
          rec[t][c] = p.z_mx + ((long long)(col < p.B ? col : 0) * cz + (l0 >> 8)) * kActRecBytes;
        }
      store_f16mx<NT, 2>(val, warp, lane, 2, p.B, reinterpret_cast<float*>(scratch), rec, idx,
                         l0 < p.L, l0 + 8 < p.L);
    }
  } else if (KIND == KIND_SGU) {
    const int i = 64 * h.rb + 8 * warp + g;
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int col = 8 * t + 2 * tig + c;
        if (col < p.B && i < p.Is)
          p.h_s[((long long)(i >> 6) * p.B + col) * 64 + (i & 63)] = silu(acc[t][c]) * acc[t][2 + c];
      }
  } else if (KIND == KIND_EGU) {
    const int i = 64 * h.rb + 8 * warp + g;
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
        rec[t][c] = p.h_mx + ((long long)(i >> 8) * p.ld_slots + pos) * kActRecBytes;
      }
    store_f16mx<NT, 1>(val, warp, lane, 4, h.ntok, reinterpret_cast<float*>(scratch), rec, idx,
                       i < p.I, false);
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

__device__ void route_tokens(const Params& p, uint8_t* scratch, int tid, int warp, int lane) {
  const int E = p.E, K = p.topk, B = p.B;
  int* cnt = reinterpret_cast<int*>(scratch);
  int* fill = cnt + E;
  int* off = fill + E;
  int* ids_s = off + E;
  for (int i = tid; i < E; i += kConsumerThreads) {
    cnt[i] = 0;
    fill[i] = 0;
  }
  named_sync(1, kConsumerThreads);
  for (int b = warp; b < B; b += kConsumerWarps) {
    int sel_id;
    float sel_w;
    warp_topk(p.logits + (long long)b * E, E, K, p.score_fn, p.bias, p.renorm, p.routed_scale, lane,
              sel_id, sel_w);
    if (lane < K) {
      p.ids[b * K + lane] = sel_id;
      p.wts[b * K + lane] = sel_w;
      ids_s[b * K + lane] = sel_id;
      atomicAdd(&cnt[sel_id], 1);
    }
  }
  named_sync(1, kConsumerThreads);
  if (warp == 0) {
    int running = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const int v = e < E ? cnt[e] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (e < E) off[e] = running + incl - v;
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  named_sync(1, kConsumerThreads);
  for (int s = tid; s < B * K; s += kConsumerThreads) {
    const int e = ids_s[s];
    const int pos = off[e] + atomicAdd(&fill[e], 1);
    p.slots_sorted[pos] = s;
  }
  if (warp == 0) {
    int running = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const int c = e < E ? cnt[e] : 0;
      const int tg = p.tg > 0 ? p.tg : 1;
      const int ng = (c + tg - 1) / tg;
      int incl = ng;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      int vs = running + incl - ng;
      for (int gi = 0; gi < ng; ++gi) {
        VExpert ve;
        ve.expert = e;
        ve.start = off[e] + gi * tg;
        ve.count = min(tg, c - gi * tg);
        ve.pad = 0;
        if (vs + gi < p.ve_max) p.ve[vs + gi] = ve;
      }
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) *p.nve = running < p.ve_max ? running : p.ve_max;
  }
  named_sync(1, kConsumerThreads);
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

// Sum the row block's pieces in piece order (the same order whatever CTA ran
// them, so the result is deterministic).
template <int NT>
__device__ __forceinline__ void sum_partials(const Params& p, const Hdr& h, float (&acc)[NT][4],
                                             int warp, int lane) {
  const int g = lane >> 2, tig = lane & 3;
  const long long first = (long long)(h.v * p.RB + h.rb) * h.ppr;
  const long long stride = NT * 8 * kRowsPerBlock;
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int col = 8 * t + 2 * tig + (q & 1);
      const int row = 16 * warp + ((q & 2) ? g + 8 : g);
      float sum = 0.f;
      if (col < h.ntok) {
        const float* src = p.partials + first * stride + col * kRowsPerBlock + row;
        int pr = 0;
        for (; pr + 8 <= h.ppr; pr += 8) {
          float v[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) v[u] = __ldcg(src + (pr + u) * stride);
#pragma unroll
          for (int u = 0; u < 8; ++u) sum += v[u];
        }
        for (; pr < h.ppr; ++pr) sum += __ldcg(src + pr * stride);
      }
      acc[t][q] = sum;
    }
}

template <int KIND, int NT>
__device__ void finalize(const Params& p, const Hdr& h, float (&acc)[NT][4], uint8_t* scratch,
                         int* sm_flag, const int* slot_tab, int tid, int warp, int lane) {
  sum_partials<NT>(p, h, acc, warp, lane);
  if (tid == 0) p.counters[h.v * p.RB + h.rb] = 0;  // ready for the next launch
  epilogue<KIND, NT>(p, h, acc, scratch, sm_flag, slot_tab, tid, warp, lane);
}

template <int KIND, int NT>
__device__ void consumer(const Params& p, uint8_t* stage_base, uint64_t* full, uint64_t* empty,
                         uint8_t* scratch, int* sm_flag, const int* slot_tab, int warp, int lane) {
  const int tid = warp * 32 + lane;
  int stage = 0;
  uint32_t phase = 0;
  int nbuf = 0;
  float acc[NT][4];
  zero_acc(acc);
  // A piece whose ticket (finalize counter) is still in flight: thread 0
  // issues the atomic after the piece's partials are written and reads its
  // result only at the next piece end, so nobody waits on the round trip.
  bool pend = false;
  Hdr pend_h;
  int ticket = 0;
  int* tflag = sm_flag + 4;  // two alternating slots
  int tslot = 0;
  // activations, routing tables and partial sums of the previous kernel are
  // read only after the dependency has resolved; the next kernel may then be
  // scheduled (it cannot overtake this one's own predecessor)
  pdl_wait();
  pdl_trigger();
  while (true) {
    if (!mbar_wait_bounded(&full[stage], phase, p.err, ERR_WAIT_FULL)) break;
    uint8_t* sb = stage_base + (size_t)stage * p.stage_bytes;
    const Hdr h = *reinterpret_cast<const Hdr*>(sb);
    if (h.flags & HDR_END) break;
    if (h.flags & HDR_FIRST) zero_acc(acc);
    const uint8_t* tile = sb + kHdrBytes;
    const uint8_t* act = sb + p.act_off;
    if (KIND == KIND_RL || KIND == KIND_SGU) {
      mma_dense_x<NT>(p, h, tile, act, acc, warp, lane);
    } else if (KIND == KIND_EGU || KIND == KIND_EDN) {
      mma_mx<NT>(p, h, tile, act, acc, warp, lane);
    } else {
      uint8_t* tbuf = scratch + 4096 + (nbuf & 1) * (16 * 320);
      ++nbuf;
      mma_tail<NT>(p, h, tile, act, tbuf, acc, warp, lane, tid);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
    if (++stage == p.nstages) {
      stage = 0;
      phase ^= 1;
    }
    if (!(h.flags & HDR_LAST)) continue;

    if (h.ppr == 1) {
      epilogue<KIND, NT>(p, h, acc, scratch, sm_flag, slot_tab, tid, warp, lane);
      continue;
    }
    write_partial<NT>(p, h.piece, h.ntok, acc, warp, lane);
    if (tid == 0 && pend) tflag[tslot] = (ticket == pend_h.ppr - 1);
    named_sync(1, kConsumerThreads);  // every warp's partials precede thread 0's release
    const bool fin = pend && tflag[tslot] != 0;
    if (tid == 0) ticket = atom_add_acqrel(p.counters + h.v * p.RB + h.rb, 1);
    const Hdr prev = pend_h;
    pend_h = h;
    pend = true;
    tslot ^= 1;
    if (fin) finalize<KIND, NT>(p, prev, acc, scratch, sm_flag, slot_tab, tid, warp, lane);
  }
  if (pend) {
    if (tid == 0) tflag[tslot] = (ticket == pend_h.ppr - 1);
    named_sync(1, kConsumerThreads);
    if (tflag[tslot] != 0) finalize<KIND, NT>(p, pend_h, acc, scratch, sm_flag, slot_tab, tid, warp, lane);
  }
}

// ---------------------------------------------------------------------------

template <int KIND, int NT>
__global__ void __launch_bounds__(kThreads, (NT <= 4 ? 2 : 1))
    moe_kernel(const __grid_constant__ Params p) {
  // shared memory: [0,128) full barriers, [128,256) empty barriers,
  // [256,512) flags, [scratch_off, ...) scratch, [table_off, ...) routing
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
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nstages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == kConsumerWarps) {
    producer<KIND>(p, ctl, stages, tables, full, empty, lane);
  } else {
    consumer<KIND, NT>(p, stages, full, empty, scratch, sm_flag, slot_tab, warp, lane);
  }
  __syncthreads();
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
// host side

template <int KIND, int NT>
static int launch_one(const Params& p, int grid, size_t smem, cudaStream_t s, bool pdl) {
  auto kfn = moe_kernel<KIND, NT>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return (int)cudaLaunchKernelEx(&cfg, kfn, p);
}

template <int KIND>
static int launch_nt(int nt, const Params& p, int grid, size_t smem, cudaStream_t s, bool pdl) {
  constexpr bool kDense = (KIND == KIND_RL || KIND == KIND_SGU);
  switch (nt) {
    case 1: return launch_one<KIND, 1>(p, grid, smem, s, pdl);
    case 2: return launch_one<KIND, 2>(p, grid, smem, s, pdl);
    case 4:
      if constexpr (KIND != KIND_TAIL) return launch_one<KIND, 4>(p, grid, smem, s, pdl);
      break;
    case 8:
      if constexpr (kDense) return launch_one<KIND, 8>(p, grid, smem, s, pdl);
      break;
    case 16:
      if constexpr (kDense) return launch_one<KIND, 16>(p, grid, smem, s, pdl);
      break;
    default: break;
  }
  return (int)cudaErrorInvalidValue;
}

template <int KIND, int NT>
static int set_attr(size_t bytes) {
  return (int)cudaFuncSetAttribute(moe_kernel<KIND, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)bytes);
}

int set_smem_limits(size_t bytes) {
  int e = 0;
  e |= set_attr<KIND_RL, 1>(bytes) | set_attr<KIND_RL, 2>(bytes) | set_attr<KIND_RL, 4>(bytes) |
       set_attr<KIND_RL, 8>(bytes) | set_attr<KIND_RL, 16>(bytes);
  e |= set_attr<KIND_SGU, 1>(bytes) | set_attr<KIND_SGU, 2>(bytes) | set_attr<KIND_SGU, 4>(bytes) |
       set_attr<KIND_SGU, 8>(bytes) | set_attr<KIND_SGU, 16>(bytes);
  e |= set_attr<KIND_EGU, 1>(bytes) | set_attr<KIND_EGU, 2>(bytes) | set_attr<KIND_EGU, 4>(bytes);
  e |= set_attr<KIND_EDN, 1>(bytes) | set_attr<KIND_EDN, 2>(bytes) | set_attr<KIND_EDN, 4>(bytes);
  e |= set_attr<KIND_TAIL, 1>(bytes) | set_attr<KIND_TAIL, 2>(bytes);
  return e;
}

int max_smem_optin() {
  int dev = 0, v = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  return v;
}

int launch_kind(int kind, int nt, const Params& p, int grid, size_t smem, void* stream, bool pdl) {
  cudaStream_t s = (cudaStream_t)stream;
  switch (kind) {
    case KIND_RL: return launch_nt<KIND_RL>(nt, p, grid, smem, s, pdl);
    case KIND_SGU: return launch_nt<KIND_SGU>(nt, p, grid, smem, s, pdl);
    case KIND_EGU: return launch_nt<KIND_EGU>(nt, p, grid, smem, s, pdl);
    case KIND_EDN: return launch_nt<KIND_EDN>(nt, p, grid, smem, s, pdl);
    case KIND_TAIL: return launch_nt<KIND_TAIL>(nt, p, grid, smem, s, pdl);
    default: return (int)cudaErrorInvalidValue;
  }
}

}  // namespace moe
