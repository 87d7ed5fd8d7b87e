// topk.cuh -- top-k expert selection for one token.
//
// Scores: softmax ranks experts by logit (the same order as by probability);
// sigmoid ranks by sigmoid(logit) + bias.  Ties go to the lower expert index.
// Combine weights come from the unbiased score, renormalised over the chosen
// experts when requested, times routed_scale.
//
// The selection is split so that several warps can share one token: each warp
// takes the top-k of a slice of the experts (warp_topk_slice), and one warp
// merges the candidates of all slices (warp_topk_merge).  With one slice the
// merge is skipped (warp_topk).
//
// A selection round is two warp reductions (redux.sync): the largest key, as
// an order-preserving unsigned integer, and the lowest expert index among the
// lanes that hold it -- instead of a five-level shuffle tree carrying key,
// index and logit.  The winner's logit then comes from its lane with one
// shuffle.
#pragma once
#include <cstdint>

namespace moe {

// Scores use the hardware exp2 and fast divide (a few ulp, far below the
// 1e-5 relative accuracy the combine weights need).
__device__ __forceinline__ float fast_sigmoid(float l) { return __fdividef(1.0f, 1.0f + __expf(-l)); }

// float -> unsigned with the same order (NaN lowest, never preferred)
__device__ __forceinline__ uint32_t key_order(float f) {
  const uint32_t b = __float_as_uint(f);
  const uint32_t o = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return f == f ? o : 0u;
}
__device__ __forceinline__ float key_value(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

struct TopkCand {
  float key, logit;
  int id, pad;
};

constexpr uint32_t kNoExpert = 0xffffffffu;

// Top-K of experts [e0, e1) of one token (K <= 16, e1 - e0 <= 32 * EPL).
// On return lane r < K holds the r-th best candidate (key-descending), and
// every lane holds the slice's logit maximum and sum of exp(logit - max)
// (softmax scoring only; they normalise the probabilities).  The logits are
// in global memory, read past L1 (other CTAs wrote them), or with kSmem in
// this CTA's shared memory.
template <int EPL, bool kSmem = false>
__device__ __forceinline__ void warp_topk_slice(const float* logits, const float* bias, int e0, int e1,
                                             int K, int score_fn, int lane, TopkCand& out,
                                             float& smax, float& ssum) {
  float lg[EPL], bs[EPL];
  uint32_t ok[EPL];
  // all loads first (one round trip), arithmetic after
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = e0 + lane + 32 * j;
    const bool in = e < e1;
    lg[j] = in ? (kSmem ? logits[e] : __ldcg(logits + e)) : 0.f;
    bs[j] = (in && bias) ? bias[e] : 0.f;  // (global or shared memory)
  }
  float mx = -INFINITY;
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = e0 + lane + 32 * j;
    ok[j] = 0u;  // below every real key
    if (e < e1) {
      if (score_fn == 1) {
        ok[j] = key_order(fast_sigmoid(lg[j]) + bs[j]);
      } else {
        ok[j] = key_order(lg[j]);
        mx = fmaxf(mx, lg[j]);
      }
    }
  }
  smax = -INFINITY;
  ssum = 0.f;
  if (score_fn == 0) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (e0 + lane + 32 * j < e1) sum += __expf(lg[j] - mx);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    smax = mx;
    ssum = sum;
  }
  out.key = -INFINITY;
  out.id = 0x7fffffff;
  out.logit = 0.f;
  out.pad = 0;
  for (int r = 0; r < K; ++r) {
    // local best: largest key, then lowest index (lower j = lower index)
    uint32_t bo = 0u, bj = 0u;
#pragma unroll
    for (int j = EPL - 1; j >= 0; --j)
      if (ok[j] >= bo) {
        bo = ok[j];
        bj = (uint32_t)j;
      }
    const uint32_t bi = bo ? (uint32_t)(e0 + lane) + 32u * bj : kNoExpert;
    const uint32_t wo = __reduce_max_sync(0xffffffffu, bo);
    const uint32_t wi = __reduce_min_sync(0xffffffffu, bo == wo ? bi : kNoExpert);
    if (wi == kNoExpert) break;  // fewer than K experts in the slice
    const int wl = (int)((wi - (uint32_t)e0) & 31u), wj = (int)((wi - (uint32_t)e0) >> 5);
    float my = 0.f;
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (j == wj) my = lg[j];
    const float wlog = __shfl_sync(0xffffffffu, my, wl);
    if (lane == wl) {
#pragma unroll
      for (int j = 0; j < EPL; ++j)
        if (j == wj) ok[j] = 0u;
    }
    if (lane == r) {
      out.key = key_value(wo);
      out.id = (int)wi;
      out.logit = wlog;
    }
  }
}

// Pick an EPL bound for a slice of n experts.
template <bool kSmem = false>
__device__ __forceinline__ void warp_topk_slice_any(const float* logits, const float* bias, int e0,
                                                    int e1, int K, int score_fn, int lane,
                                                    TopkCand& out, float& smax, float& ssum) {
  const int n = e1 - e0;
  if (n <= 32)
    warp_topk_slice<1, kSmem>(logits, bias, e0, e1, K, score_fn, lane, out, smax, ssum);
  else if (n <= 64)
    warp_topk_slice<2, kSmem>(logits, bias, e0, e1, K, score_fn, lane, out, smax, ssum);
  else if (n <= 128)
    warp_topk_slice<4, kSmem>(logits, bias, e0, e1, K, score_fn, lane, out, smax, ssum);
  else if (n <= 256)
    warp_topk_slice<8, kSmem>(logits, bias, e0, e1, K, score_fn, lane, out, smax, ssum);
  else if (n <= 384)
    warp_topk_slice<12, kSmem>(logits, bias, e0, e1, K, score_fn, lane, out, smax, ssum);
  else
    warp_topk_slice<16, kSmem>(logits, bias, e0, e1, K, score_fn, lane, out, smax, ssum);  // n <= 512
}

// K rounds over two candidates per lane (candidate slots lane and lane + 32):
// lane r < K receives the r-th expert and its combine weight.
__device__ __forceinline__ void topk_pick(uint32_t o0, uint32_t i0, float l0, uint32_t o1, uint32_t i1,
                                          float l1, int K, int E, int score_fn, int renorm,
                                          float routed_scale, float mx, float den, int lane,
                                          int& sel_id, float& sel_w) {
  sel_id = 0;
  float sel_src = 0.f, tot = 0.f;
  for (int r = 0; r < K; ++r) {
    // local best of the two slots: larger key, then lower index
    const bool second = o1 > o0 || (o1 == o0 && i1 < i0);
    const uint32_t bo = second ? o1 : o0, bi = second ? i1 : i0;
    const uint32_t wo = __reduce_max_sync(0xffffffffu, bo);
    const uint32_t wi = __reduce_min_sync(0xffffffffu, bo == wo ? bi : kNoExpert);
    // the lane that holds it: exactly one slot matches (indices are distinct)
    const bool mine0 = i0 == wi, mine1 = i1 == wi;
    const unsigned who = __ballot_sync(0xffffffffu, mine0 || mine1);
    const int wl = who ? __ffs(who) - 1 : 0;
    const float wlog = __shfl_sync(0xffffffffu, mine1 ? l1 : l0, wl);
    if (mine0) {
      o0 = 0u;
      i0 = kNoExpert;
    }
    if (mine1) {
      o1 = 0u;
      i1 = kNoExpert;
    }
    const float sv = (score_fn == 0) ? __fdividef(__expf(wlog - mx), den) : fast_sigmoid(wlog);
    tot += sv;
    if (lane == r) {
      sel_id = (wi < (uint32_t)E) ? (int)wi : 0;  // out of range only after NaN logits
      sel_src = sv;
    }
  }
  sel_w = (renorm ? __fdividef(sel_src, tot) : sel_src) * routed_scale;
}

// Final choice from P slices' candidates (cand[q * K + r], P * K <= 64) and
// their softmax partials part[q] = {max, sum}.
__device__ __forceinline__ void warp_topk_merge(const TopkCand* cand, const float2* part, int P,
                                                int K, int E, int score_fn, int renorm,
                                                float routed_scale, int lane, int& sel_id,
                                                float& sel_w) {
  const int n = P * K;
  uint32_t o0 = 0u, o1 = 0u, i0 = kNoExpert, i1 = kNoExpert;
  float l0 = 0.f, l1 = 0.f;
  if (lane < n && cand[lane].id != 0x7fffffff) {
    o0 = key_order(cand[lane].key);
    i0 = (uint32_t)cand[lane].id;
    l0 = cand[lane].logit;
  }
  if (lane + 32 < n && cand[lane + 32].id != 0x7fffffff) {
    o1 = key_order(cand[lane + 32].key);
    i1 = (uint32_t)cand[lane + 32].id;
    l1 = cand[lane + 32].logit;
  }
  float mx = -INFINITY, den = 1.f;
  if (score_fn == 0) {
    for (int q = 0; q < P; ++q) mx = fmaxf(mx, part[q].x);
    float s = 0.f;
    for (int q = 0; q < P; ++q) s += part[q].y * __expf(part[q].x - mx);
    den = s;
  }
  topk_pick(o0, i0, l0, o1, i1, l1, K, E, score_fn, renorm, routed_scale, mx, den, lane, sel_id,
            sel_w);
}

// Whole selection for one token on one warp: one slice of up to 512 experts,
// or two slices whose candidates are merged in registers (E <= 1024).
template <bool kSmem = false>
__device__ __forceinline__ void warp_topk(const float* logits, int E, int K, int score_fn,
                                          const float* bias, int renorm, float routed_scale,
                                          int lane, int& sel_id, float& sel_w) {
  const int split = E > 512 ? (E + 1) / 2 : E;
  TopkCand c0, c1;
  float m0, s0, m1 = -INFINITY, s1 = 0.f;
  warp_topk_slice_any<kSmem>(logits, bias, 0, split, K, score_fn, lane, c0, m0, s0);
  c1.key = -INFINITY;
  c1.id = 0x7fffffff;
  c1.logit = 0.f;
  if (split < E) warp_topk_slice_any<kSmem>(logits, bias, split, E, K, score_fn, lane, c1, m1, s1);
  const float mx = fmaxf(m0, m1);
  float den = 1.f;
  if (score_fn == 0) den = s0 * __expf(m0 - mx) + (split < E ? s1 * __expf(m1 - mx) : 0.f);
  const bool v0 = lane < K && c0.id != 0x7fffffff, v1 = lane < K && c1.id != 0x7fffffff;
  topk_pick(v0 ? key_order(c0.key) : 0u, v0 ? (uint32_t)c0.id : kNoExpert, c0.logit,
            v1 ? key_order(c1.key) : 0u, v1 ? (uint32_t)c1.id : kNoExpert, c1.logit, K, E,
            score_fn, renorm, routed_scale, mx, den, lane, sel_id, sel_w);
}

}  // namespace moe
