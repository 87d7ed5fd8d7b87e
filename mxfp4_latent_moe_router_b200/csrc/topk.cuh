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
#pragma once
#include <cstdint>

namespace moe {

// Scores use the hardware exp2 and fast divide (a few ulp, far below the
// 1e-5 relative accuracy the combine weights need): the selection runs once
// per forward as cold, straight-line code whose instruction footprint matters.
__device__ __forceinline__ float fast_sigmoid(float l) { return __fdividef(1.0f, 1.0f + __expf(-l)); }

__device__ __forceinline__ bool topk_better(float ka, int ia, float kb, int ib) {
  return ka > kb || (ka == kb && ia < ib);
}

// One selection round: the warp-wide best (key, index, logit) under topk_better.
__device__ __forceinline__ void warp_best(float& bk, int& bi, float& bl) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    const float ol = __shfl_xor_sync(0xffffffffu, bl, o);
    if (topk_better(ok, oi, bk, bi)) {
      bk = ok;
      bi = oi;
      bl = ol;
    }
  }
}

struct TopkCand {
  float key, logit;
  int id, pad;
};

// Top-K of experts [e0, e1) of one token (K <= 16, e1 - e0 <= 32 * EPL).
// On return lane r < K holds the r-th best candidate (key-descending), and
// every lane holds the slice's logit maximum and sum of exp(logit - max)
// (softmax scoring only; they normalise the probabilities).
template <int EPL>
__device__ __forceinline__ void warp_topk_slice(const float* logits, const float* bias, int e0, int e1,
                                             int K, int score_fn, int lane, TopkCand& out,
                                             float& smax, float& ssum) {
  float key[EPL], lg[EPL], bs[EPL];
  // all loads first (one round trip), arithmetic after
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = e0 + lane + 32 * j;
    const bool ok = e < e1;
    lg[j] = ok ? __ldcg(logits + e) : 0.f;
    bs[j] = (ok && bias) ? __ldg(bias + e) : 0.f;
  }
  float mx = -INFINITY;
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = e0 + lane + 32 * j;
    key[j] = -INFINITY;
    if (e < e1) {
      if (score_fn == 1) {
        key[j] = fast_sigmoid(lg[j]) + bs[j];
      } else {
        key[j] = lg[j];
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
    float bk = -INFINITY, bl = 0.f;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = e0 + lane + 32 * j;
      if (e < e1 && topk_better(key[j], e, bk, bi)) {
        bk = key[j];
        bi = e;
        bl = lg[j];
      }
    }
    warp_best(bk, bi, bl);
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (e0 + lane + 32 * j == bi) key[j] = -INFINITY;
    if (lane == r) {
      out.key = bk;
      out.id = bi;
      out.logit = bl;
    }
  }
}

// Pick an EPL bound for a slice of n experts.
__device__ __forceinline__ void warp_topk_slice_any(const float* logits, const float* bias, int e0,
                                                    int e1, int K, int score_fn, int lane,
                                                    TopkCand& out, float& smax, float& ssum) {
  const int n = e1 - e0;
  if (n <= 32)
    warp_topk_slice<1>(logits, bias, e0, e1, K, score_fn, lane, out, smax, ssum);
  else if (n <= 64)
    warp_topk_slice<2>(logits, bias, e0, e1, K, score_fn, lane, out, smax, ssum);
  else if (n <= 128)
    warp_topk_slice<4>(logits, bias, e0, e1, K, score_fn, lane, out, smax, ssum);
  else if (n <= 256)
    warp_topk_slice<8>(logits, bias, e0, e1, K, score_fn, lane, out, smax, ssum);
  else if (n <= 384)
    warp_topk_slice<12>(logits, bias, e0, e1, K, score_fn, lane, out, smax, ssum);
  else
    warp_topk_slice<16>(logits, bias, e0, e1, K, score_fn, lane, out, smax, ssum);  // n <= 512
}

// Final choice from P slices' candidates (cand[q * K + r], P * K <= 64) and
// their softmax partials part[q] = {max, sum}; lane r < K receives the r-th
// expert and its combine weight.
__device__ __forceinline__ void warp_topk_merge(const TopkCand* cand, const float2* part, int P,
                                                int K, int E, int score_fn, int renorm,
                                                float routed_scale, int lane, int& sel_id,
                                                float& sel_w) {
  const int n = P * K;
  float k0 = -INFINITY, k1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  int i0 = 0x7fffffff, i1 = 0x7fffffff;
  if (lane < n) {
    k0 = cand[lane].key;
    i0 = cand[lane].id;
    l0 = cand[lane].logit;
  }
  if (lane + 32 < n) {
    k1 = cand[lane + 32].key;
    i1 = cand[lane + 32].id;
    l1 = cand[lane + 32].logit;
  }
  float mx = -INFINITY, den = 1.f;
  if (score_fn == 0) {
    for (int q = 0; q < P; ++q) mx = fmaxf(mx, part[q].x);
    float s = 0.f;
    for (int q = 0; q < P; ++q) s += part[q].y * __expf(part[q].x - mx);
    den = s;
  }
  sel_id = 0;
  float sel_src = 0.f, tot = 0.f;
  for (int r = 0; r < K; ++r) {
    float bk = k0, bl = l0;
    int bi = i0;
    if (topk_better(k1, i1, bk, bi)) {
      bk = k1;
      bi = i1;
      bl = l1;
    }
    warp_best(bk, bi, bl);
    if (i0 == bi) {
      k0 = -INFINITY;
      i0 = 0x7fffffff;
    }
    if (i1 == bi) {
      k1 = -INFINITY;
      i1 = 0x7fffffff;
    }
    const float sv = (score_fn == 0) ? __fdividef(__expf(bl - mx), den) : fast_sigmoid(bl);
    tot += sv;
    if (lane == r) {
      sel_id = (bi >= 0 && bi < E) ? bi : 0;  // out of range only after NaN logits
      sel_src = sv;
    }
  }
  sel_w = (renorm ? __fdividef(sel_src, tot) : sel_src) * routed_scale;
}

// Whole selection for one token on one warp: one slice of up to 512 experts,
// or two slices whose candidates are merged in registers (E <= 1024).
__device__ __forceinline__ void warp_topk(const float* logits, int E, int K, int score_fn,
                                          const float* bias, int renorm, float routed_scale,
                                          int lane, int& sel_id, float& sel_w) {
  const int split = E > 512 ? (E + 1) / 2 : E;
  TopkCand c0, c1;
  float m0, s0, m1 = -INFINITY, s1 = 0.f;
  warp_topk_slice_any(logits, bias, 0, split, K, score_fn, lane, c0, m0, s0);
  c1.key = -INFINITY;
  c1.id = 0x7fffffff;
  c1.logit = 0.f;
  if (split < E) warp_topk_slice_any(logits, bias, split, E, K, score_fn, lane, c1, m1, s1);
  float mx = fmaxf(m0, m1), den = 1.f;
  if (score_fn == 0) den = s0 * __expf(m0 - mx) + (split < E ? s1 * __expf(m1 - mx) : 0.f);
  float k0 = lane < K ? c0.key : -INFINITY, k1 = lane < K ? c1.key : -INFINITY;
  int i0 = lane < K ? c0.id : 0x7fffffff, i1 = lane < K ? c1.id : 0x7fffffff;
  const float l0 = c0.logit, l1 = c1.logit;
  sel_id = 0;
  float sel_src = 0.f, tot = 0.f;
  for (int r = 0; r < K; ++r) {
    float bk = k0, bl = l0;
    int bi = i0;
    if (topk_better(k1, i1, bk, bi)) {
      bk = k1;
      bi = i1;
      bl = l1;
    }
    warp_best(bk, bi, bl);
    if (i0 == bi) {
      k0 = -INFINITY;
      i0 = 0x7fffffff;
    }
    if (i1 == bi) {
      k1 = -INFINITY;
      i1 = 0x7fffffff;
    }
    const float sv = (score_fn == 0) ? __fdividef(__expf(bl - mx), den) : fast_sigmoid(bl);
    tot += sv;
    if (lane == r) {
      sel_id = (bi >= 0 && bi < E) ? bi : 0;  // out of range only after NaN logits
      sel_src = sv;
    }
  }
  sel_w = (renorm ? __fdividef(sel_src, tot) : sel_src) * routed_scale;
}

}  // namespace moe
