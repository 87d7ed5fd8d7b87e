// topk.cuh -- top-k selection of one token's experts by one warp.
//
// Scores: softmax ranks experts by logit (the same order as by probability);
// sigmoid ranks by sigmoid(logit) + bias.  Ties go to the lower expert index.
// Combine weights come from the unbiased score, renormalised over the chosen
// experts when requested, times routed_scale.
#pragma once
#include <cstdint>

namespace moe {

__device__ __forceinline__ bool topk_better(float ka, int ia, float kb, int ib) {
  return ka > kb || (ka == kb && ia < ib);
}

// logits: this token's E logits (global memory written by an earlier kernel or
// by another CTA of this grid, read through L2).  After the call, lane r < K
// holds the r-th selected expert (key-descending) in sel_id and its combine
// weight in sel_w.  E <= 1024; all 32 lanes must call.
__device__ __forceinline__ void warp_topk(const float* logits, int E, int K, int score_fn,
                                          const float* bias, int renorm, float routed_scale,
                                          int lane, int& sel_id, float& sel_w) {
  constexpr int EPL = 32;
  float key[EPL], src[EPL];
  float mx = -INFINITY;
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = lane + 32 * j;
    key[j] = -INFINITY;
    src[j] = 0.f;
    if (e < E) {
      const float l = __ldcg(logits + e);
      if (score_fn == 1) {
        const float s = 1.0f / (1.0f + expf(-l));
        src[j] = s;
        key[j] = s + (bias ? bias[e] : 0.f);
      } else {
        src[j] = l;
        key[j] = l;
        mx = fmaxf(mx, l);
      }
    }
  }
  float den = 1.f;
  if (score_fn == 0) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (lane + 32 * j < E) sum += expf(src[j] - mx);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    den = sum;
  }
  sel_id = 0;
  float sel_src = 0.f, tot = 0.f;
  for (int r = 0; r < K; ++r) {
    float bk = -INFINITY, bs = 0.f;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = lane + 32 * j;
      if (e < E && topk_better(key[j], e, bk, bi)) {
        bk = key[j];
        bi = e;
        bs = src[j];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      const float os = __shfl_xor_sync(0xffffffffu, bs, o);
      if (topk_better(ok, oi, bk, bi)) {
        bk = ok;
        bi = oi;
        bs = os;
      }
    }
    if (bi < 0 || bi >= E) bi = 0;  // only reachable with NaN logits; keeps indices in range
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (lane + 32 * j == bi) key[j] = -INFINITY;
    const float sv = (score_fn == 0) ? expf(bs - mx) / den : bs;
    tot += sv;
    if (lane == r) {
      sel_id = bi;
      sel_src = sv;
    }
  }
  sel_w = (renorm ? sel_src / tot : sel_src) * routed_scale;
}

}  // namespace moe
