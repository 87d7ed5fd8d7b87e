// moe_static.cu -- router scores + top-k that allocate nothing.
//
// For callers that cannot allocate device memory themselves or through this
// library: code running inside an allocation-free region (a memory budget
// that is fixed up front, a custom allocator that must see every byte, a
// host thread that may not touch the CUDA allocator).  The caller passes the
// inputs and outputs; the only scratch is the file-scope array below, which
// every GPU that loads this library holds until the process exits.
//
// It computes what the routing part of moe_forward computes (logits = x . W_r,
// then warp_topk), but reads the canonical [H][E] router weight directly, so
// it needs no plan.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/moe.h"
#include "topk.cuh"

namespace {

constexpr int kStaticMaxTokens = 128;
constexpr int kStaticMaxExperts = 1024;
constexpr int kStaticMaxDevices = 64;

// Router logits of the current call: [tokens][experts] fp32, 512 KB.
static __device__ __align__(256) float g_static_logits[kStaticMaxTokens * kStaticMaxExperts];

// In host code g_static_logits names a host-side stand-in, not device memory:
// the device address is looked up once per device, with that device current.
float* g_scratch_addr[kStaticMaxDevices] = {};
std::mutex g_scratch_mu;

moe_status scratch_for(int dev, float** out) {
  if (dev < 0 || dev >= kStaticMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_logits);
    if (e != cudaSuccess || !ptr) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    g_scratch_addr[dev] = static_cast<float*>(ptr);
  }
  *out = g_scratch_addr[dev];
  return MOE_OK;
}

__device__ __forceinline__ float bf16f(uint16_t v) { return __uint_as_float((uint32_t)v << 16); }

// logits[b][e] = sum_h x[b][h] * W[h][e]: 64 expert columns per CTA, four row
// groups of 64 threads, tokens in groups of 8; fp32 accumulation.
__global__ void __launch_bounds__(256) static_router_logits(const uint16_t* __restrict__ x,
                                                            const uint16_t* __restrict__ w, int B,
                                                            int H, int E, float* logits) {
  __shared__ float red[4][8][64];
  const int c = threadIdx.x & 63, rg = threadIdx.x >> 6;
  const int col = blockIdx.x * 64 + c;
  for (int b0 = 0; b0 < B; b0 += 8) {
    float acc[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[t] = 0.f;
    if (col < E) {
      for (int h = rg; h < H; h += 4) {
        const float wv = bf16f(w[(long long)h * E + col]);
#pragma unroll
        for (int t = 0; t < 8; ++t)
          if (b0 + t < B) acc[t] = fmaf(bf16f(x[(long long)(b0 + t) * H + h]), wv, acc[t]);
      }
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) red[rg][t][c] = acc[t];
    __syncthreads();
    if (rg == 0 && col < E) {
#pragma unroll
      for (int t = 0; t < 8; ++t)
        if (b0 + t < B)
          logits[(b0 + t) * E + col] = ((red[0][t][c] + red[1][t][c]) + red[2][t][c]) + red[3][t][c];
    }
    __syncthreads();
  }
}

// one warp per token
__global__ void __launch_bounds__(256) static_topk(const float* logits, int B, int E, int K,
                                                   int score_fn, const float* bias, int renorm,
                                                   float routed_scale, int32_t* ids, float* wts) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x * 8 + warp;
  if (b >= B) return;
  int sel_id;
  float sel_w;
  moe::warp_topk(logits + (long long)b * E, E, K, score_fn, bias, renorm, routed_scale, lane, sel_id,
                 sel_w);
  if (lane < K) {
    ids[b * K + lane] = sel_id;
    wts[b * K + lane] = sel_w;
  }
}

}  // namespace

extern "C" moe_status moe_route_noalloc(const void* x, const void* router_w,
                                        const float* router_bias, int32_t num_tokens,
                                        int32_t hidden, int32_t num_experts, int32_t top_k,
                                        int32_t score_fn, int32_t renormalize, float routed_scale,
                                        int32_t* ids, float* weights, void* stream) {
  if (!x || !router_w || !ids || !weights) return MOE_ERR_INVALID_ARG;
  if (num_tokens < 1 || hidden < 1 || num_experts < 1 || top_k < 1 || top_k > num_experts)
    return MOE_ERR_INVALID_ARG;
  if (score_fn != MOE_SCORE_SOFTMAX && score_fn != MOE_SCORE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(router_w)) & 1)
    return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ids) | reinterpret_cast<uintptr_t>(weights) |
       reinterpret_cast<uintptr_t>(router_bias)) & 3)
    return MOE_ERR_INVALID_ARG;
  // sizes beyond the static scratch
  if (num_tokens > kStaticMaxTokens || num_experts > kStaticMaxExperts || top_k > 16)
    return MOE_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  float* logits = nullptr;
  moe_status st = scratch_for(dev, &logits);
  if (st != MOE_OK) return st;
  // each launch's own status (an error left behind by unrelated earlier work
  // on this thread is neither reported nor cleared here)
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(256);
  cfg.stream = static_cast<cudaStream_t>(stream);
  cfg.gridDim = dim3((num_experts + 63) / 64);
  cudaError_t e = cudaLaunchKernelEx(&cfg, static_router_logits, static_cast<const uint16_t*>(x),
                                     static_cast<const uint16_t*>(router_w), (int)num_tokens,
                                     (int)hidden, (int)num_experts, logits);
  if (e == cudaSuccess) {
    cfg.gridDim = dim3((num_tokens + 7) / 8);
    e = cudaLaunchKernelEx(&cfg, static_topk, static_cast<const float*>(logits), (int)num_tokens,
                           (int)num_experts, (int)top_k, (int)score_fn,
                           score_fn == MOE_SCORE_SIGMOID ? router_bias : nullptr, (int)renormalize,
                           routed_scale, ids, weights);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();  // this call's launch error: report it, leave no trace behind
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
