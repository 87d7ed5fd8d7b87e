// moe_k_front.cu -- instantiations of the dense front kernel: router rows,
// latent projection and shared-expert gate/up over x, plus the routing CTA.
#include "moe_engine.cuh"

namespace moe {

int launch_front(int nt, const Params& p, int grid, size_t smem, void* stream, bool pdl) {
  return launch_kind_nt<KIND_FRONT>(nt, p, grid, smem, (cudaStream_t)stream, pdl);
}

int set_attr_front(size_t bytes) { return set_attr_kind<KIND_FRONT>(bytes); }

// Test of the timeout path.  One thread leaves the scheduling state as a
// forward cut short by an expired wait could leave it (a router row block
// counted, a split-K ticket taken, the piece cursor advanced, the routing
// flag raised), then runs the kernels' own bounded flag wait on `never`,
// which nothing sets, with `limit` polls: the wait expires and sets the
// dependency-wait error bit.  No copy, barrier or other thread is involved,
// so the kernel always ends.
__global__ void expire_wait_kernel(int* never, int* err, int* router_done, int* ticket,
                                   Ctl* ctl, int* route_ready, uint32_t limit) {
  if (threadIdx.x != 0) return;
  atomicAdd(router_done, 1);
  atomicAdd(ticket, 1);
  atomicAdd(&ctl->cursor, 3);
  atomicExch(route_ready, 1);
  wait_flag(never, err, ERR_WAIT_DEP, 0, limit);
}

int launch_expire_wait(int* never, int* err, int* router_done, int* ticket, Ctl* ctl,
                       int* route_ready, unsigned limit, void* stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(32);
  cfg.stream = (cudaStream_t)stream;
  return (int)cudaLaunchKernelEx(&cfg, expire_wait_kernel, never, err, router_done, ticket, ctl,
                                 route_ready, (uint32_t)limit);
}

}  // namespace moe
