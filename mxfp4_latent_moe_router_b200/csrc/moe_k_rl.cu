// moe_k_rl.cu -- instantiations of the router logits + latent projection (+ top-k) kernel.
#include "moe_engine.cuh"

namespace moe {

int launch_rl(int nt, const Params& p, int grid, size_t smem, void* stream, bool pdl) {
  return launch_kind_nt<KIND_RL>(nt, p, grid, smem, (cudaStream_t)stream, pdl);
}

int set_attr_rl(size_t bytes) { return set_attr_kind<KIND_RL>(bytes); }

}  // namespace moe
