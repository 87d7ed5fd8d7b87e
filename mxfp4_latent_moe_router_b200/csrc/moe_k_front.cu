// moe_k_front.cu -- instantiations of the dense front kernel: router rows,
// latent projection and shared-expert gate/up over x, plus the routing CTA.
#include "moe_engine.cuh"

namespace moe {

int launch_front(int nt, const Params& p, int grid, size_t smem, void* stream, bool pdl) {
  return launch_kind_nt<KIND_FRONT>(nt, p, grid, smem, (cudaStream_t)stream, pdl);
}

int set_attr_front(size_t bytes) { return set_attr_kind<KIND_FRONT>(bytes); }

}  // namespace moe
