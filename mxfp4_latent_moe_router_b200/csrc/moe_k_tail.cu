// moe_k_tail.cu -- instantiations of the weighted combine + latent tail + shared down kernel.
#include "moe_engine.cuh"

namespace moe {

int launch_tail(int nt, const Params& p, int grid, size_t smem, void* stream, bool pdl) {
  return launch_kind_nt<KIND_TAIL>(nt, p, grid, smem, (cudaStream_t)stream, pdl);
}

int set_attr_tail(size_t bytes) { return set_attr_kind<KIND_TAIL>(bytes); }

}  // namespace moe
