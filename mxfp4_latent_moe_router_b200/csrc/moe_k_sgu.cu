// moe_k_sgu.cu -- instantiations of the shared expert gate/up (side stream) kernel.
#include "moe_engine.cuh"

namespace moe {

int launch_sgu(int nt, const Params& p, int grid, size_t smem, void* stream, bool pdl) {
  return launch_kind_nt<KIND_SGU>(nt, p, grid, smem, (cudaStream_t)stream, pdl);
}

int set_attr_sgu(size_t bytes) { return set_attr_kind<KIND_SGU>(bytes); }

}  // namespace moe
