// moe_k_egu.cu -- instantiations of the routed experts gate/up, MXFP4 kernel.
#include "moe_engine.cuh"

namespace moe {

int launch_egu(int nt, const Params& p, int grid, size_t smem, void* stream, bool pdl) {
  return launch_kind_nt<KIND_EGU>(nt, p, grid, smem, (cudaStream_t)stream, pdl);
}

int set_attr_egu(size_t bytes) { return set_attr_kind<KIND_EGU>(bytes); }

}  // namespace moe
