// moe_k_edn.cu -- instantiations of the routed experts down, MXFP4 kernel.
#include "moe_engine.cuh"

namespace moe {

int launch_edn(int nt, const Params& p, int grid, size_t smem, void* stream, bool pdl) {
  return launch_kind_nt<KIND_EDN>(nt, p, grid, smem, (cudaStream_t)stream, pdl);
}

int set_attr_edn(size_t bytes) { return set_attr_kind<KIND_EDN>(bytes); }

}  // namespace moe
