// moe_k_mega.cu -- instantiation of the single-launch path (B <= 8).
#include "moe_mega.cuh"

namespace moe {

int launch_mega(const MegaParams& mp, int grid, size_t smem, void* stream, bool pdl) {
  return launch_mega_nt<1>(mp, grid, smem, (cudaStream_t)stream, pdl);
}

int set_attr_mega(size_t bytes) {
  return (int)cudaFuncSetAttribute(moe_mega_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)bytes);
}

}  // namespace moe
