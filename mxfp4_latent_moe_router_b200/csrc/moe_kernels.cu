// moe_kernels.cu -- dispatch of the four kernel kinds (device code in
// moe_engine.cuh, one translation unit per kind).
#include <cuda_runtime.h>

#include "engine.cuh"

namespace moe {

int set_attr_mega(size_t bytes);

int launch_front(int nt, const Params& p, int grid, size_t smem, void* stream, bool pdl);
int launch_egu(int nt, const Params& p, int grid, size_t smem, void* stream, bool pdl);
int launch_edn(int nt, const Params& p, int grid, size_t smem, void* stream, bool pdl);
int launch_tail(int nt, const Params& p, int grid, size_t smem, void* stream, bool pdl);
int set_attr_front(size_t bytes);
int set_attr_egu(size_t bytes);
int set_attr_edn(size_t bytes);
int set_attr_tail(size_t bytes);

int set_smem_limits(size_t bytes) {
  return set_attr_front(bytes) | set_attr_egu(bytes) | set_attr_edn(bytes) | set_attr_tail(bytes) |
         set_attr_mega(bytes);
}

int max_smem_optin() {
  int dev = 0, v = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  return v;
}

int launch_kind(int kind, int nt, const Params& p, int grid, size_t smem, void* stream, bool pdl) {
  switch (kind) {
    case KIND_FRONT: return launch_front(nt, p, grid, smem, stream, pdl);
    case KIND_EGU: return launch_egu(nt, p, grid, smem, stream, pdl);
    case KIND_EDN: return launch_edn(nt, p, grid, smem, stream, pdl);
    case KIND_TAIL: return launch_tail(nt, p, grid, smem, stream, pdl);
    default: return (int)cudaErrorInvalidValue;
  }
}

}  // namespace moe
