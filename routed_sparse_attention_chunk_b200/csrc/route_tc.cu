// Tensor-core (tcgen05) routing scan for bf16 banks: not built yet; every
// shape goes to the CUDA-core kernel in route.cu.
#include "common.cuh"
#include "internal.h"

namespace msa {

cudaError_t launch_route_tc(const RouteArgs& a, cudaStream_t s, bool* handled) {
  (void)a;
  (void)s;
  *handled = false;
  return cudaSuccess;
}

}  // namespace msa
