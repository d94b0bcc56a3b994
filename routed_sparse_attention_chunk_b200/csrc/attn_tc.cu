// Tensor-core (tcgen05) attention for bf16: not built yet; every shape goes to
// the CUDA-core kernel in attn.cu.
#include "common.cuh"
#include "internal.h"

namespace msa {

size_t attn_tc_workspace_size(msa_dtype, int64_t, int, int, int, int, int, int) { return 0; }

cudaError_t launch_attn_tc(msa_dtype dt, const AttnArgs& a, cudaStream_t s, bool* handled) {
  (void)dt;
  (void)a;
  (void)s;
  *handled = false;
  return cudaSuccess;
}

}  // namespace msa
