// tcgen05 tensor-core forward for bf16 activations.
#include "paths.h"

namespace e2ttt {

bool tc_fwd_supported(const Dims&, bool) { return false; }
size_t tc_fwd_scratch_bytes(const Dims&) { return 0; }
cudaError_t tc_fwd(const Dims&, const bf16*, const bf16*, const bf16*, bf16*, const float*,
                   const float*, const float*, const float*, const float*, float*, float*, float*,
                   float*, void*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace e2ttt
