// Backward of the chunk scan.
#include "paths.h"

namespace e2ttt {

size_t bwd_workspace_bytes(const Dims&, bool) { return 256; }
template <typename TA>
cudaError_t bwd_run(const BwdArgs&) { return cudaErrorNotSupported; }
template cudaError_t bwd_run<float>(const BwdArgs&);
template cudaError_t bwd_run<bf16>(const BwdArgs&);

}  // namespace e2ttt
