// Placeholder for the tensor-core path until its kernels land: reports every
// problem as unsupported so that dispatch falls back to the CUDA-core path.
#include "gla_internal.h"

namespace gla {
bool tc_supported(const Problem&) { return false; }
size_t tc_fwd_workspace(const Problem&) { return 0; }
size_t tc_bwd_workspace(const Problem&) { return 0; }
gla_status tc_fwd(const Problem&, const void*, const void*, const void*, const float*, const float*, void*, float*,
                  Arena&, cudaStream_t) {
    return GLA_ERR_UNSUPPORTED;
}
gla_status tc_bwd(const Problem&, const void*, const void*, const void*, const float*, const float*, const void*,
                  const float*, void*, void*, void*, float*, float*, Arena&, cudaStream_t) {
    return GLA_ERR_UNSUPPORTED;
}
}  // namespace gla
