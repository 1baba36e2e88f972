// Fused tensor-core routing kernel (placeholder until the tcgen05 path lands).
#include "more_internal.cuh"

namespace more {

bool fused_tc_supports(const RouteArgs&) { return false; }

cudaError_t launch_fused_tc(const RouteArgs&) { return cudaErrorNotSupported; }

}  // namespace more
