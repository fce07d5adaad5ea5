// Tensor-core (tcgen05) attention for the Flash shape (64 heads x 512).
#include "ds4a_internal.cuh"

namespace ds4a {
bool attend_tc_supported(const AttendArgs&) { return false; }
cudaError_t launch_attend_tc(const AttendArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace ds4a
