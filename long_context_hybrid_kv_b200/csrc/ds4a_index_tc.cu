// Tensor-core (tcgen05) indexer score for the Flash shape (H_I = 64,
// D_I = 128).
#include "ds4a_internal.cuh"

namespace ds4a {
bool index_scores_tc_supported(const IndexArgs&) { return false; }
cudaError_t launch_index_scores_tc(const IndexArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace ds4a
