// gdn_chunk_tc.cu -- tensor-core (tcgen05/TMEM) chunkwise kernel: not yet built.
#include "gdn_internal.cuh"

namespace gdn {
bool chunk_tc_supported(const gdn_shape_t &) { return false; }
cudaError_t launch_chunk_tc(const PrefillArgs &, cudaStream_t, int) { return cudaErrorNotSupported; }
}  // namespace gdn
