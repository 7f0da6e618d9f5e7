// Chunkwise tcgen05 kernel (placeholder until the tensor-core path lands).
#include "gdn_internal.h"

namespace gdn {

bool chunk_tc_supported(const FwdArgs &) { return false; }

cudaError_t launch_chunk_tc(const FwdArgs &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace gdn
