// chunk_bwd.cu -- chunkwise gate-aware backward on tcgen05 (not built yet).
#include <cuda_runtime.h>

#include "internal.h"

namespace gdn2 {

cudaError_t chunk_bwd_launch(const ChunkBwdArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace gdn2
