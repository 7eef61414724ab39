// chunk_tc.cu -- bf16 chunkwise GDN forward on the tcgen05 tensor cores.
#include "common.cuh"
#include "launch.h"

namespace gdn {

bool chunk_tc_supported(const ChunkArgs&) { return false; }
cudaError_t launch_chunk_tc(const ChunkArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace gdn
