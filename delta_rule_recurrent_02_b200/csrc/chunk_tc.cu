// chunk_tc.cu -- tensor-core (tcgen05) chunk kernel: not built yet.
#include "dn_kernels.h"

namespace dn {

bool tc_supports(const ChunkArgs&) { return false; }

cudaError_t launch_chunk_tc(const ChunkArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace dn
