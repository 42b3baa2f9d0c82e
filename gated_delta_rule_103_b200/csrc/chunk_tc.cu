// Placeholder: bf16 prefill routed to the FFMA kernel until the tensor-core
// kernel lands.
#include "kda_internal.h"

namespace kda {
cudaError_t launch_chunk_tc(const ChunkArgs& a, cudaStream_t stream)
{
    return launch_chunk_simt(a, KDA_DTYPE_BF16, stream);
}
}  // namespace kda
