// Tensor-core chunkwise forward (bf16 operands, fp32 state); filled in next.
#include "gdr_internal.cuh"

namespace gdr {

bool chunk_tc_supports(const ChunkArgs &a)
{
    (void)a;
    return false;
}

cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t stream, int *launches)
{
    (void)a; (void)stream; (void)launches;
    return cudaErrorNotSupported;
}

}  // namespace gdr
