// chunk_tc.cu -- tcgen05 tensor-core chunked forward (bf16 operands, fp32 state).
#include "chunk_tc.cuh"

namespace gdr {

// Set to a non-zero code by a kernel whose bounded wait expired.
__device__ int g_tc_error = 0;

bool chunk_tc_supported(const ChunkArgs &) { return false; }

gdr_status_t launch_chunk_tc(const ChunkArgs &, cudaStream_t) { return GDR_ERR_DIM; }

cudaError_t chunk_tc_read_and_clear_error(int *err) {
    cudaError_t e = cudaMemcpyFromSymbol(err, g_tc_error, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(int));
}

}  // namespace gdr
