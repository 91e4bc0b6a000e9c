// chunk_tc.cuh -- entry points of the tcgen05 tensor-core chunked forward.
#pragma once
#include "common.cuh"

namespace gdr {

// True when the tensor-core kernel takes this call (bf16, dk = dv = 128, chunk 64).
bool chunk_tc_supported(const ChunkArgs &a);
gdr_status_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t s);
// Reads and zeroes the device error word that bounded waits set on expiry.
cudaError_t chunk_tc_read_and_clear_error(int *err);

}  // namespace gdr
