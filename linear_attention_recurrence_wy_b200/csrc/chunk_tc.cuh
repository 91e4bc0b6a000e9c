// chunk_tc.cuh -- entry points of the tcgen05 tensor-core chunked forward.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace gdr {

// True when the tensor-core kernel takes this call (bf16, dk = dv = 128, chunk 64).
bool chunk_tc_supported(const ChunkArgs &a);
gdr_status_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t s);
// Reads and zeroes the device error word that bounded waits set on expiry.
cudaError_t chunk_tc_read_and_clear_error(int *err);

// cuTensorMapEncodeTiled from the driver (looked up once; NULL when unavailable).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encode_fn();

}  // namespace gdr
