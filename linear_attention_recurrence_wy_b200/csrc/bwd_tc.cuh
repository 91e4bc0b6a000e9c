// bwd_tc.cuh -- entry points of the tcgen05 per-chunk backward (bwd_tc.cu).
#pragma once
#include "common.cuh"

namespace gdr {

// True when the tensor-core per-chunk kernel takes this call (bf16, dk = dv = 128).
bool bwd_tc_supported(const BwdArgs &a);
// One CTA per (sequence, head, 64-token chunk).  Needs the states at every 64-token
// boundary in ws_states and the state gradients at every 64-token chunk's end in
// ws_dstates; chunks with a strong cumulative decay are appended to tc_list (whose count,
// tc_list[0], must be zero before the launch).
gdr_status_t launch_bwd_tc(const BwdArgs &a, cudaStream_t s);
// Reads and zeroes the device error word that bounded waits set on expiry.
cudaError_t bwd_tc_read_and_clear_error(int *err);

}  // namespace gdr
