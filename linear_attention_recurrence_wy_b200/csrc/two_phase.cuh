// two_phase.cuh -- the two-phase chunked forward: the per-chunk record that joins its phases.
//
// Phase one (wy_prep.cu) forms, for every chunk of every sequence-head at once, the chunk's
// WY factors in the form the pages write them (Gated DeltaNet-2 Review §3-2.5 "Chunkwise WY
// training": W = T (decayed, b-scaled K), U = T (w.V)), together with the decayed query and
// key operands; none of it depends on the state.  Phase two (state_pass.cu) walks the chunks
// of each sequence-head in order and keeps only what does:
//     E = U - W S,    O = Qg S + P E,    S' = diag(e^gamma_C) (S + Kb^T E).
// The record of one chunk holds those operands as bf16 tiles in the 128-byte swizzled layout
// of tc_util.cuh (so phase two copies it into shared memory and hands it to the tensor cores
// as it is) plus e^gamma_C and the chunk's path flag.  Shape: dk = dv = 128, chunk 64.
#pragma once
#include "common.cuh"

namespace gdr {
namespace tp {

constexpr int REC_WT = 0;          // W^T  bf16 [128 d][64 t], 128-row tile            16 KB
constexpr int REC_UT = 16384;      // U^T  bf16 [128 v][64 t], 128-row tile            16 KB
constexpr int REC_QG = 32768;      // Qg   bf16 [64 t][128 d], 64-row tile             16 KB
constexpr int REC_KB = 49152;      // Kb   bf16 [64 t][128 d] (K_end on the exact path) 16 KB
constexpr int REC_P = 65536;       // P    bf16 [64 t][64 j], lower incl.               8 KB
constexpr int REC_EGC = 73728;     // e^gamma_C fp32 [128]
constexpr int REC_FLAG = 74240;    // int32: 1 = exact path (strong decay), else 0
constexpr int REC_LOAD = 74256;    // bytes phase two copies per chunk
constexpr int REC_BYTES = 74752;   // record stride (a multiple of 1024)

// Workspace of a two-phase call: records [B*H][ceil(T/64)], then the exact-path list
// (a count, then unit indices; 16-byte padded), then, for a sequence split, the split's
// three state arrays ([B*H][nseg][dk][dv] fp32 each: end states, maps, start states).
unsigned long long records_bytes(int B, int H, int T);
unsigned long long list_bytes(int B, int H, int T);

// Phase one over every chunk (units = B*H*ceil(T/64)); list = the exact-path list, whose
// count must be zero on entry.  Two launches: the tensor-core kernel for every chunk whose
// cumulative decay stays within the fast path's range, then a CUDA-core kernel for the
// chunks it listed.
gdr_status_t launch_wy_prep(const ChunkArgs &a, unsigned char *records, int *list, cudaStream_t s);
// Phase two: the roles of ChunkArgs (whole sequence, a split's passes) over the records.
gdr_status_t launch_state_pass(const ChunkArgs &a, const unsigned char *records, cudaStream_t s);
// Read and zero the device error words the kernels' bounded waits set on expiry (the
// second is the state pass's alone; the first covers both phases).
cudaError_t two_phase_read_and_clear_error(int *err);
cudaError_t state_pass_read_and_clear_error(int *err);

}  // namespace tp
}  // namespace gdr
