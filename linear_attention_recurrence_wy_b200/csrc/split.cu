// split.cu -- chaining the segment states of a sequence split.
//
// The recurrence is affine in the state: over a segment, S_end = M S_start + S_local,
// where M (dk x dk) is the product of the segment's per-token transitions
// (I - k (b.k)^T) diag(exp g) and S_local is the end state reached from S_start = 0
// (Gated DeltaNet-2 Q&A page, Q3 update equation; only the state crosses chunk and
// segment borders, Gated DeltaNet-2 Review §3-2.5).  The first pass of the split
// computes M and S_local of the inner segments in parallel; this kernel chains them
// in fp32:
//     S_start(0) = S0,  S_start(1) = S_end(0),  S_start(s+1) = M_s S_start(s) + S_local(s)
// and the second pass recomputes every segment from its S_start.
#include "bounds.cuh"
#include "common.cuh"

namespace gdr {
namespace {

constexpr int DK = 128, DV = 128, COLS = 16;   // one CTA: one sequence-head, 16 state columns

__global__ void __launch_bounds__(256) split_combine_kernel(ChunkArgs a) {
    const int slices = DV / COLS;
    const int bh = blockIdx.x / slices, c0 = (blockIdx.x % slices) * COLS;
    const int tid = threadIdx.x, i = tid >> 1, h = tid & 1;   // row i, columns c0 + 8h ..
    __shared__ float S[DK][COLS + 1];
    if (!GDR_IN_BOUNDS(bh < a.B * a.H, 501)) return;   // debug build: uniform, before any barrier
    const size_t head = (size_t)bh * a.nseg * DK * DV;
    const size_t seg_sz = (size_t)DK * DV;
    float *sstart = a.ws_sstart + head;
    // S_start(0) = S0 (zeros if absent): the second pass reads every start state from here
    for (int j = 0; j < 8; ++j) {
        const int c = c0 + 8 * h + j;
        sstart[(size_t)i * DV + c] = a.S0 ? a.S0[(size_t)bh * DK * DV + (size_t)i * DV + c] : 0.f;
        S[i][8 * h + j] = a.ws_send[head + (size_t)i * DV + c];   // S_end(0)
    }
    __syncthreads();
    for (int s = 1; s < a.nseg; ++s) {
        for (int j = 0; j < 8; ++j) sstart[s * seg_sz + (size_t)i * DV + c0 + 8 * h + j] = S[i][8 * h + j];
        if (s == a.nseg - 1) break;
        const float *M = a.ws_m + head + s * seg_sz + (size_t)i * DK;
        const float *L = a.ws_send + head + s * seg_sz + (size_t)i * DV + c0 + 8 * h;
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = L[j];
        for (int k0 = 0; k0 < DK; k0 += 4) {
            const float4 m = *reinterpret_cast<const float4 *>(M + k0);
            const float mk[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[j] = fmaf(mk[kk], S[k0 + kk][8 * h + j], acc[j]);
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < 8; ++j) S[i][8 * h + j] = acc[j];
        __syncthreads();
    }
}

// The same chaining for a sequence split across holders (ranks): segment r's start state
// from every segment's gathered maps (see launch_segment_chain).  One CTA per sequence-head
// and 16-column slice of the state, like split_combine_kernel.
__global__ void __launch_bounds__(256) segment_chain_kernel(const float *M_all, const float *S_all,
                                                            const float *S0, float *S_start, int r, int BH) {
    const int slices = DV / COLS;
    const int bh = blockIdx.x / slices, c0 = (blockIdx.x % slices) * COLS;
    const int tid = threadIdx.x, i = tid >> 1, h = tid & 1;   // row i, columns c0 + 8h ..
    __shared__ float S[DK][COLS + 1];
    const size_t st = (size_t)DK * DV;                       // one state
    const size_t per = (size_t)BH * st;                      // one holder's block of states
    if (!GDR_IN_BOUNDS(bh < BH, 502)) return;                // debug build: uniform, before any barrier
    float *out = S_start + bh * st + (size_t)i * DV + c0 + 8 * h;
    if (r == 0) {
        for (int j = 0; j < 8; ++j) out[j] = S0 ? S0[bh * st + (size_t)i * DV + c0 + 8 * h + j] : 0.f;
        return;
    }
    for (int j = 0; j < 8; ++j) S[i][8 * h + j] = S_all[bh * st + (size_t)i * DV + c0 + 8 * h + j];   // S_end(0)
    __syncthreads();
    for (int s = 1; s < r; ++s) {
        const float *M = M_all + s * per + bh * st + (size_t)i * DK;
        const float *L = S_all + s * per + bh * st + (size_t)i * DV + c0 + 8 * h;
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = L[j];
        for (int k0 = 0; k0 < DK; k0 += 4) {
            const float4 m = *reinterpret_cast<const float4 *>(M + k0);
            const float mk[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[j] = fmaf(mk[kk], S[k0 + kk][8 * h + j], acc[j]);
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < 8; ++j) S[i][8 * h + j] = acc[j];
        __syncthreads();
    }
    for (int j = 0; j < 8; ++j) out[j] = S[i][8 * h + j];
}

}  // namespace

gdr_status_t launch_segment_chain(const float *M_all, const float *S_all, const float *S0, float *S_start, int R,
                                  int r, int BH, cudaStream_t s) {
    (void)R;
    segment_chain_kernel<<<(unsigned)(BH * (DV / COLS)), 256, 0, s>>>(M_all, S_all, S0, S_start, r, BH);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

gdr_status_t launch_split_combine(const ChunkArgs &a, cudaStream_t s) {
    split_combine_kernel<<<(unsigned)(a.B * a.H * (DV / COLS)), 256, 0, s>>>(a);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

}  // namespace gdr

namespace gdr {
GDR_BOUNDS_READER(split_bounds_site)
}  // namespace gdr
