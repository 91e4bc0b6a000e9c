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
constexpr int MLD = DK + 4;                    // padded fp32 row stride of a staged map
// two maps and their segments' end-state slices (double-buffered), the state slice
constexpr int CHAIN_SMEM = (2 * DK * MLD + 2 * DK * COLS + DK * COLS) * 4;

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}
// One map M (dk x dk fp32, row-major) and the CTA's 16-column slice of the segment's local
// end state L (rows DV apart) -> shared memory by asynchronous 16-byte copies, all 256
// threads, consecutive threads on consecutive 16 bytes; one commit group per segment.
__device__ __forceinline__ void stage_map(float *dst, float *ldst, const float *M, const float *L, int tid) {
#pragma unroll
    for (int j = 0; j < DK * DK / 4 / 256; ++j) {
        const int f = tid + 256 * j, row = f >> 5, c4 = f & 31;
        cp_async16(dst + row * MLD + 4 * c4, M + (size_t)row * DK + 4 * c4);
    }
#pragma unroll
    for (int j = 0; j < DK * COLS / 4 / 256; ++j) {
        const int f = tid + 256 * j, row = f >> 2, c4 = f & 3;
        cp_async16(ldst + row * COLS + 4 * c4, L + (size_t)row * DV + 4 * c4);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}
// wait until at most n commit groups of this thread are still in flight, then a CTA barrier
template <int n>
__device__ __forceinline__ void wait_maps() {
    asm volatile("cp.async.wait_group %0;" ::"n"(n) : "memory");
    __syncthreads();
}

// S <- M S + L on the CTA's 16-column slice: thread (row i, half h) forms columns 8h .. 8h+7
// of row i; M is a staged map (rows MLD apart), L the staged slice of the local end state.  The
// slice's rows are 16 floats apart, so a thread reads its eight columns of a row of S as two
// 16-byte loads, which every thread of the same half shares (a broadcast).
__device__ __forceinline__ void apply_map(float (*S)[COLS], const float *sM, const float *sL, int i, int h) {
    const float4 l0 = *reinterpret_cast<const float4 *>(sL + i * COLS + 8 * h);
    const float4 l1 = *reinterpret_cast<const float4 *>(sL + i * COLS + 8 * h + 4);
    float acc[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
    const float *m = sM + i * MLD;
#pragma unroll 2
    for (int k0 = 0; k0 < DK; k0 += 4) {
        const float4 mv = *reinterpret_cast<const float4 *>(m + k0);
        const float mk[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const float4 s0 = *reinterpret_cast<const float4 *>(&S[k0 + kk][8 * h]);
            const float4 s1 = *reinterpret_cast<const float4 *>(&S[k0 + kk][8 * h + 4]);
            const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = fmaf(mk[kk], sv[j], acc[j]);
        }
    }
    __syncthreads();   // every thread has read S
    *reinterpret_cast<float4 *>(&S[i][8 * h]) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    *reinterpret_cast<float4 *>(&S[i][8 * h + 4]) = make_float4(acc[4], acc[5], acc[6], acc[7]);
    __syncthreads();
}

// Dynamic shared memory: the two map buffers, their two end-state slices, the state slice.
struct ChainSmem {
    float *m0, *m1, *l0, *l1;
    float (*S)[COLS];
    // the buffers of segment s, by parity
    __device__ __forceinline__ float *m(int s) const { return (s & 1) ? m1 : m0; }
    __device__ __forceinline__ float *l(int s) const { return (s & 1) ? l1 : l0; }
};
__device__ __forceinline__ ChainSmem chain_smem() {
    extern __shared__ __align__(16) float chain_raw[];
    float *l = chain_raw + 2 * DK * MLD;
    return {chain_raw, chain_raw + DK * MLD, l, l + DK * COLS, reinterpret_cast<float (*)[COLS]>(l + 2 * DK * COLS)};
}

__global__ void __launch_bounds__(256) split_combine_kernel(ChunkArgs a) {
    const int slices = DV / COLS;
    const int bh = blockIdx.x / slices, c0 = (blockIdx.x % slices) * COLS;
    const int tid = threadIdx.x, i = tid >> 1, h = tid & 1;   // row i, columns c0 + 8h ..
    if (!GDR_IN_BOUNDS(bh < a.B * a.H, 501)) return;   // debug build: uniform, before any barrier
    const ChainSmem sm = chain_smem();
    float (*S)[COLS] = sm.S;
    const size_t head = (size_t)bh * a.nseg * DK * DV;
    const size_t seg_sz = (size_t)DK * DV;
    float *sstart = a.ws_sstart + head;
    // the maps of segments 1 .. nseg-2 are applied in turn; the first travels now, each next
    // one while the current one is applied
    const int last = a.nseg - 2;
    if (last >= 1) stage_map(sm.m(1), sm.l(1), a.ws_m + head + seg_sz, a.ws_send + head + seg_sz + c0, tid);
    // S_start(0) = S0 (zeros if absent): the second pass reads every start state from here
    for (int j = 0; j < 8; ++j) {
        const int c = c0 + 8 * h + j;
        sstart[(size_t)i * DV + c] = a.S0 ? a.S0[(size_t)bh * DK * DV + (size_t)i * DV + c] : 0.f;
        S[i][8 * h + j] = a.ws_send[head + (size_t)i * DV + c];   // S_end(0)
    }
    __syncthreads();
    for (int s = 1; s < a.nseg; ++s) {
        float4 *dst = reinterpret_cast<float4 *>(sstart + s * seg_sz + (size_t)i * DV + c0 + 8 * h);
        dst[0] = *reinterpret_cast<const float4 *>(&S[i][8 * h]);
        dst[1] = *reinterpret_cast<const float4 *>(&S[i][8 * h + 4]);
        if (s > last) break;
        if (s < last) {
            stage_map(sm.m((s + 1) & 1), sm.l((s + 1) & 1), a.ws_m + head + (s + 1) * seg_sz,
                      a.ws_send + head + (s + 1) * seg_sz + c0, tid);
            wait_maps<1>();   // this segment's map has landed; the next one may still travel
        } else {
            wait_maps<0>();
        }
        apply_map(S, sm.m(s & 1), sm.l(s & 1), i, h);
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
    const size_t st = (size_t)DK * DV;                       // one state
    const size_t per = (size_t)BH * st;                      // one holder's block of states
    if (!GDR_IN_BOUNDS(bh < BH, 502)) return;                // debug build: uniform, before any barrier
    float *out = S_start + bh * st + (size_t)i * DV + c0 + 8 * h;
    if (r == 0) {
        for (int j = 0; j < 8; ++j) out[j] = S0 ? S0[bh * st + (size_t)i * DV + c0 + 8 * h + j] : 0.f;
        return;
    }
    const ChainSmem sm = chain_smem();
    float (*S)[COLS] = sm.S;
    const int last = r - 1;   // maps of holders 1 .. r-1
    if (last >= 1) stage_map(sm.m(1), sm.l(1), M_all + per + bh * st, S_all + per + bh * st + c0, tid);
    for (int j = 0; j < 8; ++j) S[i][8 * h + j] = S_all[bh * st + (size_t)i * DV + c0 + 8 * h + j];   // S_end(0)
    __syncthreads();
    for (int s = 1; s <= last; ++s) {
        if (s < last) {
            stage_map(sm.m((s + 1) & 1), sm.l((s + 1) & 1), M_all + (s + 1) * per + bh * st,
                      S_all + (s + 1) * per + bh * st + c0, tid);
            wait_maps<1>();
        } else {
            wait_maps<0>();
        }
        apply_map(S, sm.m(s & 1), sm.l(s & 1), i, h);
    }
    for (int j = 0; j < 8; ++j) out[j] = S[i][8 * h + j];
}

bool chain_attr_set(const void *kern) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, CHAIN_SMEM) == cudaSuccess;
}

}  // namespace

gdr_status_t launch_segment_chain(const float *M_all, const float *S_all, const float *S0, float *S_start, int R,
                                  int r, int BH, cudaStream_t s) {
    (void)R;
    if (!chain_attr_set((const void *)segment_chain_kernel)) return GDR_ERR_CUDA;
    segment_chain_kernel<<<(unsigned)(BH * (DV / COLS)), 256, CHAIN_SMEM, s>>>(M_all, S_all, S0, S_start, r, BH);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

gdr_status_t launch_split_combine(const ChunkArgs &a, cudaStream_t s) {
    if (!chain_attr_set((const void *)split_combine_kernel)) return GDR_ERR_CUDA;
    split_combine_kernel<<<(unsigned)(a.B * a.H * (DV / COLS)), 256, CHAIN_SMEM, s>>>(a);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

}  // namespace gdr

namespace gdr {
GDR_BOUNDS_READER(split_bounds_site)
}  // namespace gdr
