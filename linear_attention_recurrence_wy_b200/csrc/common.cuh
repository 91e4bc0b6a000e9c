// common.cuh -- shared argument block, element loads and launch helpers of libgdr.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/gdr.h"

namespace gdr {

// Everything a chunked-forward kernel needs; built once by the C-ABI layer.
struct ChunkArgs {
    const void *q, *k, *v, *b, *w;
    const float *g, *S0;
    void *o;
    float *ST;
    int B, H, T, dk, dv, chunk, mode, dtype;
    // Sequence split (tensor-core kernel only).  nseg == 1 is the plain whole-sequence call.
    // pass 0 writes outputs (segment s starts from S0 if s == 0, else from ws_sstart[bh][s]);
    // pass 1 writes only end states: the local end state of segments 0 .. nseg-2
    // (ws_send; segment 0 from S0, others from zero) and the transition matrices of
    // segments 1 .. nseg-2 (ws_m; identity start state, values taken as zero).
    int nseg, seg_len, pass;
    float *ws_send, *ws_m, *ws_sstart;   // [B*H][nseg][dk][dv] fp32 each
    // Token mixer (tensor-core kernel only).  mixer != 0: q, k, v, g, b, w hold the raw
    // projections and the kernel applies the block's activations as it loads them
    // (q, k L2-normalised per token, g = -softplus(g), b = b_range * sigmoid(b),
    // w = sigmoid(w); the tied modes' write gate is beta = b_range * sigmoid(b)), and o
    // receives y = o * rsqrt(mean_v o^2 + eps) * nw * z * sigmoid(z).
    // tstride: rows between consecutive tokens of one head, 1 for [B,H,T,D] or H for
    // [B,T,H,D] (the token-major layout of the projections).
    int mixer, tstride;
    const void *z;
    const float *nw;
    float b_range, eps;
    // The backward's checkpoints: when set, the state at the start of every chunk is written
    // to chunk_states[B*H][ceil(T/32)][dk][dv] (fp32 slots), in the slot of the chunk's
    // first 32-token chunk (a 64-token chunk c fills slot 2c), and o may be NULL.  The
    // CUDA-core kernel writes fp32; the tensor-core kernel writes the state rounded to bf16
    // ([dk][dv] bf16 at the start of the slot), its MMA operands' precision.
    float *chunk_states;
    // The backward's state-gradient pass (tensor-core kernel, reverse != 0): S0 holds dS_T,
    // ST receives dS0, dO is the output gradient [B,H,T,dv], and chunk_states receives the
    // gradient at every 64-token chunk's end (slot of its last 32-token chunk), as bf16.
    int reverse;
    const void *dO;
    // Bounded waits: polls of an mbarrier before a kernel gives up and reports
    // GDR_ERR_TIMEOUT.  first_wait_limit != 0 is a test hook: the tensor-core forward's state
    // group then gives up its very first wait after that many non-blocking polls, so the
    // expiry path runs while the WY group is merely still working.
    unsigned wait_limit = 1u << 24;
    unsigned first_wait_limit = 0;
    // The maps of one whole segment held on its own (the sequence split across GPUs;
    // tensor-core kernel, pass 1 semantics, no output): seg_maps != 0 writes the end state
    // reached from S0 (NULL: zero) to ws_send[B*H][dk][dv] and, when want_m, the segment's
    // transition map (the end state from the identity with the write term dropped) to
    // ws_m[B*H][dk][dk].
    int seg_maps = 0, want_m = 0;
};

// CTAs per sequence-head of a tensor-core forward launch: its roles (whole sequence, the
// split's segments and transfer runs, or a segment's maps).
__host__ __device__ inline int chunk_roles(const ChunkArgs &a) {
    if (a.seg_maps) return a.want_m ? 2 : 1;
    if (a.pass) return 2 * a.nseg - 3 > 1 ? 2 * a.nseg - 3 : 1;
    return a.nseg;
}

struct DecodeArgs {
    const void *q, *k, *v, *b, *w;
    const float *g;
    float *S;
    void *o;
    int N, H, dk, dv, mode, dtype;
    // bounded waits of the streaming kernel, as in ChunkArgs (first_wait_limit: a test hook
    // that makes each CTA's first wait give up after that many non-blocking polls)
    unsigned wait_limit = 1u << 24;
    unsigned first_wait_limit = 0;
};

// Gate shapes per mode: the erase gate b and the write gate w are per channel or one
// scalar per token; the scalar write gate is w itself (b-only) or beta in b (tied modes).
__host__ __device__ constexpr bool mode_b_vec(int m) { return m == GDR_MODE_GDN2 || m == GDR_MODE_BONLY; }
__host__ __device__ constexpr bool mode_w_vec(int m) { return m == GDR_MODE_GDN2 || m == GDR_MODE_WONLY; }
__host__ __device__ constexpr bool mode_uses_w(int m) {
    return m == GDR_MODE_GDN2 || m == GDR_MODE_BONLY || m == GDR_MODE_WONLY;
}
__host__ __device__ constexpr bool mode_g_vec(int m) { return m != GDR_MODE_GDN; }

__device__ __forceinline__ float ld_elem(const void *p, size_t i, int dtype) {
    if (dtype == GDR_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
    return reinterpret_cast<const float *>(p)[i];
}

__device__ __forceinline__ void st_elem(void *p, size_t i, int dtype, float x) {
    if (dtype == GDR_BF16) reinterpret_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(x);
    else reinterpret_cast<float *>(p)[i] = x;
}

// Launch wrappers (one per kernel family); each returns GDR_OK or GDR_ERR_CUDA.
gdr_status_t launch_chunk_simt(const ChunkArgs &a, cudaStream_t s);
gdr_status_t launch_decode(const DecodeArgs &a, cudaStream_t s);
// Reads and zeroes the device error word of the streaming decode kernel's bounded waits.
cudaError_t decode_read_and_clear_error(int *err);
gdr_status_t launch_state_copy(const ChunkArgs &a, cudaStream_t s);

// Backward (bwd.cu): everything the three backward kernels need.
struct BwdArgs {
    const void *q, *k, *v, *b, *w;
    const float *g, *S0;
    const void *dO;
    const float *dST;
    void *dq, *dk, *dv, *db, *dw;
    float *dg, *dS0;
    int B, H, T, dk_, dv_, mode, dtype;
    float *ws_states, *ws_dstates;   // [B*H][nchunks][dk][dv] fp32 each
    // 1: ws_dstates holds the state gradient only at the ends of 64-token spans (the
    // tensor-core state-gradient pass); the per-chunk kernel forms the middle ones
    int mid_grad;
    // [1 + B*H*nspan]: a count, then the indices (b*H + h)*nspan + span of the 64-token spans
    // the tensor-core per-chunk kernel left to the CUDA-core one; NULL: that kernel takes
    // every span
    int *tc_list;
    // 1: the tensor-core passes wrote the checkpoints (ws_states slot 2 span) and the span-end
    // state gradients (ws_dstates slot min(2 span + 1, last)) as bf16 [dk][dv]; the slots the
    // CUDA-core kernel writes itself stay fp32
    int ckpt_bf16;
    // bounded waits of the tensor-core per-chunk kernel, as in ChunkArgs (first_wait_limit: a
    // test hook that makes each CTA's first wait give up after that many non-blocking polls)
    unsigned wait_limit = 1u << 24;
    unsigned first_wait_limit = 0;
    // the tensor-core per-chunk kernel: CTAs resident at once (its SM count; 0: no prefetch).
    // The CTA that starts next on an SM is about this many grid indices ahead, so each CTA
    // prefetches that chunk's inputs to L2 once its own have landed
    int prefetch_ahead = 0;
};
constexpr int kBwdChunk = 32;   // tokens per chunk of the backward
// the two state arrays, then tc_list (16-byte multiple)
unsigned long long bwd_states_bytes(int B, int H, int T, int dk, int dv);
unsigned long long bwd_workspace_bytes(int B, int H, int T, int dk, int dv);
gdr_status_t launch_bwd(const BwdArgs &a, cudaStream_t s);
gdr_status_t launch_split_combine(const ChunkArgs &a, cudaStream_t s);
// Debug build (GDR_DEBUG): the first failed bounds-check site of each translation unit's
// kernels, read and cleared (0: none; always 0 in the release build).  See bounds.cuh.
int chunk_tc_bounds_site();
int bwd_tc_bounds_site();
int bwd_bounds_site();
int simt_bounds_site();
int decode_bounds_site();
int split_bounds_site();
int wy_prep_bounds_site();
int state_pass_bounds_site();
// Start state of segment r of a sequence split across R holders (ranks), from every
// segment's maps gathered as M_all[R][BH][dk][dk] and S_all[R][BH][dk][dv] (fp32; the end
// state of segment 0 is taken from S0 already):  r = 0: S0 (zero if NULL);  r >= 1:
// S = S_all[0];  S <- M_all[i] S + S_all[i] for i = 1 .. r-1.  dk = dv = 128.
gdr_status_t launch_segment_chain(const float *M_all, const float *S_all, const float *S0, float *S_start, int R,
                                  int r, int BH, cudaStream_t s);
// Segments the sequence split actually runs for a request of nseg (segments of whole
// chunks, none empty); 1 for T <= 0.
int split_effective_segments(int T, int chunk, int nseg);

}  // namespace gdr
