// decode.cu -- one-token recurrent step, state updated in place (bandwidth-bound).
//
// Per (sequence, head) the step reads the fp32 state once and writes it once
// (Gated DeltaNet-2 Q&A page, Q3 update equation, applied to a single token):
//   D S                 decay rows by exp(g)
//   r  = (D S)^T (b.k)  read along b.k from the decayed state
//   u  = w.v - r        the write minus what is erased
//   S' = D S + k u^T
//   o  = S'^T q = (D S)^T q + u (k.q)
// so r and (D S)^T q are two column reductions over the same pass, and the new
// state is written from registers.  One CTA of 256 threads owns one head's
// dk x dv state; each thread holds float4 column groups of several rows, the
// loads are 16-byte coalesced and all issued before any arithmetic.
#include "common.cuh"

namespace gdr {
namespace {

constexpr int kThreads = 256;

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads) decode_kernel(DecodeArgs a) {
    constexpr int TPR = DV / 4;                 // threads per state row (float4 each)
    constexpr int RPP = kThreads / TPR;         // rows covered per pass
    constexpr int NP = (DK + RPP - 1) / RPP;    // passes
    const int nh = blockIdx.x;
    const int tid = threadIdx.x;
    const int cg = tid % TPR;
    const int r0 = tid / TPR;

    __shared__ float s_q[DK], s_k[DK], s_a[DK], s_bk[DK];
    __shared__ float s_wv[DV], s_u[DV];
    __shared__ float red_r[RPP][DV + 1], red_o[RPP][DV + 1];
    __shared__ float s_kq;

    float4 *Sg = reinterpret_cast<float4 *>(a.S + (size_t)nh * DK * DV);
    float4 x[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const int row = r0 + p * RPP;
        if (row < DK) x[p] = __ldcs(Sg + row * TPR + cg);
    }
    for (int i = tid; i < DK; i += kThreads) {
        const size_t e = (size_t)nh * DK + i;
        const float kv = ld_elem(a.k, e, a.dtype);
        const float bv = (a.mode == GDR_MODE_GDN2) ? ld_elem(a.b, e, a.dtype)
                                                   : ld_elem(a.b, nh, a.dtype);
        const float gv = (a.mode == GDR_MODE_GDN) ? a.g[nh] : a.g[e];
        s_q[i] = ld_elem(a.q, e, a.dtype);
        s_k[i] = kv;
        s_bk[i] = bv * kv;
        s_a[i] = __expf(gv);
    }
    for (int j = tid; j < DV; j += kThreads) {
        const size_t e = (size_t)nh * DV + j;
        const float wv = (a.mode == GDR_MODE_GDN2) ? ld_elem(a.w, e, a.dtype)
                                                   : ld_elem(a.b, nh, a.dtype);
        s_wv[j] = wv * ld_elem(a.v, e, a.dtype);
    }
    __syncthreads();
    if (tid < 32) {
        float acc = 0.f;
        for (int i = tid; i < DK; i += 32) acc = fmaf(s_k[i], s_q[i], acc);
#pragma unroll
        for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (tid == 0) s_kq = acc;
    }
    // decay in registers; partial column sums of r = (DS)^T (b.k) and (DS)^T q
    float pr[4] = {0.f, 0.f, 0.f, 0.f}, po[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const int row = r0 + p * RPP;
        if (row < DK) {
            const float al = s_a[row], bkv = s_bk[row], qv = s_q[row];
            x[p].x *= al; x[p].y *= al; x[p].z *= al; x[p].w *= al;
            pr[0] = fmaf(x[p].x, bkv, pr[0]); pr[1] = fmaf(x[p].y, bkv, pr[1]);
            pr[2] = fmaf(x[p].z, bkv, pr[2]); pr[3] = fmaf(x[p].w, bkv, pr[3]);
            po[0] = fmaf(x[p].x, qv, po[0]); po[1] = fmaf(x[p].y, qv, po[1]);
            po[2] = fmaf(x[p].z, qv, po[2]); po[3] = fmaf(x[p].w, qv, po[3]);
        }
    }
    if (r0 < RPP) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            red_r[r0][4 * cg + c] = pr[c];
            red_o[r0][4 * cg + c] = po[c];
        }
    }
    __syncthreads();
    for (int j = tid; j < DV; j += kThreads) {
        float rs = 0.f, os = 0.f;
        const int rows = RPP < DK ? RPP : DK;
        for (int r = 0; r < rows; ++r) {
            rs += red_r[r][j];
            os += red_o[r][j];
        }
        const float u = s_wv[j] - rs;
        s_u[j] = u;
        st_elem(a.o, (size_t)nh * DV + j, a.dtype, fmaf(u, s_kq, os));
    }
    __syncthreads();
    const float u0 = s_u[4 * cg], u1 = s_u[4 * cg + 1], u2 = s_u[4 * cg + 2], u3 = s_u[4 * cg + 3];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const int row = r0 + p * RPP;
        if (row < DK) {
            const float kv = s_k[row];
            float4 y;
            y.x = fmaf(kv, u0, x[p].x); y.y = fmaf(kv, u1, x[p].y);
            y.z = fmaf(kv, u2, x[p].z); y.w = fmaf(kv, u3, x[p].w);
            __stcs(Sg + row * TPR + cg, y);
        }
    }
}

template <int DK>
gdr_status_t launch_dk(const DecodeArgs &a, cudaStream_t s) {
    const unsigned grid = (unsigned)(a.N * a.H);
    switch (a.dv) {
        case 16: decode_kernel<DK, 16><<<grid, kThreads, 0, s>>>(a); break;
        case 32: decode_kernel<DK, 32><<<grid, kThreads, 0, s>>>(a); break;
        case 64: decode_kernel<DK, 64><<<grid, kThreads, 0, s>>>(a); break;
        case 128: decode_kernel<DK, 128><<<grid, kThreads, 0, s>>>(a); break;
        default: return GDR_ERR_DIM;
    }
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

}  // namespace

gdr_status_t launch_decode(const DecodeArgs &a, cudaStream_t s) {
    switch (a.dk) {
        case 16: return launch_dk<16>(a, s);
        case 32: return launch_dk<32>(a, s);
        case 64: return launch_dk<64>(a, s);
        case 128: return launch_dk<128>(a, s);
        default: return GDR_ERR_DIM;
    }
}

}  // namespace gdr
