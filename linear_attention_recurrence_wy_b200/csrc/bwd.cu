// bwd.cu -- chunkwise backward of the gated delta rule: the launch sequence, and the
// CUDA-core kernels (fp32 arithmetic) for the shapes and chunks the tensor cores do not take.
//
// The gradient of L = sum_t <o_t, dO_t> + <S_T, dS_T> with respect to q, k, v, the decay,
// both gates and S0 (the gate-aware backward of Gated DeltaNet-2 Review §4-3 and the
// Gated DeltaNet-2 Q&A page, Q4).  It differentiates the chunkwise WY form of the forward
// (Gated DeltaNet-2 Review §3-2.5), chunk by chunk, in 32-token chunks.  For one chunk,
// with gamma the chunk-local cumulative log-decay, F_ij = exp(gamma_i - gamma_j) per key
// channel, Kh = b.k.e^gamma, Qg = q.e^gamma, Ke = k.e^(gamma_C - gamma):
//
//   forward   A = strict_lower(sum_c b_i k_i k_j F_ij)   T = (I + A)^-1
//             P = lower_incl(sum_c q_i k_j F_ij)         R = w.v - Kh S     E = T R
//             O = Qg S + P E                             S' = e^gamma_C S + Ke^T E
//   backward  dE = P^T dO + Ke dS'        dR = T^T dE      dv = dR.w   dw = dR.v
//             dS = e^gamma_C dS' + Qg^T dO - Kh^T dR
//             dP = lower_incl(dO E^T)     dA = strict_lower(-T^T (dE R^T) T^T)
//   and q, k, b, gamma collect the products' terms: dO S^T through Qg, -dR S^T through
//   Kh, E dS'^T through Ke, dP and dA through the pair decays F; the decay gradient is
//   the reverse cumulative sum of the gamma gradient over the chunk.
//
// The launches:
//   1. the states at every 64-token boundary (the forward kernel of the shape, tcgen05 or
//      CUDA cores, writing checkpoints and no output) -> workspace;
//   2. the state gradient dS' entering chunks from above, walking the chunks backwards ->
//      workspace, and dS0: for bf16 with dk = dv = 128 the tcgen05 kernel's reverse
//      instantiation (64-token chunks; gradients at the span ends), else bwd_dstate_kernel
//      (CUDA cores, 32-token chunks, every chunk's end);
//   3. for bf16 with dk = dv = 128: bwd_tc_kernel (bwd_tc.cu), the per-chunk gradients of
//      every 64-token chunk on the tensor cores, listing the chunks whose cumulative decay
//      is too strong for its factorised form;
//   4. bwd_chunk_kernel: every 64-token span in parallel, or only the listed ones (its two
//      32-token chunks in turn; the first forms the middle state for the second), from S_c
//      and dS' -> dq, dk, dv, dg, db, dw.
// Pair decays are formed as exp(gamma_i - gamma_j) with i >= j, never as a product of two
// exponentials, so no factor overflows for a forgetting decay.  The CUDA-core kernels are
// fp32 throughout (states the tensor-core passes wrote are read as stored, in bf16).
#include <algorithm>
#include <type_traits>

#include "bwd_tc.cuh"
#include "chunk_tc.cuh"
#include "bounds.cuh"
#include "common.cuh"

namespace gdr {
namespace {

constexpr int C = kBwdChunk;
constexpr int kThreadsC = 512;          // the per-chunk kernel: 16 warps
constexpr int RW = C / (kThreadsC / 32); // rows of a tiled product per warp (2)

__device__ __forceinline__ float ld_b(const BwdArgs &a, size_t tk, int c) {   // erase gate b_tc
    return mode_b_vec(a.mode) ? ld_elem(a.b, tk * a.dk_ + c, a.dtype) : ld_elem(a.b, tk, a.dtype);
}
__device__ __forceinline__ float ld_w(const BwdArgs &a, size_t tk, int j) {   // write gate w_tj
    if (mode_w_vec(a.mode)) return ld_elem(a.w, tk * a.dv_ + j, a.dtype);
    return ld_elem(a.mode == GDR_MODE_BONLY ? a.w : a.b, tk, a.dtype);
}
// element idx of a state slot: fp32, or bf16 [dk][dv] at the slot's start (the tensor-core
// passes' checkpoints and span-end state gradients)
__device__ __forceinline__ float ld_state(const float *slot, size_t idx, bool bf) {
    return bf ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(slot)[idx]) : slot[idx];
}
__device__ __forceinline__ float ld_g(const BwdArgs &a, size_t tk, int c) {
    return a.mode == GDR_MODE_GDN ? a.g[tk] : a.g[tk * a.dk_ + c];
}

// The chunk's raw q, k, b (expanded to dk channels) and gamma into shared memory ([C][dk]
// each; tokens past the end are zero, so they neither decay nor write), gamma_C, and the
// C x C matrices A (strictly lower), P (lower incl.) and T = (I + A)^-1.  All threads of
// the block call it; it ends with a barrier.
__device__ void chunk_core(const BwdArgs &a, size_t tok0, int n, float *qq, float *kk, float *bb,
                           float *gm, float *gC, float *Am, float *Tm, float *Pm) {
    const int dk = a.dk_, tid = threadIdx.x, nth = blockDim.x;
    for (int idx = tid; idx < C * dk; idx += nth) {
        const int t = idx / dk, d = idx - t * dk;
        float qv = 0.f, kv = 0.f, bv = 0.f, gv = 0.f;
        if (t < n) {
            const size_t tk = tok0 + t;
            qv = ld_elem(a.q, tk * dk + d, a.dtype);
            kv = ld_elem(a.k, tk * dk + d, a.dtype);
            bv = ld_b(a, tk, d);
            gv = ld_g(a, tk, d);
        }
        qq[idx] = qv;
        kk[idx] = kv;
        bb[idx] = bv;
        gm[idx] = gv;
    }
    __syncthreads();
    for (int d = tid; d < dk; d += nth) {
        float acc = 0.f;
        for (int t = 0; t < C; ++t) {
            acc += gm[t * dk + d];
            gm[t * dk + d] = acc;
        }
        gC[d] = acc;
    }
    __syncthreads();
    constexpr int npairs = C * (C + 1) / 2;
    for (int p = tid; p < npairs; p += nth) {
        int i = (int)((sqrtf(8.f * p + 1.f) - 1.f) * 0.5f);
        while (i * (i + 1) / 2 > p) --i;
        while ((i + 1) * (i + 2) / 2 <= p) ++i;
        const int j = p - i * (i + 1) / 2;
        float av = 0.f, pv = 0.f;
        for (int cc = 0; cc < dk; ++cc) {
            const int c = (cc + (tid & 31)) & (dk - 1);   // staggered: no bank conflicts
            const float e = kk[j * dk + c] * __expf(gm[i * dk + c] - gm[j * dk + c]);
            av = fmaf(bb[i * dk + c] * kk[i * dk + c], e, av);
            pv = fmaf(qq[i * dk + c], e, pv);
        }
        Am[i * C + j] = (j < i) ? av : 0.f;
        Am[j * C + i] = 0.f;
        Pm[i * C + j] = pv;
        if (j < i) Pm[j * C + i] = 0.f;
    }
    __syncthreads();
    for (int j = tid; j < C; j += nth) {   // T: one column per thread, forward substitution
        for (int i = 0; i <= j; ++i) Tm[i * C + j] = (i == j) ? 1.f : 0.f;
        for (int i = j + 1; i < C; ++i) {
            float acc = 0.f;
            for (int m = j; m < i; ++m) acc = fmaf(Am[i * C + m], Tm[m * C + j], acc);
            Tm[i * C + j] = -acc;
        }
    }
    __syncthreads();
}

// The state-gradient kernel keeps a whole head's dS (all dv columns) in one CTA of
// kThreadsS threads: one wave of B*H CTAs, and A, P, T formed once per chunk.
constexpr int kThreadsS = 1024;
__host__ __device__ inline int dslice(int dv) { return dv; }

// Register-tiled product over shared-memory operands, for a 32-row result: warp w owns rows
// RW w .. RW w + RW - 1 and lane l the columns l + 32 e (e < NE, columns below n only):
//   acc[r][e] += sum_{k in [k0, k1)} A(RW w + r, k) * B(k, l + 32 e)
// Per k a warp loads RW A values (one address each, broadcast) and NE B values (32
// consecutive columns) for RW * NE multiply-adds.
template <int RWT, int NE, class FA, class FB>
__device__ __forceinline__ void tile_mm_rw(float (&acc)[RWT][NE], int k0, int k1, int n, FA A, FB Bop) {
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    for (int k = k0; k < k1; ++k) {
        float av[RWT], bv[NE];
#pragma unroll
        for (int r = 0; r < RWT; ++r) av[r] = A(RWT * w + r, k);
#pragma unroll
        for (int e = 0; e < NE; ++e) bv[e] = (l + 32 * e < n) ? Bop(k, l + 32 * e) : 0.f;
#pragma unroll
        for (int r = 0; r < RWT; ++r)
#pragma unroll
            for (int e = 0; e < NE; ++e) acc[r][e] = fmaf(av[r], bv[e], acc[r][e]);
    }
}
template <int NE, class FA, class FB>
__device__ __forceinline__ void tile_mm(float (&acc)[RW][NE], int k0, int k1, int n, FA A, FB Bop) {
    tile_mm_rw<RW, NE>(acc, k0, k1, n, A, Bop);
}

__host__ __device__ inline size_t dstate_smem_floats(int dk, int VS) {
    return 4 * (size_t)C * dk + dk + 3 * (size_t)C * C + (size_t)dk * VS + 3 * (size_t)C * VS;
}

// Launch 2: the state gradient, chunks in reverse.  One CTA per sequence-head holding all
// dv columns of dS (the columns are independent, so a slice of VS columns would also do).
template <int NE>
__global__ void __launch_bounds__(kThreadsS, 1) bwd_dstate_kernel(BwdArgs a) {
    const int dk = a.dk_, dv = a.dv_, T = a.T;
    const int VS = dslice(dv);
    const int bh = blockIdx.x, v0 = blockIdx.y * VS;
    const int tid = threadIdx.x, nth = blockDim.x;
    extern __shared__ float sm[];
    float *qq = sm, *kk = qq + C * dk, *bb = kk + C * dk, *gm = bb + C * dk;
    float *gC = gm + C * dk;
    float *Am = gC + dk, *Tm = Am + C * C, *Pm = Tm + C * C;
    float *dS = Pm + C * C;          // [dk][VS]: gradient with respect to the chunk's end state
    float *dO = dS + dk * VS;        // [C][VS]
    float *dE = dO + C * VS;         // [C][VS]
    float *dR = dE + C * VS;         // [C][VS]
    const int nc = (T + C - 1) / C;
    const size_t tok0 = (size_t)bh * T;
    // debug build: this job's sequence-head and value slice exist (uniform: return before any barrier)
    if (!GDR_IN_BOUNDS(bh < a.B * a.H && v0 + VS <= dv, 401)) return;

    for (int idx = tid; idx < dk * VS; idx += nth) {
        const int d = idx / VS, j = idx - d * VS;
        dS[idx] = a.dST ? a.dST[((size_t)bh * dk + d) * dv + v0 + j] : 0.f;
    }
    for (int c = nc - 1; c >= 0; --c) {
        const int t0 = c * C, n = min(C, T - t0);
        __syncthreads();
        float *dst = a.ws_dstates + ((size_t)bh * nc + c) * dk * dv + v0;
        for (int idx = tid; idx < dk * VS; idx += nth) {
            const int d = idx / VS, j = idx - d * VS;
            dst[(size_t)d * dv + j] = dS[idx];
        }
        for (int idx = tid; idx < C * VS; idx += nth) {
            const int t = idx / VS, j = idx - t * VS;
            dO[idx] = t < n ? ld_elem(a.dO, (tok0 + t0 + t) * dv + v0 + j, a.dtype) : 0.f;
        }
        chunk_core(a, tok0 + t0, n, qq, kk, bb, gm, gC, Am, Tm, Pm);
        // decayed operands in place: Ke = k e^(gamma_C - gamma), Qg = q e^gamma, Kh = b k e^gamma
        for (int idx = tid; idx < C * dk; idx += nth) {
            const int d = idx % dk;
            const float gam = gm[idx], e = __expf(gam);
            bb[idx] *= kk[idx] * e;
            qq[idx] *= e;
            kk[idx] *= __expf(gC[d] - gam);
        }
        __syncthreads();
        // Register-tiled products (tile_mm_rw): 32 warps, row r of warp w, columns lane + 32 e
        const int w = tid >> 5, lane = tid & 31;
        // dE = P^T dO + Ke dS  (one row per warp; P is zero above its diagonal)
        {
            float acc[1][NE] = {};
            tile_mm_rw<1, NE>(acc, w, C, VS, [&](int j, int t) { return Pm[t * C + j]; },
                              [&](int t, int v) { return dO[t * VS + v]; });
            tile_mm_rw<1, NE>(acc, 0, dk, VS, [&](int j, int d) { return kk[j * dk + d]; },
                              [&](int d, int v) { return dS[d * VS + v]; });
#pragma unroll
            for (int e = 0; e < NE; ++e)
                if (lane + 32 * e < VS) dE[w * VS + lane + 32 * e] = acc[0][e];
        }
        __syncthreads();
        // dR = T^T dE  (T lower triangular)
        {
            float acc[1][NE] = {};
            tile_mm_rw<1, NE>(acc, w, C, VS, [&](int i, int j) { return Tm[j * C + i]; },
                              [&](int j, int v) { return dE[j * VS + v]; });
#pragma unroll
            for (int e = 0; e < NE; ++e)
                if (lane + 32 * e < VS) dR[w * VS + lane + 32 * e] = acc[0][e];
        }
        __syncthreads();
        // dS <- e^gamma_C dS + Qg^T dO - Kh^T dR   (the gradient with respect to S_c); four
        // key-channel rows per warp, 128 at most
        {
            float acc[4][NE] = {};
            tile_mm_rw<4, NE>(acc, 0, C, VS, [&](int d, int t) { return d < dk ? qq[t * dk + d] : 0.f; },
                              [&](int t, int v) { return dO[t * VS + v]; });
            tile_mm_rw<4, NE>(acc, 0, C, VS, [&](int d, int t) { return d < dk ? -bb[t * dk + d] : 0.f; },
                              [&](int t, int v) { return dR[t * VS + v]; });
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int d = 4 * w + r;
                if (d < dk) {
                    const float eg = __expf(gC[d]);
#pragma unroll
                    for (int e = 0; e < NE; ++e) {
                        const int v = lane + 32 * e;
                        if (v < VS) dS[d * VS + v] = fmaf(eg, dS[d * VS + v], acc[r][e]);
                    }
                }
            }
        }
    }
    __syncthreads();
    if (a.dS0) {
        for (int idx = tid; idx < dk * VS; idx += nth) {
            const int d = idx / VS, j = idx - d * VS;
            a.dS0[((size_t)bh * dk + d) * dv + v0 + j] = dS[idx];
        }
    }
}

__host__ __device__ inline size_t chunk_smem_floats(int dk, int dv) {
    return 5 * (size_t)C * dk + 2 * (size_t)dk + 5 * (size_t)C * C + 3 * (size_t)C * dv +
           (size_t)dk * (dv + 1) + 3 * (size_t)C;
}

// Launch 3: every 64-token span in parallel, its two 32-token chunks in turn.  The
// checkpoint pass stored the state at the span's start; the first chunk also forms the
// state at the span's middle, S_mid = e^gamma_C S + Ke^T E, for the second.  Thread
// (c = tid % dk, group tid / dk) owns key channel c of RPG consecutive tokens and
// accumulates their dq, dk, db and d gamma in registers.
template <int RPG, int NE>
__global__ void __launch_bounds__(kThreadsC, 1) bwd_chunk_kernel(BwdArgs a) {
    const int dk = a.dk_, dv = a.dv_, T = a.T;
    const int nc = (T + C - 1) / C, nspan = (T + 2 * C - 1) / (2 * C);
    const int tid = threadIdx.x, nth = blockDim.x;
    // this CTA's span, or with tc_list every gridDim.x-th listed span
    const int njobs = a.tc_list ? a.tc_list[0] : (int)gridDim.x;
  // debug build: the span list holds no more entries than there are spans
  if (!GDR_IN_BOUNDS(njobs <= a.B * a.H * nspan, 403)) return;
  for (int job = blockIdx.x; job < njobs; job += gridDim.x) {
    const int blk = a.tc_list ? a.tc_list[1 + job] : job;
    const int bh = blk / nspan, span = blk - bh * nspan;
    // debug build: a valid span (the same for every thread of the CTA: skipped together)
    if (!GDR_IN_BOUNDS(blk >= 0 && blk < a.B * a.H * nspan, 402)) continue;
    __syncthreads();   // the previous span's shared-memory reads are done
    if (a.mid_grad && 2 * span + 1 < nc) {
        // The state gradient at the span's middle, from its end by one step of the reverse
        // recurrence over the second chunk: dS_mid = e^gamma_C dS_end + Qg^T dO - Kh^T dR
        // with dR = T^T (P^T dO + Ke dS_end)  -> the first chunk's slot of ws_dstates.
        const int c1 = 2 * span + 1, t1 = c1 * C, n1 = min(C, T - t1);
        const size_t tk1 = (size_t)bh * T + t1;
        const int SLD = dv + 1;
        extern __shared__ float sm[];
        float *qq = sm, *kk = qq + C * dk, *bb = kk + C * dk, *gm = bb + C * dk;
        float *ex = gm + C * dk, *gC = ex + C * dk;
        float *Am = gC + 2 * dk, *Tm = Am + C * C, *Pm = Tm + C * C;
        float *X1 = Pm + 3 * C * C, *X2 = X1 + C * dv, *X3 = X2 + C * dv, *Ss = X3 + C * dv;
        const float *dSe = a.ws_dstates + ((size_t)bh * nc + c1) * dk * dv;
        float *dSm = a.ws_dstates + ((size_t)bh * nc + c1 - 1) * dk * dv;
        for (int idx = tid; idx < C * dv; idx += nth) {
            const int t = idx / dv, j = idx - t * dv;
            X1[idx] = t < n1 ? ld_elem(a.dO, (tk1 + t) * dv + j, a.dtype) : 0.f;
        }
        for (int idx = tid; idx < dk * dv; idx += nth)
            Ss[(idx / dv) * SLD + idx % dv] = ld_state(dSe, idx, a.ckpt_bf16);
        chunk_core(a, tk1, n1, qq, kk, bb, gm, gC, Am, Tm, Pm);
        for (int idx = tid; idx < C * dk; idx += nth) {   // Ke, Qg, Kh
            const int d = idx % dk;
            const float e = __expf(gm[idx]);
            ex[idx] = kk[idx] * __expf(gC[d] - gm[idx]);
            qq[idx] *= e;
            bb[idx] *= kk[idx] * e;
        }
        __syncthreads();
        const int wrow = RW * (tid >> 5), lane = tid & 31;
        {   // dE = P^T dO + Ke dS_end -> X3
            float acc[RW][NE] = {};
            tile_mm<NE>(acc, wrow, C, dv, [&](int j, int t) { return Pm[t * C + j]; },
                        [&](int t, int v) { return X1[t * dv + v]; });
            tile_mm<NE>(acc, 0, dk, dv, [&](int j, int d) { return ex[j * dk + d]; },
                        [&](int d, int v) { return Ss[d * SLD + v]; });
#pragma unroll
            for (int r = 0; r < RW; ++r)
#pragma unroll
                for (int e = 0; e < NE; ++e)
                    if (lane + 32 * e < dv) X3[(wrow + r) * dv + lane + 32 * e] = acc[r][e];
        }
        __syncthreads();
        {   // dR = T^T dE -> X2
            float acc[RW][NE] = {};
            tile_mm<NE>(acc, wrow, C, dv, [&](int i, int j) { return Tm[j * C + i]; },
                        [&](int j, int v) { return X3[j * dv + v]; });
#pragma unroll
            for (int r = 0; r < RW; ++r)
#pragma unroll
                for (int e = 0; e < NE; ++e)
                    if (lane + 32 * e < dv) X2[(wrow + r) * dv + lane + 32 * e] = acc[r][e];
        }
        __syncthreads();
        {   // dS_mid, eight key-channel rows per warp (128 at most)
            constexpr int RK = 8;
            const int w = tid >> 5;
            float acc[RK][NE] = {};
            tile_mm_rw<RK, NE>(acc, 0, C, dv, [&](int d, int t) { return d < dk ? qq[t * dk + d] : 0.f; },
                               [&](int t, int v) { return X1[t * dv + v]; });
            tile_mm_rw<RK, NE>(acc, 0, C, dv, [&](int d, int t) { return d < dk ? -bb[t * dk + d] : 0.f; },
                               [&](int t, int v) { return X2[t * dv + v]; });
#pragma unroll
            for (int r = 0; r < RK; ++r) {
                const int d = RK * w + r;
                if (d < dk) {
                    const float eg = __expf(gC[d]);
#pragma unroll
                    for (int e = 0; e < NE; ++e) {
                        const int v = lane + 32 * e;
                        if (v < dv) dSm[(size_t)d * dv + v] = fmaf(eg, Ss[d * SLD + v], acc[r][e]);
                    }
                }
            }
        }
    }
  for (int hf = 0; hf < 2; ++hf) {
    const int c_idx = 2 * span + hf;
    if (c_idx >= nc) break;
    const int t0 = c_idx * C, n = min(C, T - t0);
    const size_t tok0 = (size_t)bh * T + t0;
    const bool make_mid = hf == 0 && c_idx + 1 < nc;   // the second chunk needs S_mid
    __syncthreads();
    const int ch = tid % dk, i0 = (tid / dk) * RPG;   // this thread's channel and first token
    const int SLD = dv + 1;                            // padded row stride of the state tile

    extern __shared__ float sm[];
    float *qq = sm, *kk = qq + C * dk, *bb = kk + C * dk, *gm = bb + C * dk;
    float *ex = gm + C * dk;         // [C][dk]: Kh = b k e^gamma, later Ke = k e^(gamma_C - gamma)
    float *gC = ex + C * dk, *dgC = gC + dk;
    float *Am = dgC + dk, *Tm = Am + C * C, *Pm = Tm + C * C, *dA = Pm + C * C, *dP = dA + C * C;
    float *X1 = dP + C * C;          // [C][dv]: dO, then dR
    float *X2 = X1 + C * dv;         // [C][dv]: w.v, then R
    float *X3 = X2 + C * dv;         // [C][dv]: E, then dE
    float *Ss = X3 + C * dv;         // [dk][dv+1]: S_c, then dS', then S_c
    float *fb = Ss + dk * SLD;       // [C]: folded scalar erase-gate gradient
    float *fw = fb + C;              // [C]: folded scalar write-gate gradient
    float *fg = fw + C;              // [C]: folded scalar decay gradient
    float *Sg = a.ws_states + ((size_t)bh * nc + c_idx) * dk * dv;
    const float *dSg = a.ws_dstates + ((size_t)bh * nc + c_idx) * dk * dv;
    // slots the tensor-core passes wrote (bf16): the span's start state, and the state
    // gradient at the span's end (slot 2 span + 1, or 2 span for a one-chunk last span)
    const bool s_bf = a.ckpt_bf16 && hf == 0;
    const bool ds_bf = a.ckpt_bf16 && (hf == 1 || c_idx + 1 >= nc);

    float aq[RPG], ak[RPG], ab[RPG], ag[RPG];
#pragma unroll
    for (int r = 0; r < RPG; ++r) aq[r] = ak[r] = ab[r] = ag[r] = 0.f;

    // ---- inputs, S_c, and the chunk's A, P, T ----
    for (int idx = tid; idx < C * dv; idx += nth) {
        const int t = idx / dv, j = idx - t * dv;
        float x = 0.f, o = 0.f;
        if (t < n) {
            x = ld_w(a, tok0 + t, j) * ld_elem(a.v, (tok0 + t) * dv + j, a.dtype);
            o = ld_elem(a.dO, (tok0 + t) * dv + j, a.dtype);
        }
        X2[idx] = x;
        X1[idx] = o;
    }
    for (int idx = tid; idx < dk * dv; idx += nth) {
        const int d = idx / dv, j = idx - d * dv;
        Ss[d * SLD + j] = ld_state(Sg, idx, s_bf);
    }
    for (int i = tid; i < C; i += nth) fb[i] = fw[i] = fg[i] = 0.f;
    for (int d = tid; d < dk; d += nth) dgC[d] = 0.f;
    chunk_core(a, tok0, n, qq, kk, bb, gm, gC, Am, Tm, Pm);
    for (int idx = tid; idx < C * dk; idx += nth) ex[idx] = bb[idx] * kk[idx] * __expf(gm[idx]);
    __syncthreads();
    const int wrow = RW * (tid >> 5), lane = tid & 31;   // tile_mm's rows and first column
    // ---- R = w.v - Kh S ----
    {
        float acc[RW][NE] = {};
        tile_mm<NE>(acc, 0, dk, dv, [&](int i, int d) { return ex[i * dk + d]; },
                    [&](int d, int j) { return Ss[d * SLD + j]; });
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int e = 0; e < NE; ++e)
                if (lane + 32 * e < dv) X2[(wrow + r) * dv + lane + 32 * e] -= acc[r][e];
    }
    __syncthreads();
    // ---- E = T R  (T is zero above its diagonal);  DY = dO S^T (into dq and d gamma) ----
    {
        float acc[RW][NE] = {};
        tile_mm<NE>(acc, 0, wrow + RW, dv, [&](int i, int m) { return Tm[i * C + m]; },
                    [&](int m, int j) { return X2[m * dv + j]; });
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int e = 0; e < NE; ++e)
                if (lane + 32 * e < dv) X3[(wrow + r) * dv + lane + 32 * e] = acc[r][e];
    }
    {
        float y[RPG];
#pragma unroll
        for (int r = 0; r < RPG; ++r) y[r] = 0.f;
        for (int j = 0; j < dv; ++j) {
            const float s = Ss[ch * SLD + j];
#pragma unroll
            for (int r = 0; r < RPG; ++r) y[r] = fmaf(X1[(i0 + r) * dv + j], s, y[r]);
        }
#pragma unroll
        for (int r = 0; r < RPG; ++r) {
            const int i = i0 + r;
            const float e = __expf(gm[i * dk + ch]);
            aq[r] = fmaf(e, y[r], aq[r]);
            ag[r] = fmaf(qq[i * dk + ch] * e, y[r], ag[r]);
        }
    }
    __syncthreads();
    // Ke = k e^(gamma_C - gamma) in place of e^gamma (e^gamma is recomputed where still needed)
    for (int idx = tid; idx < C * dk; idx += nth) {
        const int d = idx % dk;
        ex[idx] = kk[idx] * __expf(gC[d] - gm[idx]);
    }
    __syncthreads();
    if (make_mid) {
        // S_mid = e^gamma_C S + Ke^T E  -> the second chunk's checkpoint slot
        float *Sm = Sg + (size_t)dk * dv;
        for (int d0 = 0; d0 < dk; d0 += C) {   // 32 rows (key channels) of S_mid at a time
            float acc[RW][NE] = {};
            tile_mm<NE>(acc, 0, C, dv, [&](int d, int t) { return d0 + d < dk ? ex[t * dk + d0 + d] : 0.f; },
                        [&](int t, int j) { return X3[t * dv + j]; });
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                const int d = d0 + wrow + r;
                if (d < dk) {
                    const float eg = __expf(gC[d]);
#pragma unroll
                    for (int e = 0; e < NE; ++e) {
                        const int j = lane + 32 * e;
                        if (j < dv) Sm[(size_t)d * dv + j] = fmaf(eg, Ss[d * SLD + j], acc[r][e]);
                    }
                }
            }
        }
        __syncthreads();
    }
    // ---- dP = lower_incl(dO E^T); dS' replaces S_c; rowsum(S_c . dS') into d gamma_C ----
    for (int p = tid; p < C * C; p += nth) {
        const int t = p / C, j = p - t * C;
        float acc = 0.f;
        if (j <= t)
            for (int v0 = 0; v0 < dv; ++v0) {
                const int v = (v0 + (tid & 31)) & (dv - 1);   // staggered: no bank conflicts
                acc = fmaf(X1[t * dv + v], X3[j * dv + v], acc);
            }
        dP[p] = acc;
    }
    for (int idx = tid; idx < dk * dv; idx += nth) {
        const int d = idx / dv, j = idx - d * dv;
        Ss[d * SLD + j] = ld_state(dSg, idx, ds_bf);
    }
    if (tid < dk) {
        float acc = 0.f;
        for (int j = 0; j < dv; ++j)
            acc = fmaf(ld_state(Sg, (size_t)tid * dv + j, s_bf), ld_state(dSg, (size_t)tid * dv + j, ds_bf), acc);
        dgC[tid] = __expf(gC[tid]) * acc;
    }
    __syncthreads();
    // ---- DK = E dS'^T (into dk, d gamma, d gamma_C), through Ke = k e^(gamma_C - gamma) ----
    {
        float y[RPG];
#pragma unroll
        for (int r = 0; r < RPG; ++r) y[r] = 0.f;
        for (int j = 0; j < dv; ++j) {
            const float s = Ss[ch * SLD + j];
#pragma unroll
            for (int r = 0; r < RPG; ++r) y[r] = fmaf(X3[(i0 + r) * dv + j], s, y[r]);
        }
        float part = 0.f;
#pragma unroll
        for (int r = 0; r < RPG; ++r) {
            const int i = i0 + r;
            const float f = __expf(gC[ch] - gm[i * dk + ch]);
            const float kf = kk[i * dk + ch] * f;
            ak[r] = fmaf(f, y[r], ak[r]);
            ag[r] = fmaf(-kf, y[r], ag[r]);
            part = fmaf(kf, y[r], part);
        }
        atomicAdd(&dgC[ch], part);
    }
    __syncthreads();
    // ---- dE = P^T dO + Ke dS'  (E is no longer needed; P is zero above its diagonal) ----
    {
        float acc[RW][NE] = {};
        tile_mm<NE>(acc, wrow, C, dv, [&](int j, int t) { return Pm[t * C + j]; },
                    [&](int t, int v) { return X1[t * dv + v]; });
        tile_mm<NE>(acc, 0, dk, dv, [&](int j, int d) { return ex[j * dk + d]; },
                    [&](int d, int v) { return Ss[d * SLD + v]; });
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int e = 0; e < NE; ++e)
                if (lane + 32 * e < dv) X3[(wrow + r) * dv + lane + 32 * e] = acc[r][e];
    }
    __syncthreads();
    // ---- dR = T^T dE (dO is no longer needed); dT = dE R^T into dA ----
    {
        float acc[RW][NE] = {};
        tile_mm<NE>(acc, wrow, C, dv, [&](int i, int j) { return Tm[j * C + i]; },
                    [&](int j, int v) { return X3[j * dv + v]; });
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int e = 0; e < NE; ++e)
                if (lane + 32 * e < dv) X1[(wrow + r) * dv + lane + 32 * e] = acc[r][e];
    }
    for (int p = tid; p < C * C; p += nth) {
        const int i = p / C, j = p - i * C;
        float acc = 0.f;
        for (int v0 = 0; v0 < dv; ++v0) {
            const int v = (v0 + (tid & 31)) & (dv - 1);
            acc = fmaf(X3[i * dv + v], X2[j * dv + v], acc);
        }
        dA[p] = acc;
    }
    __syncthreads();
    // ---- dA = strict_lower(-T^T dT T^T): M = dT T^T into Am (A itself is done with) ----
    for (int p = tid; p < C * C; p += nth) {
        const int i = p / C, j = p - i * C;
        float acc = 0.f;
        for (int m0 = 0; m0 < C; ++m0) {
            const int m = (m0 + (tid & 31)) & (C - 1);
            if (m <= j) acc = fmaf(dA[i * C + m], Tm[j * C + m], acc);
        }
        Am[p] = acc;
    }
    __syncthreads();
    for (int p = tid; p < C * C; p += nth) {
        const int i = p / C, j = p - i * C;
        float acc = 0.f;
        if (j < i)
            for (int m = i; m < C; ++m) acc = fmaf(Tm[m * C + i], Am[m * C + j], acc);
        dA[p] = -acc;
    }
    // ---- dv = dR.w, dw = dR.v (scalar write gates fold over the value channels); S_c back ----
    for (int idx = tid; idx < C * dv; idx += nth) {
        const int t = idx / dv, j = idx - t * dv;
        if (t < n) {
            const size_t tk = tok0 + t;
            const float r = X1[idx];
            st_elem(a.dv, tk * dv + j, a.dtype, r * ld_w(a, tk, j));
            const float gw = r * ld_elem(a.v, tk * dv + j, a.dtype);
            if (mode_w_vec(a.mode)) st_elem(a.dw, tk * dv + j, a.dtype, gw);
            else atomicAdd(&fw[t], gw);
        }
    }
    for (int idx = tid; idx < dk * dv; idx += nth) {
        const int d = idx / dv, j = idx - d * dv;
        Ss[d * SLD + j] = ld_state(Sg, idx, s_bf);
    }
    __syncthreads();
    // ---- DX = dR S^T (through Kh = b k e^gamma, with a minus sign: R = w.v - Kh S) ----
    {
        float y[RPG];
#pragma unroll
        for (int r = 0; r < RPG; ++r) y[r] = 0.f;
        for (int j = 0; j < dv; ++j) {
            const float s = Ss[ch * SLD + j];
#pragma unroll
            for (int r = 0; r < RPG; ++r) y[r] = fmaf(X1[(i0 + r) * dv + j], s, y[r]);
        }
#pragma unroll
        for (int r = 0; r < RPG; ++r) {
            const int i = i0 + r;
            const float e = __expf(gm[i * dk + ch]);
            const float kv = kk[i * dk + ch], bv = bb[i * dk + ch];
            ab[r] = fmaf(-kv * e, y[r], ab[r]);
            ak[r] = fmaf(-bv * e, y[r], ak[r]);
            ag[r] = fmaf(-bv * kv * e, y[r], ag[r]);
        }
    }
    // ---- pair terms of P and A, exact decays F_ij = exp(gamma_i - gamma_j), i >= j ----
#pragma unroll
    for (int r = 0; r < RPG; ++r) {
        const int i = i0 + r;
        const float gi = gm[i * dk + ch], qi = qq[i * dk + ch], ki = kk[i * dk + ch], bi = bb[i * dk + ch];
        float sq = 0.f, sk = 0.f, sb = 0.f, sg = 0.f;
        for (int j = 0; j <= i; ++j) {   // row terms: token i pairs with earlier tokens j
            const float f = __expf(gi - gm[j * dk + ch]);
            const float kj = kk[j * dk + ch] * f;
            const float p = dP[i * C + j], al = dA[i * C + j];
            sq = fmaf(p, kj, sq);
            sk = fmaf(al * bi, kj, sk);
            sb = fmaf(al * ki, kj, sb);
            sg = fmaf(p * qi + al * bi * ki, kj, sg);
        }
        float ck = 0.f, cg = 0.f;
        for (int m = i; m < C; ++m) {     // column terms: token i pairs with later tokens m
            const float f = __expf(gm[m * dk + ch] - gi);
            const float u = (dP[m * C + i] * qq[m * dk + ch] + dA[m * C + i] * bb[m * dk + ch] * kk[m * dk + ch]) * f;
            ck += u;
            cg = fmaf(-u, ki, cg);
        }
        aq[r] += sq;
        ak[r] += sk + ck;
        ab[r] += sb;
        ag[r] += sg + cg;
    }
    __syncthreads();
    // ---- d gamma -> d g (reverse cumulative sum over the chunk, gamma_C on the last token) ----
#pragma unroll
    for (int r = 0; r < RPG; ++r) qq[(i0 + r) * dk + ch] = ag[r];
    __syncthreads();
    for (int d = tid; d < dk; d += nth) {
        float acc = dgC[d];
        for (int t = C - 1; t >= 0; --t) {
            acc += qq[t * dk + d];
            qq[t * dk + d] = acc;
        }
    }
    __syncthreads();
    // ---- outputs ----
    const bool scalar_b = !mode_b_vec(a.mode), scalar_g = a.mode == GDR_MODE_GDN;
#pragma unroll
    for (int r = 0; r < RPG; ++r) {
        const int i = i0 + r;
        if (i < n) {
            const size_t tk = tok0 + i;
            st_elem(a.dq, tk * dk + ch, a.dtype, aq[r]);
            st_elem(a.dk, tk * dk + ch, a.dtype, ak[r]);
            if (scalar_b) atomicAdd(&fb[i], ab[r]);
            else st_elem(a.db, tk * dk + ch, a.dtype, ab[r]);
            if (scalar_g) atomicAdd(&fg[i], qq[i * dk + ch]);
            else a.dg[tk * dk + ch] = qq[i * dk + ch];
        }
    }
    __syncthreads();
    for (int i = tid; i < n; i += nth) {
        const size_t tk = tok0 + i;
        const bool tied = a.mode == GDR_MODE_KDA || a.mode == GDR_MODE_GDN;
        if (scalar_b) st_elem(a.db, tk, a.dtype, tied ? fb[i] + fw[i] : fb[i]);
        if (a.mode == GDR_MODE_BONLY) st_elem(a.dw, tk, a.dtype, fw[i]);
        if (scalar_g) a.dg[tk] = fg[i];
    }
  }
  }
}

}  // namespace

unsigned long long bwd_states_bytes(int B, int H, int T, int dk, int dv) {
    const unsigned long long nc = (unsigned long long)((T + C - 1) / C);
    return 2ull * (unsigned long long)B * H * nc * dk * dv * sizeof(float);
}

unsigned long long bwd_workspace_bytes(int B, int H, int T, int dk, int dv) {
    if (T <= 0) return 0;
    const unsigned long long nspan = (unsigned long long)((T + 2 * C - 1) / (2 * C));
    const unsigned long long list = (1ull + (unsigned long long)B * H * nspan) * sizeof(int);
    return bwd_states_bytes(B, H, T, dk, dv) + (list + 15) / 16 * 16;
}

gdr_status_t launch_bwd(const BwdArgs &a, cudaStream_t s) {
    // 1. checkpoints: the state at every 64-token boundary, from the forward kernel of the
    //    shape (the tcgen05 kernel for bf16, dk = dv = 128; else the fp32 CUDA-core one)
    ChunkArgs f{a.q, a.k, a.v, a.b, mode_uses_w(a.mode) ? a.w : nullptr, a.g, a.S0, nullptr, nullptr,
                a.B, a.H, a.T, a.dk_, a.dv_, 2 * C, a.mode, a.dtype,
                1, a.T, 0, nullptr, nullptr, nullptr,
                0, 1, nullptr, nullptr, 1.f, 0.f, a.ws_states, 0, nullptr};
    // the tensor-core path needs both the forward kernel (checkpoints, state gradient) and the
    // per-chunk kernel to take the shape
    const bool tc = chunk_tc_supported(f) && bwd_tc_supported(a);
    gdr_status_t st = tc ? launch_chunk_tc(f, s) : launch_chunk_simt(f, s);
    if (st != GDR_OK) return st;
    BwdArgs b = a;
    if (tc) {
        // 2. the state gradient on the tensor cores: the same kernel in reverse chunk order,
        //    writing the gradient at every 64-token span's end (the per-chunk kernel forms the
        //    middle ones) and dS0
        ChunkArgs r = f;
        r.S0 = a.dST;
        r.ST = a.dS0;
        r.chunk_states = a.ws_dstates;
        r.reverse = 1;
        r.dO = a.dO;
        if ((st = launch_chunk_tc(r, s)) != GDR_OK) return st;
        b.mid_grad = 1;
        b.ckpt_bf16 = 1;
        // 3. per-chunk gradients on the tensor cores; spans with a strong cumulative decay
        //    are listed for the CUDA-core kernel below
        b.tc_list = reinterpret_cast<int *>(reinterpret_cast<unsigned char *>(a.ws_states) +
                                            bwd_states_bytes(a.B, a.H, a.T, a.dk_, a.dv_));
        if (cudaMemsetAsync(b.tc_list, 0, sizeof(int), s) != cudaSuccess) return GDR_ERR_CUDA;
        if ((st = launch_bwd_tc(b, s)) != GDR_OK) return st;
    } else {
        // 2. state gradients on CUDA cores, chunks in reverse (every 32-token chunk's end)
        const int VS = dslice(a.dv_);
        const size_t smem2 = dstate_smem_floats(a.dk_, VS) * sizeof(float);
        auto kern2 = VS == 128 ? bwd_dstate_kernel<4> : VS == 64 ? bwd_dstate_kernel<2> : bwd_dstate_kernel<1>;
        if (cudaFuncSetAttribute(kern2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2) != cudaSuccess)
            return GDR_ERR_CUDA;
        kern2<<<dim3((unsigned)(a.B * a.H), (unsigned)(a.dv_ / VS)), kThreadsS, smem2, s>>>(a);
        if (cudaGetLastError() != cudaSuccess) return GDR_ERR_CUDA;
    }
    // 3. per-chunk gradients on CUDA cores, one CTA per 64-token span (with tc_list: the
    //    listed spans, over at most four CTAs per SM)
    const int nspan = (a.T + 2 * C - 1) / (2 * C);
    size_t grid = (size_t)a.B * a.H * nspan;
    if (b.tc_list) grid = std::min(grid, (size_t)4 * 148);
    const size_t smem3 = chunk_smem_floats(a.dk_, a.dv_) * sizeof(float);
    // RPG rows per thread for the (token, key channel) gradients; NE column groups of 32
    // for the tiled products over the value channels
    auto pick = [&](auto rpg) {
        constexpr int R = decltype(rpg)::value;
        return a.dv_ == 128 ? bwd_chunk_kernel<R, 4> : a.dv_ == 64 ? bwd_chunk_kernel<R, 2> : bwd_chunk_kernel<R, 1>;
    };
    auto kern = a.dk_ == 128 ? pick(std::integral_constant<int, C * 128 / kThreadsC>{})
              : a.dk_ == 64  ? pick(std::integral_constant<int, C * 64 / kThreadsC>{})
              : a.dk_ == 32  ? pick(std::integral_constant<int, C * 32 / kThreadsC>{})
                             : pick(std::integral_constant<int, C * 16 / kThreadsC>{});
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem3) != cudaSuccess)
        return GDR_ERR_CUDA;
    kern<<<(unsigned)grid, kThreadsC, smem3, s>>>(b);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

}  // namespace gdr

namespace gdr {
GDR_BOUNDS_READER(bwd_bounds_site)
}  // namespace gdr
