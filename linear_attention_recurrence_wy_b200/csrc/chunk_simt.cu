// chunk_simt.cu -- fp32 CUDA-core chunkwise WY forward (any supported shape, fp32 or
// bf16 storage).
//
// One CTA owns one (sequence, head) and one slice of VS value columns of the state,
// and walks the chunks in order.  Per chunk of C tokens (Gated DeltaNet-2 Review
// §3-2.5, "Chunkwise WY training"; Gated DeltaNet-2 Q&A page, Q4):
//   gamma = chunk-local cumulative sum of g_log per key channel (fp32)
//   A_ij  = sum_c b_ic k_ic k_jc exp(gamma_ic - gamma_jc)   (j < i)
//   P_ij  = sum_c q_ic k_jc exp(gamma_ic - gamma_jc)        (j <= i)
//   T     = (I + A)^-1 by forward substitution
//   W     = T (b . k . exp(gamma)),   U = T (w . v)
//   E     = U - W S                    (delta errors of the chunk's tokens)
//   O     = (q . exp(gamma)) S + P E   (read-out of the post-update state)
//   S    <- diag(exp(gamma_C)) S + (k . exp(gamma_C - gamma))^T E
// The pair decays are formed as exp(gamma_i - gamma_j) with i >= j, which is <= 1
// for a forgetting decay, so no factor can overflow however strong the decay is.
// Everything is fp32 FFMA; this kernel carries the fp32 path and every shape the
// tensor-core kernel does not take.
#include "bounds.cuh"
#include "common.cuh"

namespace gdr {
namespace {

constexpr int kThreads = 256;

__host__ __device__ inline int slice_width(int dv) { return dv < 32 ? dv : 32; }

__host__ __device__ inline size_t simt_smem_floats(int C, int dk, int VS) {
    return 4 * (size_t)C * dk + 3 * (size_t)C * C + (size_t)dk * VS + 2 * (size_t)C * VS + dk;
}

__global__ void __launch_bounds__(kThreads) chunk_simt_kernel(ChunkArgs a) {
    const int C = a.chunk, dk = a.dk, dv = a.dv, T = a.T;
    const int VS = slice_width(dv);
    const int bh = blockIdx.x;
    const int v0 = blockIdx.y * VS;
    const int tid = threadIdx.x;
    const int nth = blockDim.x;
    // debug build: this job's sequence-head and value slice exist (uniform: the barriers below
    // are reached by every thread or by none)
    if (!GDR_IN_BOUNDS(bh < a.B * a.H && v0 + VS <= dv, 601)) return;

    extern __shared__ float sm[];
    float *kk = sm;               // [C][dk]  k, later k . exp(gamma_C - gamma)
    float *bk = kk + C * dk;      // [C][dk]  b . k, later b . k . exp(gamma)
    float *qq = bk + C * dk;      // [C][dk]  q, later q . exp(gamma)
    float *gm = qq + C * dk;      // [C][dk]  gamma, later W
    float *Am = gm + C * dk;      // [C][C]   A
    float *Tm = Am + C * C;       // [C][C]   T = (I + A)^-1
    float *Pm = Tm + C * C;       // [C][C]   P
    float *Ss = Pm + C * C;       // [dk][VS] state slice
    float *Es = Ss + dk * VS;     // [C][VS]  U, then E
    float *Vs = Es + C * VS;      // [C][VS]  w . v
    float *gC = Vs + C * VS;      // [dk]     gamma at the chunk's last token

    for (int idx = tid; idx < dk * VS; idx += nth) {
        const int d = idx / VS, j = idx - d * VS;
        Ss[idx] = a.S0 ? a.S0[((size_t)bh * dk + d) * dv + v0 + j] : 0.f;
    }
    const size_t tok0 = (size_t)bh * T;
    const int npairs = C * (C + 1) / 2;

    for (int c0 = 0; c0 < T; c0 += C) {
        const int n = min(C, T - c0);
        __syncthreads();
        if (a.chunk_states) {   // checkpoint: the state this chunk starts from, in the
                                // slot of its first 32-token chunk
            float *dst = a.chunk_states + ((size_t)bh * ((T + 31) / 32) + c0 / 32) * dk * dv + v0;
            for (int idx = tid; idx < dk * VS; idx += nth) {
                const int d = idx / VS, j = idx - d * VS;
                dst[(size_t)d * dv + j] = Ss[idx];
            }
        }
        // ---- load the chunk; tokens past the end are zero (exact padding) ----
        for (int idx = tid; idx < C * dk; idx += nth) {
            const int t = idx / dk, d = idx - t * dk;
            float kv = 0.f, qv = 0.f, bv = 0.f, gv = 0.f;
            if (t < n) {
                const size_t tk = tok0 + c0 + t;
                kv = ld_elem(a.k, tk * dk + d, a.dtype);
                qv = ld_elem(a.q, tk * dk + d, a.dtype);
                bv = mode_b_vec(a.mode) ? ld_elem(a.b, tk * dk + d, a.dtype) : ld_elem(a.b, tk, a.dtype);
                gv = (a.mode == GDR_MODE_GDN) ? a.g[tk] : a.g[tk * dk + d];
            }
            kk[idx] = kv;
            qq[idx] = qv;
            bk[idx] = bv * kv;
            gm[idx] = gv;
        }
        for (int idx = tid; idx < C * VS; idx += nth) {
            const int t = idx / VS, j = idx - t * VS;
            float x = 0.f;
            if (t < n) {
                const size_t tk = tok0 + c0 + t;
                const float vv = ld_elem(a.v, tk * dv + v0 + j, a.dtype);
                const float ww = mode_w_vec(a.mode) ? ld_elem(a.w, tk * dv + v0 + j, a.dtype)
                                 : ld_elem(a.mode == GDR_MODE_BONLY ? a.w : a.b, tk, a.dtype);
                x = ww * vv;
            }
            Vs[idx] = x;
        }
        __syncthreads();
        // ---- gamma: inclusive cumulative sum over the chunk, per key channel ----
        for (int d = tid; d < dk; d += nth) {
            float acc = 0.f;
            for (int t = 0; t < C; ++t) {
                acc += gm[t * dk + d];
                gm[t * dk + d] = acc;
            }
            gC[d] = acc;
        }
        __syncthreads();
        // ---- A (strictly lower) and P (lower incl. diagonal), exact pair decays ----
        for (int p = tid; p < npairs; p += nth) {
            int i = (int)((sqrtf(8.f * p + 1.f) - 1.f) * 0.5f);
            while (i * (i + 1) / 2 > p) --i;
            while ((i + 1) * (i + 2) / 2 <= p) ++i;
            const int j = p - i * (i + 1) / 2;
            float av = 0.f, pv = 0.f;
            const float *gi = gm + i * dk, *gj = gm + j * dk;
            const float *bi = bk + i * dk, *qi = qq + i * dk, *kj = kk + j * dk;
            for (int cc = 0; cc < dk; ++cc) {
                const int c = (cc + (tid & 31)) & (dk - 1);   // staggered: no bank conflicts
                const float e = kj[c] * __expf(gi[c] - gj[c]);
                av = fmaf(bi[c], e, av);
                pv = fmaf(qi[c], e, pv);
            }
            Am[i * C + j] = (j < i) ? av : 0.f;
            Am[j * C + i] = 0.f;
            Pm[i * C + j] = pv;
            if (j < i) Pm[j * C + i] = 0.f;
        }
        __syncthreads();
        // ---- T = (I + A)^-1: one column per thread, forward substitution ----
        for (int j = tid; j < C; j += nth) {
            for (int i = 0; i <= j; ++i) Tm[i * C + j] = (i == j) ? 1.f : 0.f;
            for (int i = j + 1; i < C; ++i) {
                float acc = 0.f;
                for (int m = j; m < i; ++m) acc = fmaf(Am[i * C + m], Tm[m * C + j], acc);
                Tm[i * C + j] = -acc;
            }
        }
        __syncthreads();
        // ---- decayed operands (in place) ----
        for (int idx = tid; idx < C * dk; idx += nth) {
            const int d = idx % dk;
            const float gam = gm[idx];
            const float e = __expf(gam);
            bk[idx] *= e;                          // b . k . exp(gamma)
            qq[idx] *= e;                          // q . exp(gamma)
            kk[idx] *= __expf(gC[d] - gam);        // k . exp(gamma_C - gamma)
        }
        __syncthreads();
        // ---- W = T (b k e^gamma) into gm;  U = T (w v) into Es ----
        for (int idx = tid; idx < C * dk; idx += nth) {
            const int i = idx / dk, d = idx - i * dk;
            float acc = 0.f;
            for (int m = 0; m <= i; ++m) acc = fmaf(Tm[i * C + m], bk[m * dk + d], acc);
            gm[idx] = acc;
        }
        for (int idx = tid; idx < C * VS; idx += nth) {
            const int i = idx / VS, j = idx - i * VS;
            float acc = 0.f;
            for (int m = 0; m <= i; ++m) acc = fmaf(Tm[i * C + m], Vs[m * VS + j], acc);
            Es[idx] = acc;
        }
        __syncthreads();
        // ---- E = U - W S ----
        for (int idx = tid; idx < C * VS; idx += nth) {
            const int i = idx / VS, j = idx - i * VS;
            float acc = Es[idx];
            for (int d = 0; d < dk; ++d) acc = fmaf(-gm[i * dk + d], Ss[d * VS + j], acc);
            Es[idx] = acc;
        }
        __syncthreads();
        // ---- O = Q_g S + P E for the chunk's real tokens ----
        for (int idx = tid; a.o && idx < n * VS; idx += nth) {
            const int t = idx / VS, j = idx - t * VS;
            float acc = 0.f;
            for (int d = 0; d < dk; ++d) acc = fmaf(qq[t * dk + d], Ss[d * VS + j], acc);
            for (int m = 0; m <= t; ++m) acc = fmaf(Pm[t * C + m], Es[m * VS + j], acc);
            st_elem(a.o, (tok0 + c0 + t) * dv + v0 + j, a.dtype, acc);
        }
        __syncthreads();
        // ---- S <- diag(exp(gamma_C)) S + K_end^T E ----
        for (int idx = tid; idx < dk * VS; idx += nth) {
            const int d = idx / VS, j = idx - d * VS;
            float acc = __expf(gC[d]) * Ss[idx];
            for (int t = 0; t < C; ++t) acc = fmaf(kk[t * dk + d], Es[t * VS + j], acc);
            Ss[idx] = acc;
        }
    }
    __syncthreads();
    if (a.ST) {
        for (int idx = tid; idx < dk * VS; idx += nth) {
            const int d = idx / VS, j = idx - d * VS;
            a.ST[((size_t)bh * dk + d) * dv + v0 + j] = Ss[idx];
        }
    }
}

__global__ void state_copy_kernel(const float *S0, float *ST, size_t n) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x)
        ST[i] = S0 ? S0[i] : 0.f;
}

}  // namespace

gdr_status_t launch_chunk_simt(const ChunkArgs &a, cudaStream_t s) {
    const int VS = slice_width(a.dv);
    const size_t smem = simt_smem_floats(a.chunk, a.dk, VS) * sizeof(float);
    if (cudaFuncSetAttribute(chunk_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return GDR_ERR_CUDA;
    dim3 grid((unsigned)(a.B * a.H), (unsigned)(a.dv / VS));
    chunk_simt_kernel<<<grid, kThreads, smem, s>>>(a);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

gdr_status_t launch_state_copy(const ChunkArgs &a, cudaStream_t s) {
    if (!a.ST) return GDR_OK;
    const size_t n = (size_t)a.B * a.H * a.dk * a.dv;
    if (n == 0) return GDR_OK;
    if (a.S0 == a.ST) return GDR_OK;
    state_copy_kernel<<<(unsigned)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096), 256, 0, s>>>(
        a.S0, a.ST, n);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

}  // namespace gdr

namespace gdr {
GDR_BOUNDS_READER(simt_bounds_site)
}  // namespace gdr
