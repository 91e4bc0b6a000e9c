// tc_probe.cu -- test-only library: one tcgen05 GEMM D = (+/-) A B (optionally twice,
// accumulating) through the operand layouts and descriptors of the product kernels
// (tc_util.cuh), so each layout combination can be checked against a plain matmul.
//
// A [M x K] and B [K x N] are row-major bf16 in global memory; D [M x N] fp32.
// a_mn / b_mn select the MN-major form of the operand; r0 / pad place the operand's
// rows at an offset inside a taller tile (as the fused kernel does with stacked tiles).
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../linear_attention_recurrence_wy_b200/csrc/tc_util.cuh"

using namespace gdr::tc;

__global__ void __launch_bounds__(128) probe_kernel(const __nv_bfloat16 *A, const __nv_bfloat16 *B,
                                                    float *D, int M, int N, int K, int a_mn, int b_mn,
                                                    int neg_a, int reps, int a_r0, int a_pad,
                                                    int b_r0, int b_pad, int *status) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *base = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    // tile geometry
    const int RA = (a_mn ? K : M) + a_r0 + a_pad, CA = a_mn ? M : K;
    const int RB = (b_mn ? K : N) + b_r0 + b_pad, CB = b_mn ? N : K;
    unsigned char *tA = base;
    unsigned char *tB = tA + ((RA * CA * 2 + 1023) / 1024) * 1024;
    uint64_t *mbar = (uint64_t *)(tB + ((RB * CB * 2 + 1023) / 1024) * 1024);
    uint32_t *tslot = (uint32_t *)(mbar + 1);
    const int tid = threadIdx.x;

    for (int i = tid; i < RA * CA / 2; i += 128) ((uint32_t *)tA)[i] = 0u;
    for (int i = tid; i < RB * CB / 2; i += 128) ((uint32_t *)tB)[i] = 0u;
    __syncthreads();
    for (int i = tid; i < M * K; i += 128) {
        const int m = i / K, k = i % K;
        const int row = a_mn ? a_r0 + k : a_r0 + m, col = a_mn ? m : k;
        *(__nv_bfloat16 *)(tA + tile_off(RA, row, col)) = A[i];
    }
    for (int i = tid; i < K * N; i += 128) {
        const int k = i / N, n = i % N;
        const int row = b_mn ? b_r0 + k : b_r0 + n, col = b_mn ? n : k;
        *(__nv_bfloat16 *)(tB + tile_off(RB, row, col)) = B[i];
    }
    if (tid == 0) {
        mbar_init(smem_u32(mbar), 1);
        fence_mbar_init();
    }
    fence_async_smem();
    __syncthreads();
    if (tid < 32) {
        tmem_alloc(smem_u32(tslot), 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    if (tid == 0) {
        const uint32_t id = idesc_bf16(M, N, a_mn, b_mn, neg_a);
        for (int r = 0; r < reps; ++r)
            for (int s = 0; s < K / 16; ++s) {
                const uint64_t ad = a_mn ? desc_mnmajor(smem_u32(tA), RA, a_r0, s)
                                         : desc_kmajor(smem_u32(tA), RA, a_r0, s);
                const uint64_t bd = b_mn ? desc_mnmajor(smem_u32(tB), RB, b_r0, s)
                                         : desc_kmajor(smem_u32(tB), RB, b_r0, s);
                mma_bf16(tmem, ad, bd, id, (r > 0 || s > 0) ? 1u : 0u);
            }
        mma_commit(smem_u32(mbar));
    }
    const bool ok = mbar_wait(smem_u32(mbar), 0, 1u << 22);
    if (!ok) atomicExch(status, 1);
    tc_fence_after();
    const int warp = tid >> 5, lane = tid & 31;
    if (ok) {
        for (int c0 = 0; c0 < N; c0 += 32) {
            float v[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c0, v);
            tmem_wait_ld();
            const int row = warp * 32 + lane;
            if (row < M)
                for (int j = 0; j < 32; ++j) D[row * N + c0 + j] = v[j];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (tid < 32) tmem_dealloc(tmem, 256);
}

extern "C" int tc_probe_gemm(const void *A, const void *B, float *D, int M, int N, int K, int a_mn,
                             int b_mn, int neg_a, int reps, int a_r0, int a_pad, int b_r0, int b_pad,
                             int *status, void *stream) {
    if (M != 128 || N % 64 || N > 256 || K % 64 || K > 128 || a_r0 % 8 || b_r0 % 8 || a_pad % 8 ||
        b_pad % 8)
        return -2;
    const int RA = (a_mn ? K : M) + a_r0 + a_pad, CA = a_mn ? M : K;
    const int RB = (b_mn ? K : N) + b_r0 + b_pad, CB = b_mn ? N : K;
    const size_t smem = 1024 + ((RA * CA * 2 + 1023) / 1024) * 1024 +
                        ((RB * CB * 2 + 1023) / 1024) * 1024 + 64;
    if (smem > 227 * 1024) return -2;
    cudaFuncSetAttribute(probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    probe_kernel<<<1, 128, smem, (cudaStream_t)stream>>>(
        (const __nv_bfloat16 *)A, (const __nv_bfloat16 *)B, D, M, N, K, a_mn, b_mn, neg_a, reps,
        a_r0, a_pad, b_r0, b_pad, status);
    return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

// ---- the 64 x 64 triangular inverse of the chunk kernel, in isolation ----------------------
#include "../../linear_attention_recurrence_wy_b200/csrc/tri_inverse.cuh"

struct ProbeBar128 {
    __device__ __forceinline__ void operator()() const { asm volatile("bar.sync 1, 128;" ::: "memory"); }
};

__global__ void __launch_bounds__(128) tri_probe_kernel(const float *A, float *T) {
    __shared__ __align__(16) float sA[64 * gdr::tri::LD];
    __shared__ __align__(16) float sT[64 * gdr::tri::LD];
    __shared__ __align__(16) float sX[4 * 16 * gdr::tri::XLD];
    const float *Am = A + (size_t)blockIdx.x * 64 * 64;
    float *Tm = T + (size_t)blockIdx.x * 64 * 64;
    for (int i = threadIdx.x; i < 64 * 64; i += 128) {
        const int r = i / 64, c = i % 64;
        sA[r * gdr::tri::LD + c] = (c < r) ? Am[i] : 0.f;
    }
    __syncthreads();
    gdr::tri::inverse64(sA, sT, sX, threadIdx.x >> 5, threadIdx.x & 31, ProbeBar128{},
                         gdr::tri::NoOut{});
    __syncthreads();
    for (int i = threadIdx.x; i < 64 * 64; i += 128) {
        const int r = i / 64, c = i % 64;
        Tm[i] = (c <= r) ? sT[r * gdr::tri::LD + c] : 0.f;
    }
}

extern "C" int tc_probe_tri_inverse(const float *A, float *T, int n, void *stream) {
    if (n <= 0) return -2;
    tri_probe_kernel<<<n, 128, 0, (cudaStream_t)stream>>>(A, T);
    return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

// ---- A operand from tensor memory (TS form) ------------------------------------------------
// D = (+/-) A B (reps times, accumulating) with A [128 x K] packed into TMEM columns
// [256, 256 + K/2) and B in shared memory as in probe_kernel.
__global__ void __launch_bounds__(128) probe_ts_kernel(const __nv_bfloat16 *A, const __nv_bfloat16 *B,
                                                       float *D, int N, int K, int b_mn, int neg_a,
                                                       int reps, int *status) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *base = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int RB = b_mn ? K : N, CB = b_mn ? N : K;
    unsigned char *tB = base;
    uint64_t *mbar = (uint64_t *)(tB + ((RB * CB * 2 + 1023) / 1024) * 1024);
    uint32_t *tslot = (uint32_t *)(mbar + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < RB * CB / 2; i += 128) ((uint32_t *)tB)[i] = 0u;
    __syncthreads();
    for (int i = tid; i < K * N; i += 128) {
        const int k = i / N, n = i % N;
        const int row = b_mn ? k : n, col = b_mn ? n : k;
        *(__nv_bfloat16 *)(tB + tile_off(RB, row, col)) = B[i];
    }
    if (tid == 0) {
        mbar_init(smem_u32(mbar), 1);
        fence_mbar_init();
    }
    fence_async_smem();
    __syncthreads();
    if (tid < 32) {
        tmem_alloc(smem_u32(tslot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t lb = (uint32_t)(warp * 32) << 16;
    {
        // row tid of A -> lane tid, packed pairs along K
        const int row = tid;
        for (int k0 = 0; k0 < K; k0 += 32) {
            uint32_t r[16];
            for (int j = 0; j < 16; ++j) {
                const float lo = __bfloat162float(A[row * K + k0 + 2 * j]);
                const float hi = __bfloat162float(A[row * K + k0 + 2 * j + 1]);
                r[j] = pack_bf16(lo, hi);
            }
            tmem_st16(tmem + lb + 256 + k0 / 2, r);
        }
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        const uint32_t id = idesc_bf16(128, N, false, b_mn, neg_a);
        for (int r = 0; r < reps; ++r)
            for (int s = 0; s < K / 16; ++s) {
                const uint64_t bd = b_mn ? desc_mnmajor(smem_u32(tB), RB, 0, s)
                                         : desc_kmajor(smem_u32(tB), RB, 0, s);
                mma_bf16_ts(tmem, tmem + 256 + s * 8, bd, id, (r > 0 || s > 0) ? 1u : 0u);
            }
        mma_commit(smem_u32(mbar));
    }
    const bool ok = mbar_wait(smem_u32(mbar), 0, 1u << 22);
    if (!ok) atomicExch(status, 1);
    tc_fence_after();
    if (ok) {
        for (int c0 = 0; c0 < N; c0 += 32) {
            float v[32];
            tmem_ld32(tmem + lb + c0, v);
            tmem_wait_ld();
            for (int j = 0; j < 32; ++j) D[tid * N + c0 + j] = v[j];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (tid < 32) tmem_dealloc(tmem, 512);
}

extern "C" int tc_probe_gemm_ts(const void *A, const void *B, float *D, int N, int K, int b_mn,
                                int neg_a, int reps, int *status, void *stream) {
    if (N % 64 || N > 256 || K % 32 || K > 256) return -2;
    const int RB = b_mn ? K : N, CB = b_mn ? N : K;
    const size_t smem = 1024 + ((RB * CB * 2 + 1023) / 1024) * 1024 + 64;
    cudaFuncSetAttribute(probe_ts_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    probe_ts_kernel<<<1, 128, smem, (cudaStream_t)stream>>>((const __nv_bfloat16 *)A,
                                                              (const __nv_bfloat16 *)B, D, N, K,
                                                              b_mn, neg_a, reps, status);
    return cudaGetLastError() == cudaSuccess ? 0 : -6;
}
