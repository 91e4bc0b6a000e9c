// chunk_tc.cu -- tcgen05 tensor-core chunkwise WY forward: bf16 operands, fp32 state.
//
// Shape: dk = dv = 128, chunk C = 64, bf16 q/k/v/b/w/o, fp32 g_log and state, any mode.
// One CTA (256 threads) owns one (sequence, head); the fp32 state lives in tensor
// memory (TMEM) for the whole sequence, transposed (lane = value channel v, column =
// key channel d).  Per chunk (Gated DeltaNet-2 Review §3-2.5 "Chunkwise WY training";
// Gated DeltaNet-2 Q&A page, Q4):
//
//   gamma   = chunk-local cumulative sum of g_log (fp32, per key channel)
//   Kh      = b.k.e^gamma,  Qg = q.e^gamma,  Kb = k.e^-gamma,  WV = w.v      (bf16, smem)
//   [A; P]  = [Kh; Qg] Kb^T           one M=128 MMA; A strictly lower, P lower incl.
//   T       = (I + A)^-1              blockwise forward substitution, fp32, CUDA cores
//   W^T     = Kh^T T^T,  U^T = WV^T T^T
//   E^T     = U^T - S^T W^T           (MMA with negated A, accumulating onto U^T)
//   O^T     = S^T Qg^T + E^T P^T      (read-out of the post-update state)
//   S^T     = (S^T + E^T Kb) diag(e^gamma_C)
//
// Writing Kb = k.e^-gamma and scaling after the state MMA equals S diag(e^gamma_C) +
// (k.e^(gamma_C - gamma))^T E; both factors of every product stay within e^+-60 when
// |gamma| <= 60 on the whole chunk.  A chunk with a stronger cumulative decay takes the
// exact path instead: A and P from per-pair decays exp(gamma_i - gamma_j) on CUDA cores,
// K_end = k.e^(gamma_C - gamma) in place of Kb, and the state scaled before its MMA.
//
// Every wait on an mbarrier is bounded; on expiry the kernel records GDR_ERR_TIMEOUT in
// g_tc_error, stops issuing work, waits (bounded) for its own bulk copy and tensor-core
// work to drain, frees its TMEM and returns.
#include "chunk_tc.cuh"
#include "tc_util.cuh"

namespace gdr {

__device__ int g_tc_error = 0;

namespace {

using namespace tc;

constexpr int C = 64, DK = 128, DV = 128;
constexpr int kThreads = 256;
constexpr uint32_t kWaitLimit = 1u << 24;
constexpr float kFastLimit = 60.f;
constexpr int kAS = 68;   // fp32 row stride of the A / T scratch (bank-conflict free)

// shared memory map (byte offsets from a 1024-aligned base)
constexpr int OFF_S = 0;                       // S^T   bf16 [128 v][128 d]   32 KB
constexpr int OFF_QK = OFF_S + 32768;          // [Kh;Qg] bf16 [128][128]     32 KB
constexpr int OFF_KB = OFF_QK + 32768;         // Kb    bf16 [64 t][128 d]    16 KB
constexpr int OFF_WV = OFF_KB + 16384;         // WV    bf16 [64 t][128 v]    16 KB
constexpr int OFF_P = OFF_WV + 16384;          // P     bf16 [64 t][64 j]      8 KB
constexpr int OFF_T = OFF_P + 8192;            // T     bf16 [64 t][64 j]      8 KB
constexpr int OFF_WT = OFF_T + 8192;           // W^T   bf16 [128 d][64 t]    16 KB
constexpr int OFF_ET = OFF_WT + 16384;         // E^T   bf16 [128 v][64 t]    16 KB
constexpr int OFF_G = OFF_ET + 16384;          // g_log staging fp32 [64][128] 32 KB
constexpr int OFF_A32 = OFF_G + 32768;         // A fp32 [64][68]
constexpr int OFF_T32 = OFF_A32 + 64 * kAS * 4;  // T fp32 [64][68]
constexpr int OFF_SCAN = OFF_T32 + 64 * kAS * 4; // scan totals fp32 [16][128] / temp
constexpr int OFF_GC = OFF_SCAN + 16 * 128 * 4;  // gamma_C fp32 [128]
constexpr int OFF_EGC = OFF_GC + 512;            // exp(gamma_C) fp32 [128]
constexpr int OFF_BAR = OFF_EGC + 512;           // 2 mbarriers + TMEM slot
constexpr int SMEM_BYTES = OFF_BAR + 64 + 1024;  // + alignment slack

// TMEM columns
constexpr uint32_t TM_S = 0, TM_O = 128, TM_E = 192, TM_W = 256, TM_AP = 320, TM_COLS = 512;

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &u, float (&f)[8]) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = __bfloat1622float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}

__device__ __forceinline__ void st_chunk(uint32_t saddr, const float (&f)[8]) {
    st_shared_v4(saddr, pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                 pack_bf16(f[6], f[7]));
}

struct Waiter {
    uint32_t bar_mma, phase;
    bool ok;
    // all threads wait for the MMA barrier; false (everywhere) if any thread gave up
    __device__ __forceinline__ bool mma() {
        bool mine = mbar_wait(bar_mma, phase, kWaitLimit);
        phase ^= 1u;
        const bool all = !__syncthreads_or(!mine);
        ok = ok && all;
        tc_fence_after();
        return all;
    }
};

__global__ void __launch_bounds__(kThreads, 1) chunk_tc_kernel(ChunkArgs a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x;
    const int T = a.T, mode = a.mode;
    const size_t tok0 = (size_t)bh * T;
    const int nchunks = (T + C - 1) / C;

    float *sG = reinterpret_cast<float *>(sm + OFF_G);
    float *sA32 = reinterpret_cast<float *>(sm + OFF_A32);
    float *sT32 = reinterpret_cast<float *>(sm + OFF_T32);
    float *sScan = reinterpret_cast<float *>(sm + OFF_SCAN);
    float *sGC = reinterpret_cast<float *>(sm + OFF_GC);
    float *sEGC = reinterpret_cast<float *>(sm + OFF_EGC);
    const uint32_t bar_mma = sbase + OFF_BAR, bar_g = sbase + OFF_BAR + 8;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 16);

    const __nv_bfloat16 *Q = (const __nv_bfloat16 *)a.q, *K = (const __nv_bfloat16 *)a.k;
    const __nv_bfloat16 *V = (const __nv_bfloat16 *)a.v, *Bg = (const __nv_bfloat16 *)a.b;
    const __nv_bfloat16 *Wg = (const __nv_bfloat16 *)a.w;
    __nv_bfloat16 *O = (__nv_bfloat16 *)a.o;
    const bool vec_g = (mode != GDR_MODE_GDN);

    if (tid == 0) {
        mbar_init(bar_mma, 1);
        mbar_init(bar_g, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tslot), TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;

    // first g_log chunk in flight while the initial state is loaded
    auto issue_g = [&](int c) {
        const int t0 = c * C, n = min(C, T - t0);
        mbar_arrive_expect_tx(bar_g, (uint32_t)(n * DK * 4));
        bulk_g2s(sbase + OFF_G, a.g + (tok0 + t0) * DK, (uint32_t)(n * DK * 4), bar_g);
    };
    auto prefetch_inputs = [&](int c) {
        const int t0 = c * C, n = min(C, T - t0);
        const size_t e = (tok0 + t0) * DK;
        prefetch_l2(Q + e, n * DK * 2);
        prefetch_l2(K + e, n * DK * 2);
        prefetch_l2(V + e, n * DV * 2);
        if (mode == GDR_MODE_GDN2) {
            prefetch_l2(Bg + e, n * DK * 2);
            prefetch_l2(Wg + e, n * DV * 2);
        }
    };
    if (tid == 0) {
        if (vec_g) issue_g(0);
        prefetch_inputs(0);
        if (nchunks > 1) prefetch_inputs(1);
    }
    int g_issued = vec_g ? 1 : 0, g_done = 0;   // g_log copies issued / waited for (uniform)

    // ---- initial state -> TMEM (fp32, transposed) and the bf16 operand copy ----
    if (warp >= 4) {
        const int v = (warp - 4) * 32 + lane;
        for (int d0 = 0; d0 < DK; d0 += 32) {
            float x[32];
#pragma unroll
            for (int j = 0; j < 32; ++j)
                x[j] = a.S0 ? a.S0[((size_t)bh * DK + d0 + j) * DV + v] : 0.f;
            tmem_st32(tmem + lane_base + TM_S + d0, x);
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
                float f[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) f[j] = x[q8 * 8 + j];
                st_chunk(sbase + OFF_S + tile_chunk(128, v, d0 / 8 + q8), f);
            }
        }
        tmem_wait_st();
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    Waiter W{bar_mma, 0u, true};
    bool ok = true;
    const int tg = tid >> 4, cg = tid & 15;   // build-phase mapping: 4 tokens x 8 channels

    for (int c = 0; c < nchunks && ok; ++c) {
        const int t0 = c * C, n = min(C, T - t0);
        // ===== P1: operands =====
        uint4 rq[4], rk[4], rv[4], rb[4], rw[4];
        float bsc[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = tg * 4 + i;
            const uint4 z = make_uint4(0, 0, 0, 0);
            rq[i] = rk[i] = rv[i] = rb[i] = rw[i] = z;
            bsc[i] = 0.f;
            if (t < n) {
                const size_t e = (tok0 + t0 + t) * DK + cg * 8;
                rq[i] = *reinterpret_cast<const uint4 *>(Q + e);
                rk[i] = *reinterpret_cast<const uint4 *>(K + e);
                rv[i] = *reinterpret_cast<const uint4 *>(V + e);
                if (mode == GDR_MODE_GDN2) {
                    rb[i] = *reinterpret_cast<const uint4 *>(Bg + e);
                    rw[i] = *reinterpret_cast<const uint4 *>(Wg + e);
                } else {
                    bsc[i] = __bfloat162float(Bg[tok0 + t0 + t]);
                }
            }
        }
        float gam[4][8];
        if (vec_g) {
            const bool got = mbar_wait(bar_g, (uint32_t)(c & 1), kWaitLimit);
            if (__syncthreads_or(!got)) { ok = false; break; }
            g_done = c + 1;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = tg * 4 + i;
                if (t < n) {
                    const float4 g0 = *reinterpret_cast<const float4 *>(sG + t * DK + cg * 8);
                    const float4 g1 = *reinterpret_cast<const float4 *>(sG + t * DK + cg * 8 + 4);
                    gam[i][0] = g0.x; gam[i][1] = g0.y; gam[i][2] = g0.z; gam[i][3] = g0.w;
                    gam[i][4] = g1.x; gam[i][5] = g1.y; gam[i][6] = g1.z; gam[i][7] = g1.w;
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) gam[i][j] = 0.f;
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = tg * 4 + i;
                const float gs = (t < n) ? a.g[tok0 + t0 + t] : 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) gam[i][j] = gs;
            }
        }
        // inclusive cumulative sum over the chunk: within 4 tokens, then across groups
#pragma unroll
        for (int i = 1; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) gam[i][j] += gam[i - 1][j];
        {
            float4 *dst = reinterpret_cast<float4 *>(sScan + tg * 128 + cg * 8);
            dst[0] = make_float4(gam[3][0], gam[3][1], gam[3][2], gam[3][3]);
            dst[1] = make_float4(gam[3][4], gam[3][5], gam[3][6], gam[3][7]);
        }
        __syncthreads();
        {
            float off[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int u = 0; u < tg; ++u) {
                const float4 x0 = *reinterpret_cast<const float4 *>(sScan + u * 128 + cg * 8);
                const float4 x1 = *reinterpret_cast<const float4 *>(sScan + u * 128 + cg * 8 + 4);
                off[0] += x0.x; off[1] += x0.y; off[2] += x0.z; off[3] += x0.w;
                off[4] += x1.x; off[5] += x1.y; off[6] += x1.z; off[7] += x1.w;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) gam[i][j] += off[j];
        }
        if (tg == 15) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                sGC[cg * 8 + j] = gam[3][j];
                sEGC[cg * 8 + j] = __expf(gam[3][j]);
            }
        }
        bool big = false;
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) big |= fabsf(gam[i][j]) > kFastLimit;
        const bool exact = __syncthreads_or(big);   // also publishes sGC / sEGC
        if (exact) {
            // keep gamma for the per-pair decays; the next g_log copy waits until then
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float4 *dst = reinterpret_cast<float4 *>(sG + (tg * 4 + i) * DK + cg * 8);
                dst[0] = make_float4(gam[i][0], gam[i][1], gam[i][2], gam[i][3]);
                dst[1] = make_float4(gam[i][4], gam[i][5], gam[i][6], gam[i][7]);
            }
        } else if (c + 1 < nchunks) {
            if (vec_g) g_issued = c + 2;
            if (tid == 0) {
                fence_async_smem();
                if (vec_g) issue_g(c + 1);
                if (c + 2 < nchunks) prefetch_inputs(c + 2);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = tg * 4 + i;
            float fq[8], fk[8], fv[8], fb[8], fw[8];
            bf16x8_to_f32(rq[i], fq);
            bf16x8_to_f32(rk[i], fk);
            bf16x8_to_f32(rv[i], fv);
            if (mode == GDR_MODE_GDN2) {
                bf16x8_to_f32(rb[i], fb);
                bf16x8_to_f32(rw[i], fw);
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) fb[j] = fw[j] = bsc[i];
            }
            float kh[8], qg[8], kb[8], wv[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float e = __expf(gam[i][j]);
                kh[j] = fb[j] * fk[j] * e;
                qg[j] = fq[j] * e;
                kb[j] = exact ? fk[j] * __expf(sGC[cg * 8 + j] - gam[i][j]) : fk[j] * __expf(-gam[i][j]);
                wv[j] = fw[j] * fv[j];
            }
            st_chunk(sbase + OFF_QK + tile_chunk(128, t, cg), kh);
            st_chunk(sbase + OFF_QK + tile_chunk(128, 64 + t, cg), qg);
            st_chunk(sbase + OFF_KB + tile_chunk(64, t, cg), kb);
            st_chunk(sbase + OFF_WV + tile_chunk(64, t, cg), wv);
        }
        fence_async_smem();
        __syncthreads();

        // ===== P2: [A;P] = [Kh;Qg] Kb^T  and  O^T = S^T Qg^T =====
        if (tid == 0) {
            tc_fence_after();
            if (!exact) {
                const uint32_t id = idesc_bf16(128, 64, false, false, false);
#pragma unroll
                for (int s = 0; s < DK / 16; ++s)
                    mma_bf16(tmem + TM_AP, desc_kmajor(sbase + OFF_QK, 128, 0, s),
                             desc_kmajor(sbase + OFF_KB, 64, 0, s), id, s > 0);
            }
            const uint32_t id = idesc_bf16(128, 64, false, false, false);
#pragma unroll
            for (int s = 0; s < DK / 16; ++s)
                mma_bf16(tmem + TM_O, desc_kmajor(sbase + OFF_S, 128, 0, s),
                         desc_kmajor(sbase + OFF_QK, 128, 64, s), id, s > 0);
            mma_commit(bar_mma);
        }
        if (!W.mma()) { ok = false; break; }

        // ===== P3: A (fp32, strictly lower) and P (bf16, lower incl.) =====
        if (!exact) {
            if (warp < 4) {
                const int r = warp * 32 + lane;          // TMEM lane = row of [A; P]
                for (int j0 = 0; j0 < 64; j0 += 32) {
                    float x[32];
                    tmem_ld32(tmem + lane_base + TM_AP + j0, x);
                    tmem_wait_ld();
                    if (r < 64) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) sA32[r * kAS + j0 + j] = (j0 + j < r) ? x[j] : 0.f;
                    } else {
                        const int t = r - 64;
#pragma unroll
                        for (int q8 = 0; q8 < 4; ++q8) {
                            float f[8];
#pragma unroll
                            for (int j = 0; j < 8; ++j) f[j] = (j0 + q8 * 8 + j <= t) ? x[q8 * 8 + j] : 0.f;
                            st_chunk(sbase + OFF_P + tile_chunk(64, t, j0 / 8 + q8), f);
                        }
                    }
                }
            }
        } else {
            // exact per-pair decays (strong-decay chunks only)
            for (int p = tid; p < C * C; p += kThreads) {
                const int i = p >> 6, j = p & 63;
                float av = 0.f, pv = 0.f;
                if (j <= i && i < n) {
                    const size_t ei = (tok0 + t0 + i) * DK, ej = (tok0 + t0 + j) * DK;
                    const float bi_s = (mode == GDR_MODE_GDN2) ? 0.f : __bfloat162float(Bg[tok0 + t0 + i]);
                    for (int d = 0; d < DK; ++d) {
                        const float dec = __expf(sG[i * DK + d] - sG[j * DK + d]);
                        const float kj = __bfloat162float(K[ej + d]) * dec;
                        const float bi = (mode == GDR_MODE_GDN2) ? __bfloat162float(Bg[ei + d]) : bi_s;
                        av = fmaf(bi * __bfloat162float(K[ei + d]), kj, av);
                        pv = fmaf(__bfloat162float(Q[ei + d]), kj, pv);
                    }
                }
                sA32[i * kAS + j] = (j < i) ? av : 0.f;
                *reinterpret_cast<__nv_bfloat16 *>(sm + OFF_P + tile_off(64, i, j)) = __float2bfloat16_rn(pv);
            }
        }
        __syncthreads();
        if (exact && c + 1 < nchunks) {
            if (vec_g) g_issued = c + 2;
            if (tid == 0) {
                fence_async_smem();
                if (vec_g) issue_g(c + 1);
                if (c + 2 < nchunks) prefetch_inputs(c + 2);
            }
        }

        // ===== P4: T = (I + A)^-1, blockwise (16 x 16 blocks) =====
        if (tid < 64) {
            const int blk = tid >> 4, col = tid & 15, o = blk * 16;
            float tv[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float acc = (i == col) ? 1.f : 0.f;
#pragma unroll
                for (int m = 0; m < i; ++m) acc = fmaf(-sA32[(o + i) * kAS + o + m], tv[m], acc);
                tv[i] = acc;
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) sT32[(o + i) * kAS + o + col] = tv[i];
        }
        __syncthreads();
        {
            const int r = tid >> 4, cc = tid & 15;
            // level 1: T[I][I-1] = -T[I][I] A[I][I-1] T[I-1][I-1],  I = 1..3
            float x1[3];
#pragma unroll
            for (int I = 1; I < 4; ++I) {
                float acc = 0.f;
                for (int m = cc; m < 16; ++m)
                    acc = fmaf(sA32[(16 * I + r) * kAS + 16 * (I - 1) + m], sT32[(16 * (I - 1) + m) * kAS + 16 * (I - 1) + cc], acc);
                x1[I - 1] = acc;
            }
#pragma unroll
            for (int I = 1; I < 4; ++I) sScan[(I - 1) * 256 + r * 16 + cc] = x1[I - 1];
            __syncthreads();
#pragma unroll
            for (int I = 1; I < 4; ++I) {
                float acc = 0.f;
                for (int m = 0; m <= r; ++m)
                    acc = fmaf(sT32[(16 * I + r) * kAS + 16 * I + m], sScan[(I - 1) * 256 + m * 16 + cc], acc);
                sT32[(16 * I + r) * kAS + 16 * (I - 1) + cc] = -acc;
            }
            __syncthreads();
            // level 2: T[I][I-2] = -T[I][I] (A[I][I-2] T[I-2][I-2] + A[I][I-1] T[I-1][I-2]),  I = 2, 3
            float x2[2];
#pragma unroll
            for (int I = 2; I < 4; ++I) {
                float acc = 0.f;
                for (int m = 0; m < 32; ++m)
                    acc = fmaf(sA32[(16 * I + r) * kAS + 16 * (I - 2) + m], sT32[(16 * (I - 2) + m) * kAS + 16 * (I - 2) + cc], acc);
                x2[I - 2] = acc;
            }
#pragma unroll
            for (int I = 2; I < 4; ++I) sScan[(I - 2) * 256 + r * 16 + cc] = x2[I - 2];
            __syncthreads();
#pragma unroll
            for (int I = 2; I < 4; ++I) {
                float acc = 0.f;
                for (int m = 0; m <= r; ++m)
                    acc = fmaf(sT32[(16 * I + r) * kAS + 16 * I + m], sScan[(I - 2) * 256 + m * 16 + cc], acc);
                sT32[(16 * I + r) * kAS + 16 * (I - 2) + cc] = -acc;
            }
            __syncthreads();
            // level 3: T[3][0] = -T[3][3] (A[3][0] T[0][0] + A[3][1] T[1][0] + A[3][2] T[2][0])
            {
                float acc = 0.f;
                for (int m = 0; m < 48; ++m)
                    acc = fmaf(sA32[(48 + r) * kAS + m], sT32[m * kAS + cc], acc);
                sScan[r * 16 + cc] = acc;
            }
            __syncthreads();
            {
                float acc = 0.f;
                for (int m = 0; m <= r; ++m)
                    acc = fmaf(sT32[(48 + r) * kAS + 48 + m], sScan[m * 16 + cc], acc);
                sT32[(48 + r) * kAS + cc] = -acc;
            }
            __syncthreads();
        }
        {
            // T (unit lower triangular) -> bf16 operand, zeros above the diagonal
            const int t = tid >> 2, q = tid & 3;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int c8 = q * 2 + h;
                float f[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int col = c8 * 8 + j;
                    f[j] = (col <= t) ? sT32[t * kAS + col] : 0.f;
                }
                st_chunk(sbase + OFF_T + tile_chunk(64, t, c8), f);
            }
        }
        fence_async_smem();
        __syncthreads();

        // ===== P5: W^T = Kh^T T^T,  U^T = WV^T T^T =====
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, true, false, false);
#pragma unroll
            for (int s = 0; s < C / 16; ++s) {
                mma_bf16(tmem + TM_W, desc_mnmajor(sbase + OFF_QK, 128, 0, s),
                         desc_kmajor(sbase + OFF_T, 64, 0, s), id, s > 0);
                mma_bf16(tmem + TM_E, desc_mnmajor(sbase + OFF_WV, 64, 0, s),
                         desc_kmajor(sbase + OFF_T, 64, 0, s), id, s > 0);
            }
            mma_commit(bar_mma);
        }
        if (!W.mma()) { ok = false; break; }

        // ===== P6: W^T -> bf16 operand (MN-major B); exact chunks pre-scale the state =====
        if (warp < 4) {
            const int d = warp * 32 + lane;
            for (int t0c = 0; t0c < 64; t0c += 32) {
                float x[32];
                tmem_ld32(tmem + lane_base + TM_W + t0c, x);
                tmem_wait_ld();
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    float f[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) f[j] = x[q8 * 8 + j];
                    st_chunk(sbase + OFF_WT + tile_chunk(128, d, t0c / 8 + q8), f);
                }
            }
        } else if (exact) {
            for (int d0 = 0; d0 < DK; d0 += 32) {
                float x[32];
                tmem_ld32(tmem + lane_base + TM_S + d0, x);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) x[j] *= sEGC[d0 + j];
                tmem_st32(tmem + lane_base + TM_S + d0, x);
            }
            tmem_wait_st();
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ===== P7: E^T = U^T - S^T W^T =====
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, false, true, true);
#pragma unroll
            for (int s = 0; s < DK / 16; ++s)
                mma_bf16(tmem + TM_E, desc_kmajor(sbase + OFF_S, 128, 0, s),
                         desc_mnmajor(sbase + OFF_WT, 128, 0, s), id, 1u);
            mma_commit(bar_mma);
        }
        if (!W.mma()) { ok = false; break; }

        // ===== P8: E^T -> bf16 operand (K-major A) =====
        if (warp < 4) {
            const int v = warp * 32 + lane;
            for (int t0c = 0; t0c < 64; t0c += 32) {
                float x[32];
                tmem_ld32(tmem + lane_base + TM_E + t0c, x);
                tmem_wait_ld();
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    float f[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) f[j] = x[q8 * 8 + j];
                    st_chunk(sbase + OFF_ET + tile_chunk(128, v, t0c / 8 + q8), f);
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ===== P9: O^T += E^T P^T,  S^T += E^T Kb (or K_end) =====
        if (tid == 0) {
            tc_fence_after();
            const uint32_t ido = idesc_bf16(128, 64, false, false, false);
            const uint32_t ids = idesc_bf16(128, 128, false, true, false);
#pragma unroll
            for (int s = 0; s < C / 16; ++s) {
                mma_bf16(tmem + TM_O, desc_kmajor(sbase + OFF_ET, 128, 0, s),
                         desc_kmajor(sbase + OFF_P, 64, 0, s), ido, 1u);
                mma_bf16(tmem + TM_S, desc_kmajor(sbase + OFF_ET, 128, 0, s),
                         desc_mnmajor(sbase + OFF_KB, 64, 0, s), ids, 1u);
            }
            mma_commit(bar_mma);
        }
        if (!W.mma()) { ok = false; break; }

        // ===== P10: output rows; state scaled and copied to the bf16 operand =====
        if (warp < 4) {
            const int v = warp * 32 + lane;
            for (int t0c = 0; t0c < 64; t0c += 32) {
                float x[32];
                tmem_ld32(tmem + lane_base + TM_O + t0c, x);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (t0c + j < n) O[(tok0 + t0 + t0c + j) * DV + v] = __float2bfloat16_rn(x[j]);
            }
        } else {
            const int v = (warp - 4) * 32 + lane;
            const bool last = (c == nchunks - 1);
            for (int d0 = 0; d0 < DK; d0 += 32) {
                float x[32];
                tmem_ld32(tmem + lane_base + TM_S + d0, x);
                tmem_wait_ld();
                if (!exact) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) x[j] *= sEGC[d0 + j];
                    tmem_st32(tmem + lane_base + TM_S + d0, x);
                }
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    float f[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) f[j] = x[q8 * 8 + j];
                    st_chunk(sbase + OFF_S + tile_chunk(128, v, d0 / 8 + q8), f);
                }
                if (last && a.ST) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) a.ST[((size_t)bh * DK + d0 + j) * DV + v] = x[j];
                }
            }
            tmem_wait_st();
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (!ok) {
        if (tid == 0) atomicExch(&g_tc_error, 1);
        // drain: the last g_log copy and any committed tensor-core work (bounded)
        if (tid == 0) {
            mma_commit(bar_mma);
        }
        mbar_wait(bar_mma, W.phase, kWaitLimit);
        if (g_issued > g_done) mbar_wait(bar_g, (uint32_t)(g_done & 1), kWaitLimit);
    }
    // a g_log copy may still be in flight only when the loop stopped early
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

}  // namespace

bool chunk_tc_supported(const ChunkArgs &a) {
    return a.dtype == GDR_BF16 && a.dk == DK && a.dv == DV && a.chunk == C;
}

gdr_status_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t s) {
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
    if (cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES) != cudaSuccess)
        return GDR_ERR_CUDA;
    chunk_tc_kernel<<<(unsigned)(a.B * a.H), kThreads, SMEM_BYTES, s>>>(a);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

cudaError_t chunk_tc_read_and_clear_error(int *err) {
    cudaError_t e = cudaMemcpyFromSymbol(err, g_tc_error, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(int));
}

}  // namespace gdr
