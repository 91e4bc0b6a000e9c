// wy_prep.cu -- phase one of the two-phase chunked forward: the WY factors of every chunk.
//
// Persistent CTAs (256 threads, two per SM) take the chunks of every sequence-head in turn;
// the chunks do not depend on one another, so a call with few sequence-heads still fills
// the GPU.  Per chunk
// (Gated DeltaNet-2 Review §3-2.5 "Chunkwise WY training"; Gated DeltaNet-2 Q&A page, Q4):
//
//   gamma   = chunk-local cumulative sum of g_log           fp32, per key channel
//   Kh      = b.k.e^gamma,  Qg = q.e^gamma,  Kb = k.e^-gamma   bf16 tiles (shared memory)
//   [A; P]  = [Kh; Qg] Kb^T        one M=128 tcgen05 MMA; A strictly lower, P lower incl.
//   T       = (I + A)^-1           blocked substitution (tri_inverse.cuh)
//   W^T     = Kh^T T^T             W = T Kh: the pages' W, with the decay and b folded in
//   U^T     = (w.v)^T T^T          U = T (w.v)
//
// and the chunk's record (two_phase.cuh) goes to global memory by bulk copies.  q, k, v and
// a per-channel b arrive by tiled tensor copies (TMA, 128-byte swizzle) straight into the
// operand tiles, and the operands are built in place: each thread owns four tokens and eight
// channels, sums their g_log (read from global memory up front), scans the sums across its
// warp's token groups by shuffles (the first half of the chunk hands its totals to the second
// through shared memory), and turns its b, q, k into Kh, Qg, Kb and its v into w.v with
// 16-byte shared-memory accesses.  Once the tiles have landed, the CTA's next chunk is
// prefetched to L2.  Both factors of every product in [A; P] stay within e^+-60 when
// |gamma| <= 60 on the whole chunk; a chunk with a stronger cumulative decay is listed instead and
// wy_exact_kernel writes its record from per-pair decays exp(gamma_i - gamma_j) in fp32 on
// CUDA cores (with K_end = k.e^(gamma_C - gamma) in place of Kb, and the flag set that tells
// phase two to scale the state before its update).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <string.h>

#include "bounds.cuh"
#include "chunk_tc.cuh"
#include "tc_util.cuh"
#include "tri_inverse.cuh"
#include "two_phase.cuh"

namespace gdr {
namespace tp {

__device__ int g_tp_error = 0;

namespace {

using namespace tc;

constexpr int C = 64, DK = 128, DV = 128;
constexpr int kThreads = 256;
constexpr float kFastLimit = 60.f;

// shared memory map of the tensor-core kernel (byte offsets from a 1024-aligned base)
constexpr int OFF_QK = 0;                       // [Kh; Qg] bf16 [128][128]            32 KB
constexpr int OFF_KB = OFF_QK + 32768;          // Kb bf16 [64 t][128 d]               16 KB
constexpr int OFF_WV = OFF_KB + 16384;          // w.v bf16 [64 t][128 v], then U^T    16 KB
constexpr int OFF_P = OFF_WV + 16384;           // P bf16 [64 t][64 j]                  8 KB
constexpr int OFF_T = OFF_P + 8192;             // T bf16 [64 t][64 j]                  8 KB
constexpr int OFF_A32 = OFF_T + 8192;           // A, then T, fp32 [64][68]; then W^T bf16
constexpr int OFF_X = OFF_A32 + 64 * tri::LD * 4;   // the inverse's scratch, 4 x [16][20] fp32
constexpr int OFF_HALF = OFF_X + 4 * 16 * tri::XLD * 4;   // sum of g over tokens 0..31 [128]
constexpr int OFF_BETA = OFF_HALF + 512;        // scalar erase gate of the chunk's tokens [64]
constexpr int OFF_META = OFF_BETA + 256;        // the record's e^gamma_C [128] and flag
constexpr int OFF_BAR = OFF_META + 528 + 16;    // mbarriers (MMA, tile copies); TMEM slot
constexpr int SMEM_BYTES = OFF_BAR + 24 + 1024; // + alignment slack
static_assert(64 * tri::LD * 4 >= 16384, "W^T fits over the inverse's fp32 scratch");
static_assert(OFF_A32 % 1024 == 0 && OFF_WV % 1024 == 0, "tiles on 1024-byte boundaries");
static_assert(2 * (SMEM_BYTES + 1024) <= 228 * 1024, "two CTAs per SM");

// TMEM columns (fp32): lane = row of [A; P]; lane = key channel of W^T, value channel of U^T
constexpr uint32_t TM_AP = 0, TM_W = 64, TM_U = 128, TM_COLS = 256;

// CTA barriers that also reconverge the warp: a thread that ran code alone (an elected
// issuer, a bounded wait) may otherwise come out of the barrier still diverged from its
// warp, and every later warp-collective instruction (shuffles, warp MMAs, the .aligned
// tcgen05 loads and stores) then pays for re-synchronising it, or is not allowed at all
__device__ __forceinline__ void sync_all() {
    __syncthreads();
    __syncwarp();
}
__device__ __forceinline__ bool sync_all_and(bool v) {
    const bool r = __syncthreads_and(v);
    __syncwarp();
    return r;
}
__device__ __forceinline__ bool sync_all_or(bool v) {
    const bool r = __syncthreads_or(v);
    __syncwarp();
    return r;
}

// T = (I + A)^-1 by warps 0-3 (tri_inverse.cuh) as a call of its own: inlined into this
// kernel, whose other phases keep many registers live, its substitution chains ran several
// times slower than on their own
__device__ __noinline__ void invert(float *sA32, float *sX, int warp, int lane, uint32_t t_tile) {
    tri::inverse64(sA32, sA32, sX, warp, lane, Bar128{}, TileOut{t_tile});
}

__device__ __forceinline__ void st_bf16(unsigned char *p, float x) {
    *reinterpret_cast<__nv_bfloat16 *>(p) = __float2bfloat16_rn(x);
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 u;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w) : "r"(addr));
    return u;
}

// Tensor maps of the bf16 inputs read as tiles: [B*H*T rows][128] row-major, box {64, 64}
// with the 128-byte swizzle, so a box lands in shared memory in the operand tile layout of
// tc_util.cuh and the operands are built in place (rows past the tensor's end read zero).
struct PrepMaps {
    CUtensorMap q, k, v, b;
};

__global__ void __launch_bounds__(kThreads, 2)
    wy_prep_kernel(ChunkArgs a, unsigned char *records, int *list, const __grid_constant__ PrepMaps tm) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;

    const int nch = (a.T + C - 1) / C;
    const int units = a.B * a.H * nch;
    const int mode = a.mode;
    const bool vec_b = mode_b_vec(mode), vec_w = mode_w_vec(mode), vec_g = mode_g_vec(mode);
    const __nv_bfloat16 *Bg = (const __nv_bfloat16 *)a.b, *Wg = (const __nv_bfloat16 *)a.w;
    const __nv_bfloat16 *Wsc = mode == GDR_MODE_BONLY ? Wg : Bg;   // a scalar write gate
    float *sHalf = reinterpret_cast<float *>(sm + OFF_HALF);
    float *sBeta = reinterpret_cast<float *>(sm + OFF_BETA);
    float *sEgc = reinterpret_cast<float *>(sm + OFF_META);
    float *sA32 = reinterpret_cast<float *>(sm + OFF_A32);
    float *sX = reinterpret_cast<float *>(sm + OFF_X);
    const uint32_t bar = sbase + OFF_BAR, bar_ld = bar + 8;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 16);

    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar_ld, 1);
        fence_mbar_init();
    }
    __syncwarp();
    if (warp == 0) {
        tmem_alloc(smem_u32(tslot), TM_COLS);
        tmem_relinquish();
    }
    // T's blocks above the diagonal are never written by the inverse: cleared once
    reinterpret_cast<uint4 *>(sm + OFF_T)[tid] = make_uint4(0, 0, 0, 0);
    reinterpret_cast<uint4 *>(sm + OFF_T)[tid + kThreads] = make_uint4(0, 0, 0, 0);
    static_assert(kThreads * 32 == 8192, "two 16-byte stores per thread clear the T tile");
    tc_fence_before();
    sync_all();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t wait_limit = a.wait_limit;
    // scan and build: thread (token group tg, channel group cg) owns tokens 4 tg .. 4 tg + 3
    // and key (and value) channels 8 cg .. 8 cg + 7; a warp holds eight token groups of four
    // channel groups, so its 16-byte tile accesses spread over all the banks
    const int tgl = lane >> 2, hh = warp >> 2;   // token group within the warp, half of the chunk
    const int tg = 8 * hh + tgl, cg = 4 * (warp & 3) + (lane & 3);
    bool ok = true;
    uint32_t n_mma = 0;                          // commits on bar so far (its phase parity)
    int ld_issued = 0;                           // tile-copy batches issued (thread 0)

    // A persistent CTA: two per SM take the chunks in turn, so the code stays in the
    // instruction cache (each chunk runs every phase once, a long straight-line path).
#pragma unroll 1
    for (int it = 0, unit = blockIdx.x; unit < units; ++it, unit += gridDim.x) {
        const int bh = unit / nch, c = unit % nch;
        const int t0 = c * C, n = min(C, a.T - t0);
        const size_t row0 = (size_t)bh * a.T + t0;   // token t of the chunk is row row0 + t
        unsigned char *rec = records + (size_t)unit * REC_BYTES;
        // debug build: the chunk lies inside the inputs (a uniform condition)
        if (!GDR_IN_BOUNDS(bh < a.B * a.H && n >= 1, 701)) break;
        if (tid == 0) {
            // the chunk's q, k, v (and a per-channel b) as tiles: q into the Qg rows of the
            // stacked [Kh; Qg] tile, b into its Kh rows, k into the Kb tile, v into the w.v
            // tile (the previous chunk's copies out of these tiles have read them)
            fence_async_smem();
            mbar_arrive_expect_tx(bar_ld, (vec_b ? 8u : 6u) * 8192u);
            ++ld_issued;
            const int r = (int)row0;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                tma_load_2d(sbase + OFF_QK + h * 16384 + 8192, &tm.q, 64 * h, r, bar_ld);
                tma_load_2d(sbase + OFF_KB + h * 8192, &tm.k, 64 * h, r, bar_ld);
                tma_load_2d(sbase + OFF_WV + h * 8192, &tm.v, 64 * h, r, bar_ld);
                if (vec_b) tma_load_2d(sbase + OFF_QK + h * 16384, &tm.b, 64 * h, r, bar_ld);
            }
        }
        __syncwarp();

        // ---- global loads issued up front: g_log and the write gate of this thread's four
        //      tokens and eight channels, a scalar erase gate per token ----
        float gv[4][8];
        uint4 wr[4];
        float wsc[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = 4 * tg + i;
            const bool in = t < n;
            wr[i] = make_uint4(0, 0, 0, 0);
            wsc[i] = 0.f;
            if (vec_g) {
                float4 g0 = make_float4(0.f, 0.f, 0.f, 0.f), g1 = g0;
                if (in) {
                    const float4 *gp = reinterpret_cast<const float4 *>(a.g + (row0 + t) * DK + 8 * cg);
                    g0 = gp[0];
                    g1 = gp[1];
                }
                gv[i][0] = g0.x; gv[i][1] = g0.y; gv[i][2] = g0.z; gv[i][3] = g0.w;
                gv[i][4] = g1.x; gv[i][5] = g1.y; gv[i][6] = g1.z; gv[i][7] = g1.w;
            } else {
                const float x = in ? a.g[row0 + t] : 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) gv[i][j] = x;
            }
            if (in) {
                if (vec_w) wr[i] = *reinterpret_cast<const uint4 *>(Wg + (row0 + t) * DV + 8 * cg);
                else wsc[i] = __bfloat162float(Wsc[row0 + t]);
            }
        }
        if (!vec_b && tid < C) sBeta[tid] = tid < n ? __bfloat162float(Bg[row0 + tid]) : 0.f;
        // gamma over this half of the chunk: the thread's own four tokens, then an inclusive
        // scan over the warp's eight token groups (shuffles); the first half's totals go to
        // shared memory for the second half
#pragma unroll
        for (int i = 1; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) gv[i][j] += gv[i - 1][j];
        {
            float pre[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) pre[j] = gv[3][j];
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float y = __shfl_up_sync(0xffffffffu, pre[j], 4 * o);
                    if (tgl >= o) pre[j] += y;
                }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float excl = pre[j] - gv[3][j];   // tokens of the earlier groups of this half
#pragma unroll
                for (int i = 0; i < 4; ++i) gv[i][j] += excl;
            }
            if (hh == 0 && tgl == 7) {
                float4 *dst = reinterpret_cast<float4 *>(sHalf + 8 * cg);
                dst[0] = make_float4(pre[0], pre[1], pre[2], pre[3]);
                dst[1] = make_float4(pre[4], pre[5], pre[6], pre[7]);
            }
        }
        ok = sync_all_and(tid != 0 || mbar_wait(bar_ld, (uint32_t)(it & 1), wait_limit));
        if (!ok) break;
        if (tid == 32 && unit + (int)gridDim.x < units) {
            // this chunk's tiles have landed: the CTA's next chunk now travels to L2 while this
            // one is worked on (every CTA loads at the same time at first, so a prefetch issued
            // earlier would only compete with the loads of the current chunk)
            const int un = unit + (int)gridDim.x, bn = un / nch, cn = un % nch;
            const int nn = min(C, a.T - cn * C);
            const size_t e = ((size_t)bn * a.T + (size_t)cn * C) * DK;
            prefetch_l2((const __nv_bfloat16 *)a.q + e, (uint32_t)nn * DK * 2);
            prefetch_l2((const __nv_bfloat16 *)a.k + e, (uint32_t)nn * DK * 2);
            prefetch_l2((const __nv_bfloat16 *)a.v + e, (uint32_t)nn * DV * 2);
            if (vec_b) prefetch_l2(Bg + e, (uint32_t)nn * DK * 2);
            if (vec_w) prefetch_l2(Wg + e, (uint32_t)nn * DV * 2);
            if (vec_g) prefetch_l2(a.g + e, (uint32_t)nn * DK * 4);
        }

        // ---- the operands in place, 16 bytes at a time: b, q, k of the thread's four tokens
        //      and eight channels become Kh, Qg, Kb, and v becomes w.v (fp32 products, one bf16
        //      rounding; zero past the end) ----
        float mx = 0.f;
        if (hh == 1) {
            const float4 *src = reinterpret_cast<const float4 *>(sHalf + 8 * cg);
            const float4 h0 = src[0], h1 = src[1];
            const float hs[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) gv[i][j] += hs[j];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = 4 * tg + i;
            const bool in = t < n;
            const uint32_t okh = sbase + OFF_QK + tile_chunk(128, t, cg);
            const uint32_t oqg = sbase + OFF_QK + tile_chunk(128, 64 + t, cg);
            const uint32_t okb = sbase + OFF_KB + tile_chunk(64, t, cg);
            const uint32_t owv = sbase + OFF_WV + tile_chunk(64, t, cg);
            float fk[8], fq[8], fb[8], fv[8], fw[8];
            bf16x8_to_f32(sel(in, ld_shared_v4(okb)), fk);
            bf16x8_to_f32(sel(in, ld_shared_v4(oqg)), fq);
            bf16x8_to_f32(sel(in, ld_shared_v4(owv)), fv);
            if (vec_b) {
                bf16x8_to_f32(sel(in, ld_shared_v4(okh)), fb);
            } else {
                const float beta = sBeta[t];   // zero past the end
#pragma unroll
                for (int j = 0; j < 8; ++j) fb[j] = beta;
            }
            if (vec_w) {
                bf16x8_to_f32(wr[i], fw);
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) fw[j] = wsc[i];
            }
            float kh[8], qg[8], kb[8], wv[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                mx = fmaxf(mx, fabsf(gv[i][j]));
                const float eg = __expf(gv[i][j]);
                kh[j] = fb[j] * fk[j] * eg;
                qg[j] = fq[j] * eg;
                kb[j] = fk[j] * rcp_approx(eg);
                wv[j] = fw[j] * fv[j];
            }
            st_chunk(okh, kh);
            st_chunk(oqg, qg);
            st_chunk(okb, kb);
            st_chunk(owv, wv);
        }
        // e^gamma at the chunk's end (tokens past it add zero): the last token group's
        if (tg == 15) {
            float4 *dst = reinterpret_cast<float4 *>(sEgc + 8 * cg);
            dst[0] = make_float4(__expf(gv[3][0]), __expf(gv[3][1]), __expf(gv[3][2]), __expf(gv[3][3]));
            dst[1] = make_float4(__expf(gv[3][4]), __expf(gv[3][5]), __expf(gv[3][6]), __expf(gv[3][7]));
        }
        if (tid == 0) reinterpret_cast<int4 *>(sm + OFF_META + 512)[0] = make_int4(0, 0, 0, 0);
        if (sync_all_or(mx > kFastLimit)) {
            // strong decay: listed for the exact kernel, which writes this chunk's record
            if (tid == 0) list[1 + atomicAdd(list, 1)] = unit;
            sync_all();
            continue;
        }
        fence_async_smem();
        sync_all();
        // ---- [A; P] = [Kh; Qg] Kb^T ----
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, false, false, false);
#pragma unroll
            for (int s = 0; s < DK / 16; ++s)
                mma_bf16(tmem + TM_AP, desc_kmajor(sbase + OFF_QK, 128, 0, s), desc_kmajor(sbase + OFF_KB, 64, 0, s),
                         id, s > 0);
            mma_commit(bar);
        }
        ++n_mma;
        ok = sync_all_and(tid != 0 || mbar_wait(bar, (n_mma - 1) & 1, wait_limit));
        if (!ok) break;
        tc_fence_after();
        {
            // A (fp32, strictly lower) -> inverse scratch; P (bf16, lower incl.) -> its tile
            const int r = quarter * 32 + lane, j0 = (warp >> 2) * 32;
            float x[32];
            tmem_ld32(tmem + lane_base + TM_AP + j0, x);
            tmem_wait_ld();
            if (r < 64) {
                float4 *dst = reinterpret_cast<float4 *>(sA32 + r * tri::LD + j0);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    float y[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) y[u] = (j0 + 4 * q + u < r) ? x[4 * q + u] : 0.f;
                    dst[q] = make_float4(y[0], y[1], y[2], y[3]);
                }
            } else {
                const int t = r - 64;
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    float f[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) f[j] = (j0 + h * 8 + j <= t) ? x[h * 8 + j] : 0.f;
                    st_chunk(sbase + OFF_P + tile_chunk(64, t, j0 / 8 + h), f);
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        sync_all();
        // ---- T = (I + A)^-1 by warps 0-3, straight into the bf16 tile; meanwhile thread 128
        //      sends the record's Qg, Kb, P and tail (final once [A; P] is read out) ----
        if (warp < 4) {
            invert(sA32, sX, warp, lane, sbase + OFF_T);
        } else if (tid == 128) {
            // Qg: rows 64..127 of each column block of the stacked tile = a 64-row tile
            bulk_s2g(rec + REC_QG, sbase + OFF_QK + 8192, 8192);
            bulk_s2g(rec + REC_QG + 8192, sbase + OFF_QK + 16384 + 8192, 8192);
            bulk_s2g(rec + REC_KB, sbase + OFF_KB, 16384);
            bulk_s2g(rec + REC_P, sbase + OFF_P, 8192);
            bulk_s2g(rec + REC_EGC, sbase + OFF_META, 528);
            bulk_commit();
        }
        fence_async_smem();
        sync_all();
        // ---- W^T = Kh^T T^T and U^T = (w.v)^T T^T (A operands MN-major) ----
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, true, false, false);
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16(tmem + TM_W, desc_mnmajor(sbase + OFF_QK, 128, 0, s), desc_kmajor(sbase + OFF_T, 64, 0, s),
                         id, s > 0);
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16(tmem + TM_U, desc_mnmajor(sbase + OFF_WV, 64, 0, s), desc_kmajor(sbase + OFF_T, 64, 0, s),
                         id, s > 0);
            mma_commit(bar);
        }
        ++n_mma;
        ok = sync_all_and(tid != 0 || mbar_wait(bar, (n_mma - 1) & 1, wait_limit));
        if (!ok) break;
        tc_fence_after();
        {
            // W^T rows (warps 0-3) over the inverse's dead scratch, U^T rows (warps 4-7) over w.v
            const int r = quarter * 32 + lane;
            const uint32_t col = warp < 4 ? TM_W : TM_U;
            const uint32_t tile = sbase + (warp < 4 ? OFF_A32 : OFF_WV);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float x[32];
                tmem_ld32(tmem + lane_base + col + 32 * h, x);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float f[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) f[j] = x[8 * q + j];
                    st_chunk(tile + tile_chunk(128, r, 4 * h + q), f);
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        sync_all();
        if (tid == 0) {
            bulk_s2g(rec + REC_WT, sbase + OFF_A32, 16384);
            bulk_s2g(rec + REC_UT, sbase + OFF_WV, 16384);
            bulk_commit();
        }
        // the copies have read shared memory (each thread waits for its own) before the
        // next chunk's tiles arrive there; they land by the kernel's end
        if (tid == 0 || tid == 128) bulk_wait_read_all();
        sync_all();
    }
    if (!ok && tid == 0) {
        // a bounded wait expired: record it, and give the tile copies and the tensor cores a
        // bounded time to finish (one more commit covers every MMA issued; commits complete
        // in order, so phases n-1 and then n of it are waited for)
        atomicExch(&g_tp_error, 1);
        mbar_wait(bar_ld, (uint32_t)(ld_issued - 1) & 1, wait_limit);
        mma_commit(bar);
        if (n_mma >= 1) mbar_wait(bar, (n_mma - 1) & 1, wait_limit);
        mbar_wait(bar, n_mma & 1, wait_limit);
    }
    if (tid == 0 || tid == 128) bulk_wait_read_all();
    tc_fence_before();
    sync_all();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

// ---- the exact path: chunks whose cumulative decay leaves the fast path's range ----------
// One CTA per listed chunk (grid-stride over the list), fp32 on CUDA cores throughout, from
// the inputs in global memory: gamma by a scan per key channel, then per-pair decays
//   A_ij = sum_d b_id k_id k_jd e^(gamma_id - gamma_jd)   (i > j)
//   P_ij = sum_d q_id k_jd e^(gamma_id - gamma_jd)         (i >= j)
// T = (I + A)^-1 by forward substitution row by row, W = T Kh, U = T (w.v) with
// Kh = b.k.e^gamma, and the record's tiles written element by element.  Rarely run.
constexpr int XS = 129;   // padded fp32 row stride of the [64][128] arrays
constexpr int XOFF_G = 0;                    // gamma [64][XS]
constexpr int XOFF_K = XOFF_G + 64 * XS * 4; // k [64][XS]
constexpr int XOFF_Q = XOFF_K + 64 * XS * 4; // q, then w.v [64][XS]
constexpr int XOFF_B = XOFF_Q + 64 * XS * 4; // b.k [64][XS] (Kh before the decay)
constexpr int XOFF_A = XOFF_B + 64 * XS * 4; // A [64][65]
constexpr int XOFF_T = XOFF_A + 64 * 65 * 4; // T [64][65]
constexpr int XOFF_GC = XOFF_T + 64 * 65 * 4;   // gamma_C [128]
constexpr int XSMEM = XOFF_GC + 512;

__global__ void __launch_bounds__(kThreads, 1) wy_exact_kernel(ChunkArgs a, unsigned char *records, const int *list) {
    extern __shared__ float xs[];
    float *sG = xs + XOFF_G / 4, *sK = xs + XOFF_K / 4, *sQ = xs + XOFF_Q / 4, *sBK = xs + XOFF_B / 4;
    float *sA = xs + XOFF_A / 4, *sT = xs + XOFF_T / 4, *sGC = xs + XOFF_GC / 4;
    const int tid = threadIdx.x;
    const int nch = (a.T + C - 1) / C;
    const int count = list[0];
    const int mode = a.mode;
    const bool vec_b = mode_b_vec(mode), vec_w = mode_w_vec(mode), vec_g = mode_g_vec(mode);
    const __nv_bfloat16 *Q = (const __nv_bfloat16 *)a.q, *K = (const __nv_bfloat16 *)a.k;
    const __nv_bfloat16 *V = (const __nv_bfloat16 *)a.v, *Bg = (const __nv_bfloat16 *)a.b;
    const __nv_bfloat16 *Wg = (const __nv_bfloat16 *)a.w;
    const __nv_bfloat16 *Wsc = mode == GDR_MODE_BONLY ? Wg : Bg;
#pragma unroll 1
    for (int li = blockIdx.x; li < count; li += gridDim.x) {
        const int unit = list[1 + li];
        if (!GDR_IN_BOUNDS(unit >= 0 && unit < a.B * a.H * nch, 702)) continue;
        const int bh = unit / nch, c = unit % nch;
        const int t0 = c * C, n = min(C, a.T - t0);
        const size_t row0 = (size_t)bh * a.T + t0;
        unsigned char *rec = records + (size_t)unit * REC_BYTES;
        __syncthreads();   // the previous chunk's readers are done with the arrays
        // inputs (zero past the chunk's end) and gamma
        for (int e = tid; e < C * DK; e += kThreads) {
            const int t = e >> 7, dd = e & 127;
            const bool in = t < n;
            const size_t ge = (row0 + t) * DK + dd;
            const float kv = in ? __bfloat162float(K[ge]) : 0.f;
            const float bv = in ? __bfloat162float(vec_b ? Bg[ge] : Bg[row0 + t]) : 0.f;
            sK[t * XS + dd] = kv;
            sQ[t * XS + dd] = in ? __bfloat162float(Q[ge]) : 0.f;
            sBK[t * XS + dd] = bv * kv;
        }
        if (tid < DK) {
            float g = 0.f;
            for (int t = 0; t < C; ++t) {
                if (t < n) g += vec_g ? a.g[(row0 + t) * DK + tid] : a.g[row0 + t];
                sG[t * XS + tid] = g;
            }
            sGC[tid] = g;
        }
        __syncthreads();
        // A and P from per-pair decays; P straight into the record
        for (int p = tid; p < C * C; p += kThreads) {
            const int i = p >> 6, j = p & 63;
            float sa = 0.f, sp = 0.f;
            if (j <= i && i < n) {
                for (int dd = 0; dd < DK; ++dd) {
                    const float kd = sK[j * XS + dd] * __expf(sG[i * XS + dd] - sG[j * XS + dd]);
                    sa = fmaf(sBK[i * XS + dd], kd, sa);
                    sp = fmaf(sQ[i * XS + dd], kd, sp);
                }
            }
            sA[i * 65 + j] = j < i ? sa : 0.f;
            st_bf16(rec + REC_P + tile_off(64, i, j), sp);
        }
        __syncthreads();
        // T = (I + A)^-1 by forward substitution; thread j < 64 owns column j, whose rows
        // depend only on its own rows above: T_ij = [i == j] - sum_{j<=m<i} A_im T_mj
        if (tid < C) {
            const int j = tid;
            for (int i = 0; i < C; ++i) {
                float x = i == j ? 1.f : 0.f;
                for (int m = j; m < i; ++m) x = fmaf(-sA[i * 65 + m], sT[m * 65 + j], x);
                sT[i * 65 + j] = j <= i ? x : 0.f;
            }
        }
        __syncthreads();
        // the operands: Kh = b.k.e^gamma in place, Qg, K_end; w.v over q
        for (int e = tid; e < C * DK; e += kThreads) {
            const int t = e >> 7, dd = e & 127;
            const float gm = sG[t * XS + dd];
            const float eg = __expf(gm);
            st_bf16(rec + REC_QG + tile_off(64, t, dd), sQ[t * XS + dd] * eg);
            st_bf16(rec + REC_KB + tile_off(64, t, dd), sK[t * XS + dd] * __expf(sGC[dd] - gm));
            sBK[t * XS + dd] *= eg;
        }
        __syncthreads();
        for (int e = tid; e < C * DV; e += kThreads) {
            const int t = e >> 7, vv = e & 127;
            float x = 0.f;
            if (t < n) {
                const size_t ge = (row0 + t) * DV + vv;
                const float wv = __bfloat162float(vec_w ? Wg[ge] : Wsc[row0 + t]);
                x = wv * __bfloat162float(V[ge]);
            }
            sQ[t * XS + vv] = x;
        }
        __syncthreads();
        // W^T [d][t] = sum_j Kh[j][d] T[t][j],  U^T [v][t] = sum_j wv[j][v] T[t][j]
        for (int e = tid; e < C * DK; e += kThreads) {
            const int t = e >> 7, dd = e & 127;
            float w = 0.f, u = 0.f;
            for (int j = 0; j <= t; ++j) {
                const float tj = sT[t * 65 + j];
                w = fmaf(sBK[j * XS + dd], tj, w);
                u = fmaf(sQ[j * XS + dd], tj, u);
            }
            st_bf16(rec + REC_WT + tile_off(128, dd, t), w);
            st_bf16(rec + REC_UT + tile_off(128, dd, t), u);
        }
        if (tid < DK) reinterpret_cast<float *>(rec + REC_EGC)[tid] = __expf(sGC[tid]);
        if (tid == 0) *reinterpret_cast<int *>(rec + REC_FLAG) = 1;
    }
}

}  // namespace

unsigned long long records_bytes(int B, int H, int T) {
    return (unsigned long long)B * H * ((T + C - 1) / C) * REC_BYTES;
}
unsigned long long list_bytes(int B, int H, int T) {
    const unsigned long long n = 1ull + (unsigned long long)B * H * ((T + C - 1) / C);
    return (n * 4 + 15) / 16 * 16;
}

namespace {

// [rows][128] bf16 row-major, box {64 elements, 64 rows}, 128-byte swizzle, zero fill
bool encode_rows(CUtensorMap *m, const void *base, unsigned long long rows) {
    auto fn = tensor_map_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)DK, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)DK * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)C};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

gdr_status_t launch_wy_prep(const ChunkArgs &a, unsigned char *records, int *list, cudaStream_t s) {
    const long long units = (long long)a.B * a.H * ((a.T + C - 1) / C);
    if (units <= 0) return GDR_OK;
    const unsigned long long rows = (unsigned long long)a.B * a.H * a.T;
    PrepMaps tm;
    memset(&tm, 0, sizeof(tm));
    if (!encode_rows(&tm.q, a.q, rows) || !encode_rows(&tm.k, a.k, rows) || !encode_rows(&tm.v, a.v, rows) ||
        (mode_b_vec(a.mode) && !encode_rows(&tm.b, a.b, rows)))
        return GDR_ERR_CUDA;
    if (cudaFuncSetAttribute(wy_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) !=
            cudaSuccess ||
        cudaFuncSetAttribute(wy_exact_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, XSMEM) != cudaSuccess)
        return GDR_ERR_CUDA;
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return GDR_ERR_CUDA;
    // persistent: two CTAs per SM (their shared memory and TMEM fit twice), chunks in turn
    const long long grid = units < 2LL * sms ? units : 2LL * sms;
    wy_prep_kernel<<<(unsigned)grid, kThreads, SMEM_BYTES, s>>>(a, records, list, tm);
    wy_exact_kernel<<<(unsigned)(units < sms ? units : sms), kThreads, XSMEM, s>>>(a, records, list);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

cudaError_t two_phase_read_and_clear_error(int *err) {
    int e1 = 0, e2 = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&e1, g_tp_error, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    if ((e = cudaMemcpyToSymbol(g_tp_error, &zero, sizeof(int))) != cudaSuccess) return e;
    if ((e = state_pass_read_and_clear_error(&e2)) != cudaSuccess) return e;
    *err = e1 || e2;
    return cudaSuccess;
}

}  // namespace tp

GDR_BOUNDS_READER(wy_prep_bounds_site)

}  // namespace gdr
