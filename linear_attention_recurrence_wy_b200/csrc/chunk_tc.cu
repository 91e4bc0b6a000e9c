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
//   T       = (I + A)^-1              blocked substitution (tri_inverse.cuh)
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
// Data movement: each chunk's raw inputs arrive by bulk copies (one per tensor) into a
// staging area, issued one chunk ahead and backed by L2 prefetches two chunks ahead.
// The bf16 copies of S^T and E^T that feed the MMAs as A operands stay in TMEM.
// Schedule (16 warps): all warps build the operands; while the tensor cores form [A; P],
// warps 8-15 write the previous chunk's output rows and scale its state, whose first
// reader is this chunk's S^T Qg^T MMA, issued together with W^T and U^T.
//
// Every wait on an mbarrier is bounded; on expiry the kernel records the failure in
// g_tc_error, stops issuing work, waits (bounded) for its own bulk copies and
// tensor-core work to drain, frees its TMEM and returns.
#include "chunk_tc.cuh"
#include "tc_util.cuh"
#include "tri_inverse.cuh"

namespace gdr {

__device__ int g_tc_error = 0;

namespace {

using namespace tc;

constexpr int C = 64, DK = 128, DV = 128;
constexpr int kThreads = 512;
constexpr uint32_t kWaitLimit = 1u << 24;
constexpr float kFastLimit = 60.f;
constexpr int kAS = tri::LD;   // fp32 row stride of the A / T scratch

// shared memory map (byte offsets from a 1024-aligned base)
constexpr int RAW_Q = 0;                        // raw q bf16 [64][128]   16 KB
constexpr int RAW_K = RAW_Q + 16384;            // raw k                  16 KB
constexpr int RAW_V = RAW_K + 16384;            // raw v                  16 KB
constexpr int RAW_B = RAW_V + 16384;            // raw b (GDN-2)          16 KB
constexpr int RAW_W = RAW_B + 16384;            // raw w (GDN-2)          16 KB
constexpr int RAW_G = RAW_W + 16384;            // raw g_log fp32 [64][128] 32 KB; gamma (exact path)
constexpr int RAW_END = RAW_G + 32768;
// once a chunk's operands are built, raw v, b and w are dead: the inverse's scratch
constexpr int OFF_A32 = RAW_V;                  // A fp32 [64][68]
constexpr int OFF_T32 = OFF_A32 + 64 * kAS * 4; // T fp32 [64][68]
constexpr int OFF_X = OFF_T32 + 64 * kAS * 4;   // 4 x [16][20] fp32
static_assert(OFF_X + 4 * 16 * tri::XLD * 4 <= RAW_G, "inverse scratch must fit in raw v, b, w");
constexpr int OFF_QK = RAW_END;                 // [Kh;Qg] bf16 [128][128]  32 KB
constexpr int OFF_KB = OFF_QK + 32768;          // Kb    bf16 [64 t][128 d] 16 KB
constexpr int OFF_WV = OFF_KB + 16384;          // WV    bf16 [64 t][128 v] 16 KB
constexpr int OFF_P = OFF_WV + 16384;           // P     bf16 [64 t][64 j]   8 KB
constexpr int OFF_T = OFF_P + 8192;             // T     bf16 [64 t][64 j]   8 KB
constexpr int OFF_WT = OFF_T + 8192;            // W^T   bf16 [128 d][64 t] 16 KB
constexpr int OFF_TOT = OFF_WT + 16384;         // scan: quarter totals fp32 [4][128]
constexpr int OFF_GS = OFF_TOT + 2048;          // scalar g_log of the chunk (GDN) fp32 [64]
constexpr int OFF_GC = OFF_GS + 256;            // gamma_C fp32 [128]
constexpr int OFF_EGC = OFF_GC + 512;           // exp(gamma_C) fp32 [2][128], by chunk parity
constexpr int OFF_BAR = OFF_EGC + 1024;         // 2 mbarriers + TMEM slot
constexpr int SMEM_BYTES = OFF_BAR + 64 + 1024; // + alignment slack

// TMEM columns
constexpr uint32_t TM_S = 0;     // S^T fp32            128 cols
constexpr uint32_t TM_O = 128;   // O^T fp32             64
constexpr uint32_t TM_E = 192;   // U^T, then E^T fp32   64
constexpr uint32_t TM_W = 256;   // W^T fp32             64
constexpr uint32_t TM_AP = 320;  // [A; P] fp32          64
constexpr uint32_t TM_SB = 384;  // S^T bf16 (packed)    64
constexpr uint32_t TM_EB = 448;  // E^T bf16 (packed)    32
constexpr uint32_t TM_COLS = 512;

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

// 32 fp32 values -> 16 packed bf16 pairs -> TMEM
__device__ __forceinline__ void st_tmem_bf16(uint32_t taddr, const float (&x)[32]) {
    uint32_t r[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) r[j] = pack_bf16(x[2 * j], x[2 * j + 1]);
    tmem_st16(taddr, r);
}

// Final values of T (from the inverse) straight into the bf16 operand tile.
struct TileOut {
    uint32_t tile;   // shared address of the T tile ([64 t][64 j], 128-byte swizzled)
    __device__ __forceinline__ void chunk(int row, int c8, const float (&v)[8]) {
        st_chunk(tile + tile_chunk(64, row, c8), v);
    }
    __device__ __forceinline__ void pair(int row, int col, float v0, float v1) {
        const uint32_t x = pack_bf16(v0, v1);
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(tile + tile_off(64, row, col)), "r"(x) : "memory");
    }
};

// barrier over warps 0-3 (named barrier 1)
struct Bar128 {
    __device__ __forceinline__ void operator()() const { asm volatile("bar.sync 1, 128;" ::: "memory"); }
};

struct Waiter {
    uint32_t bar, phase;
    // all threads wait for the barrier's next phase; false (everywhere) if any gave up
    __device__ __forceinline__ bool all() {
        const bool mine = mbar_wait(bar, phase, kWaitLimit);
        phase ^= 1u;
        const bool ok = !__syncthreads_or(!mine);
        tc_fence_after();
        return ok;
    }
};

__global__ void __launch_bounds__(kThreads, 1) chunk_tc_kernel(ChunkArgs a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3;   // TMEM lanes this warp may access: 32 * quarter + [0, 32)
    // ---- this CTA's job: one sequence-head, one segment of it, one role ----
    const int roles = a.pass ? max(1, 2 * a.nseg - 3) : a.nseg;
    const int bh = blockIdx.x / roles, role = blockIdx.x % roles;
    const bool transfer = a.pass && role > a.nseg - 2;       // transition-matrix run
    const int seg = transfer ? role - (a.nseg - 2) : role;
    const int t_begin = seg * a.seg_len;
    const int T = min(a.seg_len, a.T - t_begin);              // tokens of this segment
    const int mode = a.mode;
    const size_t tok0 = (size_t)bh * a.T + t_begin;
    const int nchunks = (T + C - 1) / C;
    const size_t sidx = ((size_t)bh * a.nseg + seg) * DK * DV;
    const float *S0p = nullptr;        // initial state (NULL: zero, unless the identity)
    float *STp = nullptr;              // end state destination (NULL: not written)
    if (!a.pass) {
        S0p = a.nseg == 1 ? (a.S0 ? a.S0 + (size_t)bh * DK * DV : nullptr) : a.ws_sstart + sidx;
        STp = seg == a.nseg - 1 ? (a.ST ? a.ST + (size_t)bh * DK * DV : nullptr) : nullptr;
    } else {
        S0p = (!transfer && seg == 0 && a.S0) ? a.S0 + (size_t)bh * DK * DV : nullptr;
        STp = transfer ? a.ws_m + sidx : a.ws_send + sidx;
    }
    const bool write_o = !a.pass;

    float *sA32 = reinterpret_cast<float *>(sm + OFF_A32);
    float *sT32 = reinterpret_cast<float *>(sm + OFF_T32);
    float *sX = reinterpret_cast<float *>(sm + OFF_X);
    float *sGam = reinterpret_cast<float *>(sm + RAW_G);
    float *sTot = reinterpret_cast<float *>(sm + OFF_TOT);
    float *sGs = reinterpret_cast<float *>(sm + OFF_GS);
    float *sGC = reinterpret_cast<float *>(sm + OFF_GC);
    float *sEGC = reinterpret_cast<float *>(sm + OFF_EGC);
    const uint32_t bar_mma = sbase + OFF_BAR, bar_raw = sbase + OFF_BAR + 8;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 16);

    const __nv_bfloat16 *Q = (const __nv_bfloat16 *)a.q, *K = (const __nv_bfloat16 *)a.k;
    const __nv_bfloat16 *V = (const __nv_bfloat16 *)a.v, *Bg = (const __nv_bfloat16 *)a.b;
    const __nv_bfloat16 *Wg = (const __nv_bfloat16 *)a.w;
    __nv_bfloat16 *O = (__nv_bfloat16 *)a.o;
    const bool gdn2 = (mode == GDR_MODE_GDN2), vec_g = (mode != GDR_MODE_GDN);

    if (tid == 0) {
        mbar_init(bar_mma, 1);
        mbar_init(bar_raw, 1);
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
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;

    // raw inputs of chunk c -> staging (one bulk copy per tensor), thread 0 only
    auto issue_raw = [&](int c) {
        const int t0 = c * C, n = min(C, T - t0);
        const size_t e = (tok0 + t0) * DK;
        const uint32_t row16 = (uint32_t)n * DK * 2;
        uint32_t bytes = 3 * row16;
        if (gdn2) bytes += 2 * row16;
        if (vec_g) bytes += 2 * row16;
        fence_async_smem();
        mbar_arrive_expect_tx(bar_raw, bytes);
        bulk_g2s(sbase + RAW_Q, Q + e, row16, bar_raw);
        bulk_g2s(sbase + RAW_K, K + e, row16, bar_raw);
        bulk_g2s(sbase + RAW_V, V + e, row16, bar_raw);
        if (gdn2) {
            bulk_g2s(sbase + RAW_B, Bg + e, row16, bar_raw);
            bulk_g2s(sbase + RAW_W, Wg + e, row16, bar_raw);
        }
        if (vec_g) bulk_g2s(sbase + RAW_G, a.g + e, 2 * row16, bar_raw);
    };
    auto prefetch_inputs = [&](int c) {
        const int t0 = c * C, n = min(C, T - t0);
        const size_t e = (tok0 + t0) * DK;
        prefetch_l2(Q + e, n * DK * 2);
        prefetch_l2(K + e, n * DK * 2);
        prefetch_l2(V + e, n * DV * 2);
        if (gdn2) {
            prefetch_l2(Bg + e, n * DK * 2);
            prefetch_l2(Wg + e, n * DV * 2);
        }
        if (vec_g) prefetch_l2(a.g + e, n * DK * 4);
    };
    if (tid == 0) {
        issue_raw(0);
        if (nchunks > 1) prefetch_inputs(1);
    }
    int raw_issued = 1, raw_done = 0;   // uniform across the block

    // the T tile's blocks above the diagonal are never written: zero the tile once
    reinterpret_cast<uint4 *>(sm + OFF_T)[tid] = make_uint4(0, 0, 0, 0);
    static_assert(kThreads * 16 == 8192, "one 16-byte store per thread clears the T tile");
    // ---- initial state -> TMEM: fp32 S^T and its bf16 operand copy (warps 8-15) ----
    if (warp >= 8) {
        const int v = quarter * 32 + lane, dlo = ((warp - 8) >> 2) * 64;
        for (int d0 = dlo; d0 < dlo + 64; d0 += 32) {
            float x[32];
#pragma unroll
            for (int j = 0; j < 32; ++j)
                x[j] = transfer ? (d0 + j == v ? 1.f : 0.f) : (S0p ? S0p[(size_t)(d0 + j) * DV + v] : 0.f);
            tmem_st32(tmem + lane_base + TM_S + d0, x);
            st_tmem_bf16(tmem + lane_base + TM_SB + d0 / 2, x);
        }
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // Output rows and state update of the previous chunk (warps 8-15).  Runs while
    // warps 0-7 build the next chunk's operands: that chunk's first MMA is the first
    // reader of what is written here.
    auto finish_chunk = [&](int t0p, int np, bool exactp, const float *egc, bool last) {
        const int v = quarter * 32 + lane;
        if (warp < 12) {
            for (int t0c = 0; t0c < 64; t0c += 32) {
                float x[32];
                tmem_ld32(tmem + lane_base + TM_O + t0c, x);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (write_o && t0c + j < np) O[(tok0 + t0p + t0c + j) * DV + v] = __float2bfloat16_rn(x[j]);
            }
        } else {
            for (int d0 = 0; d0 < DK; d0 += 32) {
                float x[32];
                tmem_ld32(tmem + lane_base + TM_S + d0, x);
                tmem_wait_ld();
                if (!exactp) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) x[j] *= egc[d0 + j];
                    tmem_st32(tmem + lane_base + TM_S + d0, x);
                }
                st_tmem_bf16(tmem + lane_base + TM_SB + d0 / 2, x);
                if (last && STp) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) STp[(size_t)(d0 + j) * DV + v] = x[j];
                }
            }
            tmem_wait_st();
        }
        tc_fence_before();
    };

    Waiter Wm{bar_mma, 0u}, Wr{bar_raw, 0u};
    bool ok = true, exact_prev = false;
    int t0_prev = 0, n_prev = 0;

    for (int c = 0; c < nchunks; ++c) {
        const int t0 = c * C, n = min(C, T - t0);
        float *egc = sEGC + (c & 1) * 128;
        // ===== P1: cumulative log-decay, then operands =====
        if (!Wr.all()) { ok = false; break; }
        raw_done = c + 1;
        if (tid == 0 && c + 2 < nchunks) prefetch_inputs(c + 2);
        if (!vec_g) {
            if (tid < 64) sGs[tid] = (tid < n) ? a.g[tok0 + t0 + tid] : 0.f;
            __syncthreads();
        }
        // gamma: each thread scans 16 tokens of one key channel, then adds the totals of
        // the earlier quarters of the chunk.  Tokens past the end contribute zero.
        const int sd = tid & 127, sq = tid >> 7;
        {
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int t = sq * 16 + i;
                const float g = (t < n) ? (vec_g ? sGam[t * DK + sd] : sGs[t]) : 0.f;
                acc += g;
                sGam[t * DK + sd] = acc;
            }
            sTot[sq * 128 + sd] = acc;
        }
        __syncthreads();
        bool big = false;
        {
            float off = 0.f;
#pragma unroll
            for (int u = 0; u < 3; ++u)
                if (u < sq) off += sTot[u * 128 + sd];
            float gm = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int t = sq * 16 + i;
                gm = sGam[t * DK + sd] + off;
                sGam[t * DK + sd] = gm;
                big |= fabsf(gm) > kFastLimit;
            }
            if (sq == 3) {
                sGC[sd] = gm;
                egc[sd] = __expf(gm);
            }
        }
        const bool exact = __syncthreads_or(big);   // also publishes gamma, gamma_C

        {
            // operands: thread (tg, cg) owns tokens 2 tg, 2 tg + 1, channels 8 cg .. 8 cg + 7
            const int tg = tid >> 4, cg = tid & 15;
#pragma unroll 1
            for (int i = 0; i < 2; ++i) {
                const int t = tg * 2 + i;
                const bool in = t < n;
                const uint32_t ro = (uint32_t)(t * DK * 2 + cg * 16);
                const uint4 z = make_uint4(0, 0, 0, 0);
                const uint4 uq = in ? *reinterpret_cast<const uint4 *>(sm + RAW_Q + ro) : z;
                const uint4 uk = in ? *reinterpret_cast<const uint4 *>(sm + RAW_K + ro) : z;
                const uint4 uv = in ? *reinterpret_cast<const uint4 *>(sm + RAW_V + ro) : z;
                const float4 g0 = *reinterpret_cast<const float4 *>(sGam + t * DK + cg * 8);
                const float4 g1 = *reinterpret_cast<const float4 *>(sGam + t * DK + cg * 8 + 4);
                const float gam[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                float fq[8], fk[8], fv[8], fb[8], fw[8];
                bf16x8_to_f32(uq, fq);
                bf16x8_to_f32(uk, fk);
                bf16x8_to_f32(uv, fv);
                if (gdn2) {
                    const uint4 ub = in ? *reinterpret_cast<const uint4 *>(sm + RAW_B + ro) : z;
                    const uint4 uw = in ? *reinterpret_cast<const uint4 *>(sm + RAW_W + ro) : z;
                    bf16x8_to_f32(ub, fb);
                    bf16x8_to_f32(uw, fw);
                } else {
                    const float beta = in ? __bfloat162float(Bg[tok0 + t0 + t]) : 0.f;
#pragma unroll
                    for (int j = 0; j < 8; ++j) fb[j] = fw[j] = beta;
                }
                float kh[8], qg[8], kb[8], wv[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float e = __expf(gam[j]);
                    kh[j] = fb[j] * fk[j] * e;
                    qg[j] = fq[j] * e;
                    wv[j] = transfer ? 0.f : fw[j] * fv[j];
                }
                if (exact) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) kb[j] = fk[j] * __expf(sGC[cg * 8 + j] - gam[j]);
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) kb[j] = fk[j] * __expf(-gam[j]);
                }
                st_chunk(sbase + OFF_QK + tile_chunk(128, t, cg), kh);
                st_chunk(sbase + OFF_QK + tile_chunk(128, 64 + t, cg), qg);
                st_chunk(sbase + OFF_KB + tile_chunk(64, t, cg), kb);
                st_chunk(sbase + OFF_WV + tile_chunk(64, t, cg), wv);
            }
        }
        fence_async_smem();
        __syncthreads();

        // ===== P2: [A;P] = [Kh;Qg] Kb^T | previous chunk's outputs and state (warps 8-15) =====
        if (!exact && tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, false, false, false);
#pragma unroll
            for (int s = 0; s < DK / 16; ++s)
                mma_bf16(tmem + TM_AP, desc_kmajor(sbase + OFF_QK, 128, 0, s),
                         desc_kmajor(sbase + OFF_KB, 64, 0, s), id, s > 0);
            mma_commit(bar_mma);
        }
        if (warp >= 8 && c > 0)
            finish_chunk(t0_prev, n_prev, exact_prev, sEGC + ((c - 1) & 1) * 128, false);
        if (!exact) {
            if (!Wm.all()) { ok = false; break; }
        } else {
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
        }

        // ===== P3: A (fp32, strictly lower) and P (bf16, lower incl.) =====
        if (!exact) {
            if (warp < 8) {
                const int r = quarter * 32 + lane, j0 = (warp >> 2) * 32;   // row of [A; P], columns
                float x[32];
                tmem_ld32(tmem + lane_base + TM_AP + j0, x);
                tmem_wait_ld();
                if (r < 64) {
                    float4 *dst = reinterpret_cast<float4 *>(sA32 + r * kAS + j0);
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
        } else {
            // exact per-pair decays (strong-decay chunks only), from the staged raw inputs
            float av[8], pv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int p = tid + u * kThreads, i = p >> 6, j = p & 63;
                float sa = 0.f, sp = 0.f;
                if (j <= i && i < n) {
                    const __nv_bfloat16 *qi = (const __nv_bfloat16 *)(sm + RAW_Q) + i * DK;
                    const __nv_bfloat16 *ki = (const __nv_bfloat16 *)(sm + RAW_K) + i * DK;
                    const __nv_bfloat16 *kj = (const __nv_bfloat16 *)(sm + RAW_K) + j * DK;
                    const __nv_bfloat16 *bi = (const __nv_bfloat16 *)(sm + RAW_B) + i * DK;
                    const float bs = gdn2 ? 0.f : __bfloat162float(Bg[tok0 + t0 + i]);
                    for (int d = 0; d < DK; ++d) {
                        const float dec = __expf(sGam[i * DK + d] - sGam[j * DK + d]);
                        const float kjd = __bfloat162float(kj[d]) * dec;
                        const float bid = gdn2 ? __bfloat162float(bi[d]) : bs;
                        sa = fmaf(bid * __bfloat162float(ki[d]), kjd, sa);
                        sp = fmaf(__bfloat162float(qi[d]), kjd, sp);
                    }
                }
                av[u] = (j < i) ? sa : 0.f;
                pv[u] = sp;
            }
            __syncthreads();   // raw b is read above and overlaps the A scratch
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int p = tid + u * kThreads, i = p >> 6, j = p & 63;
                sA32[i * kAS + j] = av[u];
                *reinterpret_cast<__nv_bfloat16 *>(sm + OFF_P + tile_off(64, i, j)) = __float2bfloat16_rn(pv[u]);
            }
        }
        __syncthreads();

        // ===== P4: T = (I + A)^-1 =====
        if (warp < 4) tri::inverse64(sA32, sT32, sX, warp, lane, Bar128{}, TileOut{sbase + OFF_T});
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // the staging area is free again: the next chunk's raw inputs travel from now on
        if (c + 1 < nchunks) {
            raw_issued = c + 2;
            if (tid == 0) issue_raw(c + 1);
        }

        // ===== P5: W^T = Kh^T T^T,  U^T = WV^T T^T,  O^T = S^T Qg^T =====
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
            const uint32_t ido = idesc_bf16(128, 64, false, false, false);
#pragma unroll
            for (int s = 0; s < DK / 16; ++s)
                mma_bf16_ts(tmem + TM_O, tmem + TM_SB + s * 8, desc_kmajor(sbase + OFF_QK, 128, 64, s),
                            ido, s > 0);
            mma_commit(bar_mma);
        }
        if (!Wm.all()) { ok = false; break; }

        // ===== P6: W^T -> bf16 operand (MN-major B); exact chunks pre-scale the state =====
        if (warp < 8) {
            const int d = quarter * 32 + lane, t0c = (warp >> 2) * 32;
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
        } else if (exact) {
            const int dlo = ((warp - 8) >> 2) * 64;
            for (int d0 = dlo; d0 < dlo + 64; d0 += 32) {
                float x[32];
                tmem_ld32(tmem + lane_base + TM_S + d0, x);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) x[j] *= egc[d0 + j];
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
                mma_bf16_ts(tmem + TM_E, tmem + TM_SB + s * 8, desc_mnmajor(sbase + OFF_WT, 128, 0, s),
                            id, 1u);
            mma_commit(bar_mma);
        }
        if (!Wm.all()) { ok = false; break; }

        // ===== P8: E^T -> bf16 operand in TMEM =====
        {
            const int t0c = (warp >> 2) * 16;
            float x[16];
            tmem_ld16(tmem + lane_base + TM_E + t0c, x);
            tmem_wait_ld();
            uint32_t pk[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) pk[j] = pack_bf16(x[2 * j], x[2 * j + 1]);
            tmem_st8(tmem + lane_base + TM_EB + t0c / 2, pk);
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();

        // ===== P9: O^T += E^T P^T,  S^T += E^T Kb (or K_end) =====
        if (tid == 0) {
            tc_fence_after();
            const uint32_t ido = idesc_bf16(128, 64, false, false, false);
            const uint32_t ids = idesc_bf16(128, 128, false, true, false);
#pragma unroll
            for (int s = 0; s < C / 16; ++s) {
                mma_bf16_ts(tmem + TM_O, tmem + TM_EB + s * 8, desc_kmajor(sbase + OFF_P, 64, 0, s),
                            ido, 1u);
                mma_bf16_ts(tmem + TM_S, tmem + TM_EB + s * 8, desc_mnmajor(sbase + OFF_KB, 64, 0, s),
                            ids, 1u);
            }
            mma_commit(bar_mma);
        }
        if (!Wm.all()) { ok = false; break; }
        exact_prev = exact;
        t0_prev = t0;
        n_prev = n;
    }

    if (ok && nchunks > 0) {
        // ===== P10 of the last chunk: output rows, final state =====
        if (warp >= 8)
            finish_chunk(t0_prev, n_prev, exact_prev, sEGC + ((nchunks - 1) & 1) * 128, true);
        tc_fence_before();
        __syncthreads();
    }
    if (!ok) {
        if (tid == 0) atomicExch(&g_tc_error, 1);
        // drain: committed tensor-core work and an outstanding raw copy (bounded waits)
        if (tid == 0) mma_commit(bar_mma);
        mbar_wait(bar_mma, Wm.phase, kWaitLimit);
        if (raw_issued > raw_done) mbar_wait(bar_raw, (uint32_t)(raw_done & 1), kWaitLimit);
    }
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
    const int roles = a.pass ? (2 * a.nseg - 3 > 1 ? 2 * a.nseg - 3 : 1) : a.nseg;
    chunk_tc_kernel<<<(unsigned)(a.B * a.H * roles), kThreads, SMEM_BYTES, s>>>(a);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

cudaError_t chunk_tc_read_and_clear_error(int *err) {
    cudaError_t e = cudaMemcpyFromSymbol(err, g_tc_error, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(int));
}

}  // namespace gdr
