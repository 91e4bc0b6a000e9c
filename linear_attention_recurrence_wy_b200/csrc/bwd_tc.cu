// bwd_tc.cu -- the backward's per-chunk gradients on the tcgen05 tensor cores: bf16
// operands, fp32 accumulation in tensor memory (TMEM).
//
// Shape: dk = dv = 128, bf16 inputs, 64-token chunks, any mode.  One CTA (256 threads) per
// (sequence, head, 64-token chunk): given the state S at the chunk's start (the checkpoint
// pass) and the state gradient dS' at its end (the state-gradient pass), every chunk is
// independent.  With gamma the chunk-local cumulative log-decay, Kh = b.k.e^gamma,
// Qg = q.e^gamma, Kb = k.e^-gamma, W = w.v and dS~ = diag(e^gamma_C) dS' (the chunkwise WY
// form of Gated DeltaNet-2 Review §3-2.5, differentiated for the gate-aware backward of
// §4-3 and of the Gated DeltaNet-2 Q&A page, Q4):
//
//   forward   [A; P] = [Kh; Qg] Kb^T        T = (I + A)^-1        X^T = S^T Kh^T
//             R^T = W^T - X^T               E^T = R^T T^T          (E = T (W - Kh S))
//   backward  dE^T = dS~^T Kb^T + dO^T P    dR^T = dE^T T          (dR = T^T dE)
//             [dA; dP] = [-dR; dO] E^T      dA strictly lower, dP lower incl. (diagonal apart)
//             [dKh | dQg]^T = S [-dR; dO]^T + Kb^T [dA; dP]^T
//             dKb^T = [Kh; Qg]^T [dA; dP]   dKe^T = dS~ E^T
//
// The gradient of A needs no products with T: dA = -T^T (dE R^T) T^T = -(T^T dE)(T R)^T =
// -dR E^T, so dA and dP share one MMA.  dKe is e^gamma_C times the gradient of
// Ke = k.e^(gamma_C - gamma), the key operand of the state update, so it enters exactly
// like dKb.  The diagonal of dP pairs a token with itself, where the decay factors cancel:
// it is left out of the MMA operand (whose rounding would leave a residue in dgamma of the
// size of the whole pair term) and added as dP_tt k_t to dq and dP_tt q_t to dk.  Per
// (token, key channel), on CUDA cores:
//
//   dq = dQg e^gamma + dP_tt k      dk = dKh b e^gamma + (dKb + dKe) e^-gamma + dP_tt q
//   db = dKh k e^gamma              dgamma = dQg Qg + dKh Kh - (dKb + dKe) Kb
//   dgamma_C = sum_v S dS~ + sum_t dKe Kb       dg = dgamma_C + reverse cumulative sum of dgamma
//
// and per (token, value channel) dv = dR w, dw = dR v (scalar gates fold over channels).
// Every factor stays within e^+-60 when |gamma| <= 60 on the whole chunk.  A chunk with a
// stronger cumulative decay is left to the CUDA-core kernel (exact per-pair decays): the
// CTA appends its index to the list that kernel works through.
//
// Every wait on an mbarrier is bounded; on expiry the CTA records the failure in
// g_bwd_tc_error, waits (bounded) for its own tensor-core work and copies, frees its TMEM
// and returns.
#include "bounds.cuh"
#include "bwd_tc.cuh"
#include "tc_util.cuh"
#include "tri_inverse.cuh"

namespace gdr {

__device__ int g_bwd_tc_error = 0;

namespace {

using namespace tc;

constexpr int C = 64, DK = 128, DV = 128;
constexpr int kThreads = 256;
constexpr float kFastLimit = 60.f;

// shared memory map (byte offsets from a 1024-aligned base)
constexpr int OFF_RQ = 0;                 // raw q bf16 [64][128]                        16 KB
constexpr int OFF_RK = OFF_RQ + 16384;    // raw k                                       16 KB
constexpr int OFF_RB = OFF_RK + 16384;    // raw b (per-channel erase gate)              16 KB
constexpr int OFF_G = OFF_RB + 16384;     // raw g_log fp32 [64][128], e^gamma, dgamma   32 KB
constexpr int OFF_SB = OFF_G + 32768;     // S   bf16 [128 d][128 v]                     32 KB
constexpr int OFF_DSB = OFF_SB + 32768;   // dS~ bf16 [128 d][128 v]                     32 KB
constexpr int OFF_QK = OFF_DSB + 32768;   // [Kh; Qg] bf16 [128][128 d]                  32 KB
constexpr int OFF_KB = OFF_QK + 32768;    // Kb bf16 [64 t][128 d]                       16 KB
constexpr int OFF_P = OFF_KB + 16384;     // P bf16 [64 t][64 j]                          8 KB
constexpr int OFF_T = OFF_P + 8192;       // T bf16 [64 t][64 j]                          8 KB
// regions reused once their first contents are dead
constexpr int OFF_A32 = OFF_RQ;           // A, then T, fp32 [64][68] (after the operand build)
constexpr int OFF_X = OFF_A32 + 64 * tri::LD * 4;   // the inverse's scratch, 4 x [16][20] fp32
constexpr int OFF_DOR = OFF_RQ;           // [-dR^T | dO^T] bf16 [128 v][128] (after the inverse)
constexpr int OFF_ET = OFF_RB;            // E^T bf16 [128 v][64 t]                      16 KB
constexpr int OFF_DAP = OFF_P;            // [dA; dP] bf16 [128][64 j] (over P and T)    16 KB
constexpr int OFF_RDO = OFF_QK;           // raw dO, v, w bf16 [64][128] each (until the build)
constexpr int OFF_RV = OFF_QK + 16384;
constexpr int OFF_RW = OFF_KB;
// small arrays
constexpr int OFF_GC = OFF_T + 8192;      // gamma_C fp32 [128]
constexpr int OFF_EGC = OFF_GC + 512;     // exp(gamma_C) [128]
constexpr int OFF_DGC = OFF_EGC + 512;    // sum_v S dS' per key channel [128]
constexpr int OFF_CAR = OFF_DGC + 512;    // the epilogue's exchange between token halves [3][128]
constexpr int OFF_BETA = OFF_CAR + 1536;  // scalar erase gate of the chunk's tokens [64]
constexpr int OFF_GS = OFF_BETA + 256;    // scalar g_log (GDN) [64]
constexpr int OFF_FOLD = OFF_GS + 256;    // scalar-gate gradients [3][64]: b, w, g
constexpr int OFF_DPD = OFF_FOLD + 768;   // the diagonal of dP [64]
constexpr int OFF_FLAG = OFF_DPD + 256;   // [0] strong decay (exact path), [1] abort
constexpr int OFF_BAR = OFF_FLAG + 16;    // mbarriers: raw copies, MMA commits; TMEM slot
constexpr int SMEM_BYTES = OFF_BAR + 2 * 8 + 8 + 1024;   // + alignment slack
static_assert(OFF_X + 4 * 16 * tri::XLD * 4 <= OFF_RB, "the inverse's scratch fits over raw q and k");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");

// TMEM columns (fp32 unless noted); lane = value channel for X, E, dE, dR, lane = key
// channel for dKh, dQg, dKb, dKe, lane = row of [A; P] and [dA; dP]
constexpr uint32_t TM_AP = 0;      // [A; P], then [dA; dP]                             64
constexpr uint32_t TM_X = 64;      // X^T, then dR^T                                    64
constexpr uint32_t TM_E = 128;     // E^T                                               64
constexpr uint32_t TM_DE = 192;    // dE^T                                              64
constexpr uint32_t TM_DQK = 256;   // [dKh | dQg]^T                                    128
constexpr uint32_t TM_DKB = 384;   // dKb^T; before it, dE^T bf16 (packed)              64
constexpr uint32_t TM_DKE = 448;   // dKe^T; before it, R^T and dO^T bf16 (packed)      64
constexpr uint32_t TM_DEB = TM_DKB;
constexpr uint32_t TM_RB = TM_DKE;
constexpr uint32_t TM_DOB = TM_DKE + 32;
constexpr uint32_t TM_VB = TM_DQK;         // v and w bf16 (packed), steps 1 to 9
constexpr uint32_t TM_WB = TM_DQK + 32;
constexpr uint32_t TM_COLS = 512;

__device__ __forceinline__ float bf(const __nv_bfloat16 *p, size_t i) { return __bfloat162float(p[i]); }

// sum over the 32 lanes of a warp, returned to every lane
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// One instantiation per mode (the gate shapes are compile-time: the kernel's code is run
// once per chunk, so every branch left in it costs instruction fetch).
template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) bwd_tc_kernel(BwdArgs a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3;                       // TMEM lanes 32 quarter .. + 31
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int r = quarter * 32 + lane;                  // this thread's TMEM lane
    const int j0 = (warp >> 2) * 32;                    // and its 32 token columns

    // ---- this CTA's chunk ----
    const int T = a.T;
    const int nchunk = (T + C - 1) / C;
    const int bh = blockIdx.x / nchunk, c = blockIdx.x - bh * nchunk;
    const int t0 = c * C, n = min(C, T - t0);
    const size_t tok0 = (size_t)bh * T + t0;            // row of the chunk's first token
    // the workspace has one fp32-sized state slot per 32-token chunk: S at this chunk's start
    // is in the slot of its first 32-token chunk, dS' at its end in the slot of its last one,
    // both as bf16 [dk][dv] (the tensor-core passes write them so)
    const int nslot = (T + kBwdChunk - 1) / kBwdChunk;
    const float *Sg = a.ws_states + ((size_t)bh * nslot + 2 * c) * DK * DV;
    const float *dSg = a.ws_dstates + ((size_t)bh * nslot + min(2 * c + 1, nslot - 1)) * DK * DV;
    // debug build: this chunk and its two state slots lie inside what the arguments imply
    // (a uniform condition: a failing CTA returns before its first barrier)
    if (!GDR_IN_BOUNDS(bh < a.B * a.H && n >= 1 && t0 + n <= T && 2 * c < nslot, 301)) return;

    const __nv_bfloat16 *Q = (const __nv_bfloat16 *)a.q, *K = (const __nv_bfloat16 *)a.k;
    const __nv_bfloat16 *V = (const __nv_bfloat16 *)a.v, *Bg = (const __nv_bfloat16 *)a.b;
    const __nv_bfloat16 *Wg = (const __nv_bfloat16 *)a.w, *dOg = (const __nv_bfloat16 *)a.dO;
    __nv_bfloat16 *dQo = (__nv_bfloat16 *)a.dq, *dKo = (__nv_bfloat16 *)a.dk;
    __nv_bfloat16 *dVo = (__nv_bfloat16 *)a.dv, *dBo = (__nv_bfloat16 *)a.db, *dWo = (__nv_bfloat16 *)a.dw;
    // gate shapes: per-channel erase b (GDN-2, b-only), per-channel write w (GDN-2, w-only),
    // per-channel decay (all but GDN); a scalar write gate is w itself (b-only) or beta in b
    constexpr bool vec_b = mode_b_vec(MODE), vec_w = mode_w_vec(MODE), vec_g = mode_g_vec(MODE);
    constexpr bool tied = MODE == GDR_MODE_KDA || MODE == GDR_MODE_GDN;
    const __nv_bfloat16 *Wsc = MODE == GDR_MODE_BONLY ? Wg : Bg;

    float *sG = reinterpret_cast<float *>(sm + OFF_G);
    float *sA32 = reinterpret_cast<float *>(sm + OFF_A32);
    float *sX = reinterpret_cast<float *>(sm + OFF_X);
    float *sGC = reinterpret_cast<float *>(sm + OFF_GC);
    float *sEGC = reinterpret_cast<float *>(sm + OFF_EGC);
    float *sDGC = reinterpret_cast<float *>(sm + OFF_DGC);
    float *sCar = reinterpret_cast<float *>(sm + OFF_CAR);
    float *sBeta = reinterpret_cast<float *>(sm + OFF_BETA);
    float *sGs = reinterpret_cast<float *>(sm + OFF_GS);
    float *sFb = reinterpret_cast<float *>(sm + OFF_FOLD), *sFw = sFb + 64, *sFg = sFb + 128;
    float *sDPd = reinterpret_cast<float *>(sm + OFF_DPD);
    volatile int *sFlag = reinterpret_cast<volatile int *>(sm + OFF_FLAG);
    const uint32_t bar_raw = sbase + OFF_BAR, bar_mma = bar_raw + 8;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 16);

    if (tid == 0) {
        mbar_init(bar_raw, 1);
        mbar_init(bar_mma, 1);
        sFlag[0] = 0;
        sFlag[1] = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tslot), TM_COLS);
        tmem_relinquish();
    }
    // the T tile's blocks above the diagonal are never written by the inverse
    reinterpret_cast<uint4 *>(sm + OFF_T)[tid] = make_uint4(0, 0, 0, 0);
    reinterpret_cast<uint4 *>(sm + OFF_T)[tid + kThreads] = make_uint4(0, 0, 0, 0);
    static_assert(kThreads * 32 == 8192, "two 16-byte stores per thread clear the T tile");
    if (tid < 192) sFb[tid] = 0.f;
    // scalar gates of the chunk's tokens, zero past the end
    if (tid < 64) {
        if (!vec_g) sGs[tid] = tid < n ? a.g[tok0 + tid] : 0.f;
    } else if (tid < 128) {
        if (!vec_b) sBeta[tid - 64] = tid - 64 < n ? bf(Bg, tok0 + tid - 64) : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    int commits = 0;          // MMA commits issued on bar_mma (thread 0)
    int raw_copies = 0;       // rounds of raw input copies issued on bar_raw
    bool raw_pending = false;
    // Bounded wait for a phase of an mbarrier: thread 0 polls, the block meets at a barrier.
    // test hook (see BwdArgs): the first wait, on the raw copies, polls them right after they
    // are issued, a few non-blocking times, and gives up while they are still in flight
    bool first_expired = false;
    auto wait_bar = [&](uint32_t bar, uint32_t parity) -> bool {
        if (tid == 0 && (first_expired || !mbar_wait(bar, parity, a.wait_limit))) sFlag[1] = 1;
        first_expired = false;
        __syncthreads();
        return sFlag[1] == 0;
    };
    auto wait_mma = [&]() -> bool { return wait_bar(bar_mma, (uint32_t)((commits - 1) & 1)); };

    do {
        // ---- 1. raw q, k, b, g_log, dO, v, w of the chunk: one bulk copy per tensor (dO, v
        //      and w into the operand tiles, which the build fills only after they are read) ----
        if (tid == 0) {
            const uint32_t row16 = (uint32_t)n * DK * 2;
            fence_async_smem();
            mbar_arrive_expect_tx(bar_raw, (4 + (vec_b ? 1 : 0) + (vec_g ? 2 : 0) + (vec_w ? 1 : 0)) * row16);
            bulk_g2s(sbase + OFF_RQ, Q + tok0 * DK, row16, bar_raw);
            bulk_g2s(sbase + OFF_RK, K + tok0 * DK, row16, bar_raw);
            if (vec_b) bulk_g2s(sbase + OFF_RB, Bg + tok0 * DK, row16, bar_raw);
            if (vec_g) bulk_g2s(sbase + OFF_G, a.g + tok0 * DK, 2 * row16, bar_raw);
            bulk_g2s(sbase + OFF_RDO, dOg + tok0 * DV, row16, bar_raw);
            bulk_g2s(sbase + OFF_RV, V + tok0 * DV, row16, bar_raw);
            if (vec_w) bulk_g2s(sbase + OFF_RW, Wg + tok0 * DV, row16, bar_raw);
            if (a.first_wait_limit != 0) {
                bool got = false;
                for (uint32_t i = 0; i < a.first_wait_limit && !got; ++i) got = mbar_test_wait(bar_raw, 0u);
                first_expired = !got;
            }
        }
        ++raw_copies;
        raw_pending = true;
        // S -> bf16 tile and sum_v S dS' per key channel (both stored as bf16 [dk][dv]; warp w:
        // rows 16 w .. 16 w + 15, two per load, 16 lanes of eight channels each); dS' stays in
        // registers until gamma_C is known.  The loads are batched: no load sits behind a
        // branch, so the batch costs one latency.
        uint4 dsr[8];
        {
            const __nv_bfloat16 *Sb = reinterpret_cast<const __nv_bfloat16 *>(Sg);
            const __nv_bfloat16 *dSb = reinterpret_cast<const __nv_bfloat16 *>(dSg);
            uint4 x[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const size_t o = (size_t)(warp * 16 + 2 * i + (lane >> 4)) * DV + 8 * (lane & 15);
                x[i] = *reinterpret_cast<const uint4 *>(Sb + o);
                dsr[i] = *reinterpret_cast<const uint4 *>(dSb + o);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int d = warp * 16 + 2 * i + (lane >> 4);
                st_shared_v4(sbase + OFF_SB + tile_chunk(128, d, lane & 15), x[i].x, x[i].y, x[i].z, x[i].w);
                float fs[8], fd[8];
                bf16x8_to_f32(x[i], fs);
                bf16x8_to_f32(dsr[i], fd);
                float sd = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) sd = fmaf(fs[j], fd[j], sd);
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) sd += __shfl_xor_sync(0xffffffffu, sd, o);   // 16 lanes of row d
                if ((lane & 15) == 0) sDGC[d] = sd;
            }
        }
        // the scalar write gate of the chunk's tokens, if there is one (zero past the end)
        float wsc = 0.f;
        if (!vec_w) wsc = bf(Wsc, tok0 + min(j0 + (lane & 31), n - 1));
        if (!wait_bar(bar_raw, (uint32_t)((raw_copies - 1) & 1))) break;
        raw_pending = false;
        if (tid == 32 && a.prefetch_ahead > 0 && blockIdx.x + (unsigned)a.prefetch_ahead < gridDim.x) {
            // the chunk that starts next on an SM, about one wave of CTAs ahead: its inputs and
            // state slots travel to L2 while this chunk is worked on
            const int un = (int)blockIdx.x + a.prefetch_ahead;
            const int bn = un / nchunk, cn = un - bn * nchunk;
            const int nn = min(C, T - cn * C);
            const size_t tn = (size_t)bn * T + (size_t)cn * C;
            const uint32_t row16 = (uint32_t)nn * DK * 2;
            prefetch_l2(Q + tn * DK, row16);
            prefetch_l2(K + tn * DK, row16);
            if (vec_b) prefetch_l2(Bg + tn * DK, row16);
            if (vec_g) prefetch_l2(a.g + tn * DK, 2 * row16);
            prefetch_l2(dOg + tn * DV, row16);
            prefetch_l2(V + tn * DV, row16);
            if (vec_w) prefetch_l2(Wg + tn * DV, row16);
            prefetch_l2(a.ws_states + ((size_t)bn * nslot + 2 * cn) * DK * DV, DK * DV * 2);
            prefetch_l2(a.ws_dstates + ((size_t)bn * nslot + min(2 * cn + 1, nslot - 1)) * DK * DV, DK * DV * 2);
        }
        // dO^T, v and w of this thread's value channel and tokens -> bf16 in TMEM (v and w in
        // the [dKh | dQg] columns, first written in step 10); rows past the end are zero
        {
            const __nv_bfloat16 *rdo = reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_RDO);
            const __nv_bfloat16 *rv = reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_RV);
            const __nv_bfloat16 *rw = reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_RW);
            float x[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) x[j] = (j0 + j < n) ? __bfloat162float(rdo[(j0 + j) * DV + r]) : 0.f;
            st_tmem_bf16(tmem + lane_base + TM_DOB + j0 / 2, x);
#pragma unroll
            for (int j = 0; j < 32; ++j) x[j] = (j0 + j < n) ? __bfloat162float(rv[(j0 + j) * DV + r]) : 0.f;
            st_tmem_bf16(tmem + lane_base + TM_VB + j0 / 2, x);
#pragma unroll
            for (int j = 0; j < 32; ++j)
                x[j] = vec_w ? ((j0 + j < n) ? __bfloat162float(rw[(j0 + j) * DV + r]) : 0.f)
                             : __shfl_sync(0xffffffffu, wsc, j);
            st_tmem_bf16(tmem + lane_base + TM_WB + j0 / 2, x);
        }
        // ---- 2. cumulative log-decay: thread d < 128 scans key channel d and leaves e^gamma
        //      in place of g_log; any |gamma| > 60 sends the chunk to the exact path ----
        if (tid < DK) {
            const int d = tid;
            float acc = 0.f, mx = 0.f;
#pragma unroll 1
            for (int b = 0; b < C; b += 16) {
                float x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] = vec_g ? sG[(b + i) * DK + d] : sGs[b + i];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    acc += (b + i < n) ? x[i] : 0.f;
                    mx = fmaxf(mx, fabsf(acc));
                    x[i] = __expf(acc);
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) sG[(b + i) * DK + d] = x[i];
            }
            sGC[d] = acc;
            sEGC[d] = __expf(acc);
            if (mx > kFastLimit) sFlag[0] = 1;
        }
        __syncthreads();
        if (sFlag[0]) {
            if (tid == 0) {
                const int k = atomicAdd(a.tc_list, 1);
                // the list holds one entry per 64-token span of every sequence-head
                if (GDR_IN_BOUNDS(k < a.B * a.H * nchunk, 302)) a.tc_list[1 + k] = blockIdx.x;
            }
            break;
        }
        // ---- 3. operands: Kh, Qg, Kb (thread (tg, cg): tokens 4 tg .. + 3, channels
        //      8 cg .. + 7), and dS~ = diag(e^gamma_C) dS' ----
        {
            const int tg = tid >> 4, cg = tid & 15;
#pragma unroll 1
            for (int i = 0; i < 4; ++i) {
                const int t = tg * 4 + i;
                const bool in = t < n;
                const uint32_t ro = (uint32_t)(t * DK * 2 + cg * 16);
                float fq[8], fk[8], fb[8];
                bf16x8_to_f32(sel(in, *reinterpret_cast<const uint4 *>(sm + OFF_RQ + ro)), fq);
                bf16x8_to_f32(sel(in, *reinterpret_cast<const uint4 *>(sm + OFF_RK + ro)), fk);
                if (vec_b) {
                    bf16x8_to_f32(sel(in, *reinterpret_cast<const uint4 *>(sm + OFF_RB + ro)), fb);
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) fb[j] = sBeta[t];
                }
                const float4 g0 = *reinterpret_cast<const float4 *>(sG + t * DK + cg * 8);
                const float4 g1 = *reinterpret_cast<const float4 *>(sG + t * DK + cg * 8 + 4);
                const float e[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                float kh[8], qg[8], kb[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    kh[j] = fb[j] * fk[j] * e[j];
                    qg[j] = fq[j] * e[j];
                    kb[j] = fk[j] * rcp_approx(e[j]);
                }
                st_chunk(sbase + OFF_QK + tile_chunk(128, t, cg), kh);
                st_chunk(sbase + OFF_QK + tile_chunk(128, 64 + t, cg), qg);
                st_chunk(sbase + OFF_KB + tile_chunk(64, t, cg), kb);
            }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int d = warp * 16 + 2 * i + (lane >> 4);
            const float eg = sEGC[d];
            float f[8];
            bf16x8_to_f32(dsr[i], f);
#pragma unroll
            for (int j = 0; j < 8; ++j) f[j] *= eg;
            st_chunk(sbase + OFF_DSB + tile_chunk(128, d, lane & 15), f);
        }
        fence_async_smem();
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        // ---- 4. [A; P] = [Kh; Qg] Kb^T,  X^T = S^T Kh^T,  dE^T = dS~^T Kb^T ----
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id_kk = idesc_bf16(128, 64, false, false, false);
            const uint32_t id_mk = idesc_bf16(128, 64, true, false, false);
#pragma unroll
            for (int s = 0; s < DK / 16; ++s) {
                mma_bf16(tmem + TM_AP, desc_kmajor(sbase + OFF_QK, 128, 0, s), desc_kmajor(sbase + OFF_KB, 64, 0, s),
                         id_kk, s > 0);
                mma_bf16(tmem + TM_X, desc_mnmajor(sbase + OFF_SB, 128, 0, s), desc_kmajor(sbase + OFF_QK, 128, 0, s),
                         id_mk, s > 0);
                mma_bf16(tmem + TM_DE, desc_mnmajor(sbase + OFF_DSB, 128, 0, s), desc_kmajor(sbase + OFF_KB, 64, 0, s),
                         id_mk, s > 0);
            }
            mma_commit(bar_mma);
        }
        ++commits;
        if (!wait_mma()) break;
        tc_fence_after();
        // ---- 5. A (fp32, strictly lower) -> inverse scratch; P (lower incl.) -> bf16 tile;
        //      R^T = W^T - X^T -> bf16 in TMEM ----
        {
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
            float pv[16], pw[16];
            tmem_ld16(tmem + lane_base + TM_VB + j0 / 2, pv);
            tmem_ld16(tmem + lane_base + TM_WB + j0 / 2, pw);
            tmem_ld32(tmem + lane_base + TM_X + j0, x);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {   // W = w.v (zero past the end) from the packed pairs
                const uint32_t u = __float_as_uint(pv[j / 2]), w = __float_as_uint(pw[j / 2]);
                const float vt = __uint_as_float((j & 1) ? (u & 0xFFFF0000u) : (u << 16));
                const float wt = __uint_as_float((j & 1) ? (w & 0xFFFF0000u) : (w << 16));
                x[j] = (j0 + j < n ? vt * wt : 0.f) - x[j];
            }
            st_tmem_bf16(tmem + lane_base + TM_RB + j0 / 2, x);
        }
        fence_async_smem();
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        // ---- 6. dE^T += dO^T P; T = (I + A)^-1 by warps 0-3; then E^T = R^T T^T ----
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, false, true, false);
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16_ts(tmem + TM_DE, tmem + TM_DOB + s * 8, desc_mnmajor(sbase + OFF_P, 64, 0, s), id, 1u);
        }
        if (warp < 4) {
            tri::inverse64(sA32, sA32, sX, warp, lane, Bar128{}, TileOut{sbase + OFF_T});   // in place
            fence_async_smem();
        }
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, false, false, false);
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16_ts(tmem + TM_E, tmem + TM_RB + s * 8, desc_kmajor(sbase + OFF_T, 64, 0, s), id, s > 0);
            mma_commit(bar_mma);
        }
        ++commits;
        if (!wait_mma()) break;
        tc_fence_after();
        // ---- 7. E^T -> bf16 tile [v][t]; dE^T -> bf16 in TMEM; dO^T -> the right half of
        //      the [-dR^T | dO^T] tile ----
        {
            float x[32];
            tmem_ld32(tmem + lane_base + TM_E + j0, x);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                float f[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) f[j] = x[h * 8 + j];
                st_chunk(sbase + OFF_ET + tile_chunk(128, r, j0 / 8 + h), f);
            }
            tmem_ld32(tmem + lane_base + TM_DE + j0, x);
            tmem_wait_ld();
            st_tmem_bf16(tmem + lane_base + TM_DEB + j0 / 2, x);
            float p[16];   // packed bf16 pairs of dO^T, 8 tokens per 16-byte chunk
            tmem_ld16(tmem + lane_base + TM_DOB + j0 / 2, p);
            tmem_wait_ld();
            const uint32_t *u = reinterpret_cast<const uint32_t *>(p);
#pragma unroll
            for (int h = 0; h < 4; ++h)
                st_shared_v4(sbase + OFF_DOR + tile_chunk(128, r, 8 + j0 / 8 + h), u[4 * h], u[4 * h + 1],
                             u[4 * h + 2], u[4 * h + 3]);
        }
        fence_async_smem();
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        // ---- 8. dR^T = dE^T T,  dKe^T = dS~ E^T ----
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id_t = idesc_bf16(128, 64, false, true, false);
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16_ts(tmem + TM_X, tmem + TM_DEB + s * 8, desc_mnmajor(sbase + OFF_T, 64, 0, s), id_t, s > 0);
#pragma unroll
            for (int s = 0; s < DV / 16; ++s)
                mma_bf16(tmem + TM_DKE, desc_kmajor(sbase + OFF_DSB, 128, 0, s), desc_mnmajor(sbase + OFF_ET, 128, 0, s),
                         id_t, s > 0);
            mma_commit(bar_mma);
        }
        ++commits;
        if (!wait_mma()) break;
        tc_fence_after();
        // ---- 9. dv = dR w, dw = dR v, staged [t][v] over dS~ (free since step 8) for one
        //      bulk store each; -dR^T -> the left half of the [-dR^T | dO^T] tile ----
        {
            __nv_bfloat16 *sdv = reinterpret_cast<__nv_bfloat16 *>(sm + OFF_DSB);
#pragma unroll 1
            for (int g8 = 0; g8 < 4; ++g8) {
                const int tb = j0 + 8 * g8;
                float x[8], pv[4], pw[4];
                tmem_ld8(tmem + lane_base + TM_X + tb, x);
                tmem_ld4(tmem + lane_base + TM_VB + tb / 2, pv);
                tmem_ld4(tmem + lane_base + TM_WB + tb / 2, pw);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int t = tb + j;
                    const uint32_t u = __float_as_uint(pv[j / 2]), w = __float_as_uint(pw[j / 2]);
                    const float vt = __uint_as_float((j & 1) ? (u & 0xFFFF0000u) : (u << 16));
                    const float wt = __uint_as_float((j & 1) ? (w & 0xFFFF0000u) : (w << 16));
                    const float gw = t < n ? x[j] * vt : 0.f;
                    sdv[t * DV + r] = __float2bfloat16_rn(x[j] * wt);
                    if (vec_w) sdv[C * DV + t * DV + r] = __float2bfloat16_rn(gw);
                    if (!vec_w) {   // t is the same across the warp: fold over the value channels
                        const float s = warp_sum(gw);
                        if (lane == 0 && t < n) atomicAdd(&sFw[t], s);
                    }
                }
                float f[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) f[j] = -x[j];
                st_chunk(sbase + OFF_DOR + tile_chunk(128, r, tb / 8), f);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- 10. [dA; dP] = [-dR; dO] E^T,  [dKh | dQg]^T = S [-dR; dO]^T; dv, dw out ----
        if (tid == 0) {
            const uint32_t row16 = (uint32_t)n * DV * 2;
            bulk_s2g(dVo + tok0 * DV, sbase + OFF_DSB, row16);
            if (vec_w) bulk_s2g(dWo + tok0 * DV, sbase + OFF_DSB + C * DV * 2, row16);
            bulk_commit();
            tc_fence_after();
            const uint32_t id_ap = idesc_bf16(128, 64, true, true, false);
            const uint32_t id_qk = idesc_bf16(128, 128, false, true, false);
#pragma unroll
            for (int s = 0; s < DV / 16; ++s) {
                mma_bf16(tmem + TM_AP, desc_mnmajor(sbase + OFF_DOR, 128, 0, s), desc_mnmajor(sbase + OFF_ET, 128, 0, s),
                         id_ap, s > 0);
                mma_bf16(tmem + TM_DQK, desc_kmajor(sbase + OFF_SB, 128, 0, s), desc_mnmajor(sbase + OFF_DOR, 128, 0, s),
                         id_qk, s > 0);
            }
            mma_commit(bar_mma);
        }
        ++commits;
        if (!wait_mma()) break;
        tc_fence_after();
        // raw q, k, b again for step 13 (the first copies were overwritten), into the tiles
        // the last MMAs have released
        if (tid == 0) {
            const uint32_t row16 = (uint32_t)n * DK * 2;
            fence_async_smem();
            mbar_arrive_expect_tx(bar_raw, 2 * row16 + (vec_b ? row16 : 0));
            bulk_g2s(sbase + OFF_RQ, Q + tok0 * DK, row16, bar_raw);
            bulk_g2s(sbase + OFF_RK, K + tok0 * DK, row16, bar_raw);
            if (vec_b) bulk_g2s(sbase + OFF_RB, Bg + tok0 * DK, row16, bar_raw);
        }
        ++raw_copies;
        raw_pending = true;
        // ---- 11. dA and dP, both strictly lower, -> bf16 tile; dP's diagonal -> sDPd ----
        {
            float x[32];
            tmem_ld32(tmem + lane_base + TM_AP + j0, x);
            tmem_wait_ld();
            const int lim = r < 64 ? r : r - 64;   // columns j < lim are kept
            if (r >= 64 && lim >= j0 && lim < j0 + 32) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (j0 + j == lim) sDPd[lim] = x[j];
            }
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                float f[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) f[j] = (j0 + h * 8 + j < lim) ? x[h * 8 + j] : 0.f;
                st_chunk(sbase + OFF_DAP + tile_chunk(128, r, j0 / 8 + h), f);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- 12. [dKh | dQg]^T += Kb^T [dA; dP]^T,  dKb^T = [Kh; Qg]^T [dA; dP] ----
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id_qk = idesc_bf16(128, 128, true, false, false);
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16(tmem + TM_DQK, desc_mnmajor(sbase + OFF_KB, 64, 0, s), desc_kmajor(sbase + OFF_DAP, 128, 0, s),
                         id_qk, 1u);
            const uint32_t id_kb = idesc_bf16(128, 64, true, true, false);
#pragma unroll
            for (int s = 0; s < 128 / 16; ++s)
                mma_bf16(tmem + TM_DKB, desc_mnmajor(sbase + OFF_QK, 128, 0, s), desc_mnmajor(sbase + OFF_DAP, 128, 0, s),
                         id_kb, s > 0);
            mma_commit(bar_mma);
        }
        ++commits;
        if (!wait_mma()) break;
        tc_fence_after();
        if (!wait_bar(bar_raw, (uint32_t)((raw_copies - 1) & 1))) break;
        raw_pending = false;
        // ---- 13. per (token, key channel): thread r = d, tokens j0 .. j0 + 31; dq, dk, db
        //      staged [t][d] over S and [Kh; Qg] (both free now), dg in place of dgamma ----
        {
            const int d = r;
            const __nv_bfloat16 *rq = reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_RQ);
            const __nv_bfloat16 *rk = reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_RK);
            const __nv_bfloat16 *rb = reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_RB);
            __nv_bfloat16 *sdq = reinterpret_cast<__nv_bfloat16 *>(sm + OFF_SB), *sdk = sdq + C * DK;
            __nv_bfloat16 *sdb = reinterpret_cast<__nv_bfloat16 *>(sm + OFF_QK);
            float ske = 0.f, sdg = 0.f;   // sum_t dKe Kb, sum_t dgamma over this thread's tokens
#pragma unroll 1
            for (int g8 = 0; g8 < 4; ++g8) {
                const int tb = j0 + 8 * g8;
                float dkh[8], dqg[8], dkb[8], dke[8];
                tmem_ld8(tmem + lane_base + TM_DQK + tb, dkh);
                tmem_ld8(tmem + lane_base + TM_DQK + 64 + tb, dqg);
                tmem_ld8(tmem + lane_base + TM_DKB + tb, dkb);
                tmem_ld8(tmem + lane_base + TM_DKE + tb, dke);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int t = tb + i;
                    const bool in = t < n;
                    const float e = sG[t * DK + d], ei = rcp_approx(e);
                    const float qv = in ? __bfloat162float(rq[t * DK + d]) : 0.f;
                    const float kv = in ? __bfloat162float(rk[t * DK + d]) : 0.f;
                    const float bv = vec_b ? (in ? __bfloat162float(rb[t * DK + d]) : 0.f) : sBeta[t];
                    const float dkbt = dkb[i] + dke[i], dpd = sDPd[t];
                    const float kbv = kv * ei;
                    const float gb = dkh[i] * kv * e;
                    const float dgam = dqg[i] * qv * e + dkh[i] * bv * kv * e - dkbt * kbv;
                    ske = fmaf(dke[i], kbv, ske);
                    sdg += dgam;
                    sG[t * DK + d] = dgam;   // dgamma replaces e^gamma
                    sdq[t * DK + d] = __float2bfloat16_rn(fmaf(dqg[i], e, dpd * kv));
                    sdk[t * DK + d] = __float2bfloat16_rn(fmaf(dkh[i] * bv, e, fmaf(dkbt, ei, dpd * qv)));
                    if (vec_b) sdb[t * DK + d] = __float2bfloat16_rn(gb);
                    if (!vec_b) {   // fold over the key channels
                        const float s = warp_sum(gb);
                        if (lane == 0 && in) atomicAdd(&sFb[t], s);
                    }
                }
            }
            // dgamma_C and the later half's total reach the earlier half through shared memory
            if (j0) sCar[d] = sdg;
            sCar[128 * (1 + (j0 >> 5)) + d] = ske;
            __syncthreads();
            float acc = sEGC[d] * sDGC[d] + sCar[128 + d] + sCar[256 + d] + (j0 ? 0.f : sCar[d]);
#pragma unroll 4
            for (int i = 31; i >= 0; --i) {
                const int t = j0 + i;
                acc += sG[t * DK + d];
                if (vec_g) {
                    sG[t * DK + d] = acc;
                } else {
                    const float s = warp_sum(acc);
                    if (lane == 0 && t < n) atomicAdd(&sFg[t], s);
                }
            }
        }
        fence_async_smem();
        __syncthreads();
        // ---- 14. the staged gradients out; scalar gates: one gradient per token ----
        if (tid == 0) {
            const uint32_t row16 = (uint32_t)n * DK * 2;
            bulk_s2g(dQo + tok0 * DK, sbase + OFF_SB, row16);
            bulk_s2g(dKo + tok0 * DK, sbase + OFF_SB + C * DK * 2, row16);
            if (vec_b) bulk_s2g(dBo + tok0 * DK, sbase + OFF_QK, row16);
            if (vec_g) bulk_s2g(a.dg + tok0 * DK, sbase + OFF_G, 2 * row16);
            bulk_commit();
        }
        if (tid < n) {
            const size_t tk = tok0 + tid;
            if (!vec_b) dBo[tk] = __float2bfloat16_rn(tied ? sFb[tid] + sFw[tid] : sFb[tid]);
            if (MODE == GDR_MODE_BONLY) dWo[tk] = __float2bfloat16_rn(sFw[tid]);
            if (!vec_g) a.dg[tk] = sFg[tid];
        }
    } while (0);

    tmem_wait_st();   // an early exit can leave this thread's dO^T store in flight
    tc_fence_before();
    if (tid == 0) bulk_wait_read_all();   // the bulk stores have read their shared-memory staging
    __syncthreads();
    if (sFlag[1] && tid == 0) {
        // drain: the raw copies and every committed tensor-core operation
        atomicExch(&g_bwd_tc_error, 1);
        if (raw_pending) mbar_wait(bar_raw, (uint32_t)((raw_copies - 1) & 1), a.wait_limit);
        mma_commit(bar_mma);
        const int k = commits + 1;
        if (k >= 2) mbar_wait(bar_mma, (uint32_t)((k - 2) & 1), a.wait_limit);
        mbar_wait(bar_mma, (uint32_t)((k - 1) & 1), a.wait_limit);
    }
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

}  // namespace

bool bwd_tc_supported(const BwdArgs &a) { return a.dtype == GDR_BF16 && a.dk_ == DK && a.dv_ == DV; }

gdr_status_t launch_bwd_tc(const BwdArgs &a, cudaStream_t s) {
    static_assert(2 * kBwdChunk == C, "a chunk here is two of the backward's 32-token chunks");
    auto kern = a.mode == GDR_MODE_GDN2  ? bwd_tc_kernel<GDR_MODE_GDN2>
              : a.mode == GDR_MODE_KDA   ? bwd_tc_kernel<GDR_MODE_KDA>
              : a.mode == GDR_MODE_GDN   ? bwd_tc_kernel<GDR_MODE_GDN>
              : a.mode == GDR_MODE_BONLY ? bwd_tc_kernel<GDR_MODE_BONLY>
                                         : bwd_tc_kernel<GDR_MODE_WONLY>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) != cudaSuccess)
        return GDR_ERR_CUDA;
    const unsigned grid = (unsigned)((size_t)a.B * a.H * ((a.T + C - 1) / C));
    BwdArgs b = a;
    int dev = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        nsm = 0;
    }
    b.prefetch_ahead = a.ckpt_bf16 ? nsm : 0;   // the slots it prefetches are the bf16 ones
    kern<<<grid, kThreads, SMEM_BYTES, s>>>(b);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

cudaError_t bwd_tc_read_and_clear_error(int *err) {
    cudaError_t e = cudaMemcpyFromSymbol(err, g_bwd_tc_error, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_bwd_tc_error, &zero, sizeof(int));
}

}  // namespace gdr

namespace gdr {
GDR_BOUNDS_READER(bwd_tc_bounds_site)
}  // namespace gdr
