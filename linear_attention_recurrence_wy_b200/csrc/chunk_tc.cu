// chunk_tc.cu -- tcgen05 tensor-core chunkwise WY forward: bf16 operands, fp32 state.
//
// Shape: dk = dv = 128, chunk C = 64, bf16 q/k/v/b/w/o, fp32 g_log and state, any mode.
// One CTA (512 threads) owns one (sequence, head) -- or one segment of it under the
// sequence split -- and keeps the fp32 state in tensor memory (TMEM) for the whole run,
// transposed (lane = value channel v, column = key channel d).  Per chunk (Gated
// DeltaNet-2 Review §3-2.5 "Chunkwise WY training"; Gated DeltaNet-2 Q&A page, Q4):
//
//   gamma   = chunk-local cumulative sum of g_log (fp32, per key channel)
//   Kh      = b.k.e^gamma,  Qg = q.e^gamma,  Kb = k.e^-gamma                (bf16, smem)
//   [A; P]  = [Kh; Qg] Kb^T           one M=128 MMA; A strictly lower, P lower incl.
//   T       = (I + A)^-1              blocked substitution (tri_inverse.cuh)
//   [X | O] = S^T [Kh; Qg]^T          one N=128 MMA: X = S^T Kh^T, O = S^T Qg^T
//   R^T     = (w.v)^T - X             w.v formed in fp32 on read-out
//   E^T     = R^T T^T                 the delta errors E = T (w.v - Kh S) = U - W S
//   O^T    += E^T P^T                 (read-out of the post-update state)
//   S^T     = (S^T + E^T Kb) diag(e^gamma_C)
//
// Writing Kb = k.e^-gamma and scaling after the state MMA equals S diag(e^gamma_C) +
// (k.e^(gamma_C - gamma))^T E; both factors of every product stay within e^+-60 when
// |gamma| <= 60 on the whole chunk.  A chunk with a stronger cumulative decay takes the
// exact path instead: A and P from per-pair decays exp(gamma_i - gamma_j) on CUDA cores,
// K_end = k.e^(gamma_C - gamma) in place of Kb, and the state scaled before its MMA.
//
// Warp-specialised pipeline.  Warps 0-7 (the WY group) stage a chunk's q, k, b and g_log
// (one bulk copy per tensor), scan the log-decay, build the operands, form [A; P] on the
// tensor cores and invert (I + A).  Warps 8-15 (the state group) meanwhile run the
// state-dependent chain of an earlier chunk: X and O, R (reading v and w straight from
// global memory), E, the output and the state update, all on tcgen05 with their A
// operands (bf16 S^T, R^T, E^T) read from TMEM.  The groups hand over through mbarriers:
//   H1     operands of chunk c built           WY -> state
//   H2[2]  T and P of chunk c ready            WY -> state   (by chunk parity)
//   H3     Kh, Qg of chunk c consumed          state -> WY   (they may be rebuilt)
//   H4[2]  chunk c finished                    state -> WY   (its P, T, Kb buffers are free)
// Kb, P and T are double-buffered by chunk parity, so the WY group can run up to two
// chunks ahead of the state group.  The next chunk's raw inputs are copied as soon as
// the operands are built (fast path) or A and P are formed (exact path).
//
// Token mixer (kMixer instantiation; Gated DeltaNet-2 Review §4-3, engineering notes): the
// same pipeline on the block's raw projections.  The scan turns the decay projection into
// e^gamma as a running product of sigmoid(-x) (= e^-softplus(x)); the operand build
// L2-normalises q and k per token (16 lanes per token, shuffles) and applies b's sigmoid;
// the state group applies w's sigmoid and, after the state update, the output gate
// y = o rsqrt(mean_v o^2 + eps) weight z sigmoid(z): the sum of squares over the value
// channels is one MMA of the squared outputs against a ones operand in TMEM, and y leaves
// through the chunk's free K-bar tile by one TMA tensor store.  Either layout, [B,H,T,D]
// or the projections' [B,T,H,D] (then the raw q, k, b, g chunks arrive by TMA tensor copies).
//
// Every wait on an mbarrier is bounded.  On expiry a thread raises a CTA-wide abort flag;
// both groups leave their loops at their next wait, the kernel records the failure in
// g_tc_error, waits (bounded) for its own bulk copies and tensor-core work, frees its
// TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <string.h>

#include <mutex>

#include "bounds.cuh"
#include "chunk_tc.cuh"
#include "tc_util.cuh"
#include "tri_inverse.cuh"

namespace gdr {

__device__ int g_tc_error = 0;

namespace {

using namespace tc;

constexpr int C = 64, DK = 128, DV = 128;
constexpr int kThreads = 512;
constexpr float kFastLimit = 60.f;
constexpr float kFastProd = 8.7565108e-27f;   // e^-60: the same limit on e^gamma
constexpr int kAS = tri::LD;   // fp32 row stride of the A / T scratch

// shared memory map (byte offsets from a 1024-aligned base)
constexpr int RAW_Q = 0;                        // raw q bf16 [64][128]     16 KB
constexpr int RAW_K = RAW_Q + 16384;            // raw k                    16 KB
constexpr int RAW_B = RAW_K + 16384;            // raw b (GDN-2)            16 KB
constexpr int RAW_G = RAW_B + 16384;            // raw g_log fp32 [64][128] 32 KB, then gamma
constexpr int RAW_END = RAW_G + 32768;
constexpr int OFF_A32 = RAW_END;                // inverse scratch: A, then T, fp32 [64][68]
constexpr int OFF_X = OFF_A32 + 64 * kAS * 4;   //                  4 x [16][20] fp32
constexpr int OFF_QK = (OFF_X + 4 * 16 * tri::XLD * 4 + 1023) / 1024 * 1024;
                                                // [Kh;Qg] bf16 [128][128]  32 KB
constexpr int OFF_KB = OFF_QK + 32768;          // Kb bf16 [2][64 t][128 d] 32 KB
constexpr int OFF_P = OFF_KB + 32768;           // P  bf16 [2][64 t][64 j]  16 KB
constexpr int OFF_T = OFF_P + 16384;            // T  bf16 [2][64 t][64 j]  16 KB
constexpr int OFF_GS = OFF_T + 16384;           // scalar g_log of the chunk (GDN) fp32 [64]
constexpr int OFF_BETA = OFF_GS + 256;          // scalar beta of the chunk (KDA, GDN) fp32 [64]
constexpr int OFF_GC = OFF_BETA + 256;          // gamma_C fp32 [128]
constexpr int OFF_EGC = OFF_GC + 512;           // exp(gamma_C) fp32 [4][128], slot c % 4
constexpr int OFF_FLAG = OFF_EGC + 2048;        // exact flags [4] (slot c % 4), abort flag
constexpr int OFF_RQ = OFF_FLAG + 64;           // mixer: 1/||q_t||, 1/||k_t|| of the chunk [2][64]
constexpr int OFF_BAR = OFF_RQ + 512;           // mbarriers + TMEM slot
constexpr int NBAR = 9;
constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 8 + 1024;   // + alignment slack

// TMEM columns
constexpr uint32_t TM_S = 0;     // S^T fp32                                   128 cols
constexpr uint32_t TM_XO = 128;  // [X, then E^T | O^T] fp32                  64 + 64
constexpr uint32_t TM_AP = 256;  // [A; P] fp32                                 64
constexpr uint32_t TM_SB = 320;  // S^T bf16 (packed)                           64
constexpr uint32_t TM_XB = 384;  // R^T, then E^T bf16 (packed)                 32
constexpr uint32_t TM_DO = 416;   // state-gradient pass: dO^T bf16 (packed)      32
constexpr uint32_t TM_ONES = 448; // mixer: bf16 ones, the A operand of the output's
                                  // sum of squares over value channels        64
constexpr uint32_t TM_COLS = 512;

// named barriers (0 is __syncthreads; 1 is warps 0-3, the inverse's; 4 is warps 4-7, the scan's)
constexpr int BAR_WY = 2;    // warps 0-7
constexpr int BAR_ST = 3;    // warps 8-15

// The named barriers below are the .aligned forms: every thread of a warp must reach them
// together.  A thread that ran code alone just before (an elected issuer, a bounded wait
// inside the barrier's own argument) may still be diverged from its warp, so each helper
// first reconverges the warp (__syncwarp); the warp then also leaves the barrier converged,
// which the warp-collective instructions after it (.aligned tcgen05 loads and stores,
// shuffles, warp MMAs) need.

// barrier over the 256 threads of one warp group
__device__ __forceinline__ void group_sync(int id) {
    __syncwarp();
    asm volatile("bar.sync %0, 256;" ::"r"(id) : "memory");
}
// barrier over one warp group that also returns the AND of v over it
__device__ __forceinline__ bool group_and(int id, bool v) {
    __syncwarp();
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, 256, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id)
        : "memory");
    return r != 0;
}
// the same over 128 threads (warps 4-7 of the WY group)
__device__ __forceinline__ bool bar128_and(int id, bool v) {
    __syncwarp();
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, 128, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ bool bar128_or(int id, bool v) {
    __syncwarp();
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, %2, 128, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void mbar_arrive(uint32_t saddr) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr) : "memory");
}

// ---- token-mixer activations (Gated DeltaNet-2 Review §4-3, engineering notes) ----------
// log(1 + e^x) = max(x, 0) + log(1 + e^-|x|): the decay branch, g = -softplus(x)
__device__ __forceinline__ float softplus_f(float x) {
    return fmaxf(x, 0.f) + __logf(1.f + __expf(-fabsf(x)));
}
__device__ __forceinline__ float sigmoid_f(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }
// The gates (b, w, beta and the SiLU of z) through one tanh: sigmoid(x) = (1 + tanh(x/2)) / 2,
// with PTX tanh.approx (about 2^-11 relative error, below the bf16 rounding of the operands
// these gates scale).  The decay keeps the exp-based form: its factors multiply up over a chunk.
__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float sigmoid_gate(float x) { return fmaf(0.5f, tanh_approx(0.5f * x), 0.5f); }

// Final values of T (from the inverse) straight into the bf16 operand tile.
// After an abort: wait (bounded) until every commit issued on bar has arrived.  The
// commits complete in order; n of them were issued, so phases n-2 and n-1 are waited
// for in turn (a parity wait alone cannot tell phase n-1 from phase n-3).
__device__ __forceinline__ void drain_commits(uint32_t bar, int n, uint32_t limit) {
    if (n >= 2) mbar_wait(bar, (uint32_t)((n - 2) & 1), limit);
    if (n >= 1) mbar_wait(bar, (uint32_t)((n - 1) & 1), limit);
}

// Exact path, strong-decay chunks only: A (fp32, strictly lower) and P (bf16 tile, lower
// incl.) from per-pair decays exp(gamma_i - gamma_j), computed from the staged raw q, k, b
// and gamma on CUDA cores by the 256 threads of the WY group.  beta: the scalar b of the
// chunk's tokens in shared memory (tied modes, w-only), or NULL when b is a per-channel
// vector staged with q and k.  Mixer: rq, rk hold the tokens' 1/||q||, 1/||k|| (else
// NULL) and b_act > 0 makes a per-channel b = b_act * sigmoid(raw b).
// Kept out of line: it is rarely run and would otherwise crowd the instruction cache.
__device__ __noinline__ void exact_ap(unsigned char *sm, float *sA32, uint32_t p_off, const float *sGam,
                                      const float *beta, const float *rq, const float *rk, float b_act,
                                      int n, int wtid) {
#pragma unroll 1
    for (int u = 0; u < 16; ++u) {
        const int p = wtid + u * 256, i = p >> 6, j = p & 63;
        float sa = 0.f, sp = 0.f;
        if (j <= i && i < n) {
            const __nv_bfloat16 *qi = (const __nv_bfloat16 *)(sm + RAW_Q) + i * DK;
            const __nv_bfloat16 *ki = (const __nv_bfloat16 *)(sm + RAW_K) + i * DK;
            const __nv_bfloat16 *kj = (const __nv_bfloat16 *)(sm + RAW_K) + j * DK;
            const __nv_bfloat16 *bi = (const __nv_bfloat16 *)(sm + RAW_B) + i * DK;
            const float bs = beta ? beta[i] : 0.f;
#pragma unroll 2
            for (int d = 0; d < DK; ++d) {
                const float dec = __expf(sGam[i * DK + d] - sGam[j * DK + d]);
                const float kjd = __bfloat162float(kj[d]) * dec;
                float bid = beta ? bs : __bfloat162float(bi[d]);
                if (!beta && b_act > 0.f) bid = b_act * sigmoid_gate(bid);
                sa = fmaf(bid * __bfloat162float(ki[d]), kjd, sa);
                sp = fmaf(__bfloat162float(qi[d]), kjd, sp);
            }
            if (rq) {
                sa *= rk[i] * rk[j];
                sp *= rq[i] * rk[j];
            }
        }
        sA32[i * kAS + j] = (j < i) ? sa : 0.f;
        *reinterpret_cast<__nv_bfloat16 *>(sm + p_off + tile_off(64, i, j)) = __float2bfloat16_rn(sp);
    }
}

// Exact path: gamma of key channel d over the chunk's n tokens (zero contribution past the
// end) from the g_log in global memory, stride apart, into column d of the gamma tile
// (strong-decay chunks only; out of line like exact_ap).  act: the mixer's raw decay
// projection, g = -softplus(raw).
__device__ __noinline__ void exact_gamma(float *sGam, const float *g, size_t stride, int n, int d, bool act) {
    float acc = 0.f;
#pragma unroll 1
    for (int t = 0; t < C; ++t) {
        if (t < n) {
            const float x = g[(size_t)t * stride];
            acc += act ? -softplus_f(x) : x;
        }
        sGam[t * DK + d] = acc;
    }
}

// Exact path: S^T columns [d_begin, d_begin + 64) scaled by exp(gamma_C) in TMEM, before the
// state update (strong-decay chunks only; out of line like exact_ap).
__device__ __noinline__ void prescale_state(uint32_t taddr, const float *egc, int d_begin) {
#pragma unroll 1
    for (int d0 = d_begin; d0 < d_begin + 64; d0 += 32) {
        float x[32];
        tmem_ld32(taddr + d0, x);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] *= egc[d0 + j];
        tmem_st32(taddr + d0, x);
    }
    tmem_wait_st();
}

// Tensor maps of the mixer (one box = one chunk of one head, rows dense in shared memory).
// Token-major inputs [B, T, H, D]: dims {D, H, T, B}, box {D, 1, 64, 1}; the raw chunk
// inputs then arrive by one tiled copy per tensor (rows past the end of a sequence are
// zero-filled), and v, w, z are prefetched to L2 by box.  y, the mixer's output, is
// written by one tiled store per chunk in either layout (head-major: dims {D, T, H, B},
// box {D, 64, 1, 1}); rows past the end are clipped.
struct TokenMaps {
    CUtensorMap q, k, b, g, v, w, z, y;
};

// kMixer: the token-mixer instantiation (activations on load, output epilogue, either
// layout; ChunkArgs::mixer).  kStates: the backward's checkpoint pass, which also writes
// the state at the start of every chunk, rounded to bf16, to ChunkArgs::chunk_states (slot
// 2c of the backward's 32-token chunk slots).  kReverse: the backward's state-gradient pass
// (ChunkArgs::reverse), chunks in reverse order; see the state group.  The plain
// instantiation is the recurrence alone.
template <bool kMixer, bool kStates, bool kReverse>
__global__ void __launch_bounds__(kThreads, 1) chunk_tc_kernel(ChunkArgs a, const __grid_constant__ TokenMaps tm) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3;   // TMEM lanes this warp may access: 32 * quarter + [0, 32)
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;

    // ---- this CTA's job: one sequence-head, one segment of it, one role ----
    const bool maps = a.seg_maps != 0;                        // a whole segment's maps
    const int roles = chunk_roles(a);
    const int bh = blockIdx.x / roles, role = blockIdx.x % roles;
    const bool transfer = maps ? role == 1 : (a.pass && role > a.nseg - 2);   // transition-matrix run
    const int seg = maps ? 0 : transfer ? role - (a.nseg - 2) : role;
    const int t_begin = seg * a.seg_len;
    const int T = min(a.seg_len, a.T - t_begin);              // tokens of this segment
    const int mode = a.mode;
    // token t of this segment is row tok0 + t * ts of every [.., D] input
    const int ts = kMixer ? a.tstride : 1;
    size_t tok0 = (size_t)bh * a.T + t_begin;
    if (kMixer && ts != 1) tok0 = ((size_t)(bh / a.H) * a.T + t_begin) * a.H + bh % a.H;
    const int hc = bh % a.H, bc = bh / a.H;   // tensor-map coordinates of this head
    const int nchunks = (T + C - 1) / C;
    // iteration c (barrier phases, buffers, ring slots) works on data chunk dch(c)
    auto dch = [&](int c) { return kReverse ? nchunks - 1 - c : c; };
    const size_t sidx = ((size_t)bh * a.nseg + seg) * DK * DV;
    const float *S0p = nullptr;        // initial state (NULL: zero, unless the identity)
    float *STp = nullptr;              // end state destination (NULL: not written)
    if (maps) {
        S0p = (!transfer && a.S0) ? a.S0 + (size_t)bh * DK * DV : nullptr;
        STp = (transfer ? a.ws_m : a.ws_send) + (size_t)bh * DK * DV;
    } else if (!a.pass) {
        S0p = a.nseg == 1 ? (a.S0 ? a.S0 + (size_t)bh * DK * DV : nullptr) : a.ws_sstart + sidx;
        STp = seg == a.nseg - 1 ? (a.ST ? a.ST + (size_t)bh * DK * DV : nullptr) : nullptr;
    } else {
        S0p = (!transfer && seg == 0 && a.S0) ? a.S0 + (size_t)bh * DK * DV : nullptr;
        STp = transfer ? a.ws_m + sidx : a.ws_send + sidx;
    }
    const bool write_o = !a.pass && !kStates && !kReverse;
    // debug build: this job's rows and state slots lie inside what the arguments imply (a
    // uniform condition: a failing CTA returns before its first barrier)
    const size_t rows_total = (size_t)a.B * a.H * a.T;
    (void)rows_total;   // read by the debug build's checks only
    if (!GDR_IN_BOUNDS(bh < a.B * a.H && t_begin >= 0 && T >= 1 && tok0 + (size_t)(T - 1) * ts < rows_total &&
                           (maps || a.nseg == 1 || sidx + (size_t)DK * DV <= (size_t)a.B * a.H * a.nseg * DK * DV),
                       101))
        return;

    float *sA32 = reinterpret_cast<float *>(sm + OFF_A32);
    float *sX = reinterpret_cast<float *>(sm + OFF_X);
    float *sGam = reinterpret_cast<float *>(sm + RAW_G);
    float *sGs = reinterpret_cast<float *>(sm + OFF_GS);
    float *sBeta = reinterpret_cast<float *>(sm + OFF_BETA);
    float *sGC = reinterpret_cast<float *>(sm + OFF_GC);
    float *sEGC = reinterpret_cast<float *>(sm + OFF_EGC);
    float *sRq = reinterpret_cast<float *>(sm + OFF_RQ), *sRk = sRq + 64;
    volatile int *sExact = reinterpret_cast<volatile int *>(sm + OFF_FLAG);   // [4]
    volatile int *sAbort = reinterpret_cast<volatile int *>(sm + OFF_FLAG + 16);
    const uint32_t bar_wy = sbase + OFF_BAR;     // the WY group's MMA commits
    const uint32_t bar_st = bar_wy + 8;          // the state group's MMA commits
    const uint32_t bar_raw = bar_wy + 16;        // raw input copies
    const uint32_t bar_h1 = bar_wy + 24, bar_h3 = bar_wy + 32;
    const uint32_t bar_h2 = bar_wy + 40;         // [2], by chunk parity
    const uint32_t bar_h4 = bar_wy + 56;         // [2], by chunk parity
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + NBAR * 8);

    const __nv_bfloat16 *Q = (const __nv_bfloat16 *)a.q, *K = (const __nv_bfloat16 *)a.k;
    const __nv_bfloat16 *V = (const __nv_bfloat16 *)a.v, *Bg = (const __nv_bfloat16 *)a.b;
    const __nv_bfloat16 *Wg = (const __nv_bfloat16 *)a.w;
    __nv_bfloat16 *O = (__nv_bfloat16 *)a.o;
    const __nv_bfloat16 *Z = (const __nv_bfloat16 *)a.z;
    // gate shapes: per-channel erase b (GDN-2, b-only), per-channel write w (GDN-2, w-only),
    // per-channel decay (all but GDN); a scalar write gate is w itself (b-only) or beta
    const bool vec_b = mode_b_vec(mode), vec_w = mode_w_vec(mode), vec_g = mode_g_vec(mode);
    const __nv_bfloat16 *Wsc = mode == GDR_MODE_BONLY ? Wg : Bg;

    if (tid == 0) {
        for (int i = 0; i < NBAR; ++i) mbar_init(bar_wy + 8 * i, 1);
        sAbort[0] = 0;
        fence_mbar_init();
    }
    __syncwarp();
    if (warp == 0) {
        tmem_alloc(smem_u32(tslot), TM_COLS);
        tmem_relinquish();
    }
    // the T tiles' blocks above the diagonal are never written: zero both tiles once
    reinterpret_cast<uint4 *>(sm + OFF_T)[tid] = make_uint4(0, 0, 0, 0);
    reinterpret_cast<uint4 *>(sm + OFF_T)[tid + kThreads] = make_uint4(0, 0, 0, 0);
    static_assert(kThreads * 32 == 16384, "two 16-byte stores per thread clear the T tiles");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    // Bounded wait on an mbarrier phase; gives up early once another thread has aborted.
    // One thread per group polls; the rest of the group parks on the group's named
    // barrier (bar.red), which also carries the outcome and orders their later reads
    // after the phase completed.  Polling by every thread would steal shared-memory and
    // issue bandwidth from the other group.
    const uint32_t wait_limit = a.wait_limit;
    auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
        for (uint32_t i = 0; i < wait_limit; ++i) {
            if (mbar_try_wait(bar, parity)) return true;
            if ((i & 255) == 255 && sAbort[0]) return false;
        }
        sAbort[0] = 1;
        return false;
    };

    // L2 prefetch of chunk c's inputs (issued by the state group's first thread; contiguous
    // chunks only)
    auto prefetch_inputs = [&](int c) {
        if (kMixer && ts != 1) {
            const int tt = t_begin + dch(c) * C;
            tma_prefetch_4d(&tm.q, 0, hc, tt, bc);
            tma_prefetch_4d(&tm.k, 0, hc, tt, bc);
            tma_prefetch_4d(&tm.v, 0, hc, tt, bc);
            tma_prefetch_4d(&tm.z, 0, hc, tt, bc);
            if (vec_b) tma_prefetch_4d(&tm.b, 0, hc, tt, bc);
            if (vec_w) tma_prefetch_4d(&tm.w, 0, hc, tt, bc);
            if (vec_g) tma_prefetch_4d(&tm.g, 0, hc, tt, bc);
            return;
        }
        const int t0 = dch(c) * C, n = min(C, T - t0);
        const size_t e = (tok0 + t0) * DK;
        prefetch_l2(Q + e, n * DK * 2);
        prefetch_l2(K + e, n * DK * 2);
        if (kReverse) {
            prefetch_l2(reinterpret_cast<const __nv_bfloat16 *>(a.dO) + e, n * DV * 2);
        } else {
            prefetch_l2(V + e, n * DV * 2);
            if (vec_w) prefetch_l2(Wg + e, n * DV * 2);
        }
        if (vec_b) prefetch_l2(Bg + e, n * DK * 2);
        if (vec_g) prefetch_l2(a.g + e, n * DK * 4);
        if (kMixer) prefetch_l2(Z + e, n * DV * 2);
    };

    int raw_issued = 0, raw_done = 0;   // raw copies (WY group)
    int mma_wy = 0, mma_st = 0;         // commits issued by each group's MMA thread

    if (warp < 8) {
        // ============================================================== WY group (0-7)
        const int wtid = tid;   // 0 .. 255
        // raw q, k, b, g_log of chunk c -> staging, one bulk copy per tensor, issued by
        // lane 0 of warps 4-7 (issuing a bulk copy takes the issuing thread a while; warp 0
        // issues the MMAs)
        auto issue_raw = [&](int c) {
            if (kMixer && ts != 1) {
                // token-major: one tiled tensor copy per tensor; a box is always whole
                // (64 rows, zero-filled past the end), so its bytes are counted whole
                if (lane != 0 || warp < 4) return;
                const int tt = t_begin + dch(c) * C;
                constexpr uint32_t box16 = C * DK * 2;
                fence_async_smem();
                if (warp == 4) {
                    uint32_t bytes = 2 * box16;
                    if (vec_b) bytes += box16;
                    if (vec_g) bytes += 2 * box16;
                    mbar_arrive_expect_tx(bar_raw, bytes);
                    tma_load_4d(sbase + RAW_Q, &tm.q, 0, hc, tt, bc, bar_raw);
                } else if (warp == 5) {
                    tma_load_4d(sbase + RAW_K, &tm.k, 0, hc, tt, bc, bar_raw);
                } else if (warp == 6) {
                    if (vec_b) tma_load_4d(sbase + RAW_B, &tm.b, 0, hc, tt, bc, bar_raw);
                } else if (vec_g) {
                    tma_load_4d(sbase + RAW_G, &tm.g, 0, hc, tt, bc, bar_raw);
                }
                return;
            }
            if (lane != 0 || warp < 4) return;
            const int t0 = dch(c) * C, n = min(C, T - t0);
            const size_t e = (tok0 + t0) * DK;
            const uint32_t row16 = (uint32_t)n * DK * 2;
            // debug build: the chunk's rows lie inside this head (the copies then stay in the tensors)
            if (!GDR_IN_BOUNDS(n >= 1 && t0 >= 0 && t_begin + t0 + n <= a.T && tok0 + t0 + n <= rows_total, 102))
                return;
            fence_async_smem();
            if (warp == 4) {
                uint32_t bytes = 2 * row16;
                if (vec_b) bytes += row16;
                if (vec_g) bytes += 2 * row16;
                mbar_arrive_expect_tx(bar_raw, bytes);
                bulk_g2s(sbase + RAW_Q, Q + e, row16, bar_raw);
            } else if (warp == 5) {
                bulk_g2s(sbase + RAW_K, K + e, row16, bar_raw);
            } else if (warp == 6) {
                if (vec_b) bulk_g2s(sbase + RAW_B, Bg + e, row16, bar_raw);
            } else if (vec_g) {
                bulk_g2s(sbase + RAW_G, a.g + e, 2 * row16, bar_raw);
            }
        };
        // Cumulative log-decay of chunk c by warps 4-7 (they run it while warps 0-3 invert
        // the chunk before).  Waits for the chunk's raw inputs; thread d scans key channel d
        // (tokens past the end contribute zero) and leaves e^gamma in place of the raw g_log.
        // A chunk with |gamma| > 60 somewhere takes the exact path, which needs gamma itself:
        // then the scan is redone from the g_log in global memory (rare).  Also writes
        // gamma_C, exp(gamma_C) and the exact-path flag.  False if the wait failed.
        auto scan = [&](int c) -> bool {
            const int d = wtid - 128;   // 0 .. 127
            const int t0 = dch(c) * C, n = min(C, T - t0);
            // scalar gates (they need no staging copy): GDN's g_log by threads 0-63, a
            // scalar erase gate (beta, or w-only's b) by threads 64-127 for the operand build
            if (!vec_g && d < 64) {
                const float x = (d < n) ? a.g[tok0 + (size_t)(t0 + d) * ts] : 0.f;
                sGs[d] = kMixer ? sigmoid_f(-x) : x;   // mixer: the decay factor e^g itself
            }
            if (!vec_b && d >= 64) {
                const float x = (d - 64 < n) ? __bfloat162float(Bg[tok0 + (size_t)(t0 + d - 64) * ts]) : 0.f;
                sBeta[d - 64] = (kMixer && d - 64 < n) ? a.b_range * sigmoid_gate(x) : x;
            }
            if (!bar128_and(4, d != 0 || wait(bar_raw, (uint32_t)(c & 1)))) return false;
            if (kMixer) {
                // g = -softplus(raw) <= 0, so e^g = sigmoid(-raw) and e^gamma is the running
                // product of those factors (no logarithm per token); |gamma| peaks at the
                // chunk's last token, where the fast-path limit is checked
                float prod = 1.f;
#pragma unroll 1
                for (int b = 0; b < C; b += 16) {
                    float x[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) x[i] = vec_g ? sGam[(b + i) * DK + d] : sGs[b + i];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float e = vec_g ? sigmoid_f(-x[i]) : x[i];
                        prod *= (b + i < n) ? e : 1.f;
                        x[i] = prod;
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) sGam[(b + i) * DK + d] = x[i];
                }
                const bool any = bar128_or(4, !(prod >= kFastProd));
                float gc = 0.f;
                if (any) {
                    exact_gamma(sGam, vec_g ? a.g + (tok0 + (size_t)t0 * ts) * DK + d : a.g + tok0 + (size_t)t0 * ts,
                                vec_g ? (size_t)DK * ts : (size_t)ts, n, d, true);
                    gc = sGam[(C - 1) * DK + d];
                }
                sGC[d] = gc;
                sEGC[(c & 3) * 128 + d] = any ? __expf(gc) : prod;
                if (d == 0) sExact[c & 3] = any ? 1 : 0;
                return true;
            }
            float acc = 0.f, mx = 0.f;
#pragma unroll 1
            for (int b = 0; b < C; b += 16) {
                float x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] = vec_g ? sGam[(b + i) * DK + d] : sGs[b + i];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    acc += (b + i < n) ? x[i] : 0.f;
                    mx = fmaxf(mx, fabsf(acc));
                    x[i] = __expf(acc);
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) sGam[(b + i) * DK + d] = x[i];
            }
            const bool any = bar128_or(4, mx > kFastLimit);
            if (any) exact_gamma(sGam, vec_g ? a.g + (tok0 + t0) * DK + d : a.g + tok0 + t0, vec_g ? DK : 1, n, d, false);
            sGC[d] = acc;
            sEGC[(c & 3) * 128 + d] = __expf(acc);
            if (d == 0) sExact[c & 3] = any ? 1 : 0;
            return true;
        };
        issue_raw(0);
        raw_issued = 1;
        bool ok = true, scan_ok = true;
        // iteration c = -1 only scans chunk 0 (one call site keeps one copy of the scan)
        for (int c = -1; c < nchunks; ++c) {
          if (c >= 0) {
            const int t0 = dch(c) * C, n = min(C, T - t0);
            const int pb = c & 1;   // P, T and Kb buffer of this chunk
            // ---- W1: the scan of chunk c (warps 4-7) has finished, and the state group has
            //      consumed Kh and Qg of chunk c-1 (H3), so they may be rebuilt ----
            ok = group_and(BAR_WY, scan_ok && (c == 0 || wtid != 0 || wait(bar_h3, (uint32_t)((c - 1) & 1))));
            if (!ok) break;
            raw_done = c + 1;
            const bool exact = sExact[c & 3] != 0;
            const uint32_t kb_tile = sbase + OFF_KB + pb * 16384;
            {
                // thread (tg, cg) owns tokens 4 tg .. 4 tg + 3, channels 8 cg .. 8 cg + 7
                const int tg = wtid >> 4, cg = wtid & 15;
#pragma unroll 1
                for (int i = 0; i < 4; ++i) {
                    const int t = tg * 4 + i;
                    const bool in = t < n;
                    const uint32_t ro = (uint32_t)(t * DK * 2 + cg * 16);
                    const uint4 uq = sel(in, *reinterpret_cast<const uint4 *>(sm + RAW_Q + ro));
                    const uint4 uk = sel(in, *reinterpret_cast<const uint4 *>(sm + RAW_K + ro));
                    const float4 g0 = *reinterpret_cast<const float4 *>(sGam + t * DK + cg * 8);
                    const float4 g1 = *reinterpret_cast<const float4 *>(sGam + t * DK + cg * 8 + 4);
                    const float gm[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                    float fq[8], fk[8], fb[8];
                    bf16x8_to_f32(uq, fq);
                    bf16x8_to_f32(uk, fk);
                    if (kMixer) {
                        // L2 norms of q_t and k_t: the 16 threads of token t are 16
                        // consecutive lanes (tokens past the end are zero and stay zero)
                        float sq = 0.f, sk = 0.f;
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            sq = fmaf(fq[j], fq[j], sq);
                            sk = fmaf(fk[j], fk[j], sk);
                        }
#pragma unroll
                        for (int o = 1; o < 16; o <<= 1) {
                            sq += __shfl_xor_sync(0xffffffffu, sq, o);
                            sk += __shfl_xor_sync(0xffffffffu, sk, o);
                        }
                        const float rq = rsqrtf(sq + 1e-6f), rk = rsqrtf(sk + 1e-6f);
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            fq[j] *= rq;
                            fk[j] *= rk;
                        }
                        if (cg == 0) {
                            sRq[t] = rq;
                            sRk[t] = rk;
                        }
                    }
                    if (vec_b) {
                        bf16x8_to_f32(sel(in, *reinterpret_cast<const uint4 *>(sm + RAW_B + ro)), fb);
                        if (kMixer) {
#pragma unroll
                            for (int j = 0; j < 8; ++j) fb[j] = a.b_range * sigmoid_gate(fb[j]);
                        }
                    } else {
                        const float beta = sBeta[t];   // zero past the end
#pragma unroll
                        for (int j = 0; j < 8; ++j) fb[j] = beta;
                    }
                    // gm holds e^gamma on the fast path, gamma on the exact path
                    float kh[8], qg[8], kb[8];
                    if (!exact) {
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            kh[j] = fb[j] * fk[j] * gm[j];
                            qg[j] = fq[j] * gm[j];
                            kb[j] = fk[j] * rcp_approx(gm[j]);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const float e = __expf(gm[j]);
                            kh[j] = fb[j] * fk[j] * e;
                            qg[j] = fq[j] * e;
                            kb[j] = fk[j] * __expf(sGC[cg * 8 + j] - gm[j]);
                        }
                    }
                    st_chunk(sbase + OFF_QK + tile_chunk(128, t, cg), kh);
                    st_chunk(sbase + OFF_QK + tile_chunk(128, 64 + t, cg), qg);
                    st_chunk(kb_tile + tile_chunk(64, t, cg), kb);
                }
            }
            fence_async_smem();
            group_sync(BAR_WY);
            // ---- W4: [A; P] = [Kh; Qg] Kb^T, issued before the state group may queue its own
            //      MMAs (H1); this chunk's P and T buffers were chunk c-2's, so that chunk must
            //      have finished (H4) ----
            if (!exact) {
                if (wtid == 0) {
                    tc_fence_after();
                    const uint32_t id = idesc_bf16(128, 64, false, false, false);
#pragma unroll
                    for (int s = 0; s < DK / 16; ++s)
                        mma_bf16(tmem + TM_AP, desc_kmajor(sbase + OFF_QK, 128, 0, s),
                                 desc_kmajor(kb_tile, 64, 0, s), id, s > 0);
                    mma_commit(bar_wy);
                }
                ++mma_wy;
            }
            if (wtid == 0) mbar_arrive(bar_h1);   // H1: operands of chunk c built
            // the raw inputs are dead on the fast path: the next chunk's travel from now on
            if (!exact && c + 1 < nchunks) {
                raw_issued = c + 2;
                issue_raw(c + 1);
            }
            ok = group_and(BAR_WY, wtid != 0 ||
                                       ((exact || wait(bar_wy, (uint32_t)((mma_wy - 1) & 1))) &&
                                        (c < 2 || wait(bar_h4 + 8 * pb, (uint32_t)(((c - 2) >> 1) & 1)))));
            if (!ok) break;
            tc_fence_after();
            const uint32_t p_tile = sbase + OFF_P + pb * 8192, t_tile = sbase + OFF_T + pb * 8192;
            // ---- W6: A (fp32, strictly lower) and P (bf16, lower incl.) ----
            if (!exact) {
                const int r = quarter * 32 + lane, j0 = (warp >> 2) * 32;   // row of [A; P]
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
                        st_chunk(p_tile + tile_chunk(64, t, j0 / 8 + h), f);
                    }
                }
            } else {
                exact_ap(sm, sA32, p_tile - sbase, sGam, vec_b ? nullptr : sBeta, kMixer ? sRq : nullptr,
                         kMixer ? sRk : nullptr, (kMixer && vec_b) ? a.b_range : 0.f, n, wtid);
            }
            group_sync(BAR_WY);
            if (exact && c + 1 < nchunks) {   // raw inputs read above: now the next chunk's
                raw_issued = c + 2;
                issue_raw(c + 1);
            }
            // ---- W7: T = (I + A)^-1 by warps 0-3, straight into the bf16 tile, while
            //      warps 4-7 scan the next chunk's log-decay ----
            if (warp < 4) {
                tri::inverse64(sA32, sA32, sX, warp, lane, Bar128{}, TileOut{t_tile});   // in place
                fence_async_smem();
                Bar128{}();
                if (wtid == 0) mbar_arrive(bar_h2 + 8 * pb);   // H2: T and P of chunk c ready
            }
          }
          if (warp >= 4 && c + 1 < nchunks) scan_ok = scan(c + 1);
        }
        if (!ok) sAbort[0] = 1;
    } else {
        // =========================================================== state group (8-15)
        const int stid = tid - 256;   // 0 .. 255
        const int half = (warp - 8) >> 2;
        const int v = quarter * 32 + lane;   // value channel = TMEM lane
        const int j0 = half * 32;            // this thread's token columns of X, E and O
        const size_t vs = (size_t)DV * ts;   // elements between consecutive tokens of v, w, z, o
        // mixer: RMSNorm weight of this value channel; the write gate's activation scale
        // (the tied modes write with beta = b_range * sigmoid(b))
        const float nwv = kMixer ? a.nw[v] : 0.f;
        const float wact = (mode == GDR_MODE_KDA || mode == GDR_MODE_GDN) ? a.b_range : 1.f;
        bool ok = true;
        if (a.first_wait_limit != 0) {
            // test hook: the group's first wait (for chunk 0's operands) happens at once and
            // gives up after a few non-blocking polls, while the WY group is still loading
            bool got = stid != 0;
            for (uint32_t i = 0; i < a.first_wait_limit && !got; ++i) got = mbar_test_wait(bar_h1, 0u);
            if (!got) sAbort[0] = 1;
            ok = group_and(BAR_ST, got);
        }
        // initial state -> TMEM: fp32 S^T and its bf16 operand copy
        for (int d0 = half * 64; d0 < half * 64 + 64; d0 += 32) {
            float x[32];
#pragma unroll
            for (int j = 0; j < 32; ++j)
                x[j] = transfer ? (d0 + j == v ? 1.f : 0.f) : (S0p ? S0p[(size_t)(d0 + j) * DV + v] : 0.f);
            tmem_st32(tmem + lane_base + TM_S + d0, x);
            st_tmem_bf16(tmem + lane_base + TM_SB + d0 / 2, x);
        }
        if (kMixer) {
            float ones[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) ones[j] = __uint_as_float(0x3F803F80u);   // bf16 pair (1, 1)
            tmem_st32(tmem + lane_base + TM_ONES + half * 32, ones);
        }
        if (stid == 0 && nchunks > 1) prefetch_inputs(1);
        tmem_wait_st();
        tc_fence_before();
        group_sync(BAR_ST);
        for (int c = 0; ok && !kReverse && c < nchunks; ++c) {
            const int t0 = dch(c) * C, n = min(C, T - t0);
            const int pb = c & 1;
            const uint32_t kb_tile = sbase + OFF_KB + pb * 16384;
            const uint32_t p_tile = sbase + OFF_P + pb * 8192, t_tile = sbase + OFF_T + pb * 8192;
            const float *egc = sEGC + (c & 3) * 128;
            if (kStates && GDR_IN_BOUNDS(2 * c < (a.T + 31) / 32 && bh < a.B * a.H, 105)) {
                // checkpoint: S_c (S^T columns [64 half, +64) of this lane), before this
                // chunk's update, as bf16 [dk][dv] at the start of the slot; coalesced over
                // the value channels (lanes)
                __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(
                                         a.chunk_states + ((size_t)bh * ((a.T + 31) / 32) + 2 * c) * DK * DV) + v;
#pragma unroll 1
                for (int d0 = half * 64; d0 < half * 64 + 64; d0 += 32) {
                    float x[32];
                    tmem_ld32(tmem + lane_base + TM_S + d0, x);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) dst[(size_t)(d0 + j) * DV] = __float2bfloat16_rn(x[j]);
                }
            }
            // (w.v)^T for this thread's lane and token columns, read from global memory
            // while the S1 products run; tokens past the end give zero
            float wvt[32];
            uint32_t zp[16];   // mixer: the output gate z of the same lane and tokens, bf16 pairs
            // ---- S1: operands of chunk c (H1); [X | O] = S^T [Kh; Qg]^T ----
            ok = group_and(BAR_ST, stid != 0 || wait(bar_h1, (uint32_t)(c & 1)));
            if (!ok) break;
            const bool exact = sExact[c & 3] != 0;
            if (stid == 0) {
                tc_fence_after();
                const uint32_t id = idesc_bf16(128, 128, false, false, false);
#pragma unroll
                for (int s = 0; s < DK / 16; ++s)
                    mma_bf16_ts(tmem + TM_XO, tmem + TM_SB + s * 8, desc_kmajor(sbase + OFF_QK, 128, 0, s),
                                id, s > 0);
                mma_commit(bar_st);
                if (c + 2 < nchunks) prefetch_inputs(c + 2);
            }
            ++mma_st;
            {
                int last = transfer ? -1 : min(31, n - 1 - j0);   // last token column in range
                const size_t row = tok0 + (size_t)(t0 + j0) * ts;
                // debug build: the rows read (v, w, z) lie inside the segment and the tensors
                if (!GDR_IN_BOUNDS(last < 0 || (t0 + j0 + last < T && row + (size_t)last * ts < rows_total), 103))
                    last = -1;
                const __nv_bfloat16 *vp = V + row * DV + v;
                const __nv_bfloat16 *wp = vec_w ? Wg + row * DV + v : Wsc + row;
                const size_t ws = vec_w ? vs : (size_t)ts;
#pragma unroll
                for (int h = 0; h < 32; h += 16) {   // two halves of 16 columns bound the registers
                    __nv_bfloat16 vv[16], ww[16];
                    if (last == 31) {
                        // whole columns: fixed offsets from one base address, all loads in flight
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            vv[j] = vp[(h + j) * vs];
                            ww[j] = wp[(h + j) * ws];
                        }
                    } else if (last >= 0) {
                        // ragged end: rows past the end re-read the last row and give zero
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int jj = min(h + j, last);
                            vv[j] = vp[jj * vs];
                            ww[j] = wp[jj * ws];
                        }
                    } else {
                        // no row of these columns is in range (or a transition-matrix run)
#pragma unroll
                        for (int j = 0; j < 16; ++j) vv[j] = ww[j] = __float2bfloat16_rn(0.f);
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        float wf = __bfloat162float(ww[j]);
                        if (kMixer) wf = wact * sigmoid_gate(wf);
                        wvt[h + j] = (h + j <= last) ? wf * __bfloat162float(vv[j]) : 0.f;
                    }
                }
                if (kMixer && write_o) {
                    // loaded here, while the group waits for the operands, and kept packed
                    const __nv_bfloat16 *zq = Z + row * DV + v;
                    unsigned short zb[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        zb[j] = last >= 0 ? __bfloat16_as_ushort(zq[min(j, last) * vs]) : (unsigned short)0;
#pragma unroll
                    for (int j = 0; j < 16; ++j) zp[j] = (uint32_t)zb[2 * j] | ((uint32_t)zb[2 * j + 1] << 16);
                }
            }
            ok = group_and(BAR_ST, stid != 0 || wait(bar_st, (uint32_t)((mma_st - 1) & 1)));
            if (!ok) break;
            tc_fence_after();
            // ---- S2: R^T = (w.v)^T - X -> bf16 in TMEM; exact chunks pre-scale S ----
            {
                float x[32];
                tmem_ld32(tmem + lane_base + TM_XO + j0, x);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) x[j] = wvt[j] - x[j];
                st_tmem_bf16(tmem + lane_base + TM_XB + j0 / 2, x);
            }
            if (exact) prescale_state(tmem + lane_base + TM_S, egc, half * 64);   // strong decay
            tmem_wait_st();
            tc_fence_before();
            group_sync(BAR_ST);
            if (stid == 0) {
                // the previous chunk's output store has read its tile (a K-bar buffer the
                // WY group may rebuild once H3 has arrived)
                if (kMixer) bulk_wait_read_all();
                mbar_arrive(bar_h3);   // H3: Kh, Qg of chunk c consumed
            }
            // ---- S3: T and P of chunk c (H2); E^T = R^T T^T ----
            ok = group_and(BAR_ST, stid != 0 || wait(bar_h2 + 8 * pb, (uint32_t)((c >> 1) & 1)));
            if (!ok) break;
            if (stid == 0) {
                tc_fence_after();
                const uint32_t id = idesc_bf16(128, 64, false, false, false);
#pragma unroll
                for (int s = 0; s < C / 16; ++s)
                    mma_bf16_ts(tmem + TM_XO, tmem + TM_XB + s * 8, desc_kmajor(t_tile, 64, 0, s), id, s > 0);
                mma_commit(bar_st);
            }
            ++mma_st;
            ok = group_and(BAR_ST, stid != 0 || wait(bar_st, (uint32_t)((mma_st - 1) & 1)));
            if (!ok) break;
            tc_fence_after();
            // ---- S4: E^T -> bf16 in TMEM ----
            {
                float x[32];
                tmem_ld32(tmem + lane_base + TM_XO + j0, x);
                tmem_wait_ld();
                st_tmem_bf16(tmem + lane_base + TM_XB + j0 / 2, x);
                tmem_wait_st();
            }
            tc_fence_before();
            group_sync(BAR_ST);
            // ---- S5: O^T += E^T P^T,  S^T += E^T Kb (or K_end) ----
            if (stid == 0) {
                tc_fence_after();
                const uint32_t ido = idesc_bf16(128, 64, false, false, false);
                const uint32_t ids = idesc_bf16(128, 128, false, true, false);
#pragma unroll
                for (int s = 0; s < C / 16; ++s) {
                    mma_bf16_ts(tmem + TM_XO + 64, tmem + TM_XB + s * 8, desc_kmajor(p_tile, 64, 0, s), ido, 1u);
                    mma_bf16_ts(tmem + TM_S, tmem + TM_XB + s * 8, desc_mnmajor(kb_tile, 64, 0, s), ids, 1u);
                }
                mma_commit(bar_st);
            }
            ++mma_st;
            ok = group_and(BAR_ST, stid != 0 || wait(bar_st, (uint32_t)((mma_st - 1) & 1)));
            if (!ok) break;
            tc_fence_after();
            // ---- S6: output rows [j0, j0 + 32); state columns [64 half, +64) scaled, kept
            //      in fp32 and as the bf16 operand ----
            float xo[32];
            tmem_ld32(tmem + lane_base + TM_XO + 64 + j0, xo);
            tmem_wait_ld();
            if (!kMixer && write_o &&
                GDR_IN_BOUNDS(n - j0 <= 0 || tok0 + (size_t)(t0 + n - 1) * ts < rows_total, 104)) {
                __nv_bfloat16 *op = O + (tok0 + (size_t)(t0 + j0) * ts) * DV + v;
                const int lim = n - j0;
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (j < lim) op[j * vs] = __float2bfloat16_rn(xo[j]);
            }
            if (kMixer && write_o) {
                // RMSNorm of the output over the 128 value channels (one per TMEM lane): the
                // squares go to this chunk's K-bar buffer (free once S5 has completed) as a
                // bf16 [v][t] tile, and one MMA against a ones A operand writes sum_v o^2 of
                // every token into every lane; it runs while the state is rescaled below
                uint32_t sq[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) sq[j] = pack_bf16(xo[2 * j] * xo[2 * j], xo[2 * j + 1] * xo[2 * j + 1]);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    st_shared_v4(kb_tile + tile_chunk(128, v, j0 / 8 + q), sq[4 * q], sq[4 * q + 1], sq[4 * q + 2],
                                 sq[4 * q + 3]);
                fence_async_smem();
                tc_fence_before();
                group_sync(BAR_ST);
                if (stid == 0) {
                    tc_fence_after();
                    const uint32_t id = idesc_bf16(128, 64, false, true, false);
#pragma unroll
                    for (int s = 0; s < DV / 16; ++s)
                        mma_bf16_ts(tmem + TM_XO, tmem + TM_ONES + s * 8, desc_mnmajor(kb_tile, 128, 0, s), id, s > 0);
                    mma_commit(bar_st);
                }
                ++mma_st;
            }
            for (int d0 = half * 64; d0 < half * 64 + 64; d0 += 32) {
                float x[32];
                tmem_ld32(tmem + lane_base + TM_S + d0, x);
                tmem_wait_ld();
                if (!exact) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) x[j] *= egc[d0 + j];
                    tmem_st32(tmem + lane_base + TM_S + d0, x);
                }
                st_tmem_bf16(tmem + lane_base + TM_SB + d0 / 2, x);
            }
            tmem_wait_st();
            if (kMixer && write_o) {
                // y = o * rsqrt(mean_v o^2 + eps) * weight_v * z * sigmoid(z)
                ok = group_and(BAR_ST, stid != 0 || wait(bar_st, (uint32_t)((mma_st - 1) & 1)));
                if (!ok) break;
                tc_fence_after();
                float ss[32];
                tmem_ld32(tmem + lane_base + TM_XO + j0, ss);
                tmem_wait_ld();
                // every lane holds the same 32 sums: lane j takes token j's rsqrt, the rest by shuffle
                float mine = ss[0];
#pragma unroll
                for (int j = 1; j < 32; ++j) mine = lane == j ? ss[j] : mine;
                const float rstd = rsqrtf(fmaf(mine, 1.f / 128.f, a.eps));
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float zf = __uint_as_float((j & 1) ? (zp[j >> 1] & 0xFFFF0000u) : (zp[j >> 1] << 16));
                    xo[j] *= __shfl_sync(0xffffffffu, rstd, j) * nwv * (zf * sigmoid_gate(zf));
                }
                // y rows -> this chunk's K-bar buffer (the sum MMA has read it), row-major
                // [64 t][128 v]; one tiled store writes the chunk (rows past the end clipped)
                unsigned short *yt = reinterpret_cast<unsigned short *>(sm + (kb_tile - sbase));
#pragma unroll
                for (int j = 0; j < 32; ++j) yt[(j0 + j) * DV + v] = __bfloat16_as_ushort(__float2bfloat16_rn(xo[j]));
                fence_async_smem();
                group_sync(BAR_ST);
                if (stid == 0) {
                    const int tt = t_begin + t0;
                    if (ts != 1) tma_store_4d(&tm.y, kb_tile, 0, hc, tt, bc);
                    else tma_store_4d(&tm.y, kb_tile, 0, tt, hc, bc);
                    bulk_commit();
                }
            }
            tc_fence_before();
            group_sync(BAR_ST);
            if (stid == 0) mbar_arrive(bar_h4 + 8 * pb);   // H4: chunk c finished
        }
        // ---- the backward's state-gradient pass (kReverse): G = dL/dS walks the chunks from
        //      the last to the first.  In TMEM G^T as the state S^T is (lane = value channel);
        //      the WY group supplies the same tiles as for the forward (Kh, Qg, Kb, P, T), and
        //      per chunk (Gated DeltaNet-2 Review §3-2.5, differentiated):
        //        dE^T = (G^T diag(e^gamma_C)) Kb^T + dO^T P      (Kb: K_end on the exact path)
        //        dR^T = dE^T T
        //        G^T <- G^T diag(e^gamma_C) + dO^T Qg - dR^T Kh
        //      Before each chunk's update G is the gradient at the chunk's end: it goes to the
        //      checkpoint slot of the chunk's last 32-token chunk. ----
        for (int c = 0; ok && kReverse && c < nchunks; ++c) {
            const int cd = dch(c);
            const int t0 = cd * C, n = min(C, T - t0);
            const int pb = c & 1;
            const uint32_t kb_tile = sbase + OFF_KB + pb * 16384;
            const uint32_t p_tile = sbase + OFF_P + pb * 8192, t_tile = sbase + OFF_T + pb * 8192;
            const float *egc = sEGC + (c & 3) * 128;
            if (GDR_IN_BOUNDS(2 * cd < (T + 31) / 32 && bh < a.B * a.H, 106)) {
                const int nslot = (T + 31) / 32;
                __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(
                                         a.chunk_states + ((size_t)bh * nslot + min(2 * cd + 1, nslot - 1)) * DK * DV) + v;
#pragma unroll 1
                for (int d0 = half * 64; d0 < half * 64 + 64; d0 += 32) {
                    float x[32];
                    tmem_ld32(tmem + lane_base + TM_S + d0, x);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) dst[(size_t)(d0 + j) * DV] = __float2bfloat16_rn(x[j]);
                }
            }
            {   // dO^T of this lane and token columns -> bf16 in TMEM; tokens past the end give zero
                int last = min(31, n - 1 - j0);
                const __nv_bfloat16 *op = reinterpret_cast<const __nv_bfloat16 *>(a.dO) + (tok0 + t0 + j0) * DV + v;
                if (!GDR_IN_BOUNDS(last < 0 || (t0 + j0 + last < T && tok0 + t0 + j0 + last < rows_total), 107))
                    last = -1;
                float x[32];
                if (last >= 0) {   // rows past the end re-read the last row and give zero
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float y = __bfloat162float(op[min(j, last) * DV]);
                        x[j] = j <= last ? y : 0.f;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) x[j] = 0.f;
                }
                st_tmem_bf16(tmem + lane_base + TM_DO + j0 / 2, x);
            }
            ok = group_and(BAR_ST, stid != 0 || wait(bar_h1, (uint32_t)(c & 1)));
            if (!ok) break;
            const bool exact = sExact[c & 3] != 0;
            // G^T diag(e^gamma_C): the update's accumulator (fp32) and the operand of Kb (bf16;
            // the exact path's K_end carries the decay itself)
            for (int d0 = half * 64; d0 < half * 64 + 64; d0 += 32) {
                float x[32], y[32];
                tmem_ld32(tmem + lane_base + TM_S + d0, x);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) y[j] = x[j] * egc[d0 + j];
                tmem_st32(tmem + lane_base + TM_S + d0, y);
                st_tmem_bf16(tmem + lane_base + TM_SB + d0 / 2, exact ? x : y);
            }
            tmem_wait_st();
            tc_fence_before();
            group_sync(BAR_ST);
            if (stid == 0) {
                tc_fence_after();
                const uint32_t id64 = idesc_bf16(128, 64, false, false, false);
#pragma unroll
                for (int s = 0; s < DK / 16; ++s)   // dE^T = G~^T Kb^T
                    mma_bf16_ts(tmem + TM_XO, tmem + TM_SB + s * 8, desc_kmajor(kb_tile, 64, 0, s), id64, s > 0);
                const uint32_t id128 = idesc_bf16(128, 128, false, true, false);
#pragma unroll
                for (int s = 0; s < C / 16; ++s)    // G^T += dO^T Qg
                    mma_bf16_ts(tmem + TM_S, tmem + TM_DO + s * 8, desc_mnmajor(sbase + OFF_QK, 128, 64, s), id128, 1u);
            }
            ok = group_and(BAR_ST, stid != 0 || wait(bar_h2 + 8 * pb, (uint32_t)((c >> 1) & 1)));
            if (!ok) break;
            if (stid == 0) {
                tc_fence_after();
                const uint32_t id = idesc_bf16(128, 64, false, true, false);
#pragma unroll
                for (int s = 0; s < C / 16; ++s)    // dE^T += dO^T P
                    mma_bf16_ts(tmem + TM_XO, tmem + TM_DO + s * 8, desc_mnmajor(p_tile, 64, 0, s), id, 1u);
                mma_commit(bar_st);
            }
            ++mma_st;
            ok = group_and(BAR_ST, stid != 0 || wait(bar_st, (uint32_t)((mma_st - 1) & 1)));
            if (!ok) break;
            tc_fence_after();
            {   // dE^T -> bf16
                float x[32];
                tmem_ld32(tmem + lane_base + TM_XO + j0, x);
                tmem_wait_ld();
                st_tmem_bf16(tmem + lane_base + TM_XB + j0 / 2, x);
                tmem_wait_st();
            }
            tc_fence_before();
            group_sync(BAR_ST);
            if (stid == 0) {
                tc_fence_after();
                const uint32_t id = idesc_bf16(128, 64, false, true, false);
#pragma unroll
                for (int s = 0; s < C / 16; ++s)    // dR^T = dE^T T
                    mma_bf16_ts(tmem + TM_XO + 64, tmem + TM_XB + s * 8, desc_mnmajor(t_tile, 64, 0, s), id, s > 0);
                mma_commit(bar_st);
            }
            ++mma_st;
            ok = group_and(BAR_ST, stid != 0 || wait(bar_st, (uint32_t)((mma_st - 1) & 1)));
            if (!ok) break;
            tc_fence_after();
            {   // -dR^T -> bf16
                float x[32];
                tmem_ld32(tmem + lane_base + TM_XO + 64 + j0, x);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) x[j] = -x[j];
                st_tmem_bf16(tmem + lane_base + TM_XB + j0 / 2, x);
                tmem_wait_st();
            }
            tc_fence_before();
            group_sync(BAR_ST);
            if (stid == 0) {
                tc_fence_after();
                const uint32_t id = idesc_bf16(128, 128, false, true, false);
#pragma unroll
                for (int s = 0; s < C / 16; ++s)    // G^T -= dR^T Kh
                    mma_bf16_ts(tmem + TM_S, tmem + TM_XB + s * 8, desc_mnmajor(sbase + OFF_QK, 128, 0, s), id, 1u);
                mma_commit(bar_st);
            }
            ++mma_st;
            ok = group_and(BAR_ST, stid != 0 || wait(bar_st, (uint32_t)((mma_st - 1) & 1)));
            if (!ok) break;
            tc_fence_after();
            tc_fence_before();
            group_sync(BAR_ST);
            if (stid == 0) {
                mbar_arrive(bar_h3);            // H3: Kh, Qg of chunk c consumed
                mbar_arrive(bar_h4 + 8 * pb);   // H4: chunk c finished
            }
        }
        // end state: S^T columns [64 half, +64) of this thread's lane, from TMEM
        if (ok && STp) {
            tc_fence_after();
#pragma unroll 1
            for (int d0 = half * 64; d0 < half * 64 + 64; d0 += 16) {
                float x[16];
                tmem_ld16(tmem + lane_base + TM_S + d0, x);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) STp[(size_t)(d0 + j) * DV + v] = x[j];
            }
        }
        if (!ok) sAbort[0] = 1;
        if (kMixer && stid == 0) bulk_wait_all();   // the last output store has landed
    }

    __syncthreads();
    if (sAbort[0]) {
        // drain: committed tensor-core work of both groups and an outstanding raw copy
        if (tid == 0) {
            atomicExch(&g_tc_error, 1);
            mma_commit(bar_wy);
            drain_commits(bar_wy, mma_wy + 1, wait_limit);
            if (raw_issued > raw_done) mbar_wait(bar_raw, (uint32_t)(raw_done & 1), wait_limit);
        }
        if (tid == 256) {
            mma_commit(bar_st);
            drain_commits(bar_st, mma_st + 1, wait_limit);
        }
    }
    __syncthreads();
    __syncwarp();   // tid 0 drained alone: warp 0 reconverges for the .aligned dealloc
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

}  // namespace

bool chunk_tc_supported(const ChunkArgs &a) {
    return a.dtype == GDR_BF16 && a.dk == DK && a.dv == DV && a.chunk == C;
}

// cuTensorMapEncodeTiled from the driver, looked up once (no link against libcuda)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() { return tensor_map_encode_fn(); }

// Map of a token-major [B, T, H, D] tensor (D = 128 elements of esize bytes): dims
// {D, H, T, B}, box {D, 1, C, 1}, no swizzle, zero fill out of range.
bool encode_token_major(CUtensorMap *m, const void *base, int B, int T, int H, CUtensorMapDataType dt,
                        int esize) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)DK, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)DK * esize, (cuuint64_t)H * DK * esize,
                                   (cuuint64_t)T * H * DK * esize};
    const cuuint32_t box[4] = {(cuuint32_t)DK, 1, (cuuint32_t)C, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, dt, 4, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Map of a head-major [B, H, T, D] tensor: dims {D, T, H, B}, box {D, C, 1, 1}.
bool encode_head_major(CUtensorMap *m, const void *base, int B, int T, int H, CUtensorMapDataType dt,
                       int esize) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)DK, (cuuint64_t)T, (cuuint64_t)H, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)DK * esize, (cuuint64_t)T * DK * esize,
                                   (cuuint64_t)H * T * DK * esize};
    const cuuint32_t box[4] = {(cuuint32_t)DK, (cuuint32_t)C, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, dt, 4, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

gdr_status_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t s) {
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
    static_assert(DK == DV, "one box shape serves every per-channel tensor");
    auto kern = a.mixer ? chunk_tc_kernel<true, false, false>
              : a.reverse ? chunk_tc_kernel<false, false, true>
              : a.chunk_states ? chunk_tc_kernel<false, true, false> : chunk_tc_kernel<false, false, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) != cudaSuccess)
        return GDR_ERR_CUDA;
    TokenMaps tm;
    memset(&tm, 0, sizeof(tm));
    if (a.mixer && a.tstride != 1) {
        const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
        bool ok = encode_token_major(&tm.q, a.q, a.B, a.T, a.H, BF, 2) &&
                  encode_token_major(&tm.k, a.k, a.B, a.T, a.H, BF, 2) &&
                  encode_token_major(&tm.v, a.v, a.B, a.T, a.H, BF, 2) &&
                  encode_token_major(&tm.z, a.z, a.B, a.T, a.H, BF, 2);
        if (ok && mode_b_vec(a.mode)) ok = encode_token_major(&tm.b, a.b, a.B, a.T, a.H, BF, 2);
        if (ok && mode_w_vec(a.mode)) ok = encode_token_major(&tm.w, a.w, a.B, a.T, a.H, BF, 2);
        if (ok && mode_g_vec(a.mode))
            ok = encode_token_major(&tm.g, a.g, a.B, a.T, a.H, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4);
        if (!ok) return GDR_ERR_CUDA;
    }
    if (a.mixer) {
        const bool ok = a.tstride != 1
                            ? encode_token_major(&tm.y, a.o, a.B, a.T, a.H, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2)
                            : encode_head_major(&tm.y, a.o, a.B, a.T, a.H, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2);
        if (!ok) return GDR_ERR_CUDA;
    }
    kern<<<(unsigned)(a.B * a.H * chunk_roles(a)), kThreads, SMEM_BYTES, s>>>(a, tm);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

GDR_BOUNDS_READER(chunk_tc_bounds_site)

cudaError_t chunk_tc_read_and_clear_error(int *err) {
    cudaError_t e = cudaMemcpyFromSymbol(err, g_tc_error, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(int));
}

}  // namespace gdr
