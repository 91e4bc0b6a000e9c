// state_pass.cu -- phase two of the two-phase chunked forward: the recurrence over the
// chunk records of phase one (wy_prep.cu, two_phase.cuh).
//
// One CTA (256 threads) per sequence-head, or per segment and role of a sequence split
// (ChunkArgs: the whole sequence, a split's end-state and transition-map runs, its output
// pass).  The fp32 state stays in tensor memory, transposed (lane = value channel v, column =
// key channel d), with a bf16 copy as the A operand of the next chunk's products.  Per chunk
// (Gated DeltaNet-2 Review §3-2.5 "Chunkwise WY training": only the state crosses chunks):
//
//   X^T  = S^T W^T            MMA (W^T MN-major from the record)          -> E needs it
//   O^T  = S^T Qg^T           MMA, issued behind X^T
//   E^T  = U^T - X^T          read-out, U^T from the record, bf16 -> TMEM
//   O^T += E^T P^T,  S^T += E^T Kb      (exact chunks: S^T scaled by e^gamma_C first, Kb = K_end)
//   S^T  = S^T diag(e^gamma_C)          read-out, fp32 and its bf16 operand copy
//
// so the state's own chain is two MMA round trips per chunk.  Warp 8 copies the records in
// (one bulk copy each, two stages; a stage is refilled once the update products that last
// read it have completed) and issues the tensor-core work; warps 0-7 do the read-outs and
// hand over through mbarriers (E ready, state operand ready).  The bf16 state operand of
// the next chunk is written before the fp32 state, which is needed only by the next update.
// The output of chunk c is read out of TMEM (two buffers, by chunk parity) while chunk c+1's
// update products run, staged row-major in shared memory and written by one bulk copy.  Every wait is bounded; on expiry the kernel records the failure, drains
// its own copies and tensor-core work (bounded), frees its TMEM and returns.
#include <cuda_bf16.h>

#include "bounds.cuh"
#include "tc_util.cuh"
#include "two_phase.cuh"

namespace gdr {
namespace tp {

__device__ int g_sp_error = 0;   // a bounded wait of the state pass expired

namespace {

using namespace tc;

constexpr int C = 64, DK = 128, DV = 128;
constexpr int kCompute = 256;              // warps 0-7: TMEM read-outs and element work
constexpr int kThreads = kCompute + 32;    // warp 8: record copies and tensor-core issue
constexpr int NST = 2;                     // record stages
constexpr int BAR_CMP = 1;                 // named barrier of the compute warps

constexpr int OFF_STAGE = 0;                          // NST records            2 x 73 KB
constexpr int OFF_OT = NST * REC_BYTES;               // output rows bf16 [2][64 t][128 v]  32 KB
constexpr int OFF_EGC = OFF_OT + 2 * 16384;           // e^gamma_C of the stages [2][128] fp32
constexpr int OFF_FLAG = OFF_EGC + 1024;              // [0] abort
constexpr int OFF_BAR = OFF_FLAG + 16;                // full[2], x, s, e, sc; TMEM slot
constexpr int NBAR = 6;
constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 8 + 1024;
static_assert(REC_BYTES % 1024 == 0 && OFF_OT % 1024 == 0, "tiles on 1024-byte boundaries");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");

// TMEM columns (fp32 unless noted)
constexpr uint32_t TM_S = 0;      // S^T                               128
constexpr uint32_t TM_X = 128;    // X^T                                64
constexpr uint32_t TM_O = 192;    // O^T [2] by chunk parity           128
constexpr uint32_t TM_SB = 320;   // S^T bf16 (packed)                  64
constexpr uint32_t TM_EB = 384;   // E^T bf16 (packed)                  32
constexpr uint32_t TM_X2 = 416;   // X^T, key channels 64..127 (a second, independent
                                  // accumulation chain; X^T is the sum of both)     64
constexpr uint32_t TM_COLS = 512;

// barriers over the 256 compute threads (the .aligned forms: the warp reconverges first); the
// first also returns the AND of v over them
__device__ __forceinline__ bool cmp_and(bool v) {
    __syncwarp();
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "n"(BAR_CMP), "n"(kCompute)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void cmp_sync() {
    __syncwarp();
    asm volatile("bar.sync %0, %1;" ::"n"(BAR_CMP), "n"(kCompute) : "memory");
}
__device__ __forceinline__ void arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__global__ void __launch_bounds__(kThreads, 1) state_pass_kernel(ChunkArgs a, const unsigned char *records) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int half = (warp >> 2) & 1;        // token columns [32 half, +32), state columns [64 half, +64)
    const int v = quarter * 32 + lane;       // value channel = TMEM lane
    const int j0 = half * 32;

    // ---- this CTA's job (the roles of the fused kernel's sequence split) ----
    const bool maps = a.seg_maps != 0;
    const int roles = chunk_roles(a);
    const int bh = blockIdx.x / roles, role = blockIdx.x % roles;
    const bool transfer = maps ? role == 1 : (a.pass && role > a.nseg - 2);
    const int seg = maps ? 0 : transfer ? role - (a.nseg - 2) : role;
    const int t_begin = seg * a.seg_len;
    const int T = min(a.seg_len, a.T - t_begin);
    const int nchunks = (T + C - 1) / C;
    const int nch_all = (a.T + C - 1) / C;
    const size_t sidx = ((size_t)bh * a.nseg + seg) * DK * DV;
    const float *S0p = nullptr;
    float *STp = nullptr;
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
    const bool write_o = !a.pass && !maps;
    // debug build: the segment's records and state slots lie inside the workspace
    if (!GDR_IN_BOUNDS(bh < a.B * a.H && t_begin >= 0 && T >= 1 && t_begin % C == 0 &&
                           (maps || a.nseg == 1 || sidx + (size_t)DK * DV <= (size_t)a.B * a.H * a.nseg * DK * DV),
                       801))
        return;
    const unsigned char *rec0 = records + ((size_t)bh * nch_all + t_begin / C) * REC_BYTES;
    __nv_bfloat16 *O = (__nv_bfloat16 *)a.o;
    const size_t orow0 = (size_t)bh * a.T + t_begin;   // output row of the segment's first token

    float *sEgc = reinterpret_cast<float *>(sm + OFF_EGC);
    volatile int *sAbort = reinterpret_cast<volatile int *>(sm + OFF_FLAG);
    const uint32_t bar_full = sbase + OFF_BAR;   // [2] record c of stage c % 2 has landed
    const uint32_t bar_x = bar_full + 16;        // X^T of chunk c computed
    const uint32_t bar_s = bar_full + 24;        // chunk c's update products computed
    const uint32_t bar_e = bar_full + 32;        // E^T of chunk c in TMEM (compute -> issuer)
    const uint32_t bar_sc = bar_full + 40;       // the state's bf16 operand ready (phase 0: S0,
                                                 // phase c + 1: after chunk c)
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + NBAR * 8);

    if (tid == 0) {
        for (int i = 0; i < NBAR; ++i) mbar_init(bar_full + 8 * i, 1);
        sAbort[0] = 0;
        fence_mbar_init();
    }
    __syncwarp();
    if (warp == 0) {
        tmem_alloc(smem_u32(tslot), TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    const uint32_t wait_limit = a.wait_limit;
    auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
        for (uint32_t i = 0; i < wait_limit; ++i) {
            if (mbar_try_wait(bar, parity)) return true;
            if ((i & 255) == 255 && sAbort[0]) return false;
        }
        sAbort[0] = 1;
        return false;
    };
    int loads = 0, n_s = 0;   // (issuer) record copies issued, commits on bar_s

    if (warp == 8) {
        // ================================================ issuer: record copies and MMAs
        if (lane == 0) {
            // the parts of a record this run reads: all of it for the output pass; W^T, U^T,
            // Kb and the tail (e^gamma_C, flag) for an end-state run; without U^T for a
            // transition-map run
            auto issue_load = [&](int c) {
                const uint32_t st = sbase + OFF_STAGE + (c % NST) * REC_BYTES;
                const uint32_t full = bar_full + 8 * (c % NST);
                const unsigned char *src = rec0 + (size_t)c * REC_BYTES;
                fence_async_smem();
                if (write_o) {
                    mbar_arrive_expect_tx(full, REC_LOAD);
                    bulk_g2s(st, src, REC_LOAD, full);
                } else {
                    const uint32_t head = transfer ? REC_UT - REC_WT : REC_QG - REC_WT;
                    mbar_arrive_expect_tx(full, head + (REC_P - REC_KB) + (REC_LOAD - REC_EGC));
                    bulk_g2s(st + REC_WT, src + REC_WT, head, full);
                    bulk_g2s(st + REC_KB, src + REC_KB, REC_P - REC_KB, full);
                    bulk_g2s(st + REC_EGC, src + REC_EGC, REC_LOAD - REC_EGC, full);
                }
                ++loads;
            };
            bool ok = true;
            issue_load(0);
            if (a.first_wait_limit != 0) {
                // test hook: the first wait (for record 0) gives up after a few non-blocking
                // polls, made while the record is still on its way
                bool got = false;
                for (uint32_t i = 0; i < a.first_wait_limit && !got; ++i) got = mbar_test_wait(bar_full, 0u);
                if (!got) {
                    sAbort[0] = 1;
                    ok = false;
                }
            }
            if (nchunks > 1) issue_load(1);
            const uint32_t idx = idesc_bf16(128, 64, false, true, false);
            const uint32_t ido = idesc_bf16(128, 64, false, false, false);
            const uint32_t ids = idesc_bf16(128, 128, false, true, false);
            for (int c = 0; ok && c < nchunks; ++c) {
                const uint32_t st = sbase + OFF_STAGE + (c % NST) * REC_BYTES;
                ok = wait(bar_full + 8 * (c % NST), (uint32_t)((c / NST) & 1)) && wait(bar_sc, (uint32_t)(c & 1));
                if (!ok) break;
                tc_fence_after();
                // X^T = S^T W^T as two halves of the key channels in two accumulators (two
                // independent chains of four steps), committed on its own; then O^T = S^T Qg^T
#pragma unroll
                for (int k = 0; k < DK / 32; ++k) {
                    mma_bf16_ts(tmem + TM_X, tmem + TM_SB + k * 8, desc_mnmajor(st + REC_WT, 128, 0, k), idx, k > 0);
                    mma_bf16_ts(tmem + TM_X2, tmem + TM_SB + (k + 4) * 8, desc_mnmajor(st + REC_WT, 128, 0, k + 4), idx,
                                k > 0);
                }
                mma_commit(bar_x);
                if (write_o) {
#pragma unroll
                    for (int k = 0; k < DK / 16; ++k)
                        mma_bf16_ts(tmem + TM_O + 64 * (c & 1), tmem + TM_SB + k * 8,
                                    desc_kmajor(st + REC_QG, 64, 0, k), ido, k > 0);
                }
                ok = wait(bar_e, (uint32_t)(c & 1));
                if (!ok) break;
                tc_fence_after();
                // O^T += E^T P^T,  S^T += E^T Kb
#pragma unroll
                for (int k = 0; k < C / 16; ++k) {
                    if (write_o)
                        mma_bf16_ts(tmem + TM_O + 64 * (c & 1), tmem + TM_EB + k * 8, desc_kmajor(st + REC_P, 64, 0, k),
                                    ido, 1u);
                    mma_bf16_ts(tmem + TM_S, tmem + TM_EB + k * 8, desc_mnmajor(st + REC_KB, 64, 0, k), ids, 1u);
                }
                mma_commit(bar_s);
                ++n_s;
                if (c + NST < nchunks) {
                    // the stage is free once the update products have read it
                    ok = wait(bar_s, (uint32_t)(c & 1));
                    if (!ok) break;
                    issue_load(c + NST);
                }
            }
            if (!ok) sAbort[0] = 1;
        }
    } else {
        // ================================================ compute warps 0-7
        // initial state -> TMEM: fp32 S^T and its bf16 operand copy
        for (int d0 = half * 64; d0 < half * 64 + 64; d0 += 32) {
            float x[32];
#pragma unroll
            for (int j = 0; j < 32; ++j)
                x[j] = transfer ? (d0 + j == v ? 1.f : 0.f) : (S0p ? S0p[(size_t)(d0 + j) * DV + v] : 0.f);
            tmem_st32(tmem + lane_base + TM_S + d0, x);
            st_tmem_bf16(tmem + lane_base + TM_SB + d0 / 2, x);
        }
        tmem_wait_st();
        tc_fence_before();
        cmp_sync();
        if (tid == 0) arrive(bar_sc);   // phase 0: the start state is in place
        __syncwarp();

        // output of chunk cc: TMEM -> row-major staging (its copy goes out after the next barrier)
        auto stage_o = [&](int cc) {
            float xo[32];
            tmem_ld32(tmem + lane_base + TM_O + 64 * (cc & 1) + j0, xo);
            tmem_wait_ld();
            unsigned short *ot = reinterpret_cast<unsigned short *>(sm + OFF_OT + (cc & 1) * 16384);
#pragma unroll
            for (int j = 0; j < 32; ++j) ot[(j0 + j) * DV + v] = __bfloat16_as_ushort(__float2bfloat16_rn(xo[j]));
            fence_async_smem();
        };
        auto store_o = [&](int cc) {   // thread 0, after a barrier that follows stage_o(cc)
            const int n = min(C, T - cc * C);
            if (GDR_IN_BOUNDS(orow0 + (size_t)cc * C + n <= (size_t)a.B * a.H * a.T, 802)) {
                bulk_s2g(O + (orow0 + (size_t)cc * C) * DV, sbase + OFF_OT + (cc & 1) * 16384, (uint32_t)n * DV * 2);
                bulk_commit();
            }
        };

        bool ok = true;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NST;
            const unsigned char *rs = sm + OFF_STAGE + s * REC_BYTES;
            // ---- record c (for U^T and e^gamma_C) and X^T of chunk c ----
            // (thread 0 waits alone; its warp reconverges before the aligned barrier and the
            // warp-collective TMEM loads after it)
            bool got = true;
            if (tid == 0) got = wait(bar_full + 8 * s, (uint32_t)((c / NST) & 1)) && wait(bar_x, (uint32_t)(c & 1));
            __syncwarp();
            ok = cmp_and(got);
            if (!ok) break;
            tc_fence_after();
            if (tid < 128) sEgc[s * 128 + tid] = reinterpret_cast<const float *>(rs + REC_EGC)[tid];
            const bool exact = *reinterpret_cast<const volatile int *>(rs + REC_FLAG) != 0;
            // ---- E^T = U^T - X^T (transition-map runs: -X^T) -> bf16 in TMEM ----
            {
                float x[32], x2[32];
                tmem_ld32(tmem + lane_base + TM_X + j0, x);
                tmem_ld32(tmem + lane_base + TM_X2 + j0, x2);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) x[j] += x2[j];
                if (!transfer) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 u = *reinterpret_cast<const uint4 *>(rs + REC_UT + tile_chunk(128, v, j0 / 8 + q));
                        float f[8];
                        bf16x8_to_f32(u, f);
#pragma unroll
                        for (int j = 0; j < 8; ++j) x[8 * q + j] = f[j] - x[8 * q + j];
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) x[j] = -x[j];
                }
                st_tmem_bf16(tmem + lane_base + TM_EB + j0 / 2, x);
            }
            if (exact) {
                // strong decay: S^T columns [64 half, +64) scaled by e^gamma_C before the update
                // (this chunk's products with S^T read the bf16 copy, which stays as it was)
                cmp_sync();   // sEgc of this chunk is complete
#pragma unroll 1
                for (int d0 = half * 64; d0 < half * 64 + 64; d0 += 32) {
                    float x[32];
                    tmem_ld32(tmem + lane_base + TM_S + d0, x);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) x[j] *= sEgc[s * 128 + d0 + j];
                    tmem_st32(tmem + lane_base + TM_S + d0, x);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            // the staging buffer chunk c-1's rows go to last held chunk c-3's: read by now
            if (tid == 0 && write_o) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
            __syncwarp();
            cmp_sync();
            if (tid == 0) arrive(bar_e);
            __syncwarp();
            // ---- the previous chunk's output leaves TMEM while the update products run ----
            if (write_o && c >= 1) stage_o(c - 1);
            // ---- S^T scaled by e^gamma_C (fast path): the bf16 operand first, then fp32 ----
            got = true;
            if (tid == 0) got = wait(bar_s, (uint32_t)(c & 1));
            __syncwarp();
            ok = cmp_and(got);
            if (!ok) break;
            tc_fence_after();
            float sx[2][32];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int d0 = half * 64 + 32 * h;
                tmem_ld32(tmem + lane_base + TM_S + d0, sx[h]);
            }
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int d0 = half * 64 + 32 * h;
                if (!exact) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) sx[h][j] *= sEgc[s * 128 + d0 + j];
                }
                st_tmem_bf16(tmem + lane_base + TM_SB + d0 / 2, sx[h]);
            }
            tmem_wait_st();
            tc_fence_before();
            cmp_sync();
            if (tid == 0) {
                arrive(bar_sc);
                if (write_o && c >= 1) store_o(c - 1);
            }
            __syncwarp();
            if (!exact) {
#pragma unroll
                for (int h = 0; h < 2; ++h) tmem_st32(tmem + lane_base + TM_S + half * 64 + 32 * h, sx[h]);
                tmem_wait_st();
            }
        }
        if (ok && write_o) {
            tc_fence_after();
            if (tid == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
            __syncwarp();
            cmp_sync();
            stage_o(nchunks - 1);
            cmp_sync();
            if (tid == 0) store_o(nchunks - 1);
            __syncwarp();
        }
        // end state: S^T columns [64 half, +64) of this thread's lane
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
        if (tid == 0) bulk_wait_read_all();   // the output copies have read shared memory
    }
    __syncthreads();
    if (sAbort[0] && tid == kCompute) {
        // drain (bounded): one more commit covers every MMA the issuer made; commits complete
        // in order, so phases n-1 and then n of it are waited for (a parity wait alone cannot
        // tell phase n from n-2); then every record copy, stage by stage in issue order
        atomicExch(&g_sp_error, 1);
        mma_commit(bar_s);
        if (n_s >= 1) mbar_wait(bar_s, (uint32_t)((n_s - 1) & 1), wait_limit);
        mbar_wait(bar_s, (uint32_t)(n_s & 1), wait_limit);
        for (int c = 0; c < loads; ++c) mbar_wait(bar_full + 8 * (c % NST), (uint32_t)((c / NST) & 1), wait_limit);
    }
    tc_fence_before();
    __syncthreads();
    __syncwarp();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

}  // namespace

gdr_status_t launch_state_pass(const ChunkArgs &a, const unsigned char *records, cudaStream_t s) {
    if (cudaFuncSetAttribute(state_pass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) !=
        cudaSuccess)
        return GDR_ERR_CUDA;
    state_pass_kernel<<<(unsigned)(a.B * a.H * chunk_roles(a)), kThreads, SMEM_BYTES, s>>>(a, records);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

cudaError_t state_pass_read_and_clear_error(int *err) {
    cudaError_t e = cudaMemcpyFromSymbol(err, g_sp_error, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_sp_error, &zero, sizeof(int));
}

}  // namespace tp

GDR_BOUNDS_READER(state_pass_bounds_site)

}  // namespace gdr
