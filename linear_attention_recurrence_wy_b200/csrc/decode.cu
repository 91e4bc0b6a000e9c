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
// state is written from registers.
//
// dk = dv = 128 (decode_stream_kernel): a persistent kernel, one CTA per SM, that streams
// the heads through three 64 KB shared-memory buffers.  Each state arrives by one bulk copy
// (two heads ahead), is updated in place in shared memory, and leaves by one bulk store,
// so HBM sees a continuous read stream and write stream.  The small per-head vectors
// (q, k, v, b, w, g) come one head ahead by 16-byte asynchronous copies.  Every wait on a
// bulk copy is bounded; on expiry the kernel records the failure (read by
// gdr_last_device_error), stops issuing and drains its own copies.
//
// Other shapes (decode_kernel): one CTA of 256 threads per head; each thread holds
// float4 column groups of several rows, the loads are 16-byte coalesced and all issued
// before any arithmetic.
#include "bounds.cuh"
#include "common.cuh"
#include "tc_util.cuh"

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
        const float bv = mode_b_vec(a.mode) ? ld_elem(a.b, e, a.dtype) : ld_elem(a.b, nh, a.dtype);
        const float gv = (a.mode == GDR_MODE_GDN) ? a.g[nh] : a.g[e];
        s_q[i] = ld_elem(a.q, e, a.dtype);
        s_k[i] = kv;
        s_bk[i] = bv * kv;
        s_a[i] = __expf(gv);
    }
    for (int j = tid; j < DV; j += kThreads) {
        const size_t e = (size_t)nh * DV + j;
        const float wv = mode_w_vec(a.mode) ? ld_elem(a.w, e, a.dtype)
                         : ld_elem(a.mode == GDR_MODE_BONLY ? a.w : a.b, nh, a.dtype);
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


__device__ int g_decode_error = 0;

constexpr int SD = 128;                       // dk = dv of the streaming kernel
constexpr int kStreamThreads = 256;
constexpr int kBufs = 3;                      // state buffers
constexpr int kStateBytes = SD * SD * 4;      // 64 KB
constexpr int kVecSlot = 512;                 // one per-head vector, bf16 or fp32
constexpr int kVecBytes = 6 * kVecSlot;       // q, k, b, w, v, g
// dynamic shared memory map
constexpr int SO_BUF = 0;
constexpr int SO_VEC = kBufs * kStateBytes;                 // [2][kVecBytes]
constexpr int SO_RED = SO_VEC + 2 * kVecBytes;              // red_r, red_o [8][SD + 1] fp32
constexpr int SO_ROW = SO_RED + 2 * 8 * (SD + 1) * 4;       // s_q, s_k, s_bk, s_a, s_wv, s_u [SD]
constexpr int SO_MISC = SO_ROW + 6 * SD * 4;                // kq, abort flag, mbarriers
constexpr int kStreamSmem = SO_MISC + 64;
static_assert(kStreamSmem <= 227 * 1024, "shared memory budget");

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void *g) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(g) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_s2g(void *g, uint32_t saddr, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(g), "r"(saddr), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// the bulk stores of this thread, except the most recent one, have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_all_but_1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__global__ void __launch_bounds__(kStreamThreads, 1) decode_stream_kernel(DecodeArgs a) {
    extern __shared__ __align__(128) unsigned char sm[];
    const uint32_t sbase = tc::smem_u32(sm);
    const int tid = threadIdx.x, cg = tid & 31, r0 = tid >> 5;   // columns 4 cg .., rows r0 + 8 p
    const int NH = a.N * a.H, G = gridDim.x;
    const int iters = blockIdx.x < NH ? (NH - 1 - blockIdx.x) / G + 1 : 0;
    const bool bf = a.dtype == GDR_BF16, vec_g = mode_g_vec(a.mode);
    const bool vec_b = mode_b_vec(a.mode), vec_w = mode_w_vec(a.mode);
    const void *wsrc = a.mode == GDR_MODE_BONLY ? a.w : a.b;   // scalar write gate, when not vec_w
    const int esz = bf ? 2 : 4;   // bytes per element of q, k, v, b, w
    float *red_r = reinterpret_cast<float *>(sm + SO_RED), *red_o = red_r + 8 * (SD + 1);
    float *s_q = reinterpret_cast<float *>(sm + SO_ROW), *s_k = s_q + SD, *s_bk = s_k + SD;
    float *s_a = s_bk + SD, *s_wv = s_a + SD, *s_u = s_wv + SD;
    volatile float *s_kq = reinterpret_cast<volatile float *>(sm + SO_MISC);
    volatile int *s_abort = reinterpret_cast<volatile int *>(sm + SO_MISC + 4);
    const uint32_t bar_full = sbase + SO_MISC + 8;   // [kBufs] mbarriers, 8-byte aligned

    // per-head vectors of iteration i -> vector buffer i & 1 by 16-byte asynchronous copies;
    // scalar gates (erase, write, decay) are loaded into registers here (thread 255) and
    // stored by put_scalars once the head before no longer needs the buffer
    float pend_b = 0.f, pend_w = 0.f, pend_g = 0.f;
    auto fetch_vectors = [&](int i) {
        const int h = blockIdx.x + i * G;
        unsigned char *vb = sm + SO_VEC + (i & 1) * kVecBytes;
        const int per = SD * esz / 16;   // 16-byte pieces per vector
        // slots: 0 q, 1 k, 2 b, 3 w, 4 v, 5 g
        for (int j = tid; j < 6 * 32; j += kStreamThreads) {
            const int slot = j >> 5, piece = j & 31;
            const void *src = nullptr;
            int pieces = per;
            if (slot == 0) src = (const unsigned char *)a.q + (size_t)h * SD * esz;
            else if (slot == 1) src = (const unsigned char *)a.k + (size_t)h * SD * esz;
            else if (slot == 2) src = vec_b ? (const unsigned char *)a.b + (size_t)h * SD * esz : nullptr;
            else if (slot == 3) src = vec_w ? (const unsigned char *)a.w + (size_t)h * SD * esz : nullptr;
            else if (slot == 4) src = (const unsigned char *)a.v + (size_t)h * SD * esz;
            else { src = vec_g ? (const unsigned char *)(a.g + (size_t)h * SD) : nullptr; pieces = SD * 4 / 16; }
            if (src && piece < pieces)
                cp_async16(tc::smem_u32(vb + slot * kVecSlot + piece * 16), (const unsigned char *)src + piece * 16);
        }
        cp_async_commit();
        if (tid == kStreamThreads - 1) {
            if (!vec_b) pend_b = ld_elem(a.b, h, a.dtype);
            if (!vec_w) pend_w = ld_elem(wsrc, h, a.dtype);
            if (!vec_g) pend_g = a.g[h];
        }
    };
    auto put_scalars = [&](int i) {   // thread 255, after fetch_vectors(i)
        float *vb = reinterpret_cast<float *>(sm + SO_VEC + (i & 1) * kVecBytes);
        if (!vec_b) vb[2 * kVecSlot / 4] = pend_b;   // scalar erase gate in slot 2
        if (!vec_w) vb[3 * kVecSlot / 4] = pend_w;   // scalar write gate in slot 3
        if (!vec_g) vb[5 * kVecSlot / 4] = pend_g;   // scalar g_log in slot 5
    };
    bool first_expired = false;   // thread 0: the test hook's first wait gave up
    // bounded wait on a state buffer; gives up early once another thread has aborted
    auto wait_full = [&](int i) -> bool {
        const uint32_t bar = bar_full + 8 * (i % kBufs), parity = (uint32_t)((i / kBufs) & 1);
        if (i == 0 && a.first_wait_limit != 0 && first_expired) {
            *s_abort = 1;   // test hook: see the first load below
            return false;
        }
        for (uint32_t n = 0; n < a.wait_limit; ++n) {
            if (tc::mbar_try_wait(bar, parity)) return true;
            if ((n & 255) == 255 && *s_abort) return false;
        }
        *s_abort = 1;
        return false;
    };
    auto issue_load = [&](int i) {   // state of iteration i -> buffer i % kBufs (thread 0)
        const int h = blockIdx.x + i * G;
        if (!GDR_IN_BOUNDS(h < NH, 201)) return;   // debug build: a head of this call
        const uint32_t bar = bar_full + 8 * (i % kBufs);
        tc::mbar_arrive_expect_tx(bar, kStateBytes);
        tc::bulk_g2s(sbase + SO_BUF + (i % kBufs) * kStateBytes, a.S + (size_t)h * SD * SD, kStateBytes, bar);
    };

    if (tid == 0) {
        for (int b = 0; b < kBufs; ++b) tc::mbar_init(bar_full + 8 * b, 1);
        *s_abort = 0;
        tc::fence_mbar_init();
    }
    __syncthreads();
    int loads = 0;
    if (tid == 0) {
        for (; loads < 2 && loads < iters; ++loads) issue_load(loads);
        if (a.first_wait_limit != 0 && iters > 0) {
            // test hook: the first wait on a state copy polls it right after the issue, a few
            // non-blocking times, and gives up while the copy is still in flight
            bool got = false;
            for (uint32_t n = 0; n < a.first_wait_limit && !got; ++n) got = tc::mbar_test_wait(bar_full, 0u);
            first_expired = !got;
        }
    }
    if (iters > 0) {
        fetch_vectors(0);
        if (tid == kStreamThreads - 1) put_scalars(0);
    }

    bool ok = true;
    for (int i = 0; i < iters && ok; ++i) {
        const int h = blockIdx.x + i * G;
        float4 *buf = reinterpret_cast<float4 *>(sm + SO_BUF + (i % kBufs) * kStateBytes);
        const unsigned char *vb = sm + SO_VEC + (i & 1) * kVecBytes;
        cp_async_wait_all();
        __syncthreads();   // vectors of head i in place; the previous head is fully done
        if (i + 1 < iters) fetch_vectors(i + 1);
        // per-row values and w.v
        if (tid < SD) {
            auto vec = [&](int slot, int j) -> float {
                return bf ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(vb + slot * kVecSlot)[j])
                          : reinterpret_cast<const float *>(vb + slot * kVecSlot)[j];
            };
            const float kv = vec(1, tid);
            const float bv = vec_b ? vec(2, tid) : reinterpret_cast<const float *>(vb + 2 * kVecSlot)[0];
            const float gv = reinterpret_cast<const float *>(vb + 5 * kVecSlot)[vec_g ? tid : 0];
            s_q[tid] = vec(0, tid);
            s_k[tid] = kv;
            s_bk[tid] = bv * kv;
            s_a[tid] = __expf(gv);
            const float wv = vec_w ? vec(3, tid) : reinterpret_cast<const float *>(vb + 3 * kVecSlot)[0];
            s_wv[tid] = wv * vec(4, tid);
        }
        ok = __syncthreads_and(tid != 0 || wait_full(i));
        if (!ok) break;
        if (tid < 32) {
            float acc = 0.f;
            for (int j = tid; j < SD; j += 32) acc = fmaf(s_k[j], s_q[j], acc);
#pragma unroll
            for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (tid == 0) *s_kq = acc;
        }
        float4 x[16];
        float pr[4] = {0.f, 0.f, 0.f, 0.f}, po[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int p = 0; p < 16; ++p) {
            const int row = r0 + 8 * p;
            x[p] = buf[row * (SD / 4) + cg];
            const float al = s_a[row], bkv = s_bk[row], qv = s_q[row];
            x[p].x *= al; x[p].y *= al; x[p].z *= al; x[p].w *= al;
            pr[0] = fmaf(x[p].x, bkv, pr[0]); pr[1] = fmaf(x[p].y, bkv, pr[1]);
            pr[2] = fmaf(x[p].z, bkv, pr[2]); pr[3] = fmaf(x[p].w, bkv, pr[3]);
            po[0] = fmaf(x[p].x, qv, po[0]); po[1] = fmaf(x[p].y, qv, po[1]);
            po[2] = fmaf(x[p].z, qv, po[2]); po[3] = fmaf(x[p].w, qv, po[3]);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            red_r[r0 * (SD + 1) + 4 * cg + c] = pr[c];
            red_o[r0 * (SD + 1) + 4 * cg + c] = po[c];
        }
        __syncthreads();
        if (tid < SD) {
            float rs = 0.f, os = 0.f;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                rs += red_r[r * (SD + 1) + tid];
                os += red_o[r * (SD + 1) + tid];
            }
            const float u = s_wv[tid] - rs;
            s_u[tid] = u;
            st_elem(a.o, (size_t)h * SD + tid, a.dtype, fmaf(u, *s_kq, os));
        }
        __syncthreads();
        const float u0 = s_u[4 * cg], u1 = s_u[4 * cg + 1], u2 = s_u[4 * cg + 2], u3 = s_u[4 * cg + 3];
#pragma unroll
        for (int p = 0; p < 16; ++p) {
            const int row = r0 + 8 * p;
            const float kv = s_k[row];
            float4 y;
            y.x = fmaf(kv, u0, x[p].x); y.y = fmaf(kv, u1, x[p].y);
            y.z = fmaf(kv, u2, x[p].z); y.w = fmaf(kv, u3, x[p].w);
            buf[row * (SD / 4) + cg] = y;
        }
        if (tid == kStreamThreads - 1 && i + 1 < iters) put_scalars(i + 1);
        tc::fence_async_smem();
        __syncthreads();
        if (tid == 0 && GDR_IN_BOUNDS(h < NH, 202)) {
            bulk_s2g(a.S + (size_t)h * SD * SD, sbase + SO_BUF + (i % kBufs) * kStateBytes, kStateBytes);
            bulk_commit();
            if (loads < iters) {
                // the buffer of iteration i + 2 last held iteration i - 1, whose store must
                // have finished reading it
                bulk_wait_read_all_but_1();
                issue_load(loads);
                ++loads;
            }
        }
    }
    if (!ok) {
        if (tid == 0) {
            atomicExch(&g_decode_error, 1);
            // drain: the loads issued but not consumed, at most the last two (bounded)
            for (int i = loads > 2 ? loads - 2 : 0; i < loads; ++i)
                tc::mbar_wait(bar_full + 8 * (i % kBufs), (uint32_t)((i / kBufs) & 1), a.wait_limit);
        }
        cp_async_wait_all();
    }
    if (tid == 0) bulk_wait_all();   // stores complete before the CTA exits
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
    if (a.dk == SD && a.dv == SD) {
        int dev = 0, sms = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            return GDR_ERR_CUDA;
        if (cudaFuncSetAttribute(decode_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kStreamSmem) != cudaSuccess)
            return GDR_ERR_CUDA;
        const int nh = a.N * a.H;
        decode_stream_kernel<<<(unsigned)(nh < sms ? nh : sms), kStreamThreads, kStreamSmem, s>>>(a);
        return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
    }
    switch (a.dk) {
        case 16: return launch_dk<16>(a, s);
        case 32: return launch_dk<32>(a, s);
        case 64: return launch_dk<64>(a, s);
        case 128: return launch_dk<128>(a, s);
        default: return GDR_ERR_DIM;
    }
}

}  // namespace gdr

namespace gdr {
cudaError_t decode_read_and_clear_error(int *err) {
    cudaError_t e = cudaMemcpyFromSymbol(err, g_decode_error, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_decode_error, &zero, sizeof(int));
}
}  // namespace gdr

namespace gdr {
GDR_BOUNDS_READER(decode_bounds_site)
}  // namespace gdr
