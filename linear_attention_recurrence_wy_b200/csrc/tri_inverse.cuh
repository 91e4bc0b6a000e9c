// tri_inverse.cuh -- T = (I + A)^-1 for a 64 x 64 strictly lower triangular fp32 matrix A
// held in shared memory, computed by four warps.
//
// Blocked forward substitution on 16 x 16 blocks (the stable order of the plain
// substitution, reorganised as a 2 x 2 block recursion):
//   T_II = (I + A_II)^-1                                    substitution by rows, fp32
//   T_10 = -T_11 A_10 T_00,   T_32 = -T_33 A_32 T_22        (the two 32 x 32 diagonal blocks)
//   X    = A_[2:4,0:2] T_[0:2,0:2],  T_[2:4,0:2] = -T_[2:4,2:4] X   (the lower-left 32 x 32)
// The diagonal blocks are solved row-per-lane in registers; every off-diagonal block
// product runs on warp-level tensor-core MMAs (m16n8k8, TF32 operands rounded to nearest,
// fp32 accumulation), so the shared-memory traffic is a few fragment loads per product.
// T is rounded to bf16 by its consumers, so TF32's 2^-11 operand rounding stays below
// the final precision.
//
// A and T may be the same array (in place): every block of A is read before the block of
// T that takes its place is written, and within a phase no warp writes a block another
// warp reads (diagonal blocks: each warp its own; T_10 and T_32 replace A_10 and A_32
// after their own warp has read them; the lower-left 32 x 32 reads A_2x, A_3x in one
// phase and writes T_2x, T_3x in the next).
#pragma once
#include <stdint.h>

namespace gdr {
namespace tri {

constexpr int LD = 68;   // fp32 row stride of A and T (fragment loads are bank-conflict free)
constexpr int XLD = 20;  // row stride of a warp's 16 x 16 scratch block

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// D (16 x 8) += A (16 x 8, row-major) * B (8 x 8); fragments per the m16n8k8 TF32 layout.
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// acc (16 x 16, two n-halves of C fragments) += Am[r0:r0+16, k0:k0+K] * Bm[k0':k0'+K, c0:c0+16]
template <int K>
__device__ __forceinline__ void block_mma(float (&acc)[2][4], const float *Am, int lda, int r0, int ka,
                                          const float *Bm, int ldb, int kb, int c0, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int ks = 0; ks < K / 8; ++ks) {
        uint32_t a[4];
        const float *ap = Am + (r0 + g) * lda + ka + ks * 8 + t;
        a[0] = to_tf32(ap[0]);
        a[1] = to_tf32(ap[8 * lda]);
        a[2] = to_tf32(ap[4]);
        a[3] = to_tf32(ap[8 * lda + 4]);
#pragma unroll
        for (int nh = 0; nh < 2; ++nh) {
            uint32_t b[2];
            const float *bp = Bm + (kb + ks * 8 + t) * ldb + c0 + nh * 8 + g;
            b[0] = to_tf32(bp[0]);
            b[1] = to_tf32(bp[4 * ldb]);
            mma_tf32(acc[nh], a, b);
        }
    }
}

// store a C-fragment 16 x 16 block (optionally negated) at Dm[r0.., c0..]
__device__ __forceinline__ void block_store(float *Dm, int ldd, int r0, int c0, const float (&acc)[2][4],
                                            float sign, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
        float *p = Dm + (r0 + g) * ldd + c0 + nh * 8 + 2 * t;
        p[0] = sign * acc[nh][0];
        p[1] = sign * acc[nh][1];
        p[8 * ldd] = sign * acc[nh][2];
        p[8 * ldd + 1] = sign * acc[nh][3];
    }
}

// T_IJ = -T_II (A[I rows, J..I-1 blocks] T[J..I-1 blocks, J cols]) by one warp; the final
// block also goes to out.pair(row, col, T[row][col], T[row][col+1]) (col even).
template <int NK, class Out>
__device__ __forceinline__ void off_block(const float *A, float *T, float *X, int I, int J, int lane,
                                          Out &out) {
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    block_mma<16 * NK>(acc, A, LD, 16 * I, 16 * J, T, LD, 16 * J, 16 * J, lane);
    block_store(X, XLD, 0, 0, acc, 1.f, lane);
    __syncwarp();
    float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    block_mma<16>(acc2, T, LD, 16 * I, 16 * I, X, XLD, 0, 0, lane);
    block_store(T, LD, 16 * I, 16 * J, acc2, -1.f, lane);
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
        const int col = 16 * J + nh * 8 + 2 * t;
        out.pair(16 * I + g, col, -acc2[nh][0], -acc2[nh][1]);
        out.pair(16 * I + g + 8, col, -acc2[nh][2], -acc2[nh][3]);
    }
}

// Output hook that discards the copy (callers that only need the fp32 T).
struct NoOut {
    __device__ __forceinline__ void chunk(int, int, const float (&)[8]) {}
    __device__ __forceinline__ void pair(int, int, float, float) {}
};

// Called by four whole warps (warp = 0..3 within the group, lane = 0..31).  A, T: fp32
// [64][LD]; only the strictly lower triangle of A is read.  X: 4 x 16 x XLD fp32 scratch.
// sync() must be a barrier over exactly the four calling warps.  On return T holds the
// full lower triangle (unit diagonal) and zeros above the diagonal of each diagonal
// block; the strictly upper off-diagonal blocks of T are not written.  Every final value
// is also handed to `out`: out.chunk(row, c8, v[8]) for columns 8 c8 .. 8 c8 + 7 of the
// diagonal blocks (zeros above the diagonal included) and out.pair for the off-diagonal
// blocks.
template <class Sync, class Out>
__device__ __forceinline__ void inverse64(const float *A, float *T, float *X, int warp, int lane,
                                          Sync sync, Out out) {
    {
        // diagonal block T_ww: lane (i = lane & 15, h = lane >> 4) owns row i, columns
        // 8h..8h+7, and holds row i of A_ww in registers.  Row m of T is final after step
        // m - 1; step m broadcasts it by shuffles and updates the rows below it:
        //   T[i][:] -= A[i][m] T[m][:]   for i > m
        const int o = warp * 16, i = lane & 15, h = lane >> 4;
        float arow[16], tr[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 x = *reinterpret_cast<const float4 *>(A + (o + i) * LD + o + 4 * q);
            arow[4 * q] = x.x; arow[4 * q + 1] = x.y; arow[4 * q + 2] = x.z; arow[4 * q + 3] = x.w;
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) tr[c] = (8 * h + c == i) ? 1.f : 0.f;
#pragma unroll
        for (int m = 0; m < 15; ++m) {
            const float a = (i > m) ? arow[m] : 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float tm = __shfl_sync(0xffffffffu, tr[c], m + 16 * h);
                tr[c] = fmaf(-a, tm, tr[c]);
            }
        }
        float4 *dst = reinterpret_cast<float4 *>(T + (o + i) * LD + o + 8 * h);
        dst[0] = make_float4(tr[0], tr[1], tr[2], tr[3]);
        dst[1] = make_float4(tr[4], tr[5], tr[6], tr[7]);
        out.chunk(o + i, (o >> 3) + h, tr);
    }
    sync();
    if (warp < 2) {
        float *Xw = X + warp * 16 * XLD;
        off_block<1>(A, T, Xw, 2 * warp + 1, 2 * warp, lane, out);   // T10, T32
    }
    sync();
    // lower-left 32 x 32 block, one 16 x 16 block (I, J) per warp, I in {2, 3}, J in {0, 1}
    const int I = 2 + (warp >> 1), J = warp & 1;
    float *Xb = X + warp * 16 * XLD;   // X_IJ
    {
        // X_IJ = sum_{K=J}^{1} A_IK T_KJ  (T_01 = 0)
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        if (J == 0) block_mma<32>(acc, A, LD, 16 * I, 0, T, LD, 0, 0, lane);
        else block_mma<16>(acc, A, LD, 16 * I, 16, T, LD, 16, 16, lane);
        block_store(Xb, XLD, 0, 0, acc, 1.f, lane);
    }
    sync();
    {
        // T_IJ = -sum_{K=2}^{I} T_IK X_KJ
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        block_mma<16>(acc, T, LD, 16 * I, 16 * I, X + ((I - 2) * 2 + J) * 16 * XLD, XLD, 0, 0, lane);
        if (I == 3) block_mma<16>(acc, T, LD, 48, 32, X + J * 16 * XLD, XLD, 0, 0, lane);
        block_store(T, LD, 16 * I, 16 * J, acc, -1.f, lane);
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int nh = 0; nh < 2; ++nh) {
            const int col = 16 * J + nh * 8 + 2 * t;
            out.pair(16 * I + g, col, -acc[nh][0], -acc[nh][1]);
            out.pair(16 * I + g + 8, col, -acc[nh][2], -acc[nh][3]);
        }
    }
    sync();
}

}  // namespace tri
}  // namespace gdr
