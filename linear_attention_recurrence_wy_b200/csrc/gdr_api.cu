// gdr_api.cu -- the C ABI of libgdr: host-side validation and dispatch.
//
// Validation happens before anything is enqueued, so a rejected call launches
// nothing.  Dispatch picks one device kernel per call; there is no host or
// library fallback for any step of the computation.
#include <stdint.h>

#include "common.cuh"
#include "chunk_tc.cuh"

using namespace gdr;

namespace {

bool dim_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool chunk_ok(int c) { return c == 16 || c == 32 || c == 64; }
bool aligned16(const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

gdr_status_t check_common(int mode, int dtype, int n0, int H, int dk, int dv) {
    if (mode < GDR_MODE_GDN2 || mode > GDR_MODE_GDN) return GDR_ERR_MODE;
    if (dtype != GDR_F32 && dtype != GDR_BF16) return GDR_ERR_DTYPE;
    if (n0 < 0 || H < 0 || !dim_ok(dk) || !dim_ok(dv)) return GDR_ERR_DIM;
    return GDR_OK;
}

}  // namespace

extern "C" gdr_status_t gdr_chunk_fwd(const void *q, const void *k, const void *v,
                                      const float *g_log, const void *b, const void *w,
                                      const float *S0, void *o, float *S_T, int B, int H, int T,
                                      int dk, int dv, int chunk, gdr_mode_t mode,
                                      gdr_dtype_t dtype, void *stream) {
    gdr_status_t st = check_common(mode, dtype, B, H, dk, dv);
    if (st != GDR_OK) return st;
    if (T < 0 || !chunk_ok(chunk)) return GDR_ERR_DIM;
    if ((int64_t)B * H > INT32_MAX) return GDR_ERR_DIM;
    const bool work = (int64_t)B * H * T > 0;
    if (work) {
        if (!q || !k || !v || !g_log || !b || !o) return GDR_ERR_NULL;
        if (mode == GDR_MODE_GDN2 && !w) return GDR_ERR_NULL;
    }
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g_log) || !aligned16(b) ||
        !aligned16(w) || !aligned16(S0) || !aligned16(o) || !aligned16(S_T))
        return GDR_ERR_ALIGN;
    ChunkArgs a{q, k, v, b, mode == GDR_MODE_GDN2 ? w : nullptr, g_log, S0, o, S_T,
                B, H, T, dk, dv, chunk, (int)mode, (int)dtype};
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((int64_t)B * H == 0) return GDR_OK;
    if (T == 0) return launch_state_copy(a, s);
    if (chunk_tc_supported(a)) return launch_chunk_tc(a, s);
    return launch_chunk_simt(a, s);
}

extern "C" gdr_status_t gdr_decode_step(const void *q, const void *k, const void *v,
                                        const float *g_log, const void *b, const void *w,
                                        float *S, void *o, int N, int H, int dk, int dv,
                                        gdr_mode_t mode, gdr_dtype_t dtype, void *stream) {
    gdr_status_t st = check_common(mode, dtype, N, H, dk, dv);
    if (st != GDR_OK) return st;
    if ((int64_t)N * H > INT32_MAX) return GDR_ERR_DIM;
    if ((int64_t)N * H == 0) return GDR_OK;
    if (!q || !k || !v || !g_log || !b || !S || !o) return GDR_ERR_NULL;
    if (mode == GDR_MODE_GDN2 && !w) return GDR_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g_log) || !aligned16(b) ||
        !aligned16(w) || !aligned16(S) || !aligned16(o))
        return GDR_ERR_ALIGN;
    DecodeArgs a{q, k, v, b, mode == GDR_MODE_GDN2 ? w : nullptr, g_log, S, o,
                 N, H, dk, dv, (int)mode, (int)dtype};
    return launch_decode(a, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" gdr_status_t gdr_last_device_error(void *stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return GDR_ERR_CUDA;
    int err = 0;
    if (chunk_tc_read_and_clear_error(&err) != cudaSuccess) return GDR_ERR_CUDA;
    return err ? GDR_ERR_TIMEOUT : GDR_OK;
}

extern "C" const char *gdr_status_string(gdr_status_t status) {
    switch (status) {
        case GDR_OK: return "GDR_OK";
        case GDR_ERR_NULL: return "GDR_ERR_NULL: a required pointer is NULL";
        case GDR_ERR_DIM: return "GDR_ERR_DIM: unsupported or negative size";
        case GDR_ERR_MODE: return "GDR_ERR_MODE: unknown mode";
        case GDR_ERR_DTYPE: return "GDR_ERR_DTYPE: unknown dtype";
        case GDR_ERR_ALIGN: return "GDR_ERR_ALIGN: pointer not 16-byte aligned";
        case GDR_ERR_CUDA: return "GDR_ERR_CUDA: CUDA launch or runtime error";
        case GDR_ERR_TIMEOUT: return "GDR_ERR_TIMEOUT: a bounded device wait expired";
    }
    return "unknown gdr_status_t";
}
