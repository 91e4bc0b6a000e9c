// gdr_api.cu -- the C ABI of libgdr: host-side validation and dispatch.
//
// Validation happens before anything is enqueued, so a rejected call launches
// nothing.  Dispatch picks one device kernel per call; there is no host or
// library fallback for any step of the computation.
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "bwd_tc.cuh"
#include "chunk_tc.cuh"
#include "two_phase.cuh"

using namespace gdr;

namespace {

bool dim_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool chunk_ok(int c) { return c == 16 || c == 32 || c == 64; }
bool aligned16(const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

gdr_status_t check_common(int mode, int dtype, int n0, int H, int dk, int dv) {
    if (mode < GDR_MODE_GDN2 || mode > GDR_MODE_WONLY) return GDR_ERR_MODE;
    if (dtype != GDR_F32 && dtype != GDR_BF16) return GDR_ERR_DTYPE;
    if (n0 < 0 || H < 0 || !dim_ok(dk) || !dim_ok(dv)) return GDR_ERR_DIM;
    return GDR_OK;
}

gdr_status_t check_chunk(const void *q, const void *k, const void *v, const float *g_log,
                         const void *b, const void *w, const float *S0, const void *o,
                         const float *S_T, int B, int H, int T, int dk, int dv, int chunk,
                         int mode, int dtype) {
    gdr_status_t st = check_common(mode, dtype, B, H, dk, dv);
    if (st != GDR_OK) return st;
    if (T < 0 || !chunk_ok(chunk)) return GDR_ERR_DIM;
    if ((int64_t)B * H > INT32_MAX / 64) return GDR_ERR_DIM;
    if ((int64_t)B * H * T > 0) {
        if (!q || !k || !v || !g_log || !b || !o) return GDR_ERR_NULL;
        if (mode_uses_w(mode) && !w) return GDR_ERR_NULL;
    }
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g_log) || !aligned16(b) ||
        !aligned16(w) || !aligned16(S0) || !aligned16(o) || !aligned16(S_T))
        return GDR_ERR_ALIGN;
    return GDR_OK;
}

// Test hook (gdr_test_set_first_wait_limit): 0, the default, leaves every wait at its
// normal bound.
unsigned g_first_wait_limit = 0;

ChunkArgs make_args(const void *q, const void *k, const void *v, const float *g_log, const void *b,
                    const void *w, const float *S0, void *o, float *S_T, int B, int H, int T,
                    int dk, int dv, int chunk, int mode, int dtype) {
    ChunkArgs a{q, k, v, b, mode_uses_w(mode) ? w : nullptr, g_log, S0, o, S_T,
                B, H, T, dk, dv, chunk, mode, dtype,
                1, T, 0, nullptr, nullptr, nullptr,
                0, 1, nullptr, nullptr, 1.f, 0.f, nullptr, 0, nullptr};
    a.first_wait_limit = g_first_wait_limit;
    return a;
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return 148;
    }
    return n;
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
        if (mode_uses_w(mode) && !w) return GDR_ERR_NULL;
    }
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g_log) || !aligned16(b) ||
        !aligned16(w) || !aligned16(S0) || !aligned16(o) || !aligned16(S_T))
        return GDR_ERR_ALIGN;
    ChunkArgs a = make_args(q, k, v, g_log, b, w, S0, o, S_T, B, H, T, dk, dv, chunk, mode, dtype);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((int64_t)B * H == 0) return GDR_OK;
    if (T == 0) return launch_state_copy(a, s);
    if (chunk_tc_supported(a)) return launch_chunk_tc(a, s);
    return launch_chunk_simt(a, s);
}

// ---- sequence split -------------------------------------------------------------------
namespace {

// segment length (in chunks) and effective segment count for a requested count
void split_geometry(int nchunks, int nseg, int *seg_chunks, int *nseg_eff) {
    if (nseg > nchunks) nseg = nchunks;
    if (nseg < 1) nseg = 1;
    *seg_chunks = (nchunks + nseg - 1) / nseg;
    *nseg_eff = (nchunks + *seg_chunks - 1) / *seg_chunks;
}

}  // namespace

int gdr::split_effective_segments(int T, int chunk, int nseg) {
    if (T <= 0 || chunk <= 0) return 1;
    int sc = 1, ne = 1;
    split_geometry((T + chunk - 1) / chunk, nseg, &sc, &ne);
    return ne;
}

namespace {

// Time models in steps of the fused kernel's chunk period (one chunk of one sequence-head
// on one SM, ~10 K cycles, ~5.7 us on B200).  The fused split: its first pass (state only,
// as costly per chunk as a whole chunk, measured) in waves of units * (2 nseg - 3) CTAs, its
// second in waves of units * nseg CTAs.
double fused_split_time(int units, int sms, int nchunks, int *nseg_out) {
    double best = (double)((units + sms - 1) / sms) * nchunks;
    int best_n = 1;
    for (int n = 2; n <= 64 && n <= nchunks; ++n) {
        int sc, ne;
        split_geometry(nchunks, n, &sc, &ne);
        if (ne < 2) continue;
        const int r1 = 2 * ne - 3 > 1 ? 2 * ne - 3 : 1;
        const double t = (double)((units * r1 + sms - 1) / sms) * sc + (double)((units * ne + sms - 1) / sms) * sc;
        if (t < 0.8 * best) {   // split only for a clear gain
            best = t;
            best_n = ne;
        }
    }
    *nseg_out = best_n;
    return best;
}

// The two-phase forward, in the same unit (constants measured on B200 with per-phase clock
// stamps): phase one over every chunk, two persistent CTAs per SM, a wave of two chunks per
// SM taking kPrep (its latency-bound per-chunk path, ~21 K cycles), or bound by its traffic (the inputs, at most 112 KB per chunk, and
// the 73 KB record it writes); then the state pass, whole or split like the fused kernel,
// each CTA kState per chunk plus kFix to start, or bound by the records it reads and the
// output it writes.  kBytes: HBM bytes moved in one fused chunk period (~6 TB/s x 5 us).
constexpr double kPrep = 2.1, kState = 0.37, kFix = 0.5, kBytes = 34e6;
constexpr double kIn = 112.0 * 1024, kRec = 74752, kOut = 16.0 * 1024;
double waves(long long ctas, int sms) { return (double)((ctas + sms - 1) / sms); }
double two_phase_time(int units, int sms, int nchunks, int *nseg_out) {
    const long long un = (long long)units * nchunks;
    const double prep = fmax(kPrep * (double)((un + 2 * sms - 1) / (2 * sms)), un * (kIn + kRec) / kBytes);
    const double out_pass = un * (kRec + kOut) / kBytes;   // the output pass's traffic
    double best = prep + fmax(waves(units, sms) * (kState * nchunks + kFix), out_pass);
    int best_n = 1;
    for (int n = 2; n <= 64 && n <= nchunks; ++n) {
        int sc, ne;
        split_geometry(nchunks, n, &sc, &ne);
        if (ne < 2) continue;
        const int r1 = 2 * ne - 3 > 1 ? 2 * ne - 3 : 1;
        const double pass1 = fmax(waves((long long)units * r1, sms) * (kState * sc + kFix),
                                  (double)units * r1 * sc * kRec / kBytes);
        const double pass0 = fmax(waves((long long)units * ne, sms) * (kState * sc + kFix), out_pass);
        const double t = prep + pass1 + pass0;
        if (t < best) {
            best = t;
            best_n = ne;
        }
    }
    *nseg_out = best_n;
    return best;
}

bool two_phase_shape(int B, int H, int T, int dk, int dv, int chunk, int dtype) {
    return B > 0 && H > 0 && T > 0 && dtype == GDR_BF16 && dk == 128 && dv == 128 && chunk == 64;
}

}  // namespace

extern "C" int gdr_chunk_fwd_split_segments(int B, int H, int T, int dk, int dv, int chunk,
                                            gdr_dtype_t dtype) {
    if (!two_phase_shape(B, H, T, dk, dv, chunk, dtype)) return 1;
    int n = 1;
    fused_split_time(B * H, sm_count(), (T + chunk - 1) / chunk, &n);
    return n;
}

extern "C" int gdr_chunk_fwd_two_phase_segments(int B, int H, int T, int dk, int dv, int chunk,
                                                gdr_dtype_t dtype) {
    if (!two_phase_shape(B, H, T, dk, dv, chunk, dtype)) return 0;
    if ((long long)B * H * ((T + chunk - 1) / chunk) > INT32_MAX) return 0;
    const int units = B * H, sms = sm_count(), nchunks = (T + chunk - 1) / chunk;
    int nf = 1, nt = 1;
    const double fused = fused_split_time(units, sms, nchunks, &nf);
    const double two = two_phase_time(units, sms, nchunks, &nt);
    return two < 0.97 * fused ? nt : 0;   // where the model sees a gain beyond its rounding
}

extern "C" unsigned long long gdr_chunk_fwd_split_workspace(int B, int H, int dk, int dv, int nseg) {
    if (B < 0 || H < 0 || !dim_ok(dk) || !dim_ok(dv) || nseg < 1) return 0;
    return 3ull * (unsigned long long)B * H * nseg * dk * dv * sizeof(float);
}

extern "C" gdr_status_t gdr_chunk_fwd_split(const void *q, const void *k, const void *v,
                                            const float *g_log, const void *b, const void *w,
                                            const float *S0, void *o, float *S_T, int B, int H,
                                            int T, int dk, int dv, int chunk, gdr_mode_t mode,
                                            gdr_dtype_t dtype, int nseg, void *workspace,
                                            unsigned long long workspace_bytes, void *stream) {
    gdr_status_t st = check_chunk(q, k, v, g_log, b, w, S0, o, S_T, B, H, T, dk, dv, chunk, mode, dtype);
    if (st != GDR_OK) return st;
    if (nseg < 1) return GDR_ERR_DIM;
    ChunkArgs a = make_args(q, k, v, g_log, b, w, S0, o, S_T, B, H, T, dk, dv, chunk, mode, dtype);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int seg_chunks = 1, nseg_eff = 1;
    if (T > 0) split_geometry((T + chunk - 1) / chunk, nseg, &seg_chunks, &nseg_eff);
    if (nseg_eff > 1 && !chunk_tc_supported(a)) return GDR_ERR_DIM;
    if (nseg_eff <= 1 || (int64_t)B * H == 0)
        return gdr_chunk_fwd(q, k, v, g_log, b, w, S0, o, S_T, B, H, T, dk, dv, chunk, mode, dtype, stream);
    const unsigned long long need = gdr_chunk_fwd_split_workspace(B, H, dk, dv, nseg_eff);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return GDR_ERR_WORKSPACE;
    if ((int64_t)B * H * (2 * nseg_eff) > INT32_MAX) return GDR_ERR_DIM;
    const size_t per = (size_t)B * H * nseg_eff * dk * dv;
    float *ws = static_cast<float *>(workspace);
    a.nseg = nseg_eff;
    a.seg_len = seg_chunks * chunk;
    a.ws_send = ws;
    a.ws_m = ws + per;
    a.ws_sstart = ws + 2 * per;
    a.pass = 1;
    if ((st = launch_chunk_tc(a, s)) != GDR_OK) return st;
    if ((st = launch_split_combine(a, s)) != GDR_OK) return st;
    a.pass = 0;
    return launch_chunk_tc(a, s);
}

extern "C" unsigned long long gdr_chunk_fwd_two_phase_workspace(int B, int H, int T, int dk, int dv, int chunk,
                                                                int nseg) {
    if (B < 0 || H < 0 || T < 0 || dk != 128 || dv != 128 || chunk != 64 || nseg < 1) return 0;
    int sc = 1, ne = 1;
    if (T > 0) split_geometry((T + chunk - 1) / chunk, nseg, &sc, &ne);
    return tp::records_bytes(B, H, T) + tp::list_bytes(B, H, T) +
           (ne > 1 ? gdr_chunk_fwd_split_workspace(B, H, dk, dv, ne) : 0ull);
}

extern "C" gdr_status_t gdr_chunk_fwd_two_phase(const void *q, const void *k, const void *v,
                                                const float *g_log, const void *b, const void *w,
                                                const float *S0, void *o, float *S_T, int B, int H,
                                                int T, int dk, int dv, int chunk, gdr_mode_t mode,
                                                gdr_dtype_t dtype, int nseg, void *workspace,
                                                unsigned long long workspace_bytes, void *stream) {
    gdr_status_t st = check_chunk(q, k, v, g_log, b, w, S0, o, S_T, B, H, T, dk, dv, chunk, mode, dtype);
    if (st != GDR_OK) return st;
    if (nseg < 1) return GDR_ERR_DIM;
    ChunkArgs a = make_args(q, k, v, g_log, b, w, S0, o, S_T, B, H, T, dk, dv, chunk, mode, dtype);
    if (!chunk_tc_supported(a)) return GDR_ERR_DIM;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((int64_t)B * H == 0) return GDR_OK;
    if (T == 0) return launch_state_copy(a, s);
    const int nchunks = (T + chunk - 1) / chunk;
    if ((int64_t)B * H * nchunks > INT32_MAX || (int64_t)B * H * 2 * nseg > INT32_MAX) return GDR_ERR_DIM;
    int seg_chunks = 1, nseg_eff = 1;
    split_geometry(nchunks, nseg, &seg_chunks, &nseg_eff);
    const unsigned long long need = gdr_chunk_fwd_two_phase_workspace(B, H, T, dk, dv, chunk, nseg);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return GDR_ERR_WORKSPACE;
    unsigned char *records = static_cast<unsigned char *>(workspace);
    int *list = reinterpret_cast<int *>(records + tp::records_bytes(B, H, T));
    float *split_ws = reinterpret_cast<float *>(records + tp::records_bytes(B, H, T) + tp::list_bytes(B, H, T));
    if (cudaMemsetAsync(list, 0, sizeof(int), s) != cudaSuccess) return GDR_ERR_CUDA;
    if ((st = tp::launch_wy_prep(a, records, list, s)) != GDR_OK) return st;
    if (nseg_eff <= 1) return tp::launch_state_pass(a, records, s);
    const size_t per = (size_t)B * H * nseg_eff * dk * dv;
    a.nseg = nseg_eff;
    a.seg_len = seg_chunks * chunk;
    a.ws_send = split_ws;
    a.ws_m = split_ws + per;
    a.ws_sstart = split_ws + 2 * per;
    a.pass = 1;
    if ((st = tp::launch_state_pass(a, records, s)) != GDR_OK) return st;
    if ((st = launch_split_combine(a, s)) != GDR_OK) return st;
    a.pass = 0;
    return tp::launch_state_pass(a, records, s);
}

extern "C" gdr_status_t gdr_chunk_fwd_segment_maps(const void *q, const void *k, const void *v,
                                                   const float *g_log, const void *b, const void *w,
                                                   const float *S0, float *S_local, float *M, int B, int H,
                                                   int T, int dk, int dv, int chunk, gdr_mode_t mode,
                                                   gdr_dtype_t dtype, void *stream) {
    gdr_status_t st = check_chunk(q, k, v, g_log, b, w, S0, S_local, S_local, B, H, T, dk, dv, chunk, mode, dtype);
    if (st != GDR_OK) return st;
    if (!S_local) return GDR_ERR_NULL;
    if (!aligned16(M)) return GDR_ERR_ALIGN;
    if (T < 1) return GDR_ERR_DIM;
    ChunkArgs a = make_args(q, k, v, g_log, b, w, S0, nullptr, nullptr, B, H, T, dk, dv, chunk, mode, dtype);
    if (!chunk_tc_supported(a)) return GDR_ERR_DIM;
    if ((int64_t)B * H * 2 > INT32_MAX) return GDR_ERR_DIM;
    if ((int64_t)B * H == 0) return GDR_OK;
    a.pass = 1;   // no output
    a.seg_maps = 1;
    a.want_m = M != nullptr;
    a.seg_len = T;
    a.ws_send = S_local;
    a.ws_m = M;
    return launch_chunk_tc(a, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" gdr_status_t gdr_chain_segment_states(const float *M_all, const float *S_local_all, const float *S0,
                                                 float *S_start, int R, int r, int B, int H, int dk, int dv,
                                                 void *stream) {
    if (B < 0 || H < 0 || R < 1 || r < 0 || r >= R || dk != 128 || dv != 128) return GDR_ERR_DIM;
    if ((int64_t)B * H * (dv / 16) > INT32_MAX) return GDR_ERR_DIM;
    if (!S_start || (r >= 1 && !S_local_all) || (r >= 2 && !M_all)) return GDR_ERR_NULL;
    if (!aligned16(M_all) || !aligned16(S_local_all) || !aligned16(S0) || !aligned16(S_start)) return GDR_ERR_ALIGN;
    if ((int64_t)B * H == 0) return GDR_OK;
    return launch_segment_chain(M_all, S_local_all, S0, S_start, R, r, B * H, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" gdr_status_t gdr_mixer_fwd(const void *q, const void *k, const void *v, const float *xg,
                                      const void *xb, const void *xw, const void *z,
                                      const float *norm_weight, const float *S0, void *y,
                                      float *S_T, int B, int H, int T, int dk, int dv, int chunk,
                                      gdr_mode_t mode, gdr_dtype_t dtype, gdr_layout_t layout,
                                      float b_range, float eps, void *stream) {
    gdr_status_t st = check_chunk(q, k, v, xg, xb, xw, S0, y, S_T, B, H, T, dk, dv, chunk, mode, dtype);
    if (st != GDR_OK) return st;
    if (dtype != GDR_BF16) return GDR_ERR_DTYPE;
    if (dk != 128 || dv != 128 || chunk != 64) return GDR_ERR_DIM;
    if (layout != GDR_LAYOUT_BHTD && layout != GDR_LAYOUT_BTHD) return GDR_ERR_VALUE;
    if (!(eps > 0.f) || !(eps < INFINITY) || !(b_range >= 0.f) || !(b_range < INFINITY)) return GDR_ERR_VALUE;
    if ((int64_t)B * H * T > 0 && (!z || !norm_weight)) return GDR_ERR_NULL;
    if (!aligned16(z) || !aligned16(norm_weight)) return GDR_ERR_ALIGN;
    ChunkArgs a = make_args(q, k, v, xg, xb, xw, S0, y, S_T, B, H, T, dk, dv, chunk, mode, dtype);
    a.mixer = 1;
    a.tstride = layout == GDR_LAYOUT_BTHD ? H : 1;
    a.z = z;
    a.nw = norm_weight;
    a.b_range = b_range;
    a.eps = eps;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((int64_t)B * H == 0) return GDR_OK;
    if (T == 0) return launch_state_copy(a, s);
    return launch_chunk_tc(a, s);
}

extern "C" unsigned long long gdr_chunk_bwd_workspace(int B, int H, int T, int dk, int dv) {
    if (B < 0 || H < 0 || T < 0 || !dim_ok(dk) || !dim_ok(dv)) return 0;
    return bwd_workspace_bytes(B, H, T, dk, dv);
}

extern "C" gdr_status_t gdr_chunk_bwd(const void *q, const void *k, const void *v, const float *g_log,
                                      const void *b, const void *w, const float *S0, const void *dO,
                                      const float *dS_T, void *dq, void *dk_, void *dv_, float *dg,
                                      void *db, void *dw, float *dS0, int B, int H, int T, int dk,
                                      int dv, gdr_mode_t mode, gdr_dtype_t dtype, void *workspace,
                                      unsigned long long workspace_bytes, void *stream) {
    gdr_status_t st = check_common(mode, dtype, B, H, dk, dv);
    if (st != GDR_OK) return st;
    if (T < 0 || (int64_t)B * H > INT32_MAX / 1024) return GDR_ERR_DIM;
    const bool work = (int64_t)B * H * T > 0;
    if (work) {
        if (!q || !k || !v || !g_log || !b || !dO || !dq || !dk_ || !dv_ || !dg || !db) return GDR_ERR_NULL;
        if (mode_uses_w(mode) && (!w || !dw)) return GDR_ERR_NULL;
    }
    const void *ptrs[] = {q, k, v, g_log, b, w, S0, dO, dS_T, dq, dk_, dv_, dg, db, dw, dS0, workspace};
    for (const void *p : ptrs)
        if (!aligned16(p)) return GDR_ERR_ALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((int64_t)B * H == 0) return GDR_OK;
    if (T == 0) {   // dS0 = dS_T (or zeros); nothing else to write
        ChunkArgs a = make_args(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, dS_T, nullptr, dS0,
                                B, H, 0, dk, dv, 32, mode, dtype);
        return launch_state_copy(a, s);
    }
    const unsigned long long need = bwd_workspace_bytes(B, H, T, dk, dv);
    if (!workspace || workspace_bytes < need) return GDR_ERR_WORKSPACE;
    const size_t per = bwd_states_bytes(B, H, T, dk, dv) / 2 / sizeof(float);
    BwdArgs a{q, k, v, b, mode_uses_w(mode) ? w : nullptr, g_log, S0, dO, dS_T,
              dq, dk_, dv_, db, mode_uses_w(mode) ? dw : nullptr, dg, dS0,
              B, H, T, dk, dv, (int)mode, (int)dtype,
              static_cast<float *>(workspace), static_cast<float *>(workspace) + per, 0, nullptr};
    a.first_wait_limit = g_first_wait_limit;
    return launch_bwd(a, s);
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
    if (mode_uses_w(mode) && !w) return GDR_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g_log) || !aligned16(b) ||
        !aligned16(w) || !aligned16(S) || !aligned16(o))
        return GDR_ERR_ALIGN;
    DecodeArgs a{q, k, v, b, mode_uses_w(mode) ? w : nullptr, g_log, S, o,
                 N, H, dk, dv, (int)mode, (int)dtype};
    a.first_wait_limit = g_first_wait_limit;
    return launch_decode(a, reinterpret_cast<cudaStream_t>(stream));
}

namespace {
int g_last_bounds_site = 0;   // debug build: the site gdr_last_device_error last reported
}  // namespace

extern "C" int gdr_debug_build(void) {
#ifdef GDR_DEBUG
    return 1;
#else
    return 0;
#endif
}

extern "C" int gdr_debug_bounds_site(void) { return g_last_bounds_site; }

extern "C" gdr_status_t gdr_last_device_error(void *stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return GDR_ERR_CUDA;
    // debug build: a failed bounds check comes first (it can also starve a bounded wait)
    const int sites[] = {chunk_tc_bounds_site(), bwd_tc_bounds_site(), bwd_bounds_site(),
                         simt_bounds_site(),     decode_bounds_site(), split_bounds_site(),
                         wy_prep_bounds_site(),  state_pass_bounds_site()};
    int site = 0;
    for (int x : sites) {
        if (x < 0) return GDR_ERR_CUDA;
        if (x && !site) site = x;
    }
    if (site) {
        g_last_bounds_site = site;
        int ignore = 0;   // clear the wait error words too
        chunk_tc_read_and_clear_error(&ignore);
        decode_read_and_clear_error(&ignore);
        bwd_tc_read_and_clear_error(&ignore);
        tp::two_phase_read_and_clear_error(&ignore);
        return GDR_ERR_BOUNDS;
    }
    int err = 0, derr = 0, berr = 0, terr = 0;
    if (chunk_tc_read_and_clear_error(&err) != cudaSuccess) return GDR_ERR_CUDA;
    if (decode_read_and_clear_error(&derr) != cudaSuccess) return GDR_ERR_CUDA;
    if (bwd_tc_read_and_clear_error(&berr) != cudaSuccess) return GDR_ERR_CUDA;
    if (tp::two_phase_read_and_clear_error(&terr) != cudaSuccess) return GDR_ERR_CUDA;
    return (err || derr || berr || terr) ? GDR_ERR_TIMEOUT : GDR_OK;
}

extern "C" void gdr_test_set_first_wait_limit(unsigned polls) { g_first_wait_limit = polls; }

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
        case GDR_ERR_WORKSPACE: return "GDR_ERR_WORKSPACE: workspace missing, misaligned or too small";
        case GDR_ERR_VALUE: return "GDR_ERR_VALUE: scalar argument out of range";
        case GDR_ERR_BOUNDS: return "GDR_ERR_BOUNDS: a bounds check of the debug build failed";
    }
    return "unknown gdr_status_t";
}
