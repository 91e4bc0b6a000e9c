// split_noalloc.cu -- the sequence split with built-in scratch memory, for callers that
// cannot allocate device memory.
//
// Some callers must not allocate: plugins inside frameworks whose memory manager owns
// all device memory, and latency-critical loops where a cudaMalloc (which may
// synchronise the device) is not acceptable.  gdr_chunk_fwd_split needs a workspace
// from its caller; this entry point takes its workspace from a fixed array that lives
// in the library instead.  It calls no cudaMalloc, cudaFree or allocating routine.
#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace gdr {
namespace {

// Built-in scratch: every GPU that loads the library holds it until the process exits.
constexpr unsigned long long kScratchBytes = 24ull << 20;   // 24 MiB
static __device__ __align__(256) unsigned char g_split_scratch[kScratchBytes];

// In host code the name g_split_scratch is only a host-side stand-in, never a device
// address.  Each CUDA context loads its own copy of the module, so the array's device
// address belongs to a context: it is looked up (cudaGetSymbolAddress, with the context
// current) on every call made outside a stream capture, and remembered per context for
// calls made while a capture is in progress, when no lookup is made.
constexpr int kCacheSlots = 64;
std::mutex g_scratch_mu;
CUcontext g_cache_ctx[kCacheSlots] = {};
void *g_cache_addr[kCacheSlots] = {};
int g_cache_next = 0;

using CtxGetCurrentFn = CUresult (*)(CUcontext *);

CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

gdr_status_t scratch_address(cudaStream_t stream, void **out) {
    CtxGetCurrentFn get_ctx = ctx_get_current_fn();
    if (!get_ctx) return GDR_ERR_CUDA;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) {
        cudaGetLastError();
        return GDR_ERR_CUDA;
    }
    void *p = nullptr;
    if (cs == cudaStreamCaptureStatusNone) {
        // the lookup also makes the runtime's context current if it was not yet
        if (cudaGetSymbolAddress(&p, g_split_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return GDR_ERR_CUDA;
        }
    }
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return GDR_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    int slot = -1;
    for (int i = 0; i < kCacheSlots; ++i)
        if (g_cache_ctx[i] == ctx) slot = i;
    if (cs != cudaStreamCaptureStatusNone) {
        // capturing: no lookup; the address an earlier call in this context found
        if (slot < 0) return GDR_ERR_CUDA;
        *out = g_cache_addr[slot];
        return GDR_OK;
    }
    if (slot < 0) {
        slot = g_cache_next;
        g_cache_next = (g_cache_next + 1) % kCacheSlots;
    }
    g_cache_ctx[slot] = ctx;
    g_cache_addr[slot] = p;
    *out = p;
    return GDR_OK;
}

}  // namespace
}  // namespace gdr

extern "C" gdr_status_t gdr_chunk_fwd_split_noalloc(const void *q, const void *k, const void *v,
                                                    const float *g_log, const void *b,
                                                    const void *w, const float *S0, void *o,
                                                    float *S_T, int B, int H, int T, int dk,
                                                    int dv, int chunk, gdr_mode_t mode,
                                                    gdr_dtype_t dtype, int nseg, void *stream) {
    // Without a workspace the split validates every argument first and either returns
    // that error, or runs the calls that need no workspace (one segment, no sequence-head)
    // unsplit, or answers GDR_ERR_WORKSPACE -- in each case before anything is launched.
    gdr_status_t st = gdr_chunk_fwd_split(q, k, v, g_log, b, w, S0, o, S_T, B, H, T, dk, dv, chunk,
                                          mode, dtype, nseg, nullptr, 0, stream);
    if (st != GDR_ERR_WORKSPACE) return st;
    const int nseg_eff = gdr::split_effective_segments(T, chunk, nseg);
    if (gdr_chunk_fwd_split_workspace(B, H, dk, dv, nseg_eff) > gdr::kScratchBytes) return GDR_ERR_WORKSPACE;
    void *scratch = nullptr;
    st = gdr::scratch_address(reinterpret_cast<cudaStream_t>(stream), &scratch);
    if (st != GDR_OK) return st;
    // The split needs no zeroed scratch: every workspace byte it reads was written
    // earlier in the same call.
    return gdr_chunk_fwd_split(q, k, v, g_log, b, w, S0, o, S_T, B, H, T, dk, dv, chunk, mode,
                               dtype, nseg, scratch, gdr::kScratchBytes, stream);
}
