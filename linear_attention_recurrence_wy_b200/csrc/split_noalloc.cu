// split_noalloc.cu -- the sequence split with built-in scratch memory, for callers that
// cannot allocate device memory.
//
// Some callers must not allocate: plugins inside frameworks whose memory manager owns
// all device memory, and latency-critical loops where a cudaMalloc (which may
// synchronise the device) is not acceptable.  gdr_chunk_fwd_split needs a workspace
// from its caller; this entry point takes its workspace from a fixed array that lives
// in the library instead.  It calls no cudaMalloc, cudaFree or allocating routine.
#include <mutex>

#include "common.cuh"

namespace gdr {
namespace {

// Built-in scratch: every GPU that loads the library holds it until the process exits.
constexpr unsigned long long kScratchBytes = 24ull << 20;   // 24 MiB
static __device__ __align__(256) unsigned char g_split_scratch[kScratchBytes];

// Device address of g_split_scratch per device.  In host code the name
// g_split_scratch is only a host-side stand-in, never a device address: the address
// is looked up once per device, with that device current.
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {};

gdr_status_t scratch_for_current_device(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDR_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_split_scratch) != cudaSuccess || !p) return GDR_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
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
    void *scratch = nullptr;
    const gdr_status_t st = gdr::scratch_for_current_device(&scratch);
    if (st != GDR_OK) return st;
    // The split needs no zeroed scratch: every workspace byte it reads was written
    // earlier in the same call.  Sizes beyond the built-in array are rejected by the
    // split's own workspace check (GDR_ERR_WORKSPACE) before anything is launched.
    return gdr_chunk_fwd_split(q, k, v, g_log, b, w, S0, o, S_T, B, H, T, dk, dv, chunk, mode,
                               dtype, nseg, scratch, gdr::kScratchBytes, stream);
}
