// bounds.cuh -- in-kernel bounds checks of the debug build (compiled with -DGDR_DEBUG).
//
// A check names a site (a small integer, see the table of sites below) and a condition that
// an index or a range stays inside the extent the call's arguments imply.  In the debug
// build a failed check records the first failing site of its translation unit in a device
// word and the caller skips the access; nothing traps.  gdr_last_device_error() reports a
// recorded site as GDR_ERR_BOUNDS and gdr_debug_bounds_site() returns it.  In the release
// build every check is the constant true and the code is unchanged.
//
// Sites:  1xx chunk_tc_kernel (forward, mixer, checkpoints, reverse), 2xx decode kernels,
//         3xx bwd_tc_kernel, 4xx backward CUDA-core kernels, 5xx split chaining kernels,
//         6xx chunk_simt_kernel, 7xx the two-phase forward's phase one (wy_prep.cu),
//         8xx its state pass (state_pass.cu).
#pragma once

#ifdef GDR_DEBUG
namespace gdr {
namespace dbg {
static __device__ int g_bounds_site = 0;
__device__ __forceinline__ bool in_bounds(bool ok, int site) {
    if (!ok) atomicCAS(&g_bounds_site, 0, site);
    return ok;
}
}  // namespace dbg
}  // namespace gdr
#define GDR_IN_BOUNDS(ok, site) (::gdr::dbg::in_bounds((ok), (site)))
// Host reader of this translation unit's site word: returns the site (0: none) and clears it.
#define GDR_BOUNDS_READER(fn)                                                                \
    int fn() {                                                                               \
        int site = 0;                                                                        \
        if (cudaMemcpyFromSymbol(&site, ::gdr::dbg::g_bounds_site, sizeof(int)) != cudaSuccess) \
            return -1;                                                                       \
        const int zero = 0;                                                                  \
        cudaMemcpyToSymbol(::gdr::dbg::g_bounds_site, &zero, sizeof(int));                   \
        return site;                                                                         \
    }
#else
#define GDR_IN_BOUNDS(ok, site) (true)
#define GDR_BOUNDS_READER(fn) \
    int fn() { return 0; }
#endif
