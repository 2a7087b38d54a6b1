// gdr_chunk_fwd_noalloc: the chunked forward for callers that cannot
// allocate device memory.
//
// The tensor-core forward needs device scratch for what its UT-transform
// stage hands to its state scan (see gdr_chunk_fwd_workspace_size).  The
// normal entry point asks the caller for it.  Some callers cannot provide it:
// real-time or serving loops that forbid allocator calls on their hot path,
// code that keeps allocator calls out of a region it records as a CUDA graph,
// and hosts whose device memory is owned by another runtime or a custom pool
// that the caller cannot reach.  This entry point
// instead uses one fixed scratch array that the library itself holds as a
// file-scope __device__ variable: it calls no cudaMalloc, cudaFree or any
// allocating routine.
//
// Costs and limits:
//   - every GPU on which the library's module is loaded holds the array
//     (GDR_NOALLOC_SCRATCH_BYTES) until the process exits;
//   - problems whose workspace (gdr_chunk_fwd_workspace_size) exceeds it are
//     rejected with GDR_ERR_UNSUPPORTED before anything is launched;
//   - all calls share the one array and it keeps the last call's contents.
//     The kernels overwrite every scratch entry they read, so nothing needs
//     clearing, but two calls that overlap on the GPU (different streams
//     without ordering between them, or several host threads) race on it
//     and produce undefined results: order such calls;
//   - the device address of the array is looked up (cudaGetSymbolAddress)
//     on the first call made with each device current, and cached; make
//     that first call before any stream capture starts.
#include <mutex>

#include "gdr.h"
#include "gdr_internal.cuh"

#define GDR_API extern "C" __attribute__((visibility("default")))

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[GDR_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once per device).
cudaError_t scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        if (!p) return cudaErrorInvalidSymbol;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

GDR_API int gdr_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const float *g, const float *beta,
                                  const float *S0, void *O, float *S_T,
                                  int B, int H, int T, int dk, int dv, int C, int gate_mode, int dtype,
                                  void *stream)
{
    const size_t need = gdr_chunk_fwd_workspace_size(B, H, T, dk, dv, C, gate_mode, dtype);
    if (need > (size_t)GDR_NOALLOC_SCRATCH_BYTES) return GDR_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    if (need > 0) {
        // the set-up failed (no current device, or the module could not be
        // loaded on it): nothing was launched
        if (scratch_address(&scratch) != cudaSuccess) return GDR_ERR_CUDA;
    }
    return gdr_chunk_fwd(q, k, v, g, beta, S0, O, S_T, B, H, T, dk, dv, C, gate_mode, dtype, scratch,
                         need > 0 ? (size_t)GDR_NOALLOC_SCRATCH_BYTES : 0, stream);
}
