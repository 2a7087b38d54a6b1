// Debug-mode range check of the log-decay gate.
//
// The method takes g = log(alpha) with alpha in (0, 1], so a valid gate is a
// finite value <= 0 ("KDA vs Gated DeltaNet" (brenchcc), section 4: the state
// is multiplied by exp(decay), a decay factor in (0, 1]; values below the KDA
// bound -5 are legal and are clamped by the kernels).  When the environment
// variable GDR_DEBUG is set to anything but "" or "0" when the library first
// looks at it, every entry point that takes g runs this check before its
// kernels: one pass over g on the caller's stream, a synchronisation, and
// GDR_ERR_GATE_RANGE if any element is positive, NaN or infinite.  Without
// GDR_DEBUG nothing of this runs.
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "gdr_internal.cuh"

namespace gdr {

namespace {

__device__ int g_gate_bad;   // set by the check kernel when an element is out of range

__device__ __forceinline__ bool gate_bad(float x)
{
    // false for every finite x <= 0; true for x > 0, +-inf and NaN
    return !(x <= 0.f && x >= -3.402823466e38f);
}

__global__ void gate_range_kernel(const float *__restrict__ g, size_t n)
{
    const size_t n4 = n / 4;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    bool bad = false;
    const float4 *g4 = reinterpret_cast<const float4 *>(g);
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
        const float4 v = __ldg(g4 + i);
        bad |= gate_bad(v.x) | gate_bad(v.y) | gate_bad(v.z) | gate_bad(v.w);
    }
    for (size_t i = 4 * n4 + (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        bad |= gate_bad(__ldg(g + i));
    if (bad) g_gate_bad = 1;
}

}  // namespace

bool debug_checks_enabled()
{
    static bool on = false;
    static std::once_flag once;
    std::call_once(once, [] {
        const char *s = std::getenv("GDR_DEBUG");
        on = s && s[0] != '\0' && std::strcmp(s, "0") != 0;
    });
    return on;
}

cudaError_t check_gate_range(const float *g, size_t n, cudaStream_t stream, bool *bad)
{
    *bad = false;
    if (n == 0) return cudaSuccess;
    const int zero = 0;
    cudaError_t e = cudaMemcpyToSymbolAsync(g_gate_bad, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return e;
    const size_t blocks_needed = (n / 4 + 255) / 256;
    const int grid = (int)(blocks_needed < 1184 ? (blocks_needed > 0 ? blocks_needed : 1) : 1184);
    gate_range_kernel<<<grid, 256, 0, stream>>>(g, n);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    int v = 0;
    e = cudaMemcpyFromSymbolAsync(&v, g_gate_bad, sizeof(int), 0, cudaMemcpyDeviceToHost, stream);
    if (e != cudaSuccess) return e;
    e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    *bad = (v != 0);
    return cudaSuccess;
}

}  // namespace gdr
