// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdr {

// Arguments of one chunked forward, already validated by the C entry point.
struct ChunkArgs {
    const void *q, *k, *v;
    const float *g, *beta, *S0;
    void *O;
    float *S_T;
    int B, H, T, dk, dv, C;
    bool scalar_gate;
    bool bf16;
    void *workspace;   // device scratch of chunk_tc_workspace_bytes() bytes (tensor-core path)
};

// Arguments of one decode step, already validated.
struct StepArgs {
    const void *q, *k, *v;
    const float *g, *beta;
    float *S;
    void *o;
    int B, H, dk, dv;
    bool scalar_gate;
    bool bf16;
};

// Each launcher enqueues its kernels on `stream`, adds the number of kernels
// it launched to *launches and returns the first launch error.
cudaError_t launch_recurrent_step(const StepArgs &a, cudaStream_t stream, int *launches);
cudaError_t launch_chunk_simt(const ChunkArgs &a, cudaStream_t stream, int *launches);
cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t stream, int *launches);
bool chunk_tc_supports(const ChunkArgs &a);
size_t chunk_tc_workspace_bytes(int B, int H, int T);
// Synchronizes `stream`, then reads and clears the device status word.
cudaError_t read_device_status(cudaStream_t stream, int *status);

// The KDA lower bound on the per-channel log-decay.
constexpr float kGateMin = -5.0f;

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

}  // namespace gdr
