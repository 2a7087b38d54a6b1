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
    // Input prologue (tensor-core path only): q, k are raw and L2-normalised
    // in-kernel, g holds the bf16 gate pre-activation a (reinterpreted), the
    // log-decay is -exp(A_log[h]) * softplus(a + dt_bias) (bounded below by -5
    // per channel) and beta holds the logits of beta = sigmoid(logit).
    bool prologue = false;
    const float *A_log = nullptr, *dt_bias = nullptr;
    // Gated Delta Rule-2 (tensor-core path only): beta is unused; erase
    // [B, H, T, d_k] and write [B, H, T, d_v] are the per-channel erase and
    // write gates, in the dtype of q, k, v.
    bool gdr2 = false;
    const void *erase = nullptr, *write = nullptr;
    // Gated output (tensor-core path only): O receives
    // y = Sigmoid(ogate) * RMSNorm(o) per head and token, RMSNorm over the d_v
    // channels with weight norm_w [d_v] and epsilon eps; ogate is bf16 [B, H, T, d_v].
    bool gated_out = false;
    const void *ogate = nullptr;
    const float *norm_w = nullptr;
    float eps = 0.f;
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
    // Gated Delta Rule-2: erase [B, H, d_k] and write [B, H, d_v] gates in
    // the dtype of q, k, v (beta unused)
    bool gdr2 = false;
    const void *erase = nullptr, *write = nullptr;
};

// The tensor-core path's scratch, carved out of ChunkArgs::workspace (every
// part starts on a 256-byte boundary):
//   T, Aqk   [B*H*chunks][64][64] bf16    T' = (I + A)^{-1} Diag(beta) and Aqk
//   W        [B*H*chunks][64][128] bf16   -W, W = T' K<- (token rows, the layout of Q<-)
//   Ql       [B, H, T, 128] bf16          Q<- (chunk-relative decays)
//   Kt       [B*H*chunks][128][64] bf16   K_tail^T (key channel rows; zeros past T)
//   gam      [B*H*chunks][128] fp32       gamma_C per key channel
//   Z        [B, H, T, 128] bf16          Gated Delta Rule-2 only: w * v
struct TcWorkspace {
    __nv_bfloat16 *T, *Aqk, *W, *Ql, *Kt;
    float *gam;
    __nv_bfloat16 *Z;
};
inline size_t tc_workspace_bytes(int B, int H, int T, bool gdr2 = false)
{
    const size_t bh = (size_t)B * H, nch = (size_t)(T + 63) / 64;
    return 2 * bh * nch * 64 * 64 * 2 + 2 * bh * nch * 128 * 64 * 2 + bh * (size_t)T * 128 * 2 + bh * nch * 128 * 4 +
           (gdr2 ? bh * (size_t)T * 128 * 2 : 0);
}
inline TcWorkspace carve_tc_workspace(void *ws, int B, int H, int T, bool gdr2 = false)
{
    const size_t bh = (size_t)B * H, nch = (size_t)(T + 63) / 64;
    unsigned char *p = static_cast<unsigned char *>(ws);
    TcWorkspace w;
    w.T = reinterpret_cast<__nv_bfloat16 *>(p);
    p += bh * nch * 64 * 64 * 2;
    w.Aqk = reinterpret_cast<__nv_bfloat16 *>(p);
    p += bh * nch * 64 * 64 * 2;
    w.W = reinterpret_cast<__nv_bfloat16 *>(p);
    p += bh * nch * 128 * 64 * 2;
    w.Ql = reinterpret_cast<__nv_bfloat16 *>(p);
    p += bh * (size_t)T * 128 * 2;
    w.Kt = reinterpret_cast<__nv_bfloat16 *>(p);
    p += bh * nch * 128 * 64 * 2;
    w.gam = reinterpret_cast<float *>(p);
    p += bh * nch * 128 * 4;
    w.Z = gdr2 ? reinterpret_cast<__nv_bfloat16 *>(p) : nullptr;
    return w;
}

// Arguments of one chunked backward, already validated (d_k = d_v = D).
struct BwdArgs {
    const void *q, *k, *v, *dO;
    const float *g, *beta, *S0, *dS_T;
    void *dq, *dk, *dv;
    float *dg, *dbeta, *dS0;
    int B, H, T;
    int D;   // d_k = d_v
    bool scalar_gate;
    bool bf16;
    void *workspace;   // chunk_bwd_workspace_bytes()
};
size_t chunk_bwd_workspace_bytes(int B, int H, int T, int D);
cudaError_t launch_chunk_bwd(const BwdArgs &a, cudaStream_t stream, int *launches);

// Each launcher enqueues its kernels on `stream`, adds the number of kernels
// it launched to *launches and returns the first launch error.
cudaError_t launch_recurrent_step(const StepArgs &a, cudaStream_t stream, int *launches);
cudaError_t launch_chunk_simt(const ChunkArgs &a, cudaStream_t stream, int *launches);
cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t stream, int *launches);
bool chunk_tc_supports(const ChunkArgs &a);
size_t chunk_tc_workspace_bytes(int B, int H, int T, bool gdr2 = false);
// Synchronizes `stream`, then reads and clears the device status word.
cudaError_t read_device_status(cudaStream_t stream, int *status);
// Clock cycles each bounded device wait of later launches may take (0: the
// default, about a second); for tests of the timeout path.
void set_wait_budget(long long cycles);
// Debug mode (GDR_DEBUG set in the environment, read once): the entry points
// that take a log-decay gate check its n elements first (finite and <= 0);
// *bad is set when one is not.  Synchronizes `stream`.
bool debug_checks_enabled();
cudaError_t check_gate_range(const float *g, size_t n, cudaStream_t stream, bool *bad);

// The KDA lower bound on the per-channel log-decay.
constexpr float kGateMin = -5.0f;

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

}  // namespace gdr
