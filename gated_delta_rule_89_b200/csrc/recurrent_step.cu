// Single-token recurrent update (decode step) of the gated delta rule.
//
// Per (b, h), in one pass over the fp32 state S [dv x dk]:
//   S~ = S Diag(alpha),  p = S~ k,  delta = beta (v - p),
//   S <- S~ + delta k^T, o = S q = S~ q + delta (k . q).
// The order (decay, predict from the decayed state, delta, write, read) is
// the pseudo-code of "KDA vs Gated DeltaNet" (brenchcc), section 4; the
// orientation (o = S q, S in R^{dv x dk}) is that of "Reading notes: Kimi
// Delta Attention" (mzeromiko), section 4.
//
// Gated Delta Rule-2 ("Token Mixer I", section "Gated DeltaNet-2: Decoupling
// Erase and Write in Linear Attention", eq. (10)): the prediction reads along
// the erase-gated key and the target is the write-gated value,
//   p = S~ (b * k),  delta = w * v - p,
// with the write along k and the readout unchanged.
//
// The step is bound by HBM traffic: the state is read once and written once
// (2 * 4 * dv * dk bytes per head) and everything else is a few hundred
// bytes.  One warp owns one state row at a time: each lane holds dk/32
// consecutive channels, so a row is one coalesced 512-byte (dk = 128) load
// and store.  Both dot products S~k and S~q are reduced in a single shared
// butterfly, and o reuses S~q plus delta * (k.q), so the updated row never
// has to be read back.  Each warp keeps RPW rows in flight to cover DRAM
// latency.
#include "gdr_internal.cuh"

namespace gdr {
namespace {

constexpr int kStepThreads = 256;
constexpr int kStepWarps = kStepThreads / 32;

template <int VEC> struct VecF;
template <> struct VecF<4> {
    static __device__ __forceinline__ void load(const float *p, float *x) {
        float4 t = __ldcs(reinterpret_cast<const float4 *>(p));
        x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    }
    static __device__ __forceinline__ void store(float *p, const float *x) {
        __stcs(reinterpret_cast<float4 *>(p), make_float4(x[0], x[1], x[2], x[3]));
    }
};
template <> struct VecF<2> {
    static __device__ __forceinline__ void load(const float *p, float *x) {
        float2 t = __ldcs(reinterpret_cast<const float2 *>(p));
        x[0] = t.x; x[1] = t.y;
    }
    static __device__ __forceinline__ void store(float *p, const float *x) {
        __stcs(reinterpret_cast<float2 *>(p), make_float2(x[0], x[1]));
    }
};

template <int DK, int RPW, typename T, bool SCALAR, bool GDR2>
__global__ void __launch_bounds__(kStepThreads)
recurrent_step_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                      const float *__restrict__ g, const float *__restrict__ beta,
                      const T *__restrict__ erase, const T *__restrict__ write,
                      float *__restrict__ S, T *__restrict__ o, int dv, int blocks_per_head)
{
    constexpr int VEC = DK / 32;
    const int head = blockIdx.x / blocks_per_head;
    const int rblk = blockIdx.x - head * blocks_per_head;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int row0 = (rblk * kStepWarps + warp) * RPW;

    float s[RPW][VEC];
    float *Srow = S + ((size_t)head * dv + row0) * DK + lane * VEC;
#pragma unroll
    for (int r = 0; r < RPW; ++r) VecF<VEC>::load(Srow + (size_t)r * DK, s[r]);

    float kv[VEC], qv[VEC], av[VEC], ev[VEC];   // ev: the key the state is read along
    const size_t hk = (size_t)head * DK + lane * VEC;
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
        kv[j] = to_f32<T>(k[hk + j]);
        qv[j] = to_f32<T>(q[hk + j]);
        ev[j] = GDR2 ? to_f32<T>(erase[hk + j]) * kv[j] : kv[j];
    }
    if (SCALAR) {
        const float a = expf(g[head]);
#pragma unroll
        for (int j = 0; j < VEC; ++j) av[j] = a;
    } else {
#pragma unroll
        for (int j = 0; j < VEC; ++j) av[j] = expf(fmaxf(g[hk + j], kGateMin));
    }
    const float b = GDR2 ? 1.f : beta[head];
    float vr[RPW];   // the write target: beta v, or w * v for GDR-2
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
        const size_t iv = (size_t)head * dv + row0 + r;
        vr[r] = GDR2 ? to_f32<T>(write[iv]) * to_f32<T>(v[iv]) : to_f32<T>(v[iv]);
    }

    // k . q (identical in every warp)
    float kq = 0.f;
#pragma unroll
    for (int j = 0; j < VEC; ++j) kq = fmaf(kv[j], qv[j], kq);

    float p[RPW], rq[RPW];
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
        p[r] = 0.f;
        rq[r] = 0.f;
#pragma unroll
        for (int j = 0; j < VEC; ++j) {
            s[r][j] *= av[j];
            p[r] = fmaf(s[r][j], ev[j], p[r]);
            rq[r] = fmaf(s[r][j], qv[j], rq[r]);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        kq += __shfl_xor_sync(0xffffffffu, kq, off);
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
            p[r] += __shfl_xor_sync(0xffffffffu, p[r], off);
            rq[r] += __shfl_xor_sync(0xffffffffu, rq[r], off);
        }
    }
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
        const float delta = b * (vr[r] - p[r]);
#pragma unroll
        for (int j = 0; j < VEC; ++j) s[r][j] = fmaf(delta, kv[j], s[r][j]);
        VecF<VEC>::store(Srow + (size_t)r * DK, s[r]);
        if (lane == r) o[(size_t)head * dv + row0 + r] = from_f32<T>(fmaf(delta, kq, rq[r]));
    }
}

template <int DK, typename T, bool SCALAR, bool GDR2>
cudaError_t launch_typed(const StepArgs &a, cudaStream_t stream)
{
    constexpr int RPW = 4;
    const int rows_per_block = kStepWarps * RPW;  // 32; dv is 64 or 128
    const int blocks_per_head = a.dv / rows_per_block;
    const long long blocks = (long long)a.B * a.H * blocks_per_head;
    if (blocks == 0) return cudaSuccess;
    recurrent_step_kernel<DK, RPW, T, SCALAR, GDR2><<<(unsigned)blocks, kStepThreads, 0, stream>>>(
        (const T *)a.q, (const T *)a.k, (const T *)a.v, a.g, a.beta, (const T *)a.erase, (const T *)a.write, a.S,
        (T *)a.o, a.dv, blocks_per_head);
    return cudaGetLastError();
}

template <int DK, bool GDR2>
cudaError_t launch_dk(const StepArgs &a, cudaStream_t s)
{
    if (a.bf16) return a.scalar_gate ? launch_typed<DK, __nv_bfloat16, true, GDR2>(a, s)
                                     : launch_typed<DK, __nv_bfloat16, false, GDR2>(a, s);
    return a.scalar_gate ? launch_typed<DK, float, true, GDR2>(a, s) : launch_typed<DK, float, false, GDR2>(a, s);
}

}  // namespace

cudaError_t launch_recurrent_step(const StepArgs &a, cudaStream_t stream, int *launches)
{
    if ((long long)a.B * a.H == 0) return cudaSuccess;
    cudaError_t e = a.gdr2 ? ((a.dk == 128) ? launch_dk<128, true>(a, stream) : launch_dk<64, true>(a, stream))
                           : ((a.dk == 128) ? launch_dk<128, false>(a, stream) : launch_dk<64, false>(a, stream));
    if (e == cudaSuccess) *launches += 1;
    return e;
}

}  // namespace gdr
