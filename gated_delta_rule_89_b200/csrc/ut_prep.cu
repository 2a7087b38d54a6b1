// UT-transform preparation of the chunked forward, one CTA per chunk.
//
// For every chunk of C = 64 tokens (rows r, i) this kernel forms
//   A[r][i]   = beta_r sum_c k_rc k_ic exp(G_rc - G_ic)     (i <  r)
//   Aqk[r][i] =        sum_c q_rc k_ic exp(G_rc - G_ic)     (i <= r)
//   T' = (I + A)^{-1} Diag(beta)
// and writes T' and Aqk (bf16, row-major 64 x 64) to the workspace.  T' is
// the matrix the UT transform of "Token Mixer I", section "Kimi Delta
// Attention: Improving Delta Rule with Fine-grained Gating" calls
// M = (I + StrictTril(Diag(beta)(Gamma*K)(K/Gamma)^T))^{-1} Diag(beta), so
// W = T' (Gamma*K) and U = T' V; Aqk is the masked intra-chunk factor of the
// output equation.  Neither depends on the state, so all chunks of all heads
// run in parallel here and the sequential kernel only consumes them.
//
// Decay ratios (per-channel gate).  G is the cumulative log-decay inside the
// chunk; exp(G_r - G_i) is formed without overflow by splitting the chunk
// into four 16-token blocks.  With base_R the cumulative sum just before
// block R and bd_R = exp(base_{R+1} - base_R) the decay across block R:
//   left  (row r in block R):   Khat_r = k_r * exp(G_r - base_R)            (<= 1)
//   right (row i in block I):   Kchk_i = k_i * exp(base_{I+1} - G_i)        (<= 1)
//   exp(G_r - G_i) = e(r) * [prod_{I<J<R} bd_J] * e'(i)            (I < R)
//                  = e(r) * e'(i) / bd_R                            (I = R)
// so every stored operand is <= 1 in magnitude, the only factor above 1 is
// 1/bd_R <= exp(80) (the -5 bound on g times 16 tokens), well inside the
// bf16/fp32 range, and a factor that underflows multiplies a term that is
// below fp32 resolution anyway.  The per-channel factor of each block pair
// is applied to the B fragments in registers, so the 10 block products per
// matrix run on mma.sync (m16n8k16, bf16 in, fp32 accumulate).  The -5 bound
// is the KDA g_min; exp(G) inside a block is a running product of
// alpha = exp(max(g, -5)), one exponential per (token, channel).
// A scalar gate needs no splitting: the products use k and q as they are and
// the decay exp(G_r - G_i) multiplies each entry afterwards.
//
// Inverse.  (I + A) is unit lower triangular.  Its two 32 x 32 diagonal
// blocks are inverted by forward substitution, one thread per column, and
// the off-diagonal block is Y = -Z A_10 X (X, Z the diagonal inverses).
#include "gdr_internal.cuh"

namespace gdr {
namespace {

constexpr int kC = 64;        // chunk
constexpr int kDK = 128;      // key dim
constexpr int kLdB = kDK + 8; // padded bf16 row stride (272 B: ldmatrix conflict free)
constexpr int kLdA = kC + 1;  // padded fp32 row stride

struct PrepSmem {
    __nv_bfloat16 kh[kC][kLdB];   // Khat (left operand of A)
    __nv_bfloat16 qh[kC][kLdB];   // Qhat (left operand of Aqk)
    __nv_bfloat16 kc[kC][kLdB];   // Kchk (right operand)
    float fac[7][kDK];            // block-pair channel factors (see pair_factor)
    float A[kC][kLdA];            // A, then its inverse
    float Aq[kC][kLdA];           // Aqk
    float P[32][33];              // A_10 X
    float beta[kC];
    float G[kC];                  // scalar-gate cumulative sum
};

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void *p)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"((uint32_t)__cvta_generic_to_shared(p)));
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t v, float s0, float s1)
{
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162 *>(&v);
    float2 f = __bfloat1622float2(h);
    __nv_bfloat162 o = __floats2bfloat162_rn(f.x * s0, f.y * s1);
    return *reinterpret_cast<uint32_t *>(&o);
}

// factor row for block pair (R, I): -1 = none (adjacent blocks), else index into fac
__device__ __forceinline__ int pair_factor(int R, int I)
{
    if (R == I) return 3 + R;          // 1 / bd_R
    if (R == I + 1) return -1;         // exp(base_R - base_{I+1}) = 1
    if (R == 2 && I == 0) return 0;    // bd_1
    if (R == 3 && I == 1) return 1;    // bd_2
    return 2;                          // (3, 0): bd_1 bd_2
}

template <bool SCALAR>
__global__ void __launch_bounds__(128)
ut_prep_kernel(const __nv_bfloat16 *__restrict__ kg, const __nv_bfloat16 *__restrict__ qg,
               const float *__restrict__ gg, const float *__restrict__ betag,
               __nv_bfloat16 *__restrict__ Tout, __nv_bfloat16 *__restrict__ Aqout, int T_len, int nchunks)
{
    extern __shared__ __align__(16) unsigned char prep_raw[];
    PrepSmem &sm = *reinterpret_cast<PrepSmem *>(prep_raw);
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const size_t head = blockIdx.x / nchunks;
    const int chunk = blockIdx.x - (int)(head * nchunks);
    const int t0 = chunk * kC;
    const int n = min(kC, T_len - t0);
    const size_t row0 = head * (size_t)T_len + t0;   // first token row of this chunk

    if (tid < kC) sm.beta[tid] = tid < n ? betag[row0 + tid] : 0.f;

    // ---- operands (thread = key channel)
    {
        const int c = tid;
        if (!SCALAR) {
            float bd[4];
#pragma unroll
            for (int R = 0; R < 4; ++R) {
                float al[16], kv[16], qv[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    const int rr = R * 16 + r;
                    const bool ok = rr < n;
                    const size_t gi = (row0 + rr) * kDK + c;
                    al[r] = ok ? __expf(fmaxf(gg[gi], kGateMin)) : 1.f;
                    kv[r] = ok ? __bfloat162float(kg[gi]) : 0.f;
                    qv[r] = ok ? __bfloat162float(qg[gi]) : 0.f;
                }
                float p = 1.f;
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    p *= al[r];
                    sm.kh[R * 16 + r][c] = __float2bfloat16_rn(kv[r] * p);
                    sm.qh[R * 16 + r][c] = __float2bfloat16_rn(qv[r] * p);
                }
                bd[R] = p;
                p = 1.f;
#pragma unroll
                for (int r = 15; r >= 0; --r) {
                    sm.kc[R * 16 + r][c] = __float2bfloat16_rn(kv[r] * p);
                    p *= al[r];
                }
            }
            sm.fac[0][c] = bd[1];
            sm.fac[1][c] = bd[2];
            sm.fac[2][c] = bd[1] * bd[2];
#pragma unroll
            for (int R = 0; R < 4; ++R) sm.fac[3 + R][c] = 1.f / bd[R];
        } else {
            for (int r = 0; r < kC; ++r) {
                const bool ok = r < n;
                const size_t gi = (row0 + r) * kDK + c;
                const __nv_bfloat16 z = __float2bfloat16_rn(0.f);
                const __nv_bfloat16 kk = ok ? kg[gi] : z;
                sm.kh[r][c] = kk;
                sm.kc[r][c] = kk;
                sm.qh[r][c] = ok ? qg[gi] : z;
            }
        }
    }
    if (SCALAR && warp == 0) {
        // inclusive scan of the scalar log-decay over the chunk (2 values per lane)
        float a0 = (2 * lane < n) ? gg[row0 + 2 * lane] : 0.f;
        float a1 = (2 * lane + 1 < n) ? gg[row0 + 2 * lane + 1] : 0.f;
        float s = a0 + a1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            float o = __shfl_up_sync(0xffffffffu, s, off);
            if (lane >= off) s += o;
        }
        sm.G[2 * lane + 1] = s;
        sm.G[2 * lane] = s - a1;
    }
    for (int idx = tid; idx < kC * kLdA; idx += 128) {
        (&sm.A[0][0])[idx] = 0.f;
        (&sm.Aq[0][0])[idx] = 0.f;
    }
    __syncthreads();

    // ---- block products on tensor cores: warp (which, half)
    {
        const int which = warp >> 1;        // 0: A from Khat, 1: Aqk from Qhat
        const int half = warp & 1;
        const __nv_bfloat16(*L)[kLdB] = which ? sm.qh : sm.kh;
        float(*D)[kLdA] = which ? sm.Aq : sm.A;
        const int g = lane >> 2, t = lane & 3;
        static const int kPairs[2][5][2] = {{{0, 0}, {1, 0}, {1, 1}, {2, 0}, {2, 1}},
                                            {{2, 2}, {3, 0}, {3, 1}, {3, 2}, {3, 3}}};
#pragma unroll 1
        for (int p = 0; p < 5; ++p) {
            const int R = kPairs[half][p][0], I = kPairs[half][p][1];
            const int fi = SCALAR ? -1 : pair_factor(R, I);
            float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int s = 0; s < kDK / 16; ++s) {
                uint32_t a[4], b[4];
                ldsm_x4(a, &L[R * 16 + (lane & 15)][s * 16 + (lane >> 4) * 8]);
                ldsm_x4(b, &sm.kc[I * 16 + (lane & 7) + ((lane >> 4) << 3)][s * 16 + ((lane >> 3) & 1) * 8]);
                if (fi >= 0) {
                    const float *f = sm.fac[fi] + s * 16 + 2 * t;
                    b[0] = scale_bf16x2(b[0], f[0], f[1]);
                    b[1] = scale_bf16x2(b[1], f[8], f[9]);
                    b[2] = scale_bf16x2(b[2], f[0], f[1]);
                    b[3] = scale_bf16x2(b[3], f[8], f[9]);
                }
                mma16816(acc[0], a, b[0], b[1]);
                mma16816(acc[1], a, b[2], b[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = R * 16 + g + (e >> 1) * 8;
                    const int i = I * 16 + nt * 8 + 2 * t + (e & 1);
                    float v = acc[nt][e];
                    if (SCALAR) v *= __expf(sm.G[r] - sm.G[i]);
                    if (which == 0) v = (i < r) ? sm.beta[r] * v : 0.f;
                    else v = (i <= r) ? v : 0.f;
                    D[r][i] = v;
                }
        }
    }
    __syncthreads();

    // ---- inverse of (I + A): diagonal 32 x 32 blocks, one thread per column
    if (tid < 64) {
        const int base = (tid >> 5) * 32;   // 0: X (top-left), 32: Z (bottom-right)
        const int j = tid & 31;
        float x[32];
#pragma unroll
        for (int r = 0; r < 32; ++r) {
            float s = (r == j) ? 1.f : 0.f;
#pragma unroll
            for (int m = 0; m < r; ++m) s = fmaf(-sm.A[base + r][base + m], x[m], s);
            x[r] = s;
        }
        // every lane of this warp has finished reading its diagonal block of A
        // before any lane overwrites it (the other warp owns the other block)
        __syncwarp();
#pragma unroll
        for (int r = 0; r < 32; ++r) sm.A[base + r][base + j] = x[r];
    }
    __syncthreads();
    // P = A_10 X   (32 x 32): thread -> 8 entries
    {
        const int r = tid >> 2, c0 = (tid & 3) * 8;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        for (int m = 0; m < 32; ++m) {
            const float a = sm.A[32 + r][m];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(a, sm.A[m][c0 + e], acc[e]);
        }
        __syncthreads();
#pragma unroll
        for (int e = 0; e < 8; ++e) sm.P[r][c0 + e] = acc[e];
        __syncthreads();
        // Y = -Z P
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        for (int m = 0; m < 32; ++m) {
            const float z = sm.A[32 + r][32 + m];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(z, sm.P[m][c0 + e], acc[e]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) sm.A[32 + r][c0 + e] = -acc[e];
        // upper-right block of the inverse is zero
#pragma unroll
        for (int e = 0; e < 8; ++e) sm.A[r][32 + c0 + e] = 0.f;
    }
    __syncthreads();

    // ---- write T' = A~ Diag(beta) and Aqk (bf16, row-major 64 x 64)
    {
        const size_t cbase = ((size_t)blockIdx.x) * kC * kC;
        for (int idx = tid; idx < kC * kC / 8; idx += 128) {
            const int r = idx >> 3, c0 = (idx & 7) * 8;
            __align__(16) __nv_bfloat16 tv[8], qv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                tv[e] = __float2bfloat16_rn(sm.A[r][c0 + e] * sm.beta[c0 + e]);
                qv[e] = __float2bfloat16_rn(sm.Aq[r][c0 + e]);
            }
            *reinterpret_cast<uint4 *>(Tout + cbase + r * kC + c0) = *reinterpret_cast<uint4 *>(tv);
            *reinterpret_cast<uint4 *>(Aqout + cbase + r * kC + c0) = *reinterpret_cast<uint4 *>(qv);
        }
    }
}

}  // namespace

size_t ut_prep_smem_bytes() { return sizeof(PrepSmem); }

cudaError_t launch_ut_prep(const ChunkArgs &a, __nv_bfloat16 *Tout, __nv_bfloat16 *Aqout, cudaStream_t stream)
{
    const int nchunks = (a.T + kC - 1) / kC;
    const long long blocks = (long long)a.B * a.H * nchunks;
    if (blocks == 0) return cudaSuccess;
    const size_t smem = sizeof(PrepSmem);
    if (a.scalar_gate) {
        cudaError_t e = cudaFuncSetAttribute(ut_prep_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        ut_prep_kernel<true><<<(unsigned)blocks, 128, smem, stream>>>(
            (const __nv_bfloat16 *)a.k, (const __nv_bfloat16 *)a.q, a.g, a.beta, Tout, Aqout, a.T, nchunks);
    } else {
        cudaError_t e = cudaFuncSetAttribute(ut_prep_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        ut_prep_kernel<false><<<(unsigned)blocks, 128, smem, stream>>>(
            (const __nv_bfloat16 *)a.k, (const __nv_bfloat16 *)a.q, a.g, a.beta, Tout, Aqout, a.T, nchunks);
    }
    return cudaGetLastError();
}

}  // namespace gdr
