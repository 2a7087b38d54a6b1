// Chunkwise forward of the gated delta rule on CUDA cores, fp32 arithmetic.
//
// This is the general path: any supported d_k, d_v, C, fp32 or bf16 inputs,
// and the only path for fp32 inputs (whose 1e-5 tolerance rules out bf16 or
// tf32 tensor-core operands).  One CTA owns one (b, h) and a 32-row tile of
// the d_v rows of the state; it walks the chunks in order and keeps its
// fp32 state tile in shared memory.  Per chunk of C tokens (rows r, i), with
// G_r the inclusive cumulative sum of the (bounded) log-decay inside the
// chunk:
//
//   A[r][i]   = beta_r sum_c k_rc k_ic exp(G_rc - G_ic)        (i < r)
//   Aqk[r][i] = sum_c q_rc k_ic exp(G_rc - G_ic)                (i <= r)
//   A~ = (I + A)^{-1}                    forward substitution, row by row
//   W = A~ Diag(beta) (K * exp(G)),  U = A~ Diag(beta) V
//   V_new = U - W S^T
//   O = (Q * exp(G)) S^T + Aqk V_new
//   S <- S Diag(exp(G_C)) + V_new^T (K * exp(G_C - G))
//
// which is the UT-transform chunk form of "Token Mixer I", section "Kimi
// Delta Attention: Improving Delta Rule with Fine-grained Gating", and
// "Reading notes: Kimi Delta Attention" (mzeromiko), section 4, written in
// the d_v x d_k orientation.  Every decay ratio is formed as exp of a
// difference of cumulative sums that is <= 0, so nothing can overflow; a
// ratio that underflows to 0 is below fp32 resolution of the terms it
// multiplies.  Rows past the end of a partial last chunk are padded as
// identity tokens (k = q = v = 0, beta = 0, g = 0) and produce no output.
#include "gdr_internal.cuh"

namespace gdr {
namespace {

constexpr int kSimtThreads = 256;
constexpr int kSimtDvTile = 32;

template <int DK, int C>
struct SimtSmem {
    static constexpr int LD = DK + 1;  // padded row stride (bank spread)
    static constexpr int G = 0;                          // [C][LD] cumsum, then beta*K<-
    static constexpr int K = G + C * LD;                 // [C][LD] keys, then K_tail
    static constexpr int Q = K + C * LD;                 // [C][LD] queries, then Q<-
    static constexpr int W = Q + C * LD;                 // [C][LD] W
    static constexpr int A = W + C * LD;                 // [C][C]  A, then A~ (strict lower)
    static constexpr int AQ = A + C * C;                 // [C][C]  Aqk
    static constexpr int S = AQ + C * C;                 // [DVT][LD] state tile
    static constexpr int VN = S + kSimtDvTile * LD;      // [C][DVT] U, then V_new
    static constexpr int VB = VN + C * kSimtDvTile;      // [C][DVT] beta * V
    static constexpr int BETA = VB + C * kSimtDvTile;    // [C]
    static constexpr int GC = BETA + C;                  // [DK] G at the chunk end
    static constexpr int GAM = GC + DK;                  // [DK] exp(G_C)
    static constexpr int GS = GAM + DK;                  // [C] scalar-gate cumsum
    static constexpr int TOTAL = GS + C;
    static constexpr size_t BYTES = sizeof(float) * TOTAL;
};

template <int DK, int C, typename T, bool SCALAR>
__global__ void __launch_bounds__(kSimtThreads)
chunk_simt_kernel(const T *__restrict__ qg, const T *__restrict__ kg, const T *__restrict__ vg,
                  const float *__restrict__ gg, const float *__restrict__ betag,
                  const float *__restrict__ S0, T *__restrict__ Og, float *__restrict__ ST,
                  int T_len, int dv)
{
    using L = SimtSmem<DK, C>;
    constexpr int LD = L::LD;
    constexpr int DVT = kSimtDvTile;
    extern __shared__ float sm[];
    float *Gs = sm + L::G, *ks = sm + L::K, *qs = sm + L::Q, *Wm = sm + L::W;
    float *Am = sm + L::A, *Aq = sm + L::AQ, *Ss = sm + L::S, *Vn = sm + L::VN, *vb = sm + L::VB;
    float *bs = sm + L::BETA, *gC = sm + L::GC, *gam = sm + L::GAM, *gsc = sm + L::GS;

    const int tid = threadIdx.x;
    const size_t head = blockIdx.x;
    const int i0 = blockIdx.y * DVT;  // first state row of this tile
    const T *q = qg + head * T_len * DK;
    const T *k = kg + head * T_len * DK;
    const T *v = vg + head * T_len * dv;
    const float *beta = betag + head * T_len;
    T *O = Og + head * T_len * dv;

    for (int idx = tid; idx < DVT * DK; idx += kSimtThreads) {
        const int i = idx / DK, c = idx % DK;
        Ss[i * LD + c] = S0 ? S0[(head * dv + i0 + i) * DK + c] : 0.f;
    }

    for (int t0 = 0; t0 < T_len; t0 += C) {
        const int n = min(C, T_len - t0);
        __syncthreads();
        // ---- load the chunk (identity padding past the end)
        for (int idx = tid; idx < C * DK; idx += kSimtThreads) {
            const int r = idx / DK, c = idx % DK;
            const bool ok = r < n;
            const size_t gi = (size_t)(t0 + r) * DK + c;
            ks[r * LD + c] = ok ? to_f32<T>(k[gi]) : 0.f;
            qs[r * LD + c] = ok ? to_f32<T>(q[gi]) : 0.f;
            if (!SCALAR) Gs[r * LD + c] = ok ? fmaxf(gg[head * T_len * DK + gi], kGateMin) : 0.f;
        }
        for (int r = tid; r < C; r += kSimtThreads) {
            bs[r] = r < n ? beta[t0 + r] : 0.f;
            if (SCALAR) gsc[r] = r < n ? gg[head * T_len + t0 + r] : 0.f;
        }
        for (int idx = tid; idx < C * DVT; idx += kSimtThreads) {
            const int r = idx / DVT, i = idx % DVT;
            vb[idx] = r < n ? beta[t0 + r] * to_f32<T>(v[(size_t)(t0 + r) * dv + i0 + i]) : 0.f;
        }
        __syncthreads();
        // ---- a1: per-chunk cumulative sum of the log-decay
        if (!SCALAR) {
            for (int c = tid; c < DK; c += kSimtThreads) {
                float acc = 0.f;
                for (int r = 0; r < C; ++r) {
                    acc += Gs[r * LD + c];
                    Gs[r * LD + c] = acc;
                }
            }
        } else {
            if (tid == 0) {
                float acc = 0.f;
                for (int r = 0; r < C; ++r) {
                    acc += gsc[r];
                    gsc[r] = acc;
                }
            }
            __syncthreads();
            for (int idx = tid; idx < C * DK; idx += kSimtThreads) {
                const int r = idx / DK, c = idx % DK;
                Gs[r * LD + c] = gsc[r];
            }
        }
        __syncthreads();
        // ---- a2 (first half): A and Aqk with exact decay ratios
        for (int p = tid; p < C * C; p += kSimtThreads) {
            const int r = p / C, i = p % C;
            float aa = 0.f, aq = 0.f;
            if (i <= r) {
                const float *kr = ks + r * LD, *ki = ks + i * LD, *qr = qs + r * LD;
                const float *Gr = Gs + r * LD, *Gi = Gs + i * LD;
                for (int c = 0; c < DK; ++c) {
                    const float kk = ki[c] * expf(Gr[c] - Gi[c]);
                    aa = fmaf(kr[c], kk, aa);
                    aq = fmaf(qr[c], kk, aq);
                }
            }
            Am[p] = (i < r) ? bs[r] * aa : 0.f;
            Aq[p] = aq;
        }
        for (int c = tid; c < DK; c += kSimtThreads) {
            gC[c] = Gs[(C - 1) * LD + c];
            gam[c] = expf(Gs[(C - 1) * LD + c]);
        }
        __syncthreads();
        // ---- decayed operands: Q<- (in place), beta*K<- (over G), K_tail (over K)
        for (int idx = tid; idx < C * DK; idx += kSimtThreads) {
            const int r = idx / DK, c = idx % DK;
            const float G = Gs[r * LD + c];
            const float e = expf(G);
            const float kk = ks[r * LD + c];
            qs[r * LD + c] *= e;
            Gs[r * LD + c] = bs[r] * kk * e;
            ks[r * LD + c] = kk * expf(gC[c] - G);
        }
        // ---- a2 (second half): A~ = (I + A)^{-1}, strictly lower part, by rows
        for (int r = 1; r < C; ++r) {
            float val = 0.f;
            const int j = tid;
            if (j < r) {
                val = -Am[r * C + j];
                for (int m = j + 1; m < r; ++m) val = fmaf(-Am[r * C + m], Am[m * C + j], val);
            }
            __syncthreads();
            if (j < r) Am[r * C + j] = val;
            __syncthreads();
        }
        // ---- W = A~ (beta K<-),  U = A~ (beta V)   (unit diagonal of A~ implicit)
        for (int idx = tid; idx < C * DK; idx += kSimtThreads) {
            const int r = idx / DK, c = idx % DK;
            float acc = Gs[r * LD + c];
            for (int j = 0; j < r; ++j) acc = fmaf(Am[r * C + j], Gs[j * LD + c], acc);
            Wm[r * LD + c] = acc;
        }
        for (int idx = tid; idx < C * DVT; idx += kSimtThreads) {
            const int r = idx / DVT, i = idx % DVT;
            float acc = vb[idx];
            for (int j = 0; j < r; ++j) acc = fmaf(Am[r * C + j], vb[j * DVT + i], acc);
            Vn[idx] = acc;
        }
        __syncthreads();
        // ---- a3: V_new = U - W S^T
        for (int idx = tid; idx < C * DVT; idx += kSimtThreads) {
            const int r = idx / DVT, i = idx % DVT;
            const float *w = Wm + r * LD, *s = Ss + i * LD;
            float acc = 0.f;
            for (int c = 0; c < DK; ++c) acc = fmaf(w[c], s[c], acc);
            Vn[idx] -= acc;
        }
        __syncthreads();
        // ---- a4: O = Q<- S^T + Aqk V_new   (valid rows only)
        for (int idx = tid; idx < n * DVT; idx += kSimtThreads) {
            const int r = idx / DVT, i = idx % DVT;
            const float *qq = qs + r * LD, *s = Ss + i * LD;
            float acc = 0.f;
            for (int c = 0; c < DK; ++c) acc = fmaf(qq[c], s[c], acc);
            for (int j = 0; j <= r; ++j) acc = fmaf(Aq[r * C + j], Vn[j * DVT + i], acc);
            O[(size_t)(t0 + r) * dv + i0 + i] = from_f32<T>(acc);
        }
        __syncthreads();
        // ---- a3: S <- S Diag(gamma_C) + V_new^T K_tail
        for (int idx = tid; idx < DVT * DK; idx += kSimtThreads) {
            const int i = idx / DK, c = idx % DK;
            float acc = Ss[i * LD + c] * gam[c];
            for (int r = 0; r < C; ++r) acc = fmaf(Vn[r * DVT + i], ks[r * LD + c], acc);
            Ss[i * LD + c] = acc;
        }
    }
    __syncthreads();
    if (ST) {
        for (int idx = tid; idx < DVT * DK; idx += kSimtThreads) {
            const int i = idx / DK, c = idx % DK;
            ST[(head * dv + i0 + i) * DK + c] = Ss[i * LD + c];
        }
    }
}

template <int DK, int C, typename T, bool SCALAR>
cudaError_t launch_typed(const ChunkArgs &a, cudaStream_t stream)
{
    using L = SimtSmem<DK, C>;
    auto kern = chunk_simt_kernel<DK, C, T, SCALAR>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::BYTES);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)(a.B * a.H), (unsigned)(a.dv / kSimtDvTile));
    kern<<<grid, kSimtThreads, L::BYTES, stream>>>((const T *)a.q, (const T *)a.k, (const T *)a.v, a.g, a.beta,
                                                   a.S0, (T *)a.O, a.S_T, a.T, a.dv);
    return cudaGetLastError();
}

template <int DK, int C>
cudaError_t launch_c(const ChunkArgs &a, cudaStream_t s)
{
    if (a.bf16) return a.scalar_gate ? launch_typed<DK, C, __nv_bfloat16, true>(a, s)
                                     : launch_typed<DK, C, __nv_bfloat16, false>(a, s);
    return a.scalar_gate ? launch_typed<DK, C, float, true>(a, s) : launch_typed<DK, C, float, false>(a, s);
}

template <int DK>
cudaError_t launch_dk(const ChunkArgs &a, cudaStream_t s)
{
    switch (a.C) {
        case 16: return launch_c<DK, 16>(a, s);
        case 32: return launch_c<DK, 32>(a, s);
        default: return launch_c<DK, 64>(a, s);
    }
}

}  // namespace

cudaError_t launch_chunk_simt(const ChunkArgs &a, cudaStream_t stream, int *launches)
{
    cudaError_t e = (a.dk == 128) ? launch_dk<128>(a, stream) : launch_dk<64>(a, stream);
    if (e == cudaSuccess) *launches += 1;
    return e;
}

}  // namespace gdr
