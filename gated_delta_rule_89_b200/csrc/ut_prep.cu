// UT-transform preparation of the chunked forward.
//
// For every chunk of C = 64 tokens (rows r, i) this kernel forms
//   A[r][i]   = beta_r sum_c k_rc k_ic exp(G_rc - G_ic)     (i <  r)
//   Aqk[r][i] =        sum_c q_rc k_ic exp(G_rc - G_ic)     (i <= r)
//   T' = (I + A)^{-1} Diag(beta)
// and writes T' and Aqk (bf16, row-major 64 x 64) to the workspace, together
// with the operands of the state scan that do not depend on the state:
// -W = -T' K<- (token-major), Q<-, K_tail^T and gamma_C (defined where they
// are written).  T' is
// the matrix the UT transform of "Token Mixer I", section "Kimi Delta
// Attention: Improving Delta Rule with Fine-grained Gating" calls
// M = (I + StrictTril(Diag(beta)(Gamma*K)(K/Gamma)^T))^{-1} Diag(beta), so
// W = T' (Gamma*K) and U = T' V; Aqk is the masked intra-chunk factor of the
// output equation.  Neither depends on the state, so all chunks of all heads
// run in parallel here and the sequential kernel only consumes them.
//
// Execution.  Persistent CTAs of 8 warps, two per SM, walk the chunks
// blockIdx.x, blockIdx.x + gridDim.x, ...  The gate pass reads k, q and g of
// a chunk straight from global memory (each warp a contiguous row segment)
// and writes the scaled operands into shared memory in the 128B-swizzled
// layout, which makes the ldmatrix reads of the block products conflict
// free; the other CTA on the SM runs its own phases while one waits.

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
// Inverse of N = I + A (unit lower triangular), in 16 x 16 blocks N_im.
// D_i = N_ii^{-1} by forward substitution (one thread per column).  With
// Nt_im = D_i N_im (i > m) the blocks U_ij of N^{-1} below the diagonal
// follow column block by column block:
//   U_{i,i-1} = -Nt_{i,i-1} D_{i-1},
//   U_20 = -Nt_20 D_0 - Nt_21 U_10,   U_31 = -Nt_31 D_1 - Nt_32 U_21,
//   U_30 = -Nt_30 D_0 - Nt_31 U_10 - Nt_32 U_20,
// (from N N^{-1} = I, left-multiplied by D_i).  These 16 products of 16 x 16
// fp32 blocks run on mma.sync (m16n8k8, tf32 operands, fp32 accumulation).
// T' leaves this kernel in bf16 (8-bit mantissa), so the 10-bit tf32
// operands add well under the final rounding; a three-pass hi/lo split
// (Ootomo and Yokota, 2022) measured the same end-to-end error and was
// slower.

#include <mutex>

#include "gdr_internal.cuh"
#include "sm100_ptx.cuh"

namespace gdr {
namespace {

using namespace sm100;

constexpr int kC = 64;         // chunk
constexpr int kDK = 128;       // key dim
constexpr int kThreads = 256;  // 8 warps
constexpr int kLdA = 68;       // fp32 row stride: 16-byte rows, conflict-free fragment stores

// shared memory (offsets from a 1024-byte aligned base)
constexpr uint32_t OFF_K = 0;                      // Khat (or k), two swizzled panels   16 KB
constexpr uint32_t OFF_Q = 16384;                  // Qhat (or q); then T' bf16 [64][72]   16 KB
constexpr uint32_t OFF_KC = 32768;                 // Kchk                                 16 KB
constexpr int kLdT = 72;                           // bf16 row stride of T' (ldmatrix conflict free)
constexpr uint32_t OFF_BD = 49152;                 // bd[4][128], 1/bd[4][128] fp32         4 KB
constexpr int kLdD = 24;       // row stride of the 16 x 16 blocks (conflict-free mma B fragments)
constexpr uint32_t OFF_D = OFF_BD + 4096;          // D_i = N_ii^{-1}, [4][16][24]           6 KB
constexpr uint32_t OFF_A = OFF_D + 4 * 16 * kLdD * 4;   // A; then the -W staging tile [64][128] bf16
static_assert(kC * kLdA * 4 >= kC * kDK * 2, "the -W staging tile fits in the A tile");
constexpr uint32_t OFF_AQ = OFF_A + kC * kLdA * 4; // Aqk, then Nt / X'
constexpr uint32_t OFF_U = OFF_AQ + kC * kLdA * 4; // U_10, U_21, U_20 [3][16][24]
constexpr uint32_t OFF_BETA = OFF_U + 3 * 16 * kLdD * 4;   // beta, two buffers by chunk parity
constexpr uint32_t OFF_GC = OFF_BETA + 512;        // scalar gate: inclusive cumulative sum
constexpr uint32_t OFF_NRM = OFF_GC + 256;         // prologue: row sums of q^2, k^2 per warp half [8][2][16]
constexpr uint32_t OFF_INV = OFF_NRM + 1024;       // prologue: 1 / L2 norm of those rows [8][2][16]
constexpr uint32_t SMEM_USED = OFF_INV + 1024;
constexpr uint32_t SMEM_ALLOC = SMEM_USED + 1024;  // alignment slack
static_assert(2 * (SMEM_ALLOC + 1024) <= 233472, "two CTAs per SM must fit in shared memory");

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    __nv_bfloat162 o = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&o);
}

// bf16 pair (packed) widened to an fp32 pair
__device__ __forceinline__ float2 unpack2(uint32_t v)
{
    return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}

// bf16 pair (packed) times an fp32 pair, rounded back to a bf16 pair
__device__ __forceinline__ uint32_t scale2p(uint32_t v, float2 f)
{
    const float2 r = fmul2(make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u)), f);
    return pack2(r.x, r.y);
}

__device__ __forceinline__ uint32_t to_tf32(float x)
{
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma1688(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// One warp: c[16x16] -= A[16x16] B[16x16] (tf32 operands, fp32 accumulation).
// A, B row-major in shared memory with row strides lda, ldb.
// Fragment of c: c[nt][e] is row g + 8 (e >> 1), column 8 nt + 2 t + (e & 1),
// with g = lane / 4, t = lane % 4.
__device__ __forceinline__ void mm16_sub(float (&c)[2][4], const float *A, int lda, const float *B, int ldb, int g,
                                         int t)
{
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        uint32_t a[4];
        a[0] = to_tf32(-A[g * lda + 8 * ks + t]);
        a[1] = to_tf32(-A[(g + 8) * lda + 8 * ks + t]);
        a[2] = to_tf32(-A[g * lda + 8 * ks + t + 4]);
        a[3] = to_tf32(-A[(g + 8) * lda + 8 * ks + t + 4]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
            mma1688(c[nt], a, to_tf32(B[(8 * ks + t) * ldb + 8 * nt + g]), to_tf32(B[(8 * ks + t + 4) * ldb + 8 * nt + g]));
    }
}

// byte offset of (row, col) in a [64 rows x 128 cols] bf16 tile held as two
// 128B-swizzled panels of 64 columns
__device__ __forceinline__ uint32_t tile_off(uint32_t row, uint32_t col)
{
    return (col >> 6) * 8192u + sw128_off(row, col & 63u);
}

// channel factors of block pair (R, I) (I <= R, I != R - 1) at channels c, c + 1
// (bd holds bd[4][128] followed by 1/bd[4][128])
__device__ __forceinline__ float2 pair_factor(const float *bd, int R, int I, int c)
{
    if (I == R) return *reinterpret_cast<const float2 *>(bd + (4 + R) * kDK + c);
    if (I == R - 2) return *reinterpret_cast<const float2 *>(bd + (R - 1) * kDK + c);
    const float2 a = *reinterpret_cast<const float2 *>(bd + 1 * kDK + c);   // (3, 0): bd_1 bd_2
    const float2 b = *reinterpret_cast<const float2 *>(bd + 2 * kDK + c);
    return make_float2(a.x * b.x, a.y * b.y);
}

// softplus(z) = log(1 + e^z) = max(z, 0) + log(1 + e^-|z|), without overflow
__device__ __forceinline__ float softplus_f(float z) { return fmaxf(z, 0.f) + __logf(1.f + __expf(-fabsf(z))); }

// PRO: the input prologue.  q, k arrive raw and are L2-normalised here
// (q / sqrt(sum q^2 + 1e-6) per row), gin holds the bf16 gate
// pre-activation a, the log-decay is g = -exp(A_log[h]) * softplus(a +
// dt_bias) (per channel: bounded below by -5), and betag holds the logits of
// beta = sigmoid(logit).  Otherwise gin holds the fp32 log-decay g and betag
// beta itself.
//
// GDR2: Gated Delta Rule-2 ("Token Mixer I", section "Gated DeltaNet-2",
// subsection "Chunkwise parallel training").  The erase gate b (bf16, layout
// of k) replaces beta on the key side: A[r][i] = sum_c b_rc k_rc k_ic
// exp(G_rc - G_ic), T' = (I + A)^{-1} (no column scaling) and W = T' (b * K<-)
// (the erase-side auxiliary Y); the write gate w (layout of v) gives the
// write-side target Z = w * v, written here for the scan's U = T' Z.  So the
// left operand of A and of W becomes b * Khat; Aqk, Q<-, K_tail and gamma_C
// are those of KDA.
template <bool SCALAR, bool PRO, bool GDR2>
__global__ void __launch_bounds__(kThreads, 2)
ut_prep_kernel(const __nv_bfloat16 *__restrict__ kg, const __nv_bfloat16 *__restrict__ qg,
               const void *__restrict__ gin, const float *__restrict__ betag,
               const float *__restrict__ A_log, const float *__restrict__ dt_bias,
               const __nv_bfloat16 *__restrict__ erg, const __nv_bfloat16 *__restrict__ vg,
               const __nv_bfloat16 *__restrict__ wrg, __nv_bfloat16 *__restrict__ Zout,
               __nv_bfloat16 *__restrict__ Tout,
               __nv_bfloat16 *__restrict__ Aqout, __nv_bfloat16 *__restrict__ Wout, __nv_bfloat16 *__restrict__ Qlo,
               __nv_bfloat16 *__restrict__ Kto, float *__restrict__ gamo, int T_len, int nchunks, int total,
               int n_heads)
{
    static_assert(!(PRO && GDR2), "the fused prologue is for the tied-gate rule");
    extern __shared__ unsigned char prep_raw[];
    // aligned by an offset into the __shared__ array itself, so that the
    // compiler keeps every access through `sm` in the shared state space
    unsigned char *sm = prep_raw + ((1024u - (sm100::smem_u32(prep_raw) & 1023u)) & 1023u);
    float(*sA)[kLdA] = reinterpret_cast<float(*)[kLdA]>(sm + OFF_A);
    float(*sQ)[kLdA] = reinterpret_cast<float(*)[kLdA]>(sm + OFF_AQ);   // Aqk, later Nt
    float(*sU)[16][kLdD] = reinterpret_cast<float(*)[16][kLdD]>(sm + OFF_U);
    float *sBd = reinterpret_cast<float *>(sm + OFF_BD);              // [4][128] bd, then [4][128] 1/bd
    float(*sD)[16][kLdD] = reinterpret_cast<float(*)[16][kLdD]>(sm + OFF_D);
    float *sGc = reinterpret_cast<float *>(sm + OFF_GC);
    const float *gg = static_cast<const float *>(gin);
    const __nv_bfloat16 *ag = static_cast<const __nv_bfloat16 *>(gin);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;   // mma fragment coordinates

    // -W of chunk cw leaves the staging tile in whole 256-byte token rows (16-byte
    // chunks XOR-swizzled by token).  It runs during the next chunk's operand
    // loads, so that their latency covers it; the A tile is next written by
    // that chunk's block products.
    const unsigned char *wstg = sm + OFF_A;
    auto store_w = [&](int cw) {
        __nv_bfloat16 *wdst = Wout + (size_t)cw * kC * kDK;
#pragma unroll
        for (int q = tid; q < kC * 16; q += kThreads) {
            const int r = q >> 4, ck = q & 15;
            *reinterpret_cast<uint4 *>(wdst + r * kDK + 8 * ck) =
                *reinterpret_cast<const uint4 *>(wstg + r * 256 + ((ck ^ (r & 7)) << 4));
        }
    };
    int parity = 0;
    for (int ci = blockIdx.x; ci < total; ci += gridDim.x, parity ^= 1) {
        const int head = ci / nchunks;
        const int t0 = (ci - head * nchunks) * kC;
        const int nrows = min(kC, T_len - t0);
        const size_t row0 = (size_t)head * T_len + t0;   // first token row of this chunk
        if (tid == 0 && ci + (int)gridDim.x < total) {
            // warm L2 with the next chunk's inputs while this one is processed
            const int cn = ci + gridDim.x, hn = cn / nchunks, tn = (cn - hn * nchunks) * kC;
            const int rn = min(kC, T_len - tn);
            const size_t rown = (size_t)hn * T_len + tn;
            bulk_prefetch_l2(kg + rown * kDK, (uint32_t)rn * kDK * 2);
            bulk_prefetch_l2(qg + rown * kDK, (uint32_t)rn * kDK * 2);
            if (!SCALAR) {
                if (PRO) bulk_prefetch_l2(static_cast<const __nv_bfloat16 *>(gin) + rown * kDK, (uint32_t)rn * kDK * 2);
                else bulk_prefetch_l2(static_cast<const float *>(gin) + rown * kDK, (uint32_t)rn * kDK * 4);
            }
            if (GDR2) bulk_prefetch_l2(erg + rown * kDK, (uint32_t)rn * kDK * 2);   // (v, w are read later, once)
        }
        const size_t cbase = (size_t)ci * kC * kC;       // this chunk's T' and Aqk
        // beta alternates between two buffers: the last T' stores of the
        // previous chunk may still read theirs while this chunk starts
        float *sBeta = reinterpret_cast<float *>(sm + OFF_BETA) + kC * parity;

        // ---- operands.  Warp (R, panel) covers rows 16R..16R+15 and the 64
        // channels of one panel; lane = (half, quad): rows 16R + 8 half + 0..7,
        // channels 64 panel + 4 quad + 0..3.
        const int R = warp >> 1, half = lane >> 4;
        const uint32_t c = 64u * (warp & 1) + 4u * (lane & 15);
        const int rbase = 16 * R + 8 * half;
        uint2 kr[8], qr[8];
        uint2 br[GDR2 ? 8 : 1];             // GDR-2 erase gate b
        float4 gv[8];                       // g, then alpha = exp(max(g, -5))
        float2 oa = make_float2(1.f, 1.f), ob = oa;   // alpha product of the other half block
        // 1 / L2 norm of the rows of q, k (prologue; 1 otherwise), kept in
        // shared memory: iq(rr), ik(rr) for this thread's row rbase + rr
        const float *sinv = reinterpret_cast<const float *>(sm + OFF_INV) + (warp * 2 + half) * 16;
        auto iq = [&](int rr) { return PRO ? sinv[rr] : 1.f; };
        auto ik = [&](int rr) { return PRO ? sinv[8 + rr] : 1.f; };
        // beta of row tid (warps 0-1), loaded with the operands so that its
        // latency hides under theirs
        const float beta_ld = (!GDR2 && tid < kC) ? __ldg(betag + row0 + min(tid, nrows - 1)) : 0.f;
        {
            // Unconditional loads from rows clamped into the chunk (a
            // conditional load makes the compiler wait for each one before the
            // next); rows past T are zeroed (k, q) or given g = 0 afterwards.
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) {
                const size_t e = (row0 + min(rbase + rr, nrows - 1)) * kDK + c;
                kr[rr] = __ldg(reinterpret_cast<const uint2 *>(kg + e));
                qr[rr] = __ldg(reinterpret_cast<const uint2 *>(qg + e));
                if (GDR2) br[rr] = __ldg(reinterpret_cast<const uint2 *>(erg + e));
                if (!SCALAR) {
                    if (PRO) {   // a as four bf16, widened; the gate is formed below
                        const uint2 av = __ldg(reinterpret_cast<const uint2 *>(ag + e));
                        gv[rr] = make_float4(__uint_as_float(av.x << 16), __uint_as_float(av.x & 0xffff0000u),
                                             __uint_as_float(av.y << 16), __uint_as_float(av.y & 0xffff0000u));
                    } else {
                        gv[rr] = __ldg(reinterpret_cast<const float4 *>(gg + e));
                    }
                }
            }
            if (ci != (int)blockIdx.x) store_w(ci - (int)gridDim.x);
            if (nrows < kC) {   // only the ragged last chunk of a head (a uniform branch)
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) {
                    if (rbase + rr >= nrows) {
                        kr[rr] = make_uint2(0u, 0u);
                        qr[rr] = make_uint2(0u, 0u);
                        if (GDR2) br[rr] = make_uint2(0u, 0u);
                        if (!SCALAR) gv[rr] = make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                }
            }
            if (PRO) {
                // per-channel log-decay from the pre-activation (rows past T keep g = 0)
                const int hh = head % n_heads;   // A_log, dt_bias are per head h of [B, H]
                if (!SCALAR) {
                    const float A = __expf(__ldg(A_log + hh));
                    const float4 db = __ldg(reinterpret_cast<const float4 *>(dt_bias + (size_t)hh * kDK + c));
#pragma unroll
                    for (int rr = 0; rr < 8; ++rr) {
                        if (rbase + rr < nrows) {
                            gv[rr].x = -A * softplus_f(gv[rr].x + db.x);
                            gv[rr].y = -A * softplus_f(gv[rr].y + db.y);
                            gv[rr].z = -A * softplus_f(gv[rr].z + db.z);
                            gv[rr].w = -A * softplus_f(gv[rr].w + db.w);
                        }
                    }
                }
                // L2 norms of q and k per row: this thread's 4 channels, then the
                // 16 lanes of its half (transpose-reduce: lane v ends with row v & 7
                // of q (v < 8) or k), then the partner warp holding the other 64
                // channels (named barrier of the two warps).
                float ps[16];
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) {
                    const float q0 = __uint_as_float(qr[rr].x << 16), q1 = __uint_as_float(qr[rr].x & 0xffff0000u);
                    const float q2 = __uint_as_float(qr[rr].y << 16), q3 = __uint_as_float(qr[rr].y & 0xffff0000u);
                    const float k0 = __uint_as_float(kr[rr].x << 16), k1 = __uint_as_float(kr[rr].x & 0xffff0000u);
                    const float k2 = __uint_as_float(kr[rr].y << 16), k3 = __uint_as_float(kr[rr].y & 0xffff0000u);
                    ps[rr] = q0 * q0 + q1 * q1 + q2 * q2 + q3 * q3;
                    ps[8 + rr] = k0 * k0 + k1 * k1 + k2 * k2 + k3 * k3;
                }
                const int v = lane & 15;
#pragma unroll
                for (int w = 8; w >= 1; w >>= 1) {
                    // keep the half of the values whose index has bit w equal to this lane's
#pragma unroll
                    for (int j = 0; j < w; ++j) {
                        const bool up = (v & w) != 0;
                        const float send = up ? ps[j] : ps[j + w];
                        const float got = __shfl_xor_sync(0xffffffffu, send, w);
                        ps[j] = (up ? ps[j + w] : ps[j]) + got;
                    }
                }
                float *nrm = reinterpret_cast<float *>(sm + OFF_NRM);
                nrm[(warp * 2 + half) * 16 + v] = ps[0];
                switch (R) {   // the two warps of row block R: literal barrier ids 1..4
                case 0: asm volatile("bar.sync 1, 64;" ::: "memory"); break;
                case 1: asm volatile("bar.sync 2, 64;" ::: "memory"); break;
                case 2: asm volatile("bar.sync 3, 64;" ::: "memory"); break;
                default: asm volatile("bar.sync 4, 64;" ::: "memory"); break;
                }
                const float tot = nrm[(warp * 2 + half) * 16 + v] + nrm[((warp ^ 1) * 2 + half) * 16 + v];
                reinterpret_cast<float *>(sm + OFF_INV)[(warp * 2 + half) * 16 + v] = rsqrtf(tot + 1e-6f);
                __syncwarp();
            }
            if (tid < kC) {
                if (GDR2) {   // the gates sit in the operands; T' is (I + A)^{-1} itself
                    sBeta[tid] = tid < nrows ? 1.f : 0.f;
                } else {
                    sBeta[tid] = tid < nrows ? (PRO ? 1.f / (1.f + __expf(-beta_ld)) : beta_ld) : 0.f;
                }
            }
            if (SCALAR && warp == 0) {
                // inclusive scan of the scalar log-decay over the chunk (2 values per lane)
                auto gate_at = [&](int t) -> float {
                    if (t >= nrows) return 0.f;
                    if (!PRO) return __ldg(gg + row0 + t);
                    const int hh = head % n_heads;
                    const float z = __bfloat162float(ag[row0 + t]) + __ldg(dt_bias + hh);
                    return -__expf(__ldg(A_log + hh)) * softplus_f(z);
                };
                const float a0 = gate_at(2 * lane);
                const float a1 = gate_at(2 * lane + 1);
                float sum = a0 + a1;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float o = __shfl_up_sync(0xffffffffu, sum, off);
                    if (lane >= off) sum += o;
                }
                sGc[2 * lane + 1] = sum;
                sGc[2 * lane] = sum - a1;
            }
            if (SCALAR) {
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) {
                    const uint32_t off = tile_off(rbase + rr, c);
                    if (PRO) {
                        const float2 fk = make_float2(ik(rr), ik(rr)), fq = make_float2(iq(rr), iq(rr));
                        *reinterpret_cast<uint2 *>(sm + OFF_K + off) = make_uint2(scale2p(kr[rr].x, fk), scale2p(kr[rr].y, fk));
                        *reinterpret_cast<uint2 *>(sm + OFF_Q + off) = make_uint2(scale2p(qr[rr].x, fq), scale2p(qr[rr].y, fq));
                    } else if (GDR2) {   // left operand b * k, right operand k
                        *reinterpret_cast<uint2 *>(sm + OFF_K + off) =
                            make_uint2(scale2p(kr[rr].x, unpack2(br[rr].x)), scale2p(kr[rr].y, unpack2(br[rr].y)));
                        *reinterpret_cast<uint2 *>(sm + OFF_KC + off) = kr[rr];
                        *reinterpret_cast<uint2 *>(sm + OFF_Q + off) = qr[rr];
                    } else {
                        *reinterpret_cast<uint2 *>(sm + OFF_K + off) = kr[rr];
                        *reinterpret_cast<uint2 *>(sm + OFF_Q + off) = qr[rr];
                    }
                }
            } else {
                // alpha = exp(max(g, -5)) and the product over this thread's 8 rows
                const float2 log2e = make_float2(1.4426950408889634f, 1.4426950408889634f);
                float2 la = make_float2(1.f, 1.f), lb = make_float2(1.f, 1.f);   // channels (0,1), (2,3)
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) {
                    float2 x = fmul2(make_float2(fmaxf(gv[rr].x, kGateMin), fmaxf(gv[rr].y, kGateMin)), log2e);
                    float2 y = fmul2(make_float2(fmaxf(gv[rr].z, kGateMin), fmaxf(gv[rr].w, kGateMin)), log2e);
                    gv[rr] = make_float4(exp2f(x.x), exp2f(x.y), exp2f(y.x), exp2f(y.y));
                    la = fmul2(la, make_float2(gv[rr].x, gv[rr].y));
                    lb = fmul2(lb, make_float2(gv[rr].z, gv[rr].w));
                }
                // the other half of the 16-row block (lane ^ 16)
                oa = make_float2(__shfl_xor_sync(0xffffffffu, la.x, 16), __shfl_xor_sync(0xffffffffu, la.y, 16));
                ob = make_float2(__shfl_xor_sync(0xffffffffu, lb.x, 16), __shfl_xor_sync(0xffffffffu, lb.y, 16));
                // Khat, Qhat: inclusive running product from the block start
                float2 pa = half ? oa : make_float2(1.f, 1.f), pb = half ? ob : make_float2(1.f, 1.f);
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) {
                    const uint32_t off = tile_off(rbase + rr, c);
                    pa = fmul2(pa, make_float2(gv[rr].x, gv[rr].y));
                    pb = fmul2(pb, make_float2(gv[rr].z, gv[rr].w));
                    const float2 nk = make_float2(ik(rr), ik(rr)), nq = make_float2(iq(rr), iq(rr));
                    if (GDR2)   // Ehat = b * Khat
                        *reinterpret_cast<uint2 *>(sm + OFF_K + off) =
                            make_uint2(scale2p(kr[rr].x, fmul2(pa, unpack2(br[rr].x))),
                                       scale2p(kr[rr].y, fmul2(pb, unpack2(br[rr].y))));
                    else
                        *reinterpret_cast<uint2 *>(sm + OFF_K + off) =
                            make_uint2(scale2p(kr[rr].x, PRO ? fmul2(pa, nk) : pa), scale2p(kr[rr].y, PRO ? fmul2(pb, nk) : pb));
                    *reinterpret_cast<uint2 *>(sm + OFF_Q + off) =
                        make_uint2(scale2p(qr[rr].x, PRO ? fmul2(pa, nq) : pa), scale2p(qr[rr].y, PRO ? fmul2(pb, nq) : pb));
                }
                if (half) {   // pa, pb now hold bd_R
                    *reinterpret_cast<float4 *>(sBd + R * kDK + c) = make_float4(pa.x, pa.y, pb.x, pb.y);
                    *reinterpret_cast<float4 *>(sBd + (4 + R) * kDK + c) =
                        make_float4(1.f / pa.x, 1.f / pa.y, 1.f / pb.x, 1.f / pb.y);
                }
                // Kchk: exclusive running product to the block end
                pa = half ? make_float2(1.f, 1.f) : oa;
                pb = half ? make_float2(1.f, 1.f) : ob;
#pragma unroll
                for (int rr = 7; rr >= 0; --rr) {
                    const uint32_t off = tile_off(rbase + rr, c);
                    const float2 nk = make_float2(ik(rr), ik(rr));
                    *reinterpret_cast<uint2 *>(sm + OFF_KC + off) =
                        make_uint2(scale2p(kr[rr].x, PRO ? fmul2(pa, nk) : pa), scale2p(kr[rr].y, PRO ? fmul2(pb, nk) : pb));
                    pa = fmul2(pa, make_float2(gv[rr].x, gv[rr].y));
                    pb = fmul2(pb, make_float2(gv[rr].z, gv[rr].w));
                }
            }
        }
        __syncthreads();

        // ---- chunk-relative operands of the state scan, G counted from the
        // chunk start:
        //   Q<-_r = q_r exp(G_r)       in the layout of k ([B, H, T, 128] bf16)
        //   K_tail_r = k_r exp(G_C - G_r)   transposed per chunk ([chunks][128][64])
        // and gamma_C = exp(G_C) per key channel (fp32, [B H chunks][128]).
        // Formed in fp32 from the registers above, with the block decays bd_J.
        // (K<-_r = k_r exp(G_r) is only needed inside W = T' K<-, formed below.)
        {
            const size_t e0 = row0 * kDK + c;
            uint2 kt[8];   // K_tail of this thread's 8 rows x 4 channels (zero past T)
            if (!SCALAR) {
                float2 Fa = make_float2(1.f, 1.f), Fb = Fa, Ba = Fa, Bb = Fa;
#pragma unroll
                for (int J = 0; J < 4; ++J) {
                    const float4 bdj = *reinterpret_cast<const float4 *>(sBd + J * kDK + c);
                    if (J < R) {
                        Fa = fmul2(Fa, make_float2(bdj.x, bdj.y));
                        Fb = fmul2(Fb, make_float2(bdj.z, bdj.w));
                    } else if (J > R) {
                        Ba = fmul2(Ba, make_float2(bdj.x, bdj.y));
                        Bb = fmul2(Bb, make_float2(bdj.z, bdj.w));
                    }
                }
                float2 pa = half ? fmul2(Fa, oa) : Fa, pb = half ? fmul2(Fb, ob) : Fb;
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) {
                    pa = fmul2(pa, make_float2(gv[rr].x, gv[rr].y));
                    pb = fmul2(pb, make_float2(gv[rr].z, gv[rr].w));
                    if (rbase + rr < nrows) {
                        const size_t e = e0 + (size_t)(rbase + rr) * kDK;
                        const float2 nq = make_float2(iq(rr), iq(rr));
                        *reinterpret_cast<uint2 *>(Qlo + e) =
                            make_uint2(scale2p(qr[rr].x, PRO ? fmul2(pa, nq) : pa), scale2p(qr[rr].y, PRO ? fmul2(pb, nq) : pb));
                    }
                }
                if (R == 0 && half == 0) {   // gamma_C = product of the four block decays
                    const float4 b0 = *reinterpret_cast<const float4 *>(sBd + c);
                    const float2 ga = fmul2(Ba, make_float2(b0.x, b0.y)), gb = fmul2(Bb, make_float2(b0.z, b0.w));
                    *reinterpret_cast<float4 *>(gamo + (size_t)ci * kDK + c) = make_float4(ga.x, ga.y, gb.x, gb.y);
                }
                pa = half ? Ba : fmul2(Ba, oa);
                pb = half ? Bb : fmul2(Bb, ob);
#pragma unroll
                for (int rr = 7; rr >= 0; --rr) {
                    const float2 nk = make_float2(ik(rr), ik(rr));
                    kt[rr] = rbase + rr < nrows ? make_uint2(scale2p(kr[rr].x, PRO ? fmul2(pa, nk) : pa),
                                                             scale2p(kr[rr].y, PRO ? fmul2(pb, nk) : pb))
                                                : make_uint2(0u, 0u);
                    pa = fmul2(pa, make_float2(gv[rr].x, gv[rr].y));
                    pb = fmul2(pb, make_float2(gv[rr].z, gv[rr].w));
                }
            } else {
                const float Gl = sGc[kC - 1];   // rows past T carry g = 0
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) {
                    const int r = rbase + rr;
                    if (r < nrows) {
                        const float ef = __expf(sGc[r]), et = __expf(Gl - sGc[r]);
                        const float2 fe = make_float2(ef * iq(rr), ef * iq(rr)), ft = make_float2(et * ik(rr), et * ik(rr));
                        const size_t e = e0 + (size_t)r * kDK;
                        *reinterpret_cast<uint2 *>(Qlo + e) = make_uint2(scale2p(qr[rr].x, fe), scale2p(qr[rr].y, fe));
                        kt[rr] = make_uint2(scale2p(kr[rr].x, ft), scale2p(kr[rr].y, ft));
                    } else {
                        kt[rr] = make_uint2(0u, 0u);
                    }
                }
                if (R == 0 && half == 0) {
                    const float gl = __expf(Gl);
                    *reinterpret_cast<float4 *>(gamo + (size_t)ci * kDK + c) = make_float4(gl, gl, gl, gl);
                }
            }
            // K_tail^T [128 channels][64 tokens] per chunk, the operand layout of
            // the scan's state update: per channel, this thread's 8 consecutive
            // tokens are one 16-byte store (the two halves of a warp fill whole
            // 32-byte sectors); the tokens past T of a ragged chunk are zeros.
            {
                __nv_bfloat16 *kdst = Kto + ((size_t)ci * kDK + c) * kC + rbase;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t sel = (j & 1) ? 0x7632u : 0x5410u;   // high or low bf16 of each pair
                    uint32_t w[4];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const uint32_t a = (j < 2) ? kt[2 * m].x : kt[2 * m].y;
                        const uint32_t b = (j < 2) ? kt[2 * m + 1].x : kt[2 * m + 1].y;
                        w[m] = __byte_perm(a, b, sel);
                    }
                    *reinterpret_cast<uint4 *>(kdst + (size_t)j * kC) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            if (GDR2) {
                // write-side target Z = w * v (d_v = 128 channels, the layout of v)
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) {
                    if (rbase + rr < nrows) {
                        const size_t e = e0 + (size_t)(rbase + rr) * kDK;
                        const uint2 vv = __ldg(reinterpret_cast<const uint2 *>(vg + e));
                        const uint2 ww = __ldg(reinterpret_cast<const uint2 *>(wrg + e));
                        *reinterpret_cast<uint2 *>(Zout + e) =
                            make_uint2(scale2p(vv.x, unpack2(ww.x)), scale2p(vv.y, unpack2(ww.y)));
                    }
                }
            }
        }

        // ---- block products on tensor cores: 10 block pairs over 8 warps, each
        // pair gives both A and Aqk (the right operand and its scaling are shared)
        {
            const uint32_t left_k = smem_u32(sm + OFF_K), left_q = smem_u32(sm + OFF_Q);
            const uint32_t right = (SCALAR && !GDR2) ? left_k : smem_u32(sm + OFF_KC);
            for (int p = warp; p < 10; p += 8) {
                // pairs (R, I), I <= R, in row-major order of the lower block triangle
                const int R = p < 1 ? 0 : p < 3 ? 1 : p < 6 ? 2 : 3;
                const int I = p - R * (R + 1) / 2;
                const bool scaled = !SCALAR && I != R - 1;
                float acc[2][2][4] = {};
#pragma unroll
                for (int ks = 0; ks < kDK / 16; ++ks) {
                    uint32_t ak[4], aq[4], b[4];
                    const uint32_t aoff = tile_off(R * 16 + (lane & 15), ks * 16 + (lane >> 4) * 8);
                    ldsm_x4(ak, left_k + aoff);
                    ldsm_x4(aq, left_q + aoff);
                    ldsm_x4(b, right + tile_off(I * 16 + (lane & 7) + ((lane >> 4) << 3),
                                                ks * 16 + ((lane >> 3) & 1) * 8));
                    if (scaled) {
                        const int c = ks * 16 + 2 * t;
                        const float2 f0 = pair_factor(sBd, R, I, c), f8 = pair_factor(sBd, R, I, c + 8);
                        b[0] = scale2p(b[0], f0);
                        b[1] = scale2p(b[1], f8);
                        b[2] = scale2p(b[2], f0);
                        b[3] = scale2p(b[3], f8);
                    }
                    mma16816(acc[0][0], ak, b[0], b[1]);
                    mma16816(acc[0][1], ak, b[2], b[3]);
                    mma16816(acc[1][0], aq, b[0], b[1]);
                    mma16816(acc[1][1], aq, b[2], b[3]);
                }
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int r = R * 16 + g + h * 8;
                        const int i = I * 16 + nt * 8 + 2 * t;
                        float va[2], vq[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            va[e] = acc[0][nt][2 * h + e];
                            vq[e] = acc[1][nt][2 * h + e];
                            if (SCALAR) {
                                const float dec = __expf(sGc[r] - sGc[i + e]);   // masked below when i > r
                                va[e] *= dec;
                                vq[e] *= dec;
                            }
                            va[e] = (i + e < r) ? sBeta[r] * va[e] : 0.f;
                            vq[e] = (i + e <= r) ? vq[e] : 0.f;
                        }
                        *reinterpret_cast<float2 *>(&sA[r][i]) = make_float2(va[0], va[1]);
                        *reinterpret_cast<float2 *>(&sQ[r][i]) = make_float2(vq[0], vq[1]);
                    }
            }
        }
        __syncthreads();

        if (tid < 64) {
            // D_b = N_bb^{-1}: thread = (block b, column jc), forward substitution
            const int base = (tid >> 4) * 16, jc = tid & 15;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) x[r] = (r == jc) ? 1.f : 0.f;
            // right-looking: once x[m] is final, remove it from every later row
#pragma unroll
            for (int m = 0; m < 15; ++m)
#pragma unroll
                for (int r = m + 1; r < 16; ++r) x[r] = fmaf(-sA[base + r][base + m], x[m], x[r]);
#pragma unroll
            for (int r = 0; r < 16; ++r) sD[tid >> 4][r][jc] = x[r];
        } else {
            // Aqk out (bf16 row-major): blocks above the diagonal are zero
            for (int task = tid - 64; task < kC * 8; task += kThreads - 64) {
                const int r = task >> 3, g8 = task & 7;
                uint4 o = make_uint4(0u, 0u, 0u, 0u);
                if ((g8 >> 1) <= (r >> 4)) {
                    const float4 a0 = *reinterpret_cast<const float4 *>(&sQ[r][8 * g8]);
                    const float4 a1 = *reinterpret_cast<const float4 *>(&sQ[r][8 * g8 + 4]);
                    o.x = pack2(a0.x, a0.y);
                    o.y = pack2(a0.z, a0.w);
                    o.z = pack2(a1.x, a1.y);
                    o.w = pack2(a1.z, a1.w);
                }
                *reinterpret_cast<uint4 *>(Aqout + cbase + r * kC + 8 * g8) = o;
            }
        }
        __syncthreads();

        // T' (bf16) is also kept in shared memory as the left operand of
        // W = T' K<-; with a scalar gate its columns carry exp(G_r) there, so
        // that W = (T' Diag(exp(G))) K.
        __nv_bfloat16(*sT)[kLdT] = reinterpret_cast<__nv_bfloat16(*)[kLdT]>(sm + OFF_Q);
        auto tcol = [&](int col) { return SCALAR ? sBeta[col] * __expf(sGc[col]) : sBeta[col]; };
        // T' block (i, j) = U_ij Diag(beta_j) from a 16 x 16 accumulator fragment
        auto store_t = [&](const float (&c)[2][4], int i, int j) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int col = 16 * j + 8 * nt + 2 * t;
                const float b0 = sBeta[col], b1 = sBeta[col + 1];
                __nv_bfloat16 *dst = Tout + cbase + (size_t)(16 * i + g) * kC + col;
                *reinterpret_cast<uint32_t *>(dst) = pack2(c[nt][0] * b0, c[nt][1] * b1);
                *reinterpret_cast<uint32_t *>(dst + 8 * kC) = pack2(c[nt][2] * b0, c[nt][3] * b1);
                const float s0 = SCALAR ? tcol(col) : b0, s1 = SCALAR ? tcol(col + 1) : b1;
                *reinterpret_cast<uint32_t *>(&sT[16 * i + g][col]) = pack2(c[nt][0] * s0, c[nt][1] * s1);
                *reinterpret_cast<uint32_t *>(&sT[16 * i + g + 8][col]) = pack2(c[nt][2] * s0, c[nt][3] * s1);
            }
        };
        auto store_s = [&](const float (&c)[2][4], float (*dst)[kLdD]) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                *reinterpret_cast<float2 *>(&dst[g][8 * nt + 2 * t]) = make_float2(c[nt][0], c[nt][1]);
                *reinterpret_cast<float2 *>(&dst[g + 8][8 * nt + 2 * t]) = make_float2(c[nt][2], c[nt][3]);
            }
        };
        float acc[2][4] = {};
        if (warp < 6) {
            // Nt_im = D_i A_im for the six blocks below the diagonal (into sQ)
            const int i = warp < 1 ? 1 : warp < 3 ? 2 : 3;
            const int m = warp - i * (i - 1) / 2;
            float nt_[2][4] = {};
            mm16_sub(nt_, &sD[i][0][0], kLdD, &sA[16 * i][16 * m], kLdA, g, t);   // = -D_i A_im
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) nt_[nt][e] = -nt_[nt][e];
            float(*dst)[kLdA] = reinterpret_cast<float(*)[kLdA]>(&sQ[16 * i][16 * m]);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                *reinterpret_cast<float2 *>(&dst[g][8 * nt + 2 * t]) = make_float2(nt_[nt][0], nt_[nt][1]);
                *reinterpret_cast<float2 *>(&dst[g + 8][8 * nt + 2 * t]) = make_float2(nt_[nt][2], nt_[nt][3]);
            }
        }
        // diagonal blocks D_i Diag(beta) and the zero blocks above them, 8
        // columns of one row per task, two tasks per thread of every warp (the
        // six warps above join after their product)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int task = tid + kThreads * j;
            const int r = task >> 3, g8 = task & 7, i = r >> 4, jb = g8 >> 1;
            if (jb >= i) {
                uint4 o = make_uint4(0u, 0u, 0u, 0u), os = o;
                if (jb == i) {
                    const int ch = 8 * (g8 & 1), cl = 16 * jb + ch;
                    const float4 d0 = *reinterpret_cast<const float4 *>(&sD[i][r & 15][ch]);
                    const float4 d1 = *reinterpret_cast<const float4 *>(&sD[i][r & 15][ch + 4]);
                    o.x = pack2(d0.x * sBeta[cl + 0], d0.y * sBeta[cl + 1]);
                    o.y = pack2(d0.z * sBeta[cl + 2], d0.w * sBeta[cl + 3]);
                    o.z = pack2(d1.x * sBeta[cl + 4], d1.y * sBeta[cl + 5]);
                    o.w = pack2(d1.z * sBeta[cl + 6], d1.w * sBeta[cl + 7]);
                    if (SCALAR) {
                        os.x = pack2(d0.x * tcol(cl + 0), d0.y * tcol(cl + 1));
                        os.y = pack2(d0.z * tcol(cl + 2), d0.w * tcol(cl + 3));
                        os.z = pack2(d1.x * tcol(cl + 4), d1.y * tcol(cl + 5));
                        os.w = pack2(d1.z * tcol(cl + 6), d1.w * tcol(cl + 7));
                    } else {
                        os = o;
                    }
                }
                *reinterpret_cast<uint4 *>(Tout + cbase + r * kC + 8 * g8) = o;
                *reinterpret_cast<uint4 *>(&sT[r][8 * g8]) = os;
            }
        }
        __syncthreads();
        // first products of every block below the diagonal
        if (warp < 6) {
            // warp -> (i, j): (1,0) (2,1) (3,2) (2,0) (3,1) (3,0)
            const int i = warp < 3 ? warp + 1 : (warp == 3 ? 2 : 3);
            const int j = warp < 3 ? warp : (warp == 4 ? 1 : 0);
            mm16_sub(acc, &sQ[16 * i][16 * j], kLdA, &sD[j][0][0], kLdD, g, t);   // -Nt_ij D_j
            if (warp < 3) {
                store_t(acc, i, j);
                if (warp < 2) store_s(acc, sU[warp]);   // U_10, U_21
            }
        }
        __syncthreads();
        if (warp == 3) {          // U_20 = -Nt_20 D_0 - Nt_21 U_10
            mm16_sub(acc, &sQ[32][16], kLdA, &sU[0][0][0], kLdD, g, t);
            store_t(acc, 2, 0);
            store_s(acc, sU[2]);
        } else if (warp == 4) {   // U_31 = -Nt_31 D_1 - Nt_32 U_21
            mm16_sub(acc, &sQ[48][32], kLdA, &sU[1][0][0], kLdD, g, t);
            store_t(acc, 3, 1);
        } else if (warp == 5) {   // U_30 so far: -Nt_30 D_0 - Nt_31 U_10
            mm16_sub(acc, &sQ[48][16], kLdA, &sU[0][0][0], kLdD, g, t);
        }
        __syncthreads();
        if (warp == 5) {          // U_30 -= Nt_32 U_20
            mm16_sub(acc, &sQ[48][32], kLdA, &sU[2][0][0], kLdD, g, t);
            store_t(acc, 3, 0);
        }
        __syncthreads();

        // ---- W = T' K<- for the state scan, stored negated and token-major,
        // -W [64 tokens][128 channels] (the layout of Q<-), so that the scan takes
        // -S W^T and S Q<-^T in one product.
        // Per-channel gate: K<-_r = Khat_r * F_R with F_R = prod_{J<R} bd_J (row r
        // in block R), so W = sum_R (T'[:, block R] Khat_R) Diag(F_R): one fp32
        // accumulator per block, combined after the products.  Scalar gate: the
        // decay sits in T' (above) and Khat is k.  Warp w owns channels
        // 16w..16w+15 (two 8-channel tiles), all 64 tokens, in 4 token blocks.
        // The fragments go to the staging tile (conflict free both ways), stored
        // out during the next chunk's loads (or after the last chunk).
        {
            const int c0 = 16 * warp;
            const uint32_t khat = smem_u32(sm + OFF_K);
#pragma unroll
            for (int ct = 0; ct < 2; ++ct) {
                const int cs = c0 + 8 * ct;                  // first channel of this tile
                float2 fr[4];                                // F_R at channels cs + 2t, + 1
                fr[0] = make_float2(1.f, 1.f);
#pragma unroll
                for (int R = 1; R < 4; ++R) {
                    const float2 bdp = SCALAR ? make_float2(1.f, 1.f)
                                              : *reinterpret_cast<const float2 *>(sBd + (R - 1) * kDK + cs + 2 * t);
                    fr[R] = make_float2(fr[R - 1].x * bdp.x, fr[R - 1].y * bdp.y);
                }
                // B fragments (Khat rows of block R, channels cs..cs+7), shared by all token blocks
                uint32_t bf[4][2];
#pragma unroll
                for (int R = 0; R < 4; ++R) {
                    uint32_t r4[4];
                    ldsm_x4_trans(r4, khat + tile_off(16 * R + (lane & 15), cs));
                    bf[R][0] = r4[0];
                    bf[R][1] = r4[1];
                }
#pragma unroll
                for (int I = 0; I < 4; ++I) {
                    float w4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int R = 0; R <= I; ++R) {
                        uint32_t a[4];
                        ldsm_x4(a, smem_u32(&sT[16 * I + (lane & 15)][16 * R + (lane >> 4) * 8]));
                        float accR[4] = {0.f, 0.f, 0.f, 0.f};
                        mma16816(accR, a, bf[R][0], bf[R][1]);
                        w4[0] = fmaf(accR[0], fr[R].x, w4[0]);
                        w4[1] = fmaf(accR[1], fr[R].y, w4[1]);
                        w4[2] = fmaf(accR[2], fr[R].x, w4[2]);
                        w4[3] = fmaf(accR[3], fr[R].y, w4[3]);
                    }
                    // fragment: tokens 16I + g (+8), channels cs + 2t, + 1
                    const int r0 = 16 * I + g, ck = cs >> 3;
                    unsigned char *ws = sm + OFF_A;
                    *reinterpret_cast<uint32_t *>(ws + r0 * 256 + ((ck ^ (r0 & 7)) << 4) + 4 * t) = pack2(-w4[0], -w4[1]);
                    *reinterpret_cast<uint32_t *>(ws + (r0 + 8) * 256 + ((ck ^ (r0 & 7)) << 4) + 4 * t) =
                        pack2(-w4[2], -w4[3]);
                }
            }
        }
        // the next chunk overwrites Khat and T', and stores the staged -W
        __syncthreads();
    }
    // the -W of this CTA's last chunk (staged before the last barrier above)
    if ((int)blockIdx.x < total)
        store_w((int)blockIdx.x + ((total - 1 - (int)blockIdx.x) / (int)gridDim.x) * (int)gridDim.x);
}

int sm_count()
{
    static int counts[64];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (counts[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        counts[dev] = n;
    }
    return counts[dev];
}

}  // namespace

cudaError_t launch_ut_prep(const ChunkArgs &a, const TcWorkspace &w, cudaStream_t stream)
{
    const int nchunks = (a.T + kC - 1) / kC;
    const long long total = (long long)a.B * a.H * nchunks;
    if (total == 0) return cudaSuccess;
    if (total > 0x7fffffffLL) return cudaErrorInvalidValue;
    const long long slots = 2LL * sm_count();   // two resident CTAs per SM
    const int grid = (int)(total < slots ? total : slots);
    auto kern = a.gdr2       ? (a.scalar_gate ? ut_prep_kernel<true, false, true> : ut_prep_kernel<false, false, true>)
                : a.prologue ? (a.scalar_gate ? ut_prep_kernel<true, true, false> : ut_prep_kernel<false, true, false>)
                             : (a.scalar_gate ? ut_prep_kernel<true, false, false> : ut_prep_kernel<false, false, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, SMEM_ALLOC, stream>>>((const __nv_bfloat16 *)a.k, (const __nv_bfloat16 *)a.q,
                                                 (const void *)a.g, a.beta, a.A_log, a.dt_bias,
                                                 (const __nv_bfloat16 *)a.erase, (const __nv_bfloat16 *)a.v,
                                                 (const __nv_bfloat16 *)a.write, w.Z, w.T, w.Aqk, w.W,
                                                 w.Ql, w.Kt, w.gam, a.T, nchunks,
                                                 (int)total, a.H);
    return cudaGetLastError();
}

}  // namespace gdr
