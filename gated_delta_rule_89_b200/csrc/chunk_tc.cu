// Tensor-core chunked forward of the gated delta rule (bf16 q/k/v, fp32 state,
// d_k = d_v = 128, C = 64) on sm_100a.
//
// Two kernels per call:
//   1. ut_prep (ut_prep.cu): every chunk of every head in parallel -> the
//      UT-transform matrix T' = (I + A)^{-1} Diag(beta) and the masked
//      intra-chunk matrix Aqk, bf16, into the workspace.
//   2. chunk_scan (this file): one CTA per (b, h) walks the chunks in order.
//      The fp32 state S [d_v x d_k] lives in tensor memory for the whole
//      sequence.  Per chunk, with G the cumulative log-decay, K<- = K*exp(G),
//      Q<- = Q*exp(G), K_tail = K*exp(G_C - G) and gamma_C = exp(G_C):
//        W^T     = K<-^T T'^T                (= (T' K<-)^T)
//        V_new^T = V^T T'^T - S W^T          (U^T, then -S W^T accumulated)
//        O^T     = S Q<-^T + V_new^T Aqk^T
//        S       = S Diag(gamma_C) + V_new^T K_tail
//      which is the chunk state update and chunk output of "Reading notes:
//      Kimi Delta Attention" (mzeromiko), section 4, and of "Token Mixer I",
//      section "Kimi Delta Attention: Improving Delta Rule with Fine-grained
//      Gating", in the d_v x d_k orientation.  Every product is one
//      tcgen05.mma chain with M = 128 (rows of S, or key channels), fp32
//      accumulators in TMEM; inputs arrive by TMA with 128-byte swizzle and
//      the same tiles serve as K-major or MN-major operands.
//
// Warp roles (320 threads):
//   warp 0      TMA producer (one lane)
//   warp 1      TMEM allocation and the MMA issuer (one lane)
//   warps 2-5   "E": the gate products exp(G) and exp(G_C - G) (running
//               products of alpha = exp(g)), the scaled operands K<-, Q<-
//               (in place over the TMA tiles) and K_tail, and the output
//               epilogue (TMEM -> bf16 -> global)
//   warps 6-9   "M": the conversions on the sequential path: W^T (TMEM) ->
//               W (bf16 smem), S -> bf16 S plus S*gamma_C back into TMEM,
//               V_new^T (TMEM) -> bf16 smem
// Every wait is bounded (about a second); on timeout the kernel records
// GDR_ERR_TIMEOUT in a device status word, lets the copies and MMAs it
// issued finish, frees its tensor memory and returns.
#include <cuda.h>
#include <mutex>

#include "gdr_internal.cuh"
#include "sm100_ptx.cuh"

namespace gdr {

__device__ int g_device_status;   // 0 = OK, else the first gdr_status a kernel recorded

cudaError_t launch_ut_prep(const ChunkArgs &a, __nv_bfloat16 *Tout, __nv_bfloat16 *Aqout, cudaStream_t stream);

namespace {

using namespace sm100;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kThreads = 320;
constexpr long long kWaitBudget = 2000000000LL;   // clock cycles per wait (~1 s)

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_G = 0;                      // [64][128] fp32 gate tile          32 KB
constexpr uint32_t OFF_K = OFF_G + 32768;          // 2 x k -> K<-  (2 panels x 8 KB)   2 x 16 KB
constexpr uint32_t OFF_Q = OFF_K + 2 * 16384;      // 2 x q -> Q<-                      2 x 16 KB
constexpr uint32_t OFF_V = OFF_Q + 2 * 16384;      // v (2 panels)                      16 KB
constexpr uint32_t OFF_T = OFF_V + 16384;          // T' (1 panel)                      8 KB
constexpr uint32_t OFF_AQ = OFF_T + 8192;          // 2 x Aqk                           2 x 8 KB
constexpr uint32_t OFF_KT = OFF_AQ + 2 * 8192;     // K_tail (2 panels)                 16 KB
constexpr uint32_t OFF_W = OFF_KT + 16384;         // W, MN-major [128 ch x 64 tok]     16 KB
constexpr uint32_t OFF_S = OFF_W + 16384;          // bf16 S (2 panels x 16 KB)         32 KB
constexpr uint32_t OFF_VN = OFF_S + 32768;         // V_new^T (1 panel, 128 rows)       16 KB
constexpr uint32_t OFF_GAM = OFF_VN + 16384;       // gamma_C ring [4][128] fp32        2 KB
constexpr uint32_t OFF_BAR = OFF_GAM + 2048;       // mbarriers, TMEM slot, abort flag
constexpr uint32_t SMEM_USED = OFF_BAR + 512;
constexpr uint32_t SMEM_ALLOC = SMEM_USED + 1024;  // alignment slack
static_assert(SMEM_ALLOC <= 232448, "dynamic shared memory above the 227 KB per-block limit");

// TMEM columns (fp32)
constexpr uint32_t TM_S = 0;      // state S_n, 128 columns (written only by the conversion warps)
constexpr uint32_t TM_D = 128;    // state increment V_new^T K_tail of the last chunk, 128 columns
constexpr uint32_t TM_W = 256;    // W^T, 64 columns
constexpr uint32_t TM_V = 320;    // V_new^T accumulator, 64 columns
constexpr uint32_t TM_O = 384;    // O^T accumulators, 2 x 64 columns
constexpr uint32_t TM_COLS = 512;

enum Bar {
    B_FULL_G, B_EMPTY_G,
    B_FULL_K, B_FULL_K1, B_EMPTY_K, B_EMPTY_K1,
    B_FULL_Q, B_FULL_Q1, B_EMPTY_Q, B_EMPTY_Q1,
    B_FULL_V, B_EMPTY_V, B_FULL_T, B_EMPTY_T,
    B_FULL_AQ, B_FULL_AQ1, B_EMPTY_AQ, B_EMPTY_AQ1,
    B_KQ_READY, B_KQ_READY1, B_KT_READY, B_KT_FREE,
    B_WT_FULL, B_WT_EMPTY, B_W_READY, B_W_FREE,
    B_S_READY, B_S_FULL, B_X_FULL, B_VN_READY,
    B_VACC_EMPTY, B_O_FULL, B_O_FULL1, B_OACC_EMPTY, B_OACC_EMPTY1,
    B_XCH, B_XCH1,
    B_FINAL,
    B_COUNT
};
static_assert(8 * B_COUNT + 8 <= 512, "barrier area");

struct Maps {
    CUtensorMap k, q, v, g, t, aq;
};

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_device_status, 0, code); }

// Optional phase timestamps of block 0 (SM clock), compiled only with -DGDR_TRACE.
#ifdef GDR_TRACE
__device__ long long g_trace[16][1024];
#define GDR_TRACE_AT(ev, n)                                                   \
    do {                                                                      \
        if (blockIdx.x == 0 && (n) < 1024) g_trace[(ev)][(n)] = clock64();    \
    } while (0)
#else
#define GDR_TRACE_AT(ev, n) \
    do {                    \
    } while (0)
#endif

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Eight bf16 (one 16-byte chunk) times eight fp32 factors, rounded back to bf16.
__device__ __forceinline__ uint4 scale8(uint4 v, const float (&f)[8])
{
    uint4 o;
    o.x = pack_bf16(__uint_as_float(v.x << 16) * f[0], __uint_as_float(v.x & 0xffff0000u) * f[1]);
    o.y = pack_bf16(__uint_as_float(v.y << 16) * f[2], __uint_as_float(v.y & 0xffff0000u) * f[3]);
    o.z = pack_bf16(__uint_as_float(v.z << 16) * f[4], __uint_as_float(v.z & 0xffff0000u) * f[5]);
    o.w = pack_bf16(__uint_as_float(v.w << 16) * f[6], __uint_as_float(v.w & 0xffff0000u) * f[7]);
    return o;
}

// Sixteen fp32 TMEM words -> two 16-byte bf16 chunks.
__device__ __forceinline__ void pack16(const uint32_t (&r)[16], uint4 &lo, uint4 &hi)
{
    lo.x = pack_bf16(__uint_as_float(r[0]), __uint_as_float(r[1]));
    lo.y = pack_bf16(__uint_as_float(r[2]), __uint_as_float(r[3]));
    lo.z = pack_bf16(__uint_as_float(r[4]), __uint_as_float(r[5]));
    lo.w = pack_bf16(__uint_as_float(r[6]), __uint_as_float(r[7]));
    hi.x = pack_bf16(__uint_as_float(r[8]), __uint_as_float(r[9]));
    hi.y = pack_bf16(__uint_as_float(r[10]), __uint_as_float(r[11]));
    hi.z = pack_bf16(__uint_as_float(r[12]), __uint_as_float(r[13]));
    hi.w = pack_bf16(__uint_as_float(r[14]), __uint_as_float(r[15]));
}

template <bool SCALAR>
__global__ void __launch_bounds__(kThreads, 1)
chunk_scan_kernel(const __grid_constant__ Maps maps, const float *__restrict__ g_scalar,
                  const float *__restrict__ S0, __nv_bfloat16 *__restrict__ O, float *__restrict__ ST,
                  int T_len, int nchunks)
{
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                          ~static_cast<uintptr_t>(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 8 * B_COUNT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_BAR + 8 * B_COUNT + 4);
    float *gam = reinterpret_cast<float *>(sm + OFF_GAM);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int head = blockIdx.x;
    const size_t tok0 = (size_t)head * T_len;

    if (tid == 0) {
        const uint32_t counts[B_COUNT] = {
            1, 128,             // g full / empty (E threads release)
            1, 1, 1, 1,         // k full x2, empty x2
            1, 1, 1, 1,         // q
            1, 1, 1, 1,         // v full/empty, T' full/empty
            1, 1, 1, 1,         // Aqk
            128, 128, 128, 1,   // kq ready (E) x2, kt ready (E), kt free (MMA)
            1, 128, 128, 1,     // wt full (MMA), wt empty (M), w ready (M), w free (MMA)
            128, 1, 1, 128,     // s ready (M), s full (MMA), x full (MMA), vn ready (M)
            128, 1, 1, 128, 128,        // vacc empty (M), o full (MMA) x2, oacc empty (E) x2
            128, 128,                   // row-group exchange (E) x2
            1};
        for (int i = 0; i < B_COUNT; ++i) mbar_init(&bar[i], counts[i]);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t sbase = smem_u32(sm);

    // Single-thread roles (TMA producer, MMA issuer) wait with `wait`.
    auto wait = [&](int b, uint32_t parity) -> bool {
        if (*abort_flag) return false;
        if (mbar_wait(&bar[b], parity, kWaitBudget)) return true;
        record_error(6 /* GDR_ERR_TIMEOUT */);
        *abort_flag = 1;
        return false;
    };
    // Warp-wide roles wait with `waitw`: every lane acquires the barrier
    // phase, the result is made warp-uniform, and the warp reconverges -- the
    // tcgen05.ld/st that follow are .sync.aligned and need all 32 lanes
    // converged (lanes leave a spin loop at different times).
    auto waitw = [&](int b, uint32_t parity) -> bool {
        bool ok = wait(b, parity);
        ok = __all_sync(0xffffffffu, ok);
        __syncwarp();
        return ok;
    };

    if (warp == 0) {
        // ================================================================ TMA producer
        if (lane == 0) {
            for (int i = 0; i < 6; ++i) tma_prefetch_desc(&maps.k + i);
            int issued = 0;
            for (int n = 0; n < nchunks; ++n) {
                const int t0 = n * kC;
                const int b = n & 1;
                const uint32_t par = (uint32_t)(n & 1), upar = (uint32_t)((n >> 1) & 1);
                const int crow = (head * nchunks + n) * kC;   // row of this chunk in the workspace
                if (!SCALAR) {
                    if (!wait(B_EMPTY_G, par ^ 1)) break;
                    mbar_arrive_expect_tx(&bar[B_FULL_G], 32768);
                    tma_load_3d(sm + OFF_G, &maps.g, &bar[B_FULL_G], 0, t0, head);
                }
                if (!wait(B_EMPTY_K + b, upar ^ 1)) break;
                mbar_arrive_expect_tx(&bar[B_FULL_K + b], 16384);
                tma_load_3d(sm + OFF_K + b * 16384, &maps.k, &bar[B_FULL_K + b], 0, t0, head);
                tma_load_3d(sm + OFF_K + b * 16384 + 8192, &maps.k, &bar[B_FULL_K + b], 64, t0, head);
                if (!wait(B_EMPTY_Q + b, upar ^ 1)) break;
                mbar_arrive_expect_tx(&bar[B_FULL_Q + b], 16384);
                tma_load_3d(sm + OFF_Q + b * 16384, &maps.q, &bar[B_FULL_Q + b], 0, t0, head);
                tma_load_3d(sm + OFF_Q + b * 16384 + 8192, &maps.q, &bar[B_FULL_Q + b], 64, t0, head);
                if (!wait(B_EMPTY_T, par ^ 1)) break;
                mbar_arrive_expect_tx(&bar[B_FULL_T], 8192);
                tma_load_2d(sm + OFF_T, &maps.t, &bar[B_FULL_T], 0, crow);
                if (!wait(B_EMPTY_V, par ^ 1)) break;
                mbar_arrive_expect_tx(&bar[B_FULL_V], 16384);
                tma_load_3d(sm + OFF_V, &maps.v, &bar[B_FULL_V], 0, t0, head);
                tma_load_3d(sm + OFF_V + 8192, &maps.v, &bar[B_FULL_V], 64, t0, head);
                if (!wait(B_EMPTY_AQ + b, upar ^ 1)) break;
                mbar_arrive_expect_tx(&bar[B_FULL_AQ + b], 8192);
                tma_load_2d(sm + OFF_AQ + b * 8192, &maps.aq, &bar[B_FULL_AQ + b], 0, crow);
                GDR_TRACE_AT(0, n);
                issued = n + 1;
            }
            if (*abort_flag && issued > 0) {
                // let the copies of the last issued chunk land before the CTA exits
                const int n = issued - 1, b = n & 1;
                const uint32_t par = (uint32_t)(n & 1), upar = (uint32_t)((n >> 1) & 1);
                const long long small = kWaitBudget / 4;
                if (!SCALAR) mbar_wait(&bar[B_FULL_G], par, small);
                mbar_wait(&bar[B_FULL_K + b], upar, small);
                mbar_wait(&bar[B_FULL_Q + b], upar, small);
                mbar_wait(&bar[B_FULL_T], par, small);
                mbar_wait(&bar[B_FULL_V], par, small);
                mbar_wait(&bar[B_FULL_AQ + b], upar, small);
            }
        }
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_WU = idesc_bf16(128, 64, true, false);         // A MN-major, B K-major
            constexpr uint32_t ID_X = idesc_bf16(128, 64, false, true, true);    // -A, B (W) MN-major
            constexpr uint32_t ID_O = idesc_bf16(128, 64, false, false);
            constexpr uint32_t ID_S = idesc_bf16(128, 128, false, true);         // B MN-major
            for (int n = 0; n < nchunks; ++n) {
                const int b = n & 1;
                const uint32_t par = (uint32_t)(n & 1), upar = (uint32_t)((n >> 1) & 1);
                // ---- W^T = K<-^T T'^T ; U^T = V^T T'^T
                if (!wait(B_KQ_READY + b, upar) || !wait(B_FULL_T, par) || !wait(B_FULL_V, par) ||
                    !wait(B_WT_EMPTY, par ^ 1) || !wait(B_VACC_EMPTY, par ^ 1))
                    break;
                tc_fence_after();
                GDR_TRACE_AT(1, n);
                const uint32_t kb = sbase + OFF_K + b * 16384;
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tmem + TM_W, sdesc_sw128(kb + s * 2048, 8192, 1024),
                             sdesc_sw128(sbase + OFF_T + s * 32, 16, 1024), ID_WU, s > 0);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tmem + TM_V, sdesc_sw128(sbase + OFF_V + s * 2048, 8192, 1024),
                             sdesc_sw128(sbase + OFF_T + s * 32, 16, 1024), ID_WU, s > 0);
                mma_commit(&bar[B_WT_FULL]);
                mma_commit(&bar[B_EMPTY_K + b]);
                mma_commit(&bar[B_EMPTY_V]);
                mma_commit(&bar[B_EMPTY_T]);
                // ---- V_new^T += -S W^T ; O^T = S Q<-^T
                if (!wait(B_S_READY, par) || !wait(B_W_READY, par) || !wait(B_OACC_EMPTY + b, upar ^ 1)) break;
                tc_fence_after();
                GDR_TRACE_AT(2, n);
                const uint32_t qb = sbase + OFF_Q + b * 16384;
                // V_new^T first: it is on the sequential path
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_bf16(tmem + TM_V, sdesc_sw128(sbase + OFF_S + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024),
                             sdesc_sw128(sbase + OFF_W + s * 2048, 8192, 1024), ID_X, 1);
                mma_commit(&bar[B_X_FULL]);
                mma_commit(&bar[B_W_FREE]);
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_bf16(tmem + TM_O + 64 * b, sdesc_sw128(sbase + OFF_S + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024),
                             sdesc_sw128(qb + (s >> 2) * 8192 + (s & 3) * 32, 16, 1024), ID_O, s > 0);
                mma_commit(&bar[B_EMPTY_Q + b]);
                // ---- O^T += V_new^T Aqk^T ; S += V_new^T K_tail
                if (!wait(B_VN_READY, par) || !wait(B_FULL_AQ + b, upar) || !wait(B_KT_READY, par)) break;
                tc_fence_after();
                GDR_TRACE_AT(3, n);
                // the state increment first: it is on the sequential path
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tmem + TM_D, sdesc_sw128(sbase + OFF_VN + s * 32, 16, 1024),
                             sdesc_sw128(sbase + OFF_KT + s * 2048, 8192, 1024), ID_S, s > 0);
                mma_commit(&bar[B_S_FULL]);
                mma_commit(&bar[B_KT_FREE]);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tmem + TM_O + 64 * b, sdesc_sw128(sbase + OFF_VN + s * 32, 16, 1024),
                             sdesc_sw128(sbase + OFF_AQ + b * 8192 + s * 32, 16, 1024), ID_O, 1);
                mma_commit(&bar[B_O_FULL + b]);
                mma_commit(&bar[B_EMPTY_AQ + b]);
            }
            // every MMA issued above has completed before TMEM is released
            mma_commit(&bar[B_FINAL]);
            mbar_wait(&bar[B_FINAL], 0, kWaitBudget);
        }
    } else if (warp < 6) {
        // ================================================================ E: gate products, operands, epilogue
        const uint32_t lq = 32u * (warp & 3);        // TMEM lane quarter of this warp
        const int orow = (int)lq + lane;             // d_v index for the epilogue
        auto epilogue = [&](int m) -> bool {
            const int bb = m & 1;
            if (!waitw(B_O_FULL + bb, (uint32_t)((m >> 1) & 1))) return false;
            tc_fence_after();
            const int nvalid = min(kC, T_len - m * kC);
            __nv_bfloat16 *orow_ptr = O + (tok0 + (size_t)m * kC) * kD + orow;
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                uint32_t r[16];
                __syncwarp();   // the bounded stores below diverge the warp; tcgen05.ld needs it converged
                tmem_ld16(tmem + (lq << 16) + TM_O + 64 * bb + 16 * cb, r);
                tmem_ld_wait(r);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int t = 16 * cb + j;
                    if (t < nvalid) orow_ptr[(size_t)t * kD] = __float2bfloat16_rn(__uint_as_float(r[j]));
                }
            }
            tc_fence_before();
            mbar_arrive(&bar[B_OACC_EMPTY + bb]);
            return true;
        };
        // Vectorised gate pass: thread (rg, cg) owns rows 8rg..8rg+7 and key
        // channels 8cg..8cg+7, so every shared access is one 16-byte chunk of
        // a 128B-swizzled row.  The running products exp(G_r) and exp(G_C - G_r)
        // per channel combine the thread's own 8 rows with the products of the
        // other row groups, exchanged through shared memory once per chunk.
        const int et = tid - 64;
        const int cg = et & 15, rg = et >> 4;
        const uint32_t pan = (uint32_t)(cg >> 3) * 8192u;   // panel holding this channel group
        bool ok = true;
        for (int n = 0; n < nchunks && ok; ++n) {
            const int b = n & 1;
            const uint32_t par = (uint32_t)(n & 1), upar = (uint32_t)((n >> 1) & 1);
            const int t0 = n * kC;
            if (!SCALAR && !waitw(B_FULL_G, par)) break;
            if (!waitw(B_FULL_K + b, upar) || !waitw(B_FULL_Q + b, upar)) break;
            if (tid == 64) GDR_TRACE_AT(4, n);
            float a[8][8];
            if (!SCALAR) {
                const float *gt = reinterpret_cast<const float *>(sm + OFF_G) + (8 * rg) * kD + 8 * cg;
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) {
                    const float4 x0 = *reinterpret_cast<const float4 *>(gt + rr * kD);
                    const float4 x1 = *reinterpret_cast<const float4 *>(gt + rr * kD + 4);
                    a[rr][0] = __expf(fmaxf(x0.x, kGateMin)); a[rr][1] = __expf(fmaxf(x0.y, kGateMin));
                    a[rr][2] = __expf(fmaxf(x0.z, kGateMin)); a[rr][3] = __expf(fmaxf(x0.w, kGateMin));
                    a[rr][4] = __expf(fmaxf(x1.x, kGateMin)); a[rr][5] = __expf(fmaxf(x1.y, kGateMin));
                    a[rr][6] = __expf(fmaxf(x1.z, kGateMin)); a[rr][7] = __expf(fmaxf(x1.w, kGateMin));
                }
            } else {
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) {
                    const int t = t0 + 8 * rg + rr;
                    const float e = (t < T_len) ? __expf(__ldg(g_scalar + tok0 + t)) : 1.f;
#pragma unroll
                    for (int c = 0; c < 8; ++c) a[rr][c] = e;
                }
            }
            // product of this row group, exchanged with the other seven
            float L[8], F[8], Bk[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                L[c] = a[0][c];
#pragma unroll
                for (int rr = 1; rr < 8; ++rr) L[c] *= a[rr][c];
                F[c] = 1.f;
                Bk[c] = 1.f;
            }
            // Exchange area: with per-channel gates, row 8j of the g tile, which
            // only the threads of row group j read, and which they overwrite
            // after reading it; the tile is released after the exchange.  With
            // a scalar gate the g region holds no tile, so two [8][128] buffers
            // live there.
            float *xb = reinterpret_cast<float *>(sm + OFF_G) + (SCALAR ? b * 8 * kD : 0);
            constexpr int xrow = SCALAR ? kD : 8 * kD;
            *reinterpret_cast<float4 *>(xb + rg * xrow + 8 * cg) = make_float4(L[0], L[1], L[2], L[3]);
            *reinterpret_cast<float4 *>(xb + rg * xrow + 8 * cg + 4) = make_float4(L[4], L[5], L[6], L[7]);
            mbar_arrive(&bar[B_XCH + b]);
            if (!waitw(B_XCH + b, upar)) break;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (j == rg) continue;
                const float4 y0 = *reinterpret_cast<const float4 *>(xb + j * xrow + 8 * cg);
                const float4 y1 = *reinterpret_cast<const float4 *>(xb + j * xrow + 8 * cg + 4);
                const float y[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    if (j < rg) F[c] *= y[c];
                    else Bk[c] *= y[c];
                }
            }
            if (!SCALAR) {
                // The next TMA load overwrites the g tile as soon as this
                // barrier completes; an arrive does not wait for this thread's
                // shared loads, so order them before the async-proxy write.
                fence_async_smem();
                mbar_arrive(&bar[B_EMPTY_G]);
            }
            // K<- = k exp(G_r), Q<- = q exp(G_r) in place; raw k kept for K_tail
            unsigned char *kp = sm + OFF_K + b * 16384 + pan;
            unsigned char *qp = sm + OFF_Q + b * 16384 + pan;
            uint4 kraw[8];
            float pf[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) pf[c] = F[c];
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) {
                const uint32_t r = (uint32_t)(8 * rg + rr);
                const uint32_t off = r * 128u + ((((uint32_t)(cg & 7)) ^ (r & 7u)) << 4);
                const uint4 kv = *reinterpret_cast<const uint4 *>(kp + off);
                const uint4 qv = *reinterpret_cast<const uint4 *>(qp + off);
                kraw[rr] = kv;
#pragma unroll
                for (int c = 0; c < 8; ++c) pf[c] *= a[rr][c];
                *reinterpret_cast<uint4 *>(kp + off) = scale8(kv, pf);
                *reinterpret_cast<uint4 *>(qp + off) = scale8(qv, pf);
            }
            if (rg == 0) {   // gamma_C = product over all 64 rows
                float *gw = gam + (n & 3) * kD + 8 * cg;
                *reinterpret_cast<float4 *>(gw) = make_float4(L[0] * Bk[0], L[1] * Bk[1], L[2] * Bk[2], L[3] * Bk[3]);
                *reinterpret_cast<float4 *>(gw + 4) = make_float4(L[4] * Bk[4], L[5] * Bk[5], L[6] * Bk[6], L[7] * Bk[7]);
            }
            fence_async_smem();
            mbar_arrive(&bar[B_KQ_READY + b]);
            if (tid == 64) GDR_TRACE_AT(5, n);
            // K_tail = k exp(G_C - G_r): exclusive running product from the end
            if (!waitw(B_KT_FREE, par ^ 1)) break;
            if (tid == 64) GDR_TRACE_AT(6, n);
            unsigned char *ktp = sm + OFF_KT + pan;
            float sf[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) sf[c] = Bk[c];
#pragma unroll
            for (int rr = 7; rr >= 0; --rr) {
                const uint32_t r = (uint32_t)(8 * rg + rr);
                const uint32_t off = r * 128u + ((((uint32_t)(cg & 7)) ^ (r & 7u)) << 4);
                *reinterpret_cast<uint4 *>(ktp + off) = scale8(kraw[rr], sf);
#pragma unroll
                for (int c = 0; c < 8; ++c) sf[c] *= a[rr][c];
            }
            fence_async_smem();
            mbar_arrive(&bar[B_KT_READY]);
            if (tid == 64) GDR_TRACE_AT(7, n);
            if (n > 0) ok = epilogue(n - 1);
            if (tid == 64 && n > 0) GDR_TRACE_AT(8, n - 1);
        }
        if (ok && !*abort_flag && nchunks > 0) epilogue(nchunks - 1);
    } else {
        // ================================================================ M: sequential-path conversions
        // The state S_n lives at TM_S and is written only here.  At chunk n
        // (n > 0) this group forms S_n = S_{n-1} * gamma_{n-1} + dS_{n-1}, with
        // dS_{n-1} = V_new^T K_tail of chunk n-1 taken from TM_D, stores it
        // back, and writes its bf16 copy for the MMAs of chunk n.
        const uint32_t lq = 32u * (warp & 3);
        const int i = (int)lq + lane;                // TMEM lane: row of S / V_new^T, key channel of W^T
        const uint32_t trow = tmem + (lq << 16);
        // initial state into TMEM
#pragma unroll
        for (int cb = 0; cb < 8; ++cb) {
            uint32_t r[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
                r[j] = __float_as_uint(S0 ? S0[((size_t)head * kD + i) * kD + 16 * cb + j] : 0.f);
            tmem_st16(trow + TM_S + 16 * cb, r);
        }
        tmem_st_wait();
        // S_{n} = S_{n-1} * gamma_{n-1} + dS_{n-1}, in TMEM and (optionally) as bf16 in smem
        auto advance_state = [&](int n, bool to_smem) {
            const float *gm = gam + ((n - 1) & 3) * kD;
#pragma unroll
            for (int cb = 0; cb < 8; cb += 2) {
                uint32_t r0[16], r1[16], d0[16], d1[16];
                tmem_ld16(trow + TM_S + 16 * cb, r0);
                tmem_ld16(trow + TM_S + 16 * cb + 16, r1);
                tmem_ld16(trow + TM_D + 16 * cb, d0);
                tmem_ld16(trow + TM_D + 16 * cb + 16, d1);
                tmem_ld_wait(r0);
                reg_touch(r1);
                reg_touch(d0);
                reg_touch(d1);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    r0[j] = __float_as_uint(fmaf(__uint_as_float(r0[j]), gm[16 * cb + j], __uint_as_float(d0[j])));
                    r1[j] = __float_as_uint(fmaf(__uint_as_float(r1[j]), gm[16 * cb + 16 + j], __uint_as_float(d1[j])));
                }
                tmem_st16(trow + TM_S + 16 * cb, r0);
                tmem_st16(trow + TM_S + 16 * cb + 16, r1);
                if (to_smem) {
                    unsigned char *sp = sm + OFF_S + (cb >> 2) * 16384;
                    const uint32_t col = (uint32_t)((16 * cb) & 63);
                    uint4 lo, hi;
                    pack16(r0, lo, hi);
                    *reinterpret_cast<uint4 *>(sp + sw128_off(i, col)) = lo;
                    *reinterpret_cast<uint4 *>(sp + sw128_off(i, col + 8)) = hi;
                    pack16(r1, lo, hi);
                    *reinterpret_cast<uint4 *>(sp + sw128_off(i, col + 16)) = lo;
                    *reinterpret_cast<uint4 *>(sp + sw128_off(i, col + 24)) = hi;
                }
            }
            tmem_st_wait();
        };
        bool ok = true;
        for (int n = 0; n < nchunks; ++n) {
            const uint32_t par = (uint32_t)(n & 1);
            // ---- W^T -> W (bf16, K-major [64 tokens x 128 channels])
            // KQ_READY(n) has completed (W^T(n) needed it); waiting on it here only
            // acquires gamma_C(n), which the next chunk boundary reads.
            if (!waitw(B_WT_FULL, par) || !waitw(B_W_FREE, par ^ 1) ||
                !waitw(B_KQ_READY + (n & 1), (uint32_t)((n >> 1) & 1))) { ok = false; break; }
            tc_fence_after();
            if (tid == 192) GDR_TRACE_AT(9, n);
            {
                // W^T row of key channel i = 64 tokens = one 128-byte row of the
                // MN-major W operand
                uint32_t r0[16], r1[16];
                tmem_ld16(trow + TM_W, r0);
                tmem_ld16(trow + TM_W + 16, r1);
                tmem_ld_wait(r0);
                reg_touch(r1);
                uint4 lo, hi;
                pack16(r0, lo, hi);
                *reinterpret_cast<uint4 *>(sm + OFF_W + sw128_off(i, 0)) = lo;
                *reinterpret_cast<uint4 *>(sm + OFF_W + sw128_off(i, 8)) = hi;
                pack16(r1, lo, hi);
                *reinterpret_cast<uint4 *>(sm + OFF_W + sw128_off(i, 16)) = lo;
                *reinterpret_cast<uint4 *>(sm + OFF_W + sw128_off(i, 24)) = hi;
                tmem_ld16(trow + TM_W + 32, r0);
                tmem_ld16(trow + TM_W + 48, r1);
                tmem_ld_wait(r0);
                reg_touch(r1);
                pack16(r0, lo, hi);
                *reinterpret_cast<uint4 *>(sm + OFF_W + sw128_off(i, 32)) = lo;
                *reinterpret_cast<uint4 *>(sm + OFF_W + sw128_off(i, 40)) = hi;
                pack16(r1, lo, hi);
                *reinterpret_cast<uint4 *>(sm + OFF_W + sw128_off(i, 48)) = lo;
                *reinterpret_cast<uint4 *>(sm + OFF_W + sw128_off(i, 56)) = hi;
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bar[B_W_READY]);
            mbar_arrive(&bar[B_WT_EMPTY]);
            if (tid == 192) GDR_TRACE_AT(10, n);
            // ---- state of this chunk -> bf16 smem
            if (n > 0) {
                if (!waitw(B_S_FULL, par ^ 1)) { ok = false; break; }
                tc_fence_after();
                if (tid == 192) GDR_TRACE_AT(11, n);
                advance_state(n, true);
            } else {
                if (tid == 192) GDR_TRACE_AT(11, n);
#pragma unroll
                for (int cb = 0; cb < 8; ++cb) {
                    uint32_t r[16];
                    tmem_ld16(trow + TM_S + 16 * cb, r);
                    tmem_ld_wait(r);
                    unsigned char *sp = sm + OFF_S + (cb >> 2) * 16384;
                    uint4 lo, hi;
                    lo.x = pack_bf16(__uint_as_float(r[0]), __uint_as_float(r[1]));
                    lo.y = pack_bf16(__uint_as_float(r[2]), __uint_as_float(r[3]));
                    lo.z = pack_bf16(__uint_as_float(r[4]), __uint_as_float(r[5]));
                    lo.w = pack_bf16(__uint_as_float(r[6]), __uint_as_float(r[7]));
                    hi.x = pack_bf16(__uint_as_float(r[8]), __uint_as_float(r[9]));
                    hi.y = pack_bf16(__uint_as_float(r[10]), __uint_as_float(r[11]));
                    hi.z = pack_bf16(__uint_as_float(r[12]), __uint_as_float(r[13]));
                    hi.w = pack_bf16(__uint_as_float(r[14]), __uint_as_float(r[15]));
                    *reinterpret_cast<uint4 *>(sp + sw128_off(i, (16 * cb) & 63)) = lo;
                    *reinterpret_cast<uint4 *>(sp + sw128_off(i, ((16 * cb) & 63) + 8)) = hi;
                }
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bar[B_S_READY]);
            if (tid == 192) GDR_TRACE_AT(12, n);
            // ---- V_new^T (TMEM) -> bf16 smem
            if (!waitw(B_X_FULL, par)) { ok = false; break; }
            tc_fence_after();
            if (tid == 192) GDR_TRACE_AT(13, n);
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                uint32_t r[16];
                tmem_ld16(trow + TM_V + 16 * cb, r);
                tmem_ld_wait(r);
                uint4 lo, hi;
                lo.x = pack_bf16(__uint_as_float(r[0]), __uint_as_float(r[1]));
                lo.y = pack_bf16(__uint_as_float(r[2]), __uint_as_float(r[3]));
                lo.z = pack_bf16(__uint_as_float(r[4]), __uint_as_float(r[5]));
                lo.w = pack_bf16(__uint_as_float(r[6]), __uint_as_float(r[7]));
                hi.x = pack_bf16(__uint_as_float(r[8]), __uint_as_float(r[9]));
                hi.y = pack_bf16(__uint_as_float(r[10]), __uint_as_float(r[11]));
                hi.z = pack_bf16(__uint_as_float(r[12]), __uint_as_float(r[13]));
                hi.w = pack_bf16(__uint_as_float(r[14]), __uint_as_float(r[15]));
                *reinterpret_cast<uint4 *>(sm + OFF_VN + sw128_off(i, 16 * cb)) = lo;
                *reinterpret_cast<uint4 *>(sm + OFF_VN + sw128_off(i, 16 * cb + 8)) = hi;
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bar[B_VN_READY]);
            mbar_arrive(&bar[B_VACC_EMPTY]);
            if (tid == 192) GDR_TRACE_AT(14, n);
        }
        // ---- final state S_N = S_{N-1} gamma_{N-1} + dS_{N-1}
        if (ok && nchunks > 0 && waitw(B_S_FULL, (uint32_t)((nchunks - 1) & 1))) {
            tc_fence_after();
            advance_state(nchunks, false);
            if (ST) {
#pragma unroll
                for (int cb = 0; cb < 8; ++cb) {
                    uint32_t r[16];
                    tmem_ld16(trow + TM_S + 16 * cb, r);
                    tmem_ld_wait(r);
                    float4 *dst = reinterpret_cast<float4 *>(ST + ((size_t)head * kD + i) * kD + 16 * cb);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        dst[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                             __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, TM_COLS);
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool make_map(CUtensorMap *m, CUtensorMapDataType dt, int rank, void *ptr, const cuuint64_t *dims,
              const cuuint64_t *strides, const cuuint32_t *box, CUtensorMapSwizzle sw)
{
    const cuuint32_t estr[3] = {1, 1, 1};
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    return f(m, dt, (cuuint32_t)rank, ptr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool chunk_tc_supports(const ChunkArgs &a)
{
    return a.bf16 && a.dk == kD && a.dv == kD && a.C == kC;
}

size_t chunk_tc_workspace_bytes(int B, int H, int T)
{
    const size_t nchunks = (size_t)(T + kC - 1) / kC;
    return 2 * (size_t)B * H * nchunks * kC * kC * sizeof(__nv_bfloat16);
}

cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t stream, int *launches)
{
    const int BH = a.B * a.H;
    const int nchunks = (a.T + kC - 1) / kC;
    __nv_bfloat16 *Tw = static_cast<__nv_bfloat16 *>(a.workspace);
    __nv_bfloat16 *Aw = Tw + (size_t)BH * nchunks * kC * kC;

    Maps maps;
    {
        const cuuint64_t dims3[3] = {(cuuint64_t)kD, (cuuint64_t)a.T, (cuuint64_t)BH};
        const cuuint64_t str_bf[2] = {(cuuint64_t)kD * 2, (cuuint64_t)a.T * kD * 2};
        const cuuint32_t box_bf[3] = {64, 64, 1};
        if (!make_map(&maps.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(a.k), dims3, str_bf, box_bf,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&maps.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(a.q), dims3, str_bf, box_bf,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&maps.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(a.v), dims3, str_bf, box_bf,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        if (!a.scalar_gate) {
            const cuuint64_t str_f[2] = {(cuuint64_t)kD * 4, (cuuint64_t)a.T * kD * 4};
            const cuuint32_t box_f[3] = {128, 64, 1};
            if (!make_map(&maps.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(a.g), dims3, str_f, box_f,
                          CU_TENSOR_MAP_SWIZZLE_NONE))
                return cudaErrorInvalidValue;
        } else {
            maps.g = maps.k;   // unused in scalar mode
        }
        const cuuint64_t dims2[2] = {(cuuint64_t)kC, (cuuint64_t)BH * nchunks * kC};
        const cuuint64_t str2[1] = {(cuuint64_t)kC * 2};
        const cuuint32_t box2[2] = {64, 64};
        if (!make_map(&maps.t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Tw, dims2, str2, box2, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&maps.aq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Aw, dims2, str2, box2, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }

    cudaError_t e = launch_ut_prep(a, Tw, Aw, stream);
    if (e != cudaSuccess) return e;
    *launches += 1;

    auto kern = a.scalar_gate ? chunk_scan_kernel<true> : chunk_scan_kernel<false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    kern<<<BH, kThreads, SMEM_ALLOC, stream>>>(maps, a.g, a.S0, static_cast<__nv_bfloat16 *>(a.O), a.S_T, a.T,
                                              nchunks);
    e = cudaGetLastError();
    if (e == cudaSuccess) *launches += 1;
    return e;
}

#ifdef GDR_TRACE
extern "C" __attribute__((visibility("default"))) int gdr_trace_dump(long long *host)
{
    return (int)cudaMemcpyFromSymbol(host, g_trace, sizeof(g_trace));
}
#endif

cudaError_t read_device_status(cudaStream_t stream, int *status)
{
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int));
    if (e != cudaSuccess) return e;
    if (v != 0) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
    }
    *status = v;
    return e;
}

}  // namespace gdr
