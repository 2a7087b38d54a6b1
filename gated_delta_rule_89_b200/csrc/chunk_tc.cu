// Tensor-core chunked forward of the gated delta rule (bf16 q/k/v, fp32 state,
// d_k = d_v = 128, C = 64) on sm_100a.
//
// Two kernels per call:
//   1. ut_prep (ut_prep.cu): every chunk of every head in parallel -> the
//      UT-transform matrix T' = (I + A)^{-1} Diag(beta), the masked
//      intra-chunk matrix Aqk and, with G the cumulative log-decay inside the
//      chunk, -W = -T' (K*exp(G)), Q<- = Q*exp(G), K_tail = K*exp(G_C - G)
//      (stored transposed) and gamma_C = exp(G_C), all into the workspace.
//   2. chunk_scan (this file): one CTA per (b, h) walks the chunks in order.
//      The fp32 state S [d_v x d_k] lives in tensor memory for the whole
//      sequence.  Per chunk:
//        [O^T | V_new^T] = [0 | V^T T'^T] + S [Q<-; -W]^T          (N = 128)
//        [S   | O^T    ] = [S Diag(gamma_C) | O^T] + V_new^T [K_tail^T; Aqk]^T
//                                                                   (N = 192)
//      (the scaling of S by the conversion warps, the increment accumulated
//      onto it by the MMA; S alternates between two TMEM regions so that each
//      pair of accumulators is contiguous), which is the chunk state update and chunk output of "Reading notes:
//      Kimi Delta Attention" (mzeromiko), section 4, and of "Token Mixer I",
//      section "Kimi Delta Attention: Improving Delta Rule with Fine-grained
//      Gating", in the d_v x d_k orientation.  Every product is one
//      tcgen05.mma chain with M = 128 (rows of S, or key channels), fp32
//      accumulators in TMEM; all inputs arrive by TMA with 128-byte swizzle
//      into double-buffered tiles, and the same tiles serve as K-major or
//      MN-major operands.
//
// Warp roles (448 threads):
//   warp 0      TMA producer (lane 0): all tiles of a chunk land in one of
//               two stages and complete one barrier; gamma_C in two slots.
//               Lane 1 issues the TMA stores of the output tiles (for the
//               gated output instead the loads of the gate tiles).
//   warp 1      TMEM allocation and the MMA issuer (one lane), in the order
//               XO(n) = S_n [Q<-; -W]^T (in two halves, each issued once its
//               half of the bf16 S_n is in smem), SO(n) = V_new^T(n)
//               [K_tail^T; Aqk]^T, U^T(n+1), so the product that does not
//               depend on the state runs while the conversion warps work
//   warps 2-9   the state conversions, split by columns between warps 2-5
//               and 6-9: on the sequential path S (TMEM) -> bf16 smem and
//               V_new^T (TMEM) -> bf16 smem; off it, in the gaps while the
//               tensor core runs, gamma_C S into the other TMEM region.
//   warps 10-13 the output epilogue, one chunk behind the MMAs (the
//               TMEM regions alternate by chunk): O^T (TMEM) -> bf16 staging
//               tile -> TMA store, then the O^T columns are zeroed for the
//               chunk after next.  With OEPI the layer's gated output is
//               fused in (and stored by these warps themselves):
//               y_t = Sigmoid(gate_t) * RMSNorm(o_t) per head
//               ("Token Mixer I", section "The Kimi Linear Model
//               Architecture", the output equation before W_o), RMSNorm over
//               the d_v channels in fp32 straight from the accumulator.
// The sequential chain per chunk is SO -> S to bf16 -> XO -> V_new -> SO.
// Every wait is bounded (about a second); on timeout the kernel records
// GDR_ERR_TIMEOUT in a device status word, lets the copies and MMAs it
// issued finish, frees its tensor memory and returns.
#include <cuda.h>
#include <atomic>
#include <mutex>

#include "gdr_internal.cuh"
#include "sm100_ptx.cuh"

namespace gdr {

__device__ int g_device_status;   // 0 = OK, else the first gdr_status a kernel recorded

cudaError_t launch_ut_prep(const ChunkArgs &a, const TcWorkspace &w, cudaStream_t stream);

namespace {

using namespace sm100;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kThreads = 448;   // 14 warps: TMA, MMA, 8 conversion warps, 4 output-epilogue warps
constexpr long long kWaitBudget = 2000000000LL;   // default clock cycles per wait (~1 s)
constexpr long long kDrainBudget = 500000000LL;   // waits for copies and MMAs already issued, on the way out

// shared memory map (bytes from a 1024-aligned base).  The input tiles of a
// chunk form one stage (gamma_C in a slot of its own); two stages alternate
// by chunk parity.
constexpr uint32_t ST_WQ = 0;                      // [Q<-; -W]: per 64-channel panel (16 KB) the 64
                                                   // token rows of Q<-, then the 64 of -W  32 KB
constexpr uint32_t ST_V = 32768;                   // v                                    16 KB
constexpr uint32_t ST_T = 49152;                   // T' (1 panel)                          8 KB
constexpr uint32_t ST_KT = 57344;                  // [K_tail^T; Aqk]: the 128 key-channel rows of
                                                   // K_tail^T, then the 64 token rows of Aqk  24 KB
constexpr uint32_t ST_AQ = 73728;
constexpr uint32_t STAGE = 81920;                  // stage stride (1024-aligned)
constexpr uint32_t STAGE_TX = 4 * 16384 + 2 * 8192;   // bytes one stage receives
constexpr uint32_t OFF_OST = 2 * STAGE;            // O^T staging for the TMA store (2 panels) 16 KB
constexpr uint32_t OFF_S = OFF_OST + 16384;        // bf16 S (2 panels x 16 KB)             32 KB
constexpr uint32_t OFF_VN = OFF_S + 32768;         // V_new^T (1 panel, 128 rows)           16 KB
constexpr uint32_t OFF_GAM = OFF_VN + 16384;       // gamma_C of each stage, [2][128] fp32   1 KB
constexpr uint32_t OFF_BAR = OFF_GAM + 1024;       // mbarriers, TMEM slot, abort flag
constexpr uint32_t OFF_RED = OFF_BAR + 256;        // gated output: partial sums [4 warps][32 tokens] fp32
constexpr uint32_t OFF_RSTD = OFF_RED + 512;       // gated output: 1 / RMS of the 64 tokens
constexpr uint32_t SMEM_USED = OFF_RSTD + 256;
constexpr uint32_t SMEM_ALLOC = SMEM_USED + 1024;  // alignment slack
static_assert(SMEM_ALLOC <= 232448, "dynamic shared memory above the 227 KB per-block limit");

// TMEM columns (fp32): one region of 256 columns per chunk parity b, at
// TM_REG * b.  For chunk n (b = n & 1) the region holds
//   + TM_S  (128)  gamma_C(n) S_n, written by the conversion warps, onto which
//                  the MMA accumulates the increment: S_{n+1} stays here while
//                  chunk n + 1 reads it (and writes its own region)
//   + TM_O  (64)   O^T(n)      } contiguous, so that [S | O^T] and
//   + TM_V  (64)   V_new^T(n)  } [O^T | V_new^T] are each one accumulator
constexpr uint32_t TM_REG = 256;
constexpr uint32_t TM_S = 0;
constexpr uint32_t TM_O = 128;
constexpr uint32_t TM_V = 192;
constexpr uint32_t TM_COLS = 512;

enum Bar {
    B_FULL, B_FULL1,          // stage landed (TMA transaction bytes)
    B_EMPTY, B_EMPTY1,        // stage released (MMA commit)
    B_GFULL, B_GFULL1,        // gamma_C slot landed
    B_GEMPTY, B_GEMPTY1,      // gamma_C slot read by the state-update threads
    B_SW_LO, B_SW_HI,         // S_n (bf16) in smem: columns 0-31 and 64-95, then 32-63 and 96-127
    B_X_FULL,                 // XO(n) done: V_new^T(n) in TMEM, the S Q<-^T part of O^T(n) in place
    B_VN_READY,               // V_new^T(n) bf16 in smem, V part read, S_n scaled by gamma_C(n)
    B_S_FULL,                 // S_{n+1} complete in TMEM (and O^T(n))
    B_O_FULL, B_O_FULL1,      // O^T(n) complete
    B_OACC_EMPTY, B_OACC_EMPTY1,   // O^T accumulator drained by the epilogue
    B_EPI_FULL,               // O^T staging tile written (warps 2-9)
    B_EPI_FREE,               // O^T staging tile free again (the previous store has read it)
    B_GATE_FULL,              // gated output: the gate tile of the next chunk landed in the staging tile
    B_FINAL,
    B_COUNT
};
static_assert(8 * B_COUNT + 8 <= 256, "barrier area");

struct Maps {
    CUtensorMap w, q, kt, v, t, aq, o;   // Q<-, K_tail, v, O: [BH][T][128]; T', Aqk: [chunks*64][64];
                                         // -W: [chunks*64][128]; K_tail^T: [chunks*128][64]
    CUtensorMap og;                      // output gate [BH][T][128] (gated output only)
};

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_device_status, 0, code); }

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
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

// One barrier of the 128 threads of the output-epilogue warps that also
// returns whether every one of them passed ok (so they leave together).
__device__ __forceinline__ bool epi_all(bool ok)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)ok)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <bool SCALAR, bool OEPI>
__global__ void __launch_bounds__(kThreads, 1)
chunk_scan_kernel(const __grid_constant__ Maps maps, const float *__restrict__ gamma_c,
                  const float *__restrict__ S0, __nv_bfloat16 *__restrict__ O, float *__restrict__ ST,
                  int T_len, int nchunks, const __nv_bfloat16 *__restrict__ ogate,
                  const float *__restrict__ norm_w, float eps, long long wait_budget)
{
    extern __shared__ unsigned char smem_raw[];
    // aligned by an offset into the __shared__ array itself, so that the
    // compiler keeps every access through `sm` in the shared state space
    unsigned char *sm = smem_raw + ((1024u - (sm100::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 8 * B_COUNT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_BAR + 8 * B_COUNT + 4);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int head = blockIdx.x;

    if (tid == 0) {
        const uint32_t counts[B_COUNT] = {
            1, 1, 1, 1,       // stage full (TMA), stage empty (MMA commit)
            1, 1, 8, 8,       // gamma full (TMA), gamma empty (warps 2-9)
            8, 8, 1, 8,       // sw ready (warps 2-9, two halves), x full (MMA), vn ready (warps 2-9)
            1,                // s full (MMA)
            1, 1, 4, 4,       // o full (MMA) x2, oacc empty (epilogue warps) x2
            4, 1,             // epilogue tile written (epilogue warps), free (warp 0 lane 1)
            1,                // gate tile landed (TMA)
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

    // Single-thread roles (TMA producer, MMA issuer) wait with `wait`: one
    // try first, and only a thread that has to wait looks at the abort flag.
    auto wait = [&](int b, uint32_t parity) -> bool {
        if (mbar_try_wait(&bar[b], parity)) return true;
        if (*abort_flag) return false;
        if (mbar_wait(&bar[b], parity, wait_budget)) return true;
        record_error(6 /* GDR_ERR_TIMEOUT */);
        *abort_flag = 1;
        return false;
    };
    // Warp-wide roles arrive once per warp: the warp barrier orders every
    // lane's prior writes (after its proxy and tcgen05 fences) before lane 0's
    // arrive.  An arrive is an atomic on one shared word, so 32 of them from a
    // warp would queue behind each other on the hand-offs of the chain.
    auto warp_arrive = [&](int b) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[b]);
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
        // ================================================================ TMA producer, output stores
        if (lane == 1 && OEPI) {
            // Gated output: the staging tile receives the gate tile of chunk m (TMA);
            // the epilogue writes y(m) to global memory itself, and as soon as it has
            // read the gate values the gate tile of chunk m + 1 goes in.
            auto load_gate = [&](int m) {
                mbar_arrive_expect_tx(&bar[B_GATE_FULL], 16384);
                tma_load_3d(sm + OFF_OST, &maps.og, &bar[B_GATE_FULL], 0, m * kC, head);
                tma_load_3d(sm + OFF_OST + 8192, &maps.og, &bar[B_GATE_FULL], 64, m * kC, head);
            };
            int loaded = 0;
            if (nchunks > 0) {
                load_gate(0);
                loaded = 1;
            }
            for (int m = 0; m + 1 < nchunks; ++m) {
                if (!wait(B_EPI_FULL, (uint32_t)(m & 1))) break;   // the gate tile of m has been read
                load_gate(m + 1);
                loaded = m + 2;
            }
            if (*abort_flag && loaded > 0)   // a gate tile still in flight lands before exit
                mbar_wait(&bar[B_GATE_FULL], (uint32_t)((loaded - 1) & 1), kDrainBudget);
        }
        if (lane == 1 && !OEPI) {
            // Output tile m: stored once the epilogue has written it; the tile
            // is handed back once the store has read it.  (The gated output is
            // written by the epilogue warps themselves.)
            mbar_arrive(&bar[B_EPI_FREE]);
            for (int m = 0; m < nchunks; ++m) {
                if (!wait(B_EPI_FULL, (uint32_t)(m & 1))) break;
                tma_store_3d(&maps.o, sm + OFF_OST, 0, m * kC, head);
                tma_store_3d(&maps.o, sm + OFF_OST + 8192, 64, m * kC, head);
                bulk_commit_group();
                bulk_wait_read_all();
                mbar_arrive(&bar[B_EPI_FREE]);
            }
            bulk_wait_all();   // the last store has completed before the CTA exits
        }
        if (lane == 0) {
            for (int i = 0; i < 6; ++i) tma_prefetch_desc(&maps.w + i);
            if (OEPI) tma_prefetch_desc(&maps.og);
            int issued = 0;
            for (int n = 0; n < nchunks; ++n) {
                const int t0 = n * kC;
                const int b = n & 1;
                const uint32_t upar = (uint32_t)((n >> 1) & 1);
                const int crow = (head * nchunks + n) * kC;   // row of this chunk in T' / Aqk
                unsigned char *st = sm + b * STAGE;
                uint64_t *full = &bar[B_FULL + b];
                if (!wait(B_EMPTY + b, upar ^ 1)) break;
                mbar_arrive_expect_tx(full, STAGE_TX);
                tma_load_3d(st + ST_WQ, &maps.q, full, 0, t0, head);
                tma_load_3d(st + ST_WQ + 16384, &maps.q, full, 64, t0, head);
                tma_load_2d(st + ST_WQ + 8192, &maps.w, full, 0, crow);
                tma_load_2d(st + ST_WQ + 16384 + 8192, &maps.w, full, 64, crow);
                tma_load_3d(st + ST_V, &maps.v, full, 0, t0, head);
                tma_load_3d(st + ST_V + 8192, &maps.v, full, 64, t0, head);
                tma_load_2d(st + ST_T, &maps.t, full, 0, crow);
                tma_load_2d(st + ST_KT, &maps.kt, full, 0, 2 * crow);   // key-channel rows of this chunk
                tma_load_2d(st + ST_AQ, &maps.aq, full, 0, crow);
                if (OEPI) {   // the epilogue's gate tile, warmed in L2 a chunk ahead of its load
                    tma_prefetch_l2_3d(&maps.og, 0, t0, head);
                    tma_prefetch_l2_3d(&maps.og, 64, t0, head);
                }
                // gamma_C has its own slots, released by the state update, so the
                // stage itself only waits for the MMAs that read it
                if (!wait(B_GEMPTY + b, upar ^ 1)) break;
                mbar_arrive_expect_tx(&bar[B_GFULL + b], 512);
                bulk_load(sm + OFF_GAM + b * 512, gamma_c + (size_t)(head * nchunks + n) * kD, 512, &bar[B_GFULL + b]);
                issued = n + 1;
            }
            if (*abort_flag) {
                // let the copies of the (at most two) stages still in flight land
                // before the CTA exits
                for (int n = issued - 1; n >= 0 && n >= issued - 2; --n) {
                    mbar_wait(&bar[B_FULL + (n & 1)], (uint32_t)((n >> 1) & 1), kDrainBudget);
                    mbar_wait(&bar[B_GFULL + (n & 1)], (uint32_t)((n >> 1) & 1), kDrainBudget);
                }
            }
        }
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_WU = idesc_bf16(128, 64, true, false);         // A (v) MN-major, B K-major
            constexpr uint32_t ID_XO = idesc_bf16(128, 128, false, false);       // S [Q<-; -W]^T
            constexpr uint32_t ID_SO = idesc_bf16(128, 192, false, false);       // V_new^T [K_tail^T; Aqk]^T
            // descriptors of the two operand layouts at the base of shared memory:
            // the address field counts 16-byte units, so a byte offset adds directly
            const uint64_t d16 = sdesc_sw128(sbase, 16, 1024), d8k = sdesc_sw128(sbase, 8192, 1024);
            auto K16 = [&](uint32_t off) { return d16 + (uint64_t)(off >> 4); };   // K-major tile
            auto MN = [&](uint32_t off) { return d8k + (uint64_t)(off >> 4); };    // MN-major tile, panels 8 KB apart
            // U^T = V^T T'^T of chunk n into V_new^T of region n & 1, tokens 16 s .. 16 s + 15
            auto mma_u = [&](int n, int s) {
                const uint32_t st = (n & 1) * STAGE;
                mma_bf16(tmem + TM_REG * (n & 1) + TM_V, MN(st + ST_V + s * 2048), K16(st + ST_T + s * 32), ID_WU, s > 0);
            };
            // [O^T | V_new^T] += S [Q<-; -W]^T, key channels 16 s .. 16 s + 15
            auto mma_xo = [&](uint32_t st, uint32_t reg, int s) {
                mma_bf16(reg + TM_O, K16(OFF_S + (s >> 2) * 16384 + (s & 3) * 32),
                         K16(st + ST_WQ + (s >> 2) * 16384 + (s & 3) * 32), ID_XO, 1);
            };
            bool ok = nchunks > 0 && wait(B_FULL, 0);
            if (ok) {
                tc_fence_after();
                for (int s = 0; s < 4; ++s) mma_u(0, s);
            }
            // U^T(n + 1) does not depend on the state; it is issued last, when
            // the stage of chunk n + 1 (loaded once the MMAs of chunk n - 1 had
            // released it) has landed, and runs while S_{n+1} is converted.
            for (int n = 0; n < nchunks && ok; ++n) {
                const int b = n & 1;
                const uint32_t par = (uint32_t)(n & 1), upar = (uint32_t)((n >> 1) & 1);
                const uint32_t st = b * STAGE;
                const uint32_t reg = tmem + TM_REG * b;
                const bool more = n + 1 < nchunks;
                // ---- O^T = S Q<-^T and V_new^T = U^T - S W^T in one product (the O^T
                // part was zeroed by the epilogue), the half of S converted first first
                if (!wait(B_SW_LO, par) || !wait(B_OACC_EMPTY + b, upar ^ 1)) break;
                tc_fence_after();
                mma_xo(st, reg, 0);
                mma_xo(st, reg, 1);
                mma_xo(st, reg, 4);
                mma_xo(st, reg, 5);
                if (!wait(B_SW_HI, par)) break;
                tc_fence_after();
                mma_xo(st, reg, 2);
                mma_xo(st, reg, 3);
                mma_xo(st, reg, 6);
                mma_xo(st, reg, 7);
                mma_commit(&bar[B_X_FULL]);
                // ---- [S | O^T] += V_new^T [K_tail^T; Aqk]^T: the state increment
                // (the sequential path; S already scaled by gamma_C) and the
                // intra-chunk part of the output in one product
                if (!wait(B_VN_READY, par)) break;
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 4; ++s) mma_bf16(reg + TM_S, K16(OFF_VN + s * 32), K16(st + ST_KT + s * 32), ID_SO, 1);
                mma_commit(&bar[B_S_FULL]);
                mma_commit(&bar[B_O_FULL + b]);
                mma_commit(&bar[B_EMPTY + b]);   // every read of this stage is issued
                // ---- U^T(n + 1)
                if (more) {
                    if (!wait(B_FULL + (b ^ 1), (uint32_t)(((n + 1) >> 1) & 1))) break;
                    tc_fence_after();
                    for (int s = 0; s < 4; ++s) mma_u(n + 1, s);
                }
            }
            // every MMA issued above has completed before TMEM is released
            mma_commit(&bar[B_FINAL]);
            mbar_wait(&bar[B_FINAL], 0, kWaitBudget);
        }
    } else if (warp < 10) {
        // ================================================================ state update, conversions, epilogue
        // The state S_n lives in region (n + 1) & 1.  At chunk n these warps copy
        // it to bf16 smem for the MMAs of chunk n (on the sequential path), then
        // store gamma_C(n) S_n into region n & 1 (off the path, while XO(n)
        // runs); the MMA of S += V_new^T K_tail then leaves S_{n+1} there.
        // Warps 2-5 take key channels 64..127 of S and tokens 32..63 of V_new^T,
        // warps 6-9 the other halves.
        const bool ga = warp < 6;                     // warps 2-5
        const uint32_t lq = 32u * (warp & 3);         // TMEM lane quarter of this warp
        const int i = (int)lq + lane;                 // TMEM lane: row of S / V_new^T / O^T
        const uint32_t trow = tmem + (lq << 16);
        const int sc0 = ga ? 64 : 0;                  // first state column of this warp
        const int vc0 = ga ? 32 : 0;                  // first V_new^T / O^T column (token)
        // initial state into TMEM
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            uint32_t r[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
                r[j] = __float_as_uint(S0 ? S0[((size_t)head * kD + i) * kD + sc0 + 16 * cb + j] : 0.f);
            tmem_st16(trow + TM_REG + TM_S + sc0 + 16 * cb, r);   // read by chunk 0 from region 1
        }
        // the O^T parts of both regions start at zero (the first products
        // accumulate onto them; later the epilogue zeroes what it drained)
        {
            uint32_t z[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) z[j] = 0u;
#pragma unroll
            for (int bb = 0; bb < 2; ++bb)
#pragma unroll
                for (int cb = 0; cb < 2; ++cb) tmem_st16(trow + TM_REG * bb + TM_O + vc0 + 16 * cb, z);
        }
        tmem_st_wait();
        // One pass over this warp's 64 columns of S_n (TMEM, region (n + 1) & 1):
        // the bf16 copy goes to smem and is released to the MMAs at once, in two
        // halves (the sequential path); then gamma_C(n) S_n is stored into
        // region n & 1 for the accumulation of chunk n's increment.
        auto state_pass = [&](int n) -> bool {
            unsigned char *sp = sm + OFF_S + (sc0 >> 6) * 16384;
            uint32_t r[4][16];
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) tmem_ld16(trow + TM_REG * ((n + 1) & 1) + TM_S + sc0 + 16 * cb, r[cb]);
            tmem_ld_wait(r[0]);
            reg_touch(r[1]);
            reg_touch(r[2]);
            reg_touch(r[3]);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
                for (int cb = 2 * hf; cb < 2 * hf + 2; ++cb) {
                    uint4 lo, hi;
                    pack16(r[cb], lo, hi);
                    *reinterpret_cast<uint4 *>(sp + sw128_off(i, 16 * cb)) = lo;
                    *reinterpret_cast<uint4 *>(sp + sw128_off(i, 16 * cb + 8)) = hi;
                }
                fence_async_smem();
                tc_fence_before();
                warp_arrive(hf ? B_SW_HI : B_SW_LO);
            }
            if (!waitw(B_GFULL + (n & 1), (uint32_t)((n >> 1) & 1))) return false;
            const float4 *gm = reinterpret_cast<const float4 *>(sm + OFF_GAM + (n & 1) * 512) + (sc0 >> 2);
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 gv = gm[4 * cb + q];
                    r[cb][4 * q + 0] = __float_as_uint(__uint_as_float(r[cb][4 * q + 0]) * gv.x);
                    r[cb][4 * q + 1] = __float_as_uint(__uint_as_float(r[cb][4 * q + 1]) * gv.y);
                    r[cb][4 * q + 2] = __float_as_uint(__uint_as_float(r[cb][4 * q + 2]) * gv.z);
                    r[cb][4 * q + 3] = __float_as_uint(__uint_as_float(r[cb][4 * q + 3]) * gv.w);
                }
                tmem_st16(trow + TM_REG * (n & 1) + TM_S + sc0 + 16 * cb, r[cb]);
            }
            tmem_st_wait();
            warp_arrive(B_GEMPTY + (n & 1));
            return true;
        };
        bool ok = true;
        for (int n = 0; n < nchunks && ok; ++n) {
            const uint32_t par = (uint32_t)(n & 1);
            // ---- S_n -> bf16 smem (the MMAs of chunk n - 1 that read the old
            // copy completed before S_FULL(n - 1), which also completed S_n)
            if (n > 0) {
                if (!waitw(B_S_FULL, par ^ 1)) { ok = false; break; }
                tc_fence_after();
            }
            if (!state_pass(n)) { ok = false; break; }
            // ---- V_new^T (TMEM) -> bf16 smem (the MMAs of chunk n - 1 that read
            // the old copy completed before X_FULL(n))
            if (!waitw(B_X_FULL, par)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                uint32_t r[16];
                tmem_ld16(trow + TM_REG * (n & 1) + TM_V + vc0 + 16 * cb, r);
                tmem_ld_wait(r);
                uint4 lo, hi;
                pack16(r, lo, hi);
                *reinterpret_cast<uint4 *>(sm + OFF_VN + sw128_off(i, vc0 + 16 * cb)) = lo;
                *reinterpret_cast<uint4 *>(sm + OFF_VN + sw128_off(i, vc0 + 16 * cb + 8)) = hi;
            }
            fence_async_smem();
            tc_fence_before();
            warp_arrive(B_VN_READY);   // also: S_n scaled
        }
        // ---- final state S_N: the last accumulation has completed
        if (ok && nchunks > 0 && waitw(B_S_FULL, (uint32_t)((nchunks - 1) & 1))) {
            tc_fence_after();
            if (ST) {
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) {
                    uint32_t r[16];
                    tmem_ld16(trow + TM_REG * ((nchunks - 1) & 1) + TM_S + sc0 + 16 * cb, r);
                    tmem_ld_wait(r);
                    float4 *dst = reinterpret_cast<float4 *>(ST + ((size_t)head * kD + i) * kD + sc0 + 16 * cb);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        dst[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                             __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
                }
            }
        }
    } else {
        // ================================================================ output epilogue (warps 10-13)
        // Warp w holds d_v channels 32 (w & 3) .. + 31 (its TMEM lane quarter)
        // of all 64 tokens of O^T(m).
        // Plain: O^T -> bf16 staging tile -> TMA store (warp 0, lane 1).
        // OEPI: the gate tile of chunk m is TMA-loaded into the staging tile
        // (same layout as the output); per token the sum of squares over the 128
        // channels (lanes, then the four warps); the gate values are read into
        // registers, which frees the tile for the next gate load, and
        // y = o * rsqrt(mean o^2 + eps) * norm_w * Sigmoid(gate) is stored to
        // global memory straight from registers (32 consecutive channels per
        // warp and token).
        const uint32_t lq = 32u * (warp & 3);
        const int i = (int)lq + lane;
        const uint32_t trow = tmem + (lq << 16);
        unsigned char *ost = sm + OFF_OST + (i >> 6) * 8192 + (i & 7) * 2;
        const uint32_t c8 = (uint32_t)((i & 63) >> 3);
        const float nw = OEPI ? __ldg(norm_w + i) : 1.f;
        float *red = reinterpret_cast<float *>(sm + OFF_RED);     // [4 warps][32 tokens]
        float *rstd = reinterpret_cast<float *>(sm + OFF_RSTD);   // [64 tokens]
        for (int m = 0; m < nchunks; ++m) {
            const int bb = m & 1;
            // the gate tile is only needed by pass 2: its load overlaps pass 1
            bool ok = (OEPI || waitw(B_EPI_FREE, (uint32_t)(m & 1))) && waitw(B_O_FULL + bb, (uint32_t)((m >> 1) & 1));
            if (OEPI) ok = epi_all(ok);   // the four warps go on (or stop) together
            if (!ok) break;
            tc_fence_after();
            const uint32_t oc = trow + TM_REG * bb + TM_O;
            // after the last read of O^T(m) its columns are zeroed: the next
            // product into this accumulator adds onto them
            auto zero_oacc = [&]() {
                uint32_t z[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) z[j] = 0u;
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) tmem_st16(oc + 16 * cb, z);
                tmem_st_wait();
            };
            if (!OEPI) {
#pragma unroll 2
                for (int cb = 0; cb < 8; ++cb) {
                    uint32_t r[8];
                    tmem_ld8(oc + 8 * cb, r);
                    tmem_ld_wait8(r);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<__nv_bfloat16 *>(ost + cb * 1024 + j * 128 + ((c8 ^ (uint32_t)j) << 4)) =
                            __float2bfloat16_rn(__uint_as_float(r[j]));
                }
                zero_oacc();
                tc_fence_before();
                warp_arrive(B_OACC_EMPTY + bb);
                fence_async_smem();
                warp_arrive(B_EPI_FULL);
            } else {
                // pass 1, per 32 tokens: lane L ends with this warp's partial sum of
                // token 32 h + L; warp (w & 3) == 0 adds the four up
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float ps[32];
                    {
                        uint32_t r0[8], r1[8], r2[8], r3[8];
                        tmem_ld8(oc + 32 * h, r0);
                        tmem_ld8(oc + 32 * h + 8, r1);
                        tmem_ld8(oc + 32 * h + 16, r2);
                        tmem_ld8(oc + 32 * h + 24, r3);
                        tmem_ld_wait8(r0);
                        reg_touch8(r1);
                        reg_touch8(r2);
                        reg_touch8(r3);
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            ps[j] = __uint_as_float(r0[j]) * __uint_as_float(r0[j]);
                            ps[8 + j] = __uint_as_float(r1[j]) * __uint_as_float(r1[j]);
                            ps[16 + j] = __uint_as_float(r2[j]) * __uint_as_float(r2[j]);
                            ps[24 + j] = __uint_as_float(r3[j]) * __uint_as_float(r3[j]);
                        }
                    }
                    // transpose-reduce: keep the half of the values whose index has bit w
                    // equal to this lane's, add the partner's copy of it
#pragma unroll
                    for (int w = 16; w >= 1; w >>= 1) {
#pragma unroll
                        for (int j = 0; j < w; ++j) {
                            const bool up = (lane & w) != 0;
                            const float send = up ? ps[j] : ps[j + w];
                            const float got = __shfl_xor_sync(0xffffffffu, send, w);
                            ps[j] = (up ? ps[j + w] : ps[j]) + got;
                        }
                    }
                    red[(warp & 3) * 32 + lane] = ps[0];
                    epi_sync();
                    if ((warp & 3) == 0)   // half the reciprocal RMS: Sigmoid(z) = (1 + tanh(z / 2)) / 2
                        rstd[32 * h + lane] =
                            0.5f * rsqrtf((red[lane] + red[32 + lane] + red[64 + lane] + red[96 + lane]) * (1.f / kD) + eps);
                    epi_sync();   // red is free again, rstd of these tokens written
                }
                if (!epi_all(waitw(B_GATE_FULL, (uint32_t)(m & 1)))) break;
                // the chunk's 64 gate values of this channel, packed in token pairs;
                // then the tile goes back for the next chunk's gate
                uint32_t zp[32];
#pragma unroll
                for (int jp = 0; jp < 32; ++jp) {
                    const uint32_t t0 = 2u * jp, t1 = t0 + 1u;
                    const uint32_t lo = *reinterpret_cast<const unsigned short *>(
                        ost + (t0 >> 3) * 1024 + (t0 & 7) * 128 + ((c8 ^ (t0 & 7)) << 4));
                    const uint32_t hi = *reinterpret_cast<const unsigned short *>(
                        ost + (t1 >> 3) * 1024 + (t1 & 7) * 128 + ((c8 ^ (t1 & 7)) << 4));
                    zp[jp] = lo | (hi << 16);
                }
                fence_async_smem();   // the next gate tile (TMA) overwrites what was read
                warp_arrive(B_EPI_FULL);
                // pass 2: 16 tokens per step; y goes to global memory from registers,
                // 32 consecutive channels per warp and token (tokens past T dropped)
                __nv_bfloat16 *yrow = O + ((size_t)head * T_len + (size_t)m * kC) * kD + i;
                const int tvalid = T_len - m * kC;
#pragma unroll
                for (int cs = 0; cs < 4; ++cs) {
                    uint32_t r0[8], r1[8];
                    tmem_ld8(oc + 16 * cs, r0);
                    tmem_ld8(oc + 16 * cs + 8, r1);
                    float f[16], z[16];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float4 fv = *reinterpret_cast<const float4 *>(rstd + 16 * cs + 4 * q4);
                        f[4 * q4] = fv.x;
                        f[4 * q4 + 1] = fv.y;
                        f[4 * q4 + 2] = fv.z;
                        f[4 * q4 + 3] = fv.w;
                    }
#pragma unroll
                    for (int j = 0; j < 16; j += 2) {
                        z[j] = __uint_as_float(zp[8 * cs + j / 2] << 16);
                        z[j + 1] = __uint_as_float(zp[8 * cs + j / 2] & 0xffff0000u);
                    }
                    tmem_ld_wait8(r0);
                    reg_touch8(r1);
                    // two tokens at a time: a = o * rstd / 2 * norm_w, y = a (1 + tanh(z / 2))
#pragma unroll
                    for (int j = 0; j < 16; j += 2) {
                        const float2 o2 = make_float2(__uint_as_float(j < 8 ? r0[j] : r1[j - 8]),
                                                      __uint_as_float(j < 8 ? r0[j + 1] : r1[j - 7]));
                        const float2 a = fmul2(fmul2(o2, make_float2(f[j], f[j + 1])), make_float2(nw, nw));
                        const float2 hz = fmul2(make_float2(z[j], z[j + 1]), make_float2(0.5f, 0.5f));
                        const float2 y = ffma2(a, make_float2(tanh_approx(hz.x), tanh_approx(hz.y)), a);
                        const uint32_t yb = pack2_bf16(y.x, y.y);
                        const int tt = 16 * cs + j;
                        if (tt < tvalid) *reinterpret_cast<unsigned short *>(yrow + (size_t)tt * kD) = (unsigned short)(yb & 0xffffu);
                        if (tt + 1 < tvalid)
                            *reinterpret_cast<unsigned short *>(yrow + (size_t)(tt + 1) * kD) = (unsigned short)(yb >> 16);
                    }
                }
                zero_oacc();
                tc_fence_before();
                warp_arrive(B_OACC_EMPTY + bb);
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

namespace {
std::atomic<long long> g_wait_budget{0};   // 0: the default budget
long long wait_budget_now()
{
    const long long v = g_wait_budget.load(std::memory_order_relaxed);
    return v > 0 ? v : kWaitBudget;
}
}  // namespace

void set_wait_budget(long long cycles) { g_wait_budget.store(cycles > 0 ? cycles : 0, std::memory_order_relaxed); }

bool chunk_tc_supports(const ChunkArgs &a)
{
    return a.bf16 && a.dk == kD && a.dv == kD && a.C == kC;
}

size_t chunk_tc_workspace_bytes(int B, int H, int T, bool gdr2) { return tc_workspace_bytes(B, H, T, gdr2); }

cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t stream, int *launches)
{
    const int BH = a.B * a.H;
    const int nchunks = (a.T + kC - 1) / kC;
    const TcWorkspace w = carve_tc_workspace(a.workspace, a.B, a.H, a.T, a.gdr2);

    Maps maps;
    {
        const cuuint64_t dims3[3] = {(cuuint64_t)kD, (cuuint64_t)a.T, (cuuint64_t)BH};
        const cuuint64_t str_bf[2] = {(cuuint64_t)kD * 2, (cuuint64_t)a.T * kD * 2};
        const cuuint32_t box_bf[3] = {64, 64, 1};
        // Gated Delta Rule-2: U = T' Z with Z = w * v, formed by the prep kernel
        void *tiles[3] = {w.Ql, a.gdr2 ? static_cast<void *>(w.Z) : const_cast<void *>(a.v), a.O};
        CUtensorMap *dst[3] = {&maps.q, &maps.v, &maps.o};
        for (int i = 0; i < 3; ++i)
            if (!make_map(dst[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, tiles[i], dims3, str_bf, box_bf,
                          CU_TENSOR_MAP_SWIZZLE_128B))
                return cudaErrorInvalidValue;
        if (a.gated_out && !make_map(&maps.og, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(a.ogate), dims3,
                                     str_bf, box_bf, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        const cuuint64_t dims2[2] = {(cuuint64_t)kC, (cuuint64_t)BH * nchunks * kC};
        const cuuint64_t str2[1] = {(cuuint64_t)kC * 2};
        const cuuint32_t box2[2] = {64, 64};
        // -W: [chunks * 64 token rows][128 channels], boxes of 64 x 64
        const cuuint64_t dimsw[2] = {(cuuint64_t)kD, (cuuint64_t)BH * nchunks * kC};
        const cuuint64_t strw[1] = {(cuuint64_t)kD * 2};
        // K_tail^T: [chunks * 128 key-channel rows][64 tokens], one box of 64 x 128
        const cuuint64_t dimsk[2] = {(cuuint64_t)kC, (cuuint64_t)BH * nchunks * kD};
        const cuuint32_t boxk[2] = {64, 128};
        if (!make_map(&maps.w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w.W, dimsw, strw, box2, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&maps.kt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w.Kt, dimsk, str2, boxk, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&maps.t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w.T, dims2, str2, box2, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&maps.aq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w.Aqk, dims2, str2, box2, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }

    cudaError_t e = launch_ut_prep(a, w, stream);
    if (e != cudaSuccess) return e;
    *launches += 1;

    auto kern = a.gated_out ? (a.scalar_gate ? chunk_scan_kernel<true, true> : chunk_scan_kernel<false, true>)
                            : (a.scalar_gate ? chunk_scan_kernel<true, false> : chunk_scan_kernel<false, false>);
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    kern<<<BH, kThreads, SMEM_ALLOC, stream>>>(
        maps, w.gam, a.S0, static_cast<__nv_bfloat16 *>(a.O), a.S_T, a.T, nchunks,
        static_cast<const __nv_bfloat16 *>(a.ogate), a.norm_w, a.eps, wait_budget_now());
    e = cudaGetLastError();
    if (e == cudaSuccess) *launches += 1;
    return e;
}

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
        if (e != cudaSuccess) return e;
    }
    *status = v;
    return cudaSuccess;
}

}  // namespace gdr
