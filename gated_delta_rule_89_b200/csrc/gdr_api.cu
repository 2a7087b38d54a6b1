// C entry points of libgdr.so: argument validation, dispatch, status codes.
// The declarations and the contract of every call are in include/gdr.h.
#include <stdint.h>

#include "gdr.h"
#include "gdr_internal.cuh"

#define GDR_API extern "C" __attribute__((visibility("default")))

namespace {

thread_local int tl_last_cuda_error = 0;
thread_local int tl_last_launches = 0;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int finish(cudaError_t e, int launches)
{
    if (e != cudaSuccess) {
        tl_last_cuda_error = (int)e;
        return GDR_ERR_CUDA;
    }
    tl_last_launches = launches;
    return GDR_OK;
}

bool size_ok(int d) { return d == 64 || d == 128; }

// Debug mode only: GDR_ERR_GATE_RANGE when an element of g is positive or not
// finite (n elements), GDR_ERR_CUDA when the check itself failed, else GDR_OK.
int gate_guard(const float *g, size_t n, cudaStream_t st)
{
    if (!gdr::debug_checks_enabled()) return GDR_OK;
    bool bad = false;
    const cudaError_t e = gdr::check_gate_range(g, n, st, &bad);
    if (e != cudaSuccess) {
        tl_last_cuda_error = (int)e;
        return GDR_ERR_CUDA;
    }
    return bad ? GDR_ERR_GATE_RANGE : GDR_OK;
}

size_t gate_elems(long long heads, int T, int dk, int gate_mode)
{
    return (size_t)heads * (size_t)T * (gate_mode == GDR_GATE_PER_CHANNEL ? (size_t)dk : 1u);
}

}  // namespace

GDR_API const char *gdr_status_string(int status)
{
    switch (status) {
        case GDR_OK: return "GDR_OK";
        case GDR_ERR_INVALID_ARG: return "GDR_ERR_INVALID_ARG";
        case GDR_ERR_UNSUPPORTED: return "GDR_ERR_UNSUPPORTED";
        case GDR_ERR_ALIGNMENT: return "GDR_ERR_ALIGNMENT";
        case GDR_ERR_CUDA: return "GDR_ERR_CUDA";
        case GDR_ERR_GATE_RANGE: return "GDR_ERR_GATE_RANGE";
        case GDR_ERR_TIMEOUT: return "GDR_ERR_TIMEOUT";
        default: return "GDR_ERR_UNKNOWN";
    }
}

GDR_API int gdr_last_cuda_error(void) { return tl_last_cuda_error; }

GDR_API int gdr_last_launch_count(void) { return tl_last_launches; }

GDR_API void gdr_debug_set_wait_budget(long long cycles) { gdr::set_wait_budget(cycles); }

GDR_API size_t gdr_chunk_fwd_workspace_size(int B, int H, int T, int dk, int dv, int C, int gate_mode, int dtype)
{
    if (B <= 0 || H <= 0 || T <= 0) return 0;
    if (gate_mode != GDR_GATE_PER_CHANNEL && gate_mode != GDR_GATE_SCALAR) return 0;
    gdr::ChunkArgs a = {};
    a.B = B; a.H = H; a.T = T; a.dk = dk; a.dv = dv; a.C = C;
    a.scalar_gate = (gate_mode == GDR_GATE_SCALAR);
    a.bf16 = (dtype == GDR_BF16);
    return gdr::chunk_tc_supports(a) ? gdr::chunk_tc_workspace_bytes(B, H, T) : 0;
}

GDR_API int gdr_device_status(void *stream)
{
    int v = 0;
    cudaError_t e = gdr::read_device_status(static_cast<cudaStream_t>(stream), &v);
    if (e != cudaSuccess) {
        tl_last_cuda_error = (int)e;
        return GDR_ERR_CUDA;
    }
    return v;
}

GDR_API int gdr_chunk_fwd(const void *q, const void *k, const void *v, const float *g, const float *beta,
                          const float *S0, void *O, float *S_T,
                          int B, int H, int T, int dk, int dv, int C, int gate_mode, int dtype,
                          void *workspace, size_t ws_bytes, void *stream)
{
    if (B < 0 || H < 0 || T < 0) return GDR_ERR_INVALID_ARG;
    if (gate_mode != GDR_GATE_PER_CHANNEL && gate_mode != GDR_GATE_SCALAR) return GDR_ERR_INVALID_ARG;
    if (dtype != GDR_F32 && dtype != GDR_BF16) return GDR_ERR_INVALID_ARG;
    if (dk <= 0 || dv <= 0 || C <= 0) return GDR_ERR_INVALID_ARG;
    if (!size_ok(dk) || !size_ok(dv) || !(C == 16 || C == 32 || C == 64)) return GDR_ERR_UNSUPPORTED;
    if ((long long)B * H * T * (dk > dv ? dk : dv) >= (1LL << 40)) return GDR_ERR_UNSUPPORTED;
    const size_t ws_need = gdr_chunk_fwd_workspace_size(B, H, T, dk, dv, C, gate_mode, dtype);
    if (ws_bytes < ws_need || (ws_need && !workspace)) return GDR_ERR_INVALID_ARG;
    const long long heads = (long long)B * H;
    if (heads == 0) {
        tl_last_launches = 0;
        return GDR_OK;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        // nothing to read or write per token; the final state is the initial one
        if (S_T && !aligned16(S_T)) return GDR_ERR_ALIGNMENT;
        if (S0 && !aligned16(S0)) return GDR_ERR_ALIGNMENT;
        cudaError_t e = cudaSuccess;
        const size_t bytes = sizeof(float) * (size_t)heads * dv * dk;
        if (S_T && S0 && S_T != S0) e = cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, st);
        else if (S_T && !S0) e = cudaMemsetAsync(S_T, 0, bytes, st);
        return finish(e, 0);
    }
    if (!q || !k || !v || !g || !beta || !O) return GDR_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, g, beta, S0, O, S_T, workspace};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDR_ERR_ALIGNMENT;

    gdr::ChunkArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S0 = S0; a.O = O; a.S_T = S_T;
    a.B = B; a.H = H; a.T = T; a.dk = dk; a.dv = dv; a.C = C;
    a.scalar_gate = (gate_mode == GDR_GATE_SCALAR);
    a.bf16 = (dtype == GDR_BF16);
    a.workspace = workspace;
    if (const int gs = gate_guard(g, gate_elems(heads, T, dk, gate_mode), st)) return gs;
    int launches = 0;
    cudaError_t e = gdr::chunk_tc_supports(a) ? gdr::launch_chunk_tc(a, st, &launches)
                                              : gdr::launch_chunk_simt(a, st, &launches);
    return finish(e, launches);
}

GDR_API int gdr_chunk_fwd_prologue(const void *q_raw, const void *k_raw, const void *v, const void *a,
                                   const float *A_log, const float *dt_bias, const float *b_logit,
                                   const float *S0, void *O, float *S_T,
                                   int B, int H, int T, int dk, int dv, int C, int gate_mode, int dtype,
                                   void *workspace, size_t ws_bytes, void *stream)
{
    if (B < 0 || H < 0 || T < 0) return GDR_ERR_INVALID_ARG;
    if (gate_mode != GDR_GATE_PER_CHANNEL && gate_mode != GDR_GATE_SCALAR) return GDR_ERR_INVALID_ARG;
    if (dtype != GDR_F32 && dtype != GDR_BF16) return GDR_ERR_INVALID_ARG;
    if (dk <= 0 || dv <= 0 || C <= 0) return GDR_ERR_INVALID_ARG;
    gdr::ChunkArgs a_;
    a_.dk = dk; a_.dv = dv; a_.C = C; a_.bf16 = (dtype == GDR_BF16);
    if (!gdr::chunk_tc_supports(a_)) return GDR_ERR_UNSUPPORTED;   // bf16, d_k = d_v = 128, C = 64 only
    if ((long long)B * H * T * 128 >= (1LL << 40)) return GDR_ERR_UNSUPPORTED;
    const size_t ws_need = gdr_chunk_fwd_workspace_size(B, H, T, dk, dv, C, gate_mode, dtype);
    if (ws_bytes < ws_need || (ws_need && !workspace)) return GDR_ERR_INVALID_ARG;
    const long long heads = (long long)B * H;
    if (heads == 0) {
        tl_last_launches = 0;
        return GDR_OK;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (S_T && !aligned16(S_T)) return GDR_ERR_ALIGNMENT;
        if (S0 && !aligned16(S0)) return GDR_ERR_ALIGNMENT;
        cudaError_t e = cudaSuccess;
        const size_t bytes = sizeof(float) * (size_t)heads * dv * dk;
        if (S_T && S0 && S_T != S0) e = cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, st);
        else if (S_T && !S0) e = cudaMemsetAsync(S_T, 0, bytes, st);
        return finish(e, 0);
    }
    if (!q_raw || !k_raw || !v || !a || !A_log || !dt_bias || !b_logit || !O) return GDR_ERR_INVALID_ARG;
    const void *ptrs[] = {q_raw, k_raw, v, a, dt_bias, S0, O, S_T, workspace};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDR_ERR_ALIGNMENT;
    if (reinterpret_cast<uintptr_t>(A_log) % 4 || reinterpret_cast<uintptr_t>(b_logit) % 4) return GDR_ERR_ALIGNMENT;

    gdr::ChunkArgs c;
    c.q = q_raw; c.k = k_raw; c.v = v;
    c.g = static_cast<const float *>(a);   // the bf16 pre-activation, reinterpreted by the prologue kernel
    c.beta = b_logit; c.S0 = S0; c.O = O; c.S_T = S_T;
    c.B = B; c.H = H; c.T = T; c.dk = dk; c.dv = dv; c.C = C;
    c.scalar_gate = (gate_mode == GDR_GATE_SCALAR);
    c.bf16 = true;
    c.workspace = workspace;
    c.prologue = true;
    c.A_log = A_log;
    c.dt_bias = dt_bias;
    int launches = 0;
    cudaError_t e = gdr::launch_chunk_tc(c, st, &launches);
    return finish(e, launches);
}

GDR_API int gdr_chunk_fwd_gated(const void *q, const void *k, const void *v, const float *g, const float *beta,
                                const void *gate, const float *norm_w, float eps,
                                const float *S0, void *Y, float *S_T,
                                int B, int H, int T, int dk, int dv, int C, int gate_mode, int dtype,
                                void *workspace, size_t ws_bytes, void *stream)
{
    if (B < 0 || H < 0 || T < 0) return GDR_ERR_INVALID_ARG;
    if (gate_mode != GDR_GATE_PER_CHANNEL && gate_mode != GDR_GATE_SCALAR) return GDR_ERR_INVALID_ARG;
    if (dtype != GDR_F32 && dtype != GDR_BF16) return GDR_ERR_INVALID_ARG;
    if (dk <= 0 || dv <= 0 || C <= 0) return GDR_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || eps > 1e30f) return GDR_ERR_INVALID_ARG;   // also rejects NaN
    gdr::ChunkArgs a_;
    a_.dk = dk; a_.dv = dv; a_.C = C; a_.bf16 = (dtype == GDR_BF16);
    if (!gdr::chunk_tc_supports(a_)) return GDR_ERR_UNSUPPORTED;   // bf16, d_k = d_v = 128, C = 64 only
    if ((long long)B * H * T * 128 >= (1LL << 40)) return GDR_ERR_UNSUPPORTED;
    const size_t ws_need = gdr_chunk_fwd_workspace_size(B, H, T, dk, dv, C, gate_mode, dtype);
    if (ws_bytes < ws_need || (ws_need && !workspace)) return GDR_ERR_INVALID_ARG;
    const long long heads = (long long)B * H;
    if (heads == 0) {
        tl_last_launches = 0;
        return GDR_OK;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (S_T && !aligned16(S_T)) return GDR_ERR_ALIGNMENT;
        if (S0 && !aligned16(S0)) return GDR_ERR_ALIGNMENT;
        cudaError_t e = cudaSuccess;
        const size_t bytes = sizeof(float) * (size_t)heads * dv * dk;
        if (S_T && S0 && S_T != S0) e = cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, st);
        else if (S_T && !S0) e = cudaMemsetAsync(S_T, 0, bytes, st);
        return finish(e, 0);
    }
    if (!q || !k || !v || !g || !beta || !gate || !norm_w || !Y) return GDR_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, g, beta, gate, S0, Y, S_T, workspace};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDR_ERR_ALIGNMENT;
    if (reinterpret_cast<uintptr_t>(norm_w) % 4) return GDR_ERR_ALIGNMENT;

    gdr::ChunkArgs c;
    c.q = q; c.k = k; c.v = v; c.g = g; c.beta = beta; c.S0 = S0; c.O = Y; c.S_T = S_T;
    c.B = B; c.H = H; c.T = T; c.dk = dk; c.dv = dv; c.C = C;
    c.scalar_gate = (gate_mode == GDR_GATE_SCALAR);
    c.bf16 = true;
    c.workspace = workspace;
    c.gated_out = true;
    c.ogate = gate;
    c.norm_w = norm_w;
    c.eps = eps;
    if (const int gs = gate_guard(g, gate_elems(heads, T, dk, gate_mode), st)) return gs;
    int launches = 0;
    cudaError_t e = gdr::launch_chunk_tc(c, st, &launches);
    return finish(e, launches);
}

GDR_API size_t gdr_chunk_bwd_workspace_size(int B, int H, int T, int dk, int dv, int C, int gate_mode, int dtype)
{
    if (B <= 0 || H <= 0 || T <= 0) return 0;
    if (gate_mode != GDR_GATE_PER_CHANNEL && gate_mode != GDR_GATE_SCALAR) return 0;
    if (dtype != GDR_F32 && dtype != GDR_BF16) return 0;
    if (dk != dv || !size_ok(dk) || C != 64) return 0;
    return gdr::chunk_bwd_workspace_bytes(B, H, T, dk);
}

GDR_API int gdr_chunk_bwd(const void *q, const void *k, const void *v, const float *g, const float *beta,
                          const float *S0, const void *dO, const float *dS_T,
                          void *dq, void *dk, void *dv, float *dg, float *dbeta, float *dS0,
                          int B, int H, int T, int dk_, int dv_, int C, int gate_mode, int dtype,
                          void *workspace, size_t ws_bytes, void *stream)
{
    if (B < 0 || H < 0 || T < 0) return GDR_ERR_INVALID_ARG;
    if (gate_mode != GDR_GATE_PER_CHANNEL && gate_mode != GDR_GATE_SCALAR) return GDR_ERR_INVALID_ARG;
    if (dtype != GDR_F32 && dtype != GDR_BF16) return GDR_ERR_INVALID_ARG;
    if (dk_ <= 0 || dv_ <= 0 || C <= 0) return GDR_ERR_INVALID_ARG;
    if (dk_ != dv_ || !size_ok(dk_) || C != 64) return GDR_ERR_UNSUPPORTED;
    if ((long long)B * H * T * dk_ >= (1LL << 40)) return GDR_ERR_UNSUPPORTED;
    const long long heads = (long long)B * H;
    if (heads == 0) {
        tl_last_launches = 0;
        return GDR_OK;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        // no tokens: S_T = S0, so dS0 = dS_T
        if (dS0 && !aligned16(dS0)) return GDR_ERR_ALIGNMENT;
        if (dS_T && !aligned16(dS_T)) return GDR_ERR_ALIGNMENT;
        cudaError_t e = cudaSuccess;
        const size_t bytes = sizeof(float) * (size_t)heads * dv_ * dk_;
        if (dS0 && dS_T && dS0 != dS_T) e = cudaMemcpyAsync(dS0, dS_T, bytes, cudaMemcpyDeviceToDevice, st);
        else if (dS0 && !dS_T) e = cudaMemsetAsync(dS0, 0, bytes, st);
        return finish(e, 0);
    }
    const size_t ws_need = gdr_chunk_bwd_workspace_size(B, H, T, dk_, dv_, C, gate_mode, dtype);
    if (ws_bytes < ws_need || !workspace) return GDR_ERR_INVALID_ARG;
    if (!q || !k || !v || !g || !beta || !dO || !dq || !dk || !dv || !dg || !dbeta) return GDR_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, g, beta, S0, dO, dS_T, dq, dk, dv, dg, dbeta, dS0, workspace};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDR_ERR_ALIGNMENT;
    gdr::BwdArgs a;
    a.q = q; a.k = k; a.v = v; a.dO = dO; a.g = g; a.beta = beta; a.S0 = S0; a.dS_T = dS_T;
    a.dq = dq; a.dk = dk; a.dv = dv; a.dg = dg; a.dbeta = dbeta; a.dS0 = dS0;
    a.B = B; a.H = H; a.T = T; a.D = dk_;
    a.scalar_gate = (gate_mode == GDR_GATE_SCALAR);
    a.bf16 = (dtype == GDR_BF16);
    a.workspace = workspace;
    if (const int gs = gate_guard(g, gate_elems(heads, T, dk_, gate_mode), st)) return gs;
    int launches = 0;
    cudaError_t e = gdr::launch_chunk_bwd(a, st, &launches);
    return finish(e, launches);
}

GDR_API size_t gdr2_chunk_fwd_workspace_size(int B, int H, int T, int dk, int dv, int C, int gate_mode, int dtype)
{
    if (B <= 0 || H <= 0 || T <= 0) return 0;
    if (gate_mode != GDR_GATE_PER_CHANNEL && gate_mode != GDR_GATE_SCALAR) return 0;
    gdr::ChunkArgs a = {};
    a.dk = dk; a.dv = dv; a.C = C;
    a.bf16 = (dtype == GDR_BF16);
    return gdr::chunk_tc_supports(a) ? gdr::chunk_tc_workspace_bytes(B, H, T, true) : 0;
}

GDR_API int gdr2_chunk_fwd(const void *q, const void *k, const void *v, const float *g, const void *b,
                           const void *w, const float *S0, void *O, float *S_T,
                           int B, int H, int T, int dk, int dv, int C, int gate_mode, int dtype,
                           void *workspace, size_t ws_bytes, void *stream)
{
    if (B < 0 || H < 0 || T < 0) return GDR_ERR_INVALID_ARG;
    if (gate_mode != GDR_GATE_PER_CHANNEL && gate_mode != GDR_GATE_SCALAR) return GDR_ERR_INVALID_ARG;
    if (dtype != GDR_F32 && dtype != GDR_BF16) return GDR_ERR_INVALID_ARG;
    if (dk <= 0 || dv <= 0 || C <= 0) return GDR_ERR_INVALID_ARG;
    gdr::ChunkArgs a_;
    a_.dk = dk; a_.dv = dv; a_.C = C; a_.bf16 = (dtype == GDR_BF16);
    if (!gdr::chunk_tc_supports(a_)) return GDR_ERR_UNSUPPORTED;   // bf16, d_k = d_v = 128, C = 64 only
    if ((long long)B * H * T * 128 >= (1LL << 40)) return GDR_ERR_UNSUPPORTED;
    const size_t ws_need = gdr2_chunk_fwd_workspace_size(B, H, T, dk, dv, C, gate_mode, dtype);
    if (ws_bytes < ws_need || (ws_need && !workspace)) return GDR_ERR_INVALID_ARG;
    const long long heads = (long long)B * H;
    if (heads == 0) {
        tl_last_launches = 0;
        return GDR_OK;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (S_T && !aligned16(S_T)) return GDR_ERR_ALIGNMENT;
        if (S0 && !aligned16(S0)) return GDR_ERR_ALIGNMENT;
        cudaError_t e = cudaSuccess;
        const size_t bytes = sizeof(float) * (size_t)heads * dv * dk;
        if (S_T && S0 && S_T != S0) e = cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, st);
        else if (S_T && !S0) e = cudaMemsetAsync(S_T, 0, bytes, st);
        return finish(e, 0);
    }
    if (!q || !k || !v || !g || !b || !w || !O) return GDR_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, g, b, w, S0, O, S_T, workspace};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDR_ERR_ALIGNMENT;

    gdr::ChunkArgs c;
    c.q = q; c.k = k; c.v = v; c.g = g; c.beta = nullptr; c.S0 = S0; c.O = O; c.S_T = S_T;
    c.B = B; c.H = H; c.T = T; c.dk = dk; c.dv = dv; c.C = C;
    c.scalar_gate = (gate_mode == GDR_GATE_SCALAR);
    c.bf16 = true;
    c.workspace = workspace;
    c.gdr2 = true;
    c.erase = b;
    c.write = w;
    if (const int gs = gate_guard(g, gate_elems(heads, T, dk, gate_mode), st)) return gs;
    int launches = 0;
    cudaError_t e = gdr::launch_chunk_tc(c, st, &launches);
    return finish(e, launches);
}

GDR_API int gdr2_recurrent_step(const void *q, const void *k, const void *v, const float *g, const void *b,
                                const void *w, float *S, void *o, int B, int H, int dk, int dv, int gate_mode,
                                int dtype, void *stream)
{
    if (B < 0 || H < 0) return GDR_ERR_INVALID_ARG;
    if (gate_mode != GDR_GATE_PER_CHANNEL && gate_mode != GDR_GATE_SCALAR) return GDR_ERR_INVALID_ARG;
    if (dtype != GDR_F32 && dtype != GDR_BF16) return GDR_ERR_INVALID_ARG;
    if (dk <= 0 || dv <= 0) return GDR_ERR_INVALID_ARG;
    if (!size_ok(dk) || !size_ok(dv)) return GDR_ERR_UNSUPPORTED;
    if ((long long)B * H * dv * dk >= (1LL << 40)) return GDR_ERR_UNSUPPORTED;
    if ((long long)B * H == 0) {
        tl_last_launches = 0;
        return GDR_OK;
    }
    if (!q || !k || !v || !g || !b || !w || !S || !o) return GDR_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, g, b, w, S, o};
    for (const void *p : ptrs)
        if (!aligned16(p)) return GDR_ERR_ALIGNMENT;
    gdr::StepArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = nullptr; a.S = S; a.o = o;
    a.B = B; a.H = H; a.dk = dk; a.dv = dv;
    a.scalar_gate = (gate_mode == GDR_GATE_SCALAR);
    a.bf16 = (dtype == GDR_BF16);
    a.gdr2 = true;
    a.erase = b;
    a.write = w;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (const int gs = gate_guard(g, gate_elems((long long)B * H, 1, dk, gate_mode), st)) return gs;
    int launches = 0;
    cudaError_t e = gdr::launch_recurrent_step(a, st, &launches);
    return finish(e, launches);
}

GDR_API int gdr_recurrent_step(const void *q, const void *k, const void *v, const float *g, const float *beta,
                               float *S, void *o, int B, int H, int dk, int dv, int gate_mode, int dtype,
                               void *stream)
{
    if (B < 0 || H < 0) return GDR_ERR_INVALID_ARG;
    if (gate_mode != GDR_GATE_PER_CHANNEL && gate_mode != GDR_GATE_SCALAR) return GDR_ERR_INVALID_ARG;
    if (dtype != GDR_F32 && dtype != GDR_BF16) return GDR_ERR_INVALID_ARG;
    if (dk <= 0 || dv <= 0) return GDR_ERR_INVALID_ARG;
    if (!size_ok(dk) || !size_ok(dv)) return GDR_ERR_UNSUPPORTED;
    if ((long long)B * H * dv * dk >= (1LL << 40)) return GDR_ERR_UNSUPPORTED;
    if ((long long)B * H == 0) {
        tl_last_launches = 0;
        return GDR_OK;
    }
    if (!q || !k || !v || !g || !beta || !S || !o) return GDR_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, g, beta, S, o};
    for (const void *p : ptrs)
        if (!aligned16(p)) return GDR_ERR_ALIGNMENT;
    gdr::StepArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S = S; a.o = o;
    a.B = B; a.H = H; a.dk = dk; a.dv = dv;
    a.scalar_gate = (gate_mode == GDR_GATE_SCALAR);
    a.bf16 = (dtype == GDR_BF16);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (const int gs = gate_guard(g, gate_elems((long long)B * H, 1, dk, gate_mode), st)) return gs;
    int launches = 0;
    cudaError_t e = gdr::launch_recurrent_step(a, st, &launches);
    return finish(e, launches);
}
