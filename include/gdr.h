/*
 * gdr.h -- C ABI of the B200 (sm_100a) gated delta rule library (libgdr.so).
 *
 * The method (d_v x d_k orientation, o_t = S_t q_t):
 *
 *     S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *
 * as written in "Reading notes: Kimi Delta Attention" (mzeromiko), section 4
 * "Forward pass" (KDA: alpha_t in (0,1)^{d_k}, one decay per key channel) and
 * in "Token Mixer I", section "Gated Delta Networks" (Gated DeltaNet: one
 * scalar alpha_t per head).  The gate is passed as its logarithm g = log alpha
 * ("KDA vs Gated DeltaNet" (brenchcc), section 4: the state is multiplied by
 * exp(decay)).  In per-channel mode the library applies the KDA lower bound
 * g >= -5 ("Lightweight LLM reproduction: Linear Attention" (aitujian),
 * section 3.1 [7a], g_min = -5) by computing with max(g, -5); scalar gates
 * are used as given.
 *
 * Conventions shared by every call
 *   - Every tensor pointer is a DEVICE pointer owned by the caller; the
 *     library never allocates, frees or keeps a pointer after the call.
 *   - Tensors are dense, row-major (last index fastest), with the shapes
 *     given per argument below, and must be 16-byte aligned.
 *   - dtype GDR_F32 means q, k, v and the output are float; GDR_BF16 means
 *     they are bfloat16.  g, beta and every state tensor are always float.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  Argument errors are detected on the host and
 *     returned before anything is launched; a launch failure returns
 *     GDR_ERR_CUDA and the CUDA error code is kept for gdr_last_cuda_error().
 *   - Outputs must not overlap inputs, except where an argument says so.
 *   - Supported sizes: d_k, d_v in {64, 128}; chunk C in {16, 32, 64};
 *     any T >= 0, B >= 0, H >= 0.  Other sizes return GDR_ERR_UNSUPPORTED.
 *   - Functions return a gdr_status value as int.
 *   - Debug mode: when the environment variable GDR_DEBUG is set (to
 *     anything but "" or "0") at the library's first call, every entry point
 *     that takes a log-decay g first checks it on the device: a valid gate is
 *     a finite value <= 0 (alpha = exp(g) in (0, 1]).  The check synchronizes
 *     `stream`; if an element is positive, NaN or infinite the call returns
 *     GDR_ERR_GATE_RANGE and launches nothing else.  Per-channel values below
 *     -5 are legal (the -5 bound clamps them).  Debug mode adds a pass over g
 *     and a host synchronization per call, so it is not for timed or
 *     graph-captured code.
 */
#ifndef GDR_H_
#define GDR_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gdr_status {
    GDR_OK = 0,
    GDR_ERR_INVALID_ARG = 1,  /* null pointer, negative size, bad enum, short workspace */
    GDR_ERR_UNSUPPORTED = 2,  /* valid but unsupported size (d_k, d_v, C) */
    GDR_ERR_ALIGNMENT = 3,    /* a tensor pointer is not 16-byte aligned */
    GDR_ERR_CUDA = 4,         /* a CUDA call failed; see gdr_last_cuda_error() */
    GDR_ERR_GATE_RANGE = 5,   /* debug mode (GDR_DEBUG): an element of g is > 0, NaN or infinite */
    GDR_ERR_TIMEOUT = 6       /* a bounded device wait ran out (see gdr_device_status) */
} gdr_status;

typedef enum gdr_dtype { GDR_F32 = 0, GDR_BF16 = 1 } gdr_dtype;

typedef enum gdr_gate_mode {
    GDR_GATE_PER_CHANNEL = 0, /* KDA: g has one value per key channel */
    GDR_GATE_SCALAR = 1       /* Gated DeltaNet: g has one value per head and token */
} gdr_gate_mode;

/*
 * Bytes of device workspace gdr_chunk_fwd needs for these sizes (0 when the
 * chosen kernels need none).  Returns 0 for unsupported arguments too; the
 * forward call itself reports those.
 */
size_t gdr_chunk_fwd_workspace_size(int B, int H, int T, int dk, int dv, int C,
                                    int gate_mode, int dtype);

/*
 * Chunkwise-parallel forward over a whole sequence.
 *
 * Computes, for every (b, h), O[t] = S_t q_t for t = 0..T-1 and the final
 * state S_T, starting from S0.  The work follows the chunk form of "Reading
 * notes: Kimi Delta Attention", section 4 (also "Token Mixer I", section
 * "Kimi Delta Attention: Improving Delta Rule with Fine-grained Gating", the
 * UT transform, chunk state update and chunk output equations): chunks of C
 * tokens, a per-chunk log-gate cumulative sum, the UT transform
 * A~ = (I + StrictTril(Diag(beta) (Gamma*K)(K/Gamma)^T))^{-1}, W = A~ Diag(beta)(Gamma*K),
 * U = A~ Diag(beta) V, then sequentially over chunks
 * V_new = U - W S^T,  O = (Gamma*Q) S^T + Tril((Gamma*Q)(K/Gamma)^T) V_new,
 * S <- S Diag(gamma_C) + V_new^T (K * gamma_C/Gamma).
 * The result equals the token recurrence above up to rounding; a last
 * partial chunk (T not a multiple of C) is handled exactly.
 *
 *   q, k   [B,H,T,dk]  dtype           queries / keys (not normalised here)
 *   v      [B,H,T,dv]  dtype           values
 *   g      [B,H,T,dk] (per-channel) or [B,H,T] (scalar), float: log-decay
 *   beta   [B,H,T]     float           write strength
 *   S0     [B,H,dv,dk] float           initial state; NULL = zeros
 *   O      [B,H,T,dv]  dtype           output (written)
 *   S_T    [B,H,dv,dk] float           final state (written); NULL = not
 *                                      written; may be the same pointer as
 *                                      S0 (in-place update of the state)
 *   C                                   chunk size (64 is the tuned size)
 *   workspace / ws_bytes                device scratch of at least
 *                                      gdr_chunk_fwd_workspace_size() bytes
 *                                      (may be NULL when that is 0)
 *   stream                              cudaStream_t
 */
int gdr_chunk_fwd(const void *q, const void *k, const void *v, const float *g, const float *beta,
                  const float *S0, void *O, float *S_T,
                  int B, int H, int T, int dk, int dv, int C, int gate_mode, int dtype,
                  void *workspace, size_t ws_bytes, void *stream);

/*
 * One single-token recurrent update per (b, h): the decode step.
 *
 * Follows the order of the pseudo-code in "KDA vs Gated DeltaNet", section 4
 * (decay the state, predict from the decayed state, delta, write, read), in a
 * single pass over S: S~ = S Diag(alpha); p = S~ k; delta = beta (v - p);
 * S <- S~ + delta k^T; o = S q.
 *
 *   q, k   [B,H,dk]    dtype
 *   v      [B,H,dv]    dtype
 *   g      [B,H,dk] (per-channel) or [B,H] (scalar), float
 *   beta   [B,H]       float
 *   S      [B,H,dv,dk] float           state, updated IN PLACE
 *   o      [B,H,dv]    dtype           output (written)
 */
int gdr_recurrent_step(const void *q, const void *k, const void *v, const float *g, const float *beta,
                       float *S, void *o, int B, int H, int dk, int dv, int gate_mode, int dtype,
                       void *stream);

/*
 * Chunkwise-parallel forward with the layer's input prologue fused in:
 *   q = L2Norm(q_raw), k = L2Norm(k_raw)          per head and token,
 *                                                 L2Norm(x) = x / sqrt(sum x^2 + 1e-6)
 *   g = max(-exp(A_log[h]) * softplus(a + dt_bias[h][c]), -5)   (per-channel gate)
 *   g = -exp(A_log[h]) * softplus(a + dt_bias[h])               (scalar gate)
 *   beta = sigmoid(b_logit)
 * then the same forward as gdr_chunk_fwd.  "Token Mixer I", section "Kimi
 * Delta Attention", Neural Parameterization (L2Norm of q, k; Sigmoid beta);
 * the gate of the Kimi Linear notes (-exp(A_log) softplus(. + dt_bias), A_log
 * of shape [H], dt_bias [H * d_k]); the lower bound g_min = -5 of KDA.
 *
 * Arguments as gdr_chunk_fwd, except:
 *   q_raw, k_raw   [B,H,T,d_k]  not normalised
 *   a              [B,H,T,d_k] (per-channel) or [B,H,T] (scalar), dtype as q
 *   A_log          [H] fp32; dt_bias [H,d_k] (per-channel) or [H] (scalar) fp32
 *   b_logit        [B,H,T] fp32
 * Only the tensor-core configuration (bf16, d_k = d_v = 128, C = 64) runs;
 * anything else returns GDR_ERR_UNSUPPORTED.  Same workspace as
 * gdr_chunk_fwd (gdr_chunk_fwd_workspace_size).  a and dt_bias must be
 * 16-byte aligned like the other tensors; A_log and b_logit 4-byte aligned.
 */
int gdr_chunk_fwd_prologue(const void *q_raw, const void *k_raw, const void *v, const void *a,
                           const float *A_log, const float *dt_bias, const float *b_logit,
                           const float *S0, void *O, float *S_T,
                           int B, int H, int T, int dk, int dv, int C, int gate_mode, int dtype,
                           void *workspace, size_t ws_bytes, void *stream);

/*
 * Chunkwise forward with the layer's output epilogue fused in ("Token Mixer
 * I", section "The Kimi Linear Model Architecture": before the output
 * projection W_o, a per-head RMSNorm of the output and a data-dependent
 * sigmoid gate):
 *   Y[b,h,t,:] = Sigmoid(gate[b,h,t,:]) * RMSNorm(o_t),
 *   RMSNorm(x) = x / sqrt(mean_c x_c^2 + eps) * norm_w        (c over the d_v channels)
 * with o_t the output gdr_chunk_fwd would write.  The normalisation is taken
 * in fp32 from the accumulator, before any rounding of o_t.
 *
 * Arguments as gdr_chunk_fwd, plus
 *   gate     [B,H,T,d_v]   dtype       pre-activation of the output gate
 *   norm_w   [d_v]         float       RMSNorm weight (shared by the heads)
 *   eps      >= 0                      RMSNorm epsilon
 * and Y [B,H,T,d_v] (dtype) in place of O.  Only the tensor-core
 * configuration (bf16, d_k = d_v = 128, C = 64) runs; anything else returns
 * GDR_ERR_UNSUPPORTED.  Same workspace as gdr_chunk_fwd.  norm_w must be
 * 4-byte aligned, the other tensors 16-byte aligned.
 */
int gdr_chunk_fwd_gated(const void *q, const void *k, const void *v, const float *g, const float *beta,
                        const void *gate, const float *norm_w, float eps,
                        const float *S0, void *Y, float *S_T,
                        int B, int H, int T, int dk, int dv, int C, int gate_mode, int dtype,
                        void *workspace, size_t ws_bytes, void *stream);

/*
 * Backward pass of the chunkwise forward: the gradients of
 *   L = <dO, O> + <dS_T, S_T>
 * with respect to q, k, v, g, beta and S0, where (O, S_T) is what
 * gdr_chunk_fwd returns for the same inputs.  It differentiates the same
 * chunk form (UT transform, chunk state recurrence and output: "Token Mixer
 * I", section "Kimi Delta Attention: Improving Delta Rule with Fine-grained
 * Gating"; the training path of the section "Gated Delta Networks"): the
 * states at chunk boundaries are recomputed, the state gradient runs through
 * the chunks in reverse, and the rest is parallel over chunks.  fp32
 * arithmetic; for bf16 inputs at d = 128 the matrix products take tf32
 * operands (rounded from fp32) on the tensor cores, accumulating in fp32.
 * The -5 bound on a per-channel g passes the gradient where g >= -5 and
 * blocks it below.
 *
 *   q, k, v, g, beta, S0   as gdr_chunk_fwd (S0 NULL -> zeros)
 *   dO     [B,H,T,d_v]   dtype                  gradient of O
 *   dS_T   [B,H,d_v,d_k] float or NULL (zeros)  gradient of S_T
 *   dq, dk [B,H,T,d_k], dv [B,H,T,d_v]   dtype  (written)
 *   dg     layout of g, float                   (written)
 *   dbeta  [B,H,T] float                        (written)
 *   dS0    [B,H,d_v,d_k] float or NULL          (written if given)
 * Supported: d_k = d_v in {64, 128}, C = 64, fp32 or bf16; anything else
 * returns GDR_ERR_UNSUPPORTED.  The workspace (device, >=
 * gdr_chunk_bwd_workspace_size() bytes, 16-byte aligned) holds the
 * recomputed chunk quantities and the per-chunk states and state gradients:
 * 384 KB per 64-token chunk at d = 128.
 */
size_t gdr_chunk_bwd_workspace_size(int B, int H, int T, int dk, int dv, int C, int gate_mode, int dtype);

int gdr_chunk_bwd(const void *q, const void *k, const void *v, const float *g, const float *beta,
                  const float *S0, const void *dO, const float *dS_T,
                  void *dq, void *dk, void *dv, float *dg, float *dbeta, float *dS0,
                  int B, int H, int T, int dk_, int dv_, int C, int gate_mode, int dtype,
                  void *workspace, size_t ws_bytes, void *stream);

/*
 * Gated Delta Rule-2: the erase and write decisions of the delta rule get
 * their own per-channel gates ("Token Mixer I", section "Gated DeltaNet-2:
 * Decoupling Erase and Write in Linear Attention", eq. (10)).  With
 * S~ = S_{t-1} Diag(alpha_t), in the d_v x d_k orientation of gdr_chunk_fwd:
 *   delta = w_t * v_t - S~ (b_t * k_t),   S_t = S~ + delta k_t^T,   o_t = S_t q_t
 * b_t in [0,1]^d_k is the erase gate (the key coordinates the old content is
 * read along), w_t in [0,1]^d_v the write gate (the value coordinates
 * written).  b = w = beta 1 gives gdr_chunk_fwd / gdr_recurrent_step.  The
 * chunked form follows the section's "Chunkwise parallel training": T' =
 * (I + StrictTril((b * K<-) K->^T))^{-1}, Y = T' (b * K<-), U = T' (w * V).
 *
 * gdr2_chunk_fwd: arguments as gdr_chunk_fwd, with beta replaced by
 *   b   [B,H,T,d_k]   dtype (as q, k)     erase gate
 *   w   [B,H,T,d_v]   dtype (as v)        write gate
 * Only the tensor-core configuration (bf16, d_k = d_v = 128, C = 64) runs;
 * anything else returns GDR_ERR_UNSUPPORTED.  The -5 lower bound applies to
 * a per-channel gate as in gdr_chunk_fwd.  Its workspace is larger than
 * gdr_chunk_fwd's (it also holds w * v): size it with
 * gdr2_chunk_fwd_workspace_size (0 for unsupported arguments).
 */
size_t gdr2_chunk_fwd_workspace_size(int B, int H, int T, int dk, int dv, int C,
                                     int gate_mode, int dtype);

int gdr2_chunk_fwd(const void *q, const void *k, const void *v, const float *g, const void *b, const void *w,
                   const float *S0, void *O, float *S_T,
                   int B, int H, int T, int dk, int dv, int C, int gate_mode, int dtype,
                   void *workspace, size_t ws_bytes, void *stream);

/*
 * gdr2_recurrent_step: one Gated Delta Rule-2 decode step, arguments as
 * gdr_recurrent_step with beta replaced by
 *   b   [B,H,d_k]   dtype     erase gate
 *   w   [B,H,d_v]   dtype     write gate
 * Same sizes and dtypes as gdr_recurrent_step (d_k, d_v in {64, 128}; fp32
 * or bf16); S is updated in place.
 */
int gdr2_recurrent_step(const void *q, const void *k, const void *v, const float *g, const void *b, const void *w,
                        float *S, void *o, int B, int H, int dk, int dv, int gate_mode, int dtype,
                        void *stream);

/*
 * Chunked forward that allocates nothing, for callers that cannot allocate
 * device memory or pass a workspace at the point of the call: serving or
 * real-time loops that forbid allocator calls on their hot path, code that
 * keeps allocator calls out of a region it records as a CUDA graph, hosts
 * whose device memory belongs to another runtime or a pool the caller cannot
 * reach.  The pages have no counterpart to this call; it is an interface
 * convenience of this library.
 *
 * Same arguments, layouts and results as gdr_chunk_fwd, without the
 * workspace: the scratch the tensor-core path needs comes from one fixed
 * array the library holds in device memory, GDR_NOALLOC_SCRATCH_BYTES on
 * every GPU where the library is loaded, until the process exits.
 *   - Problems whose gdr_chunk_fwd_workspace_size() exceeds
 *     GDR_NOALLOC_SCRATCH_BYTES are rejected with GDR_ERR_UNSUPPORTED before
 *     any launch (bf16 d=128 needs 66,048 bytes per 64-token chunk, so at
 *     most 508 full chunks, B*H*ceil(T/64) <= 508, fit).
 *   - Every call shares that array.  Calls that may overlap on the GPU
 *     (unordered streams, several host threads) race on it and give
 *     undefined results; order them.  Nothing has to be cleared between
 *     calls.
 *   - The first call made with a given device current looks up the array's
 *     device address (cudaGetSymbolAddress) and caches it; make that first
 *     call before any stream capture begins.  A failed look-up returns
 *     GDR_ERR_CUDA without launching anything.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define GDR_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

int gdr_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const float *g, const float *beta,
                          const float *S0, void *O, float *S_T,
                          int B, int H, int T, int dk, int dv, int C, int gate_mode, int dtype,
                          void *stream);

/*
 * Device-side status.  Kernels that wait on other warps of their own block
 * bound every wait (about a second); when one runs out the kernel records
 * GDR_ERR_TIMEOUT in a device status word, stops, and leaves its outputs
 * undefined.  This call synchronizes `stream`, returns that word (GDR_OK if
 * no kernel recorded anything since the last call) and clears it.  It may
 * return GDR_ERR_CUDA if the synchronization itself fails.
 */
int gdr_device_status(void *stream);

/*
 * Testing aid for the timeout path: the number of SM clock cycles each
 * bounded device wait of the kernels launched after this call may take
 * before it gives up (process-wide; cycles <= 0 restores the default of
 * about two billion cycles, about a second).  With a budget far below the
 * time the pipeline's hand-offs take, a call's waits run out: the kernel
 * records GDR_ERR_TIMEOUT (read it with gdr_device_status), lets the copies
 * and tensor-core operations it issued finish, frees its tensor memory and
 * returns; its outputs are undefined.  Not for production use.
 */
void gdr_debug_set_wait_budget(long long cycles);

/* Human-readable name of a status value (static string, never NULL). */
const char *gdr_status_string(int status);

/* The last cudaError_t value a call of this thread met (0 if none). */
int gdr_last_cuda_error(void);

/*
 * Number of kernel launches the last successful call of this thread issued
 * (lets a caller count device launches without a profiler).
 */
int gdr_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H_ */
