/*
 * ckda.h: C ABI of the CKDA (Complex Kimi Delta Attention) CUDA library for
 * NVIDIA B200 (sm_100a).
 *
 * The operation (Semidirect Fourier Delta Attention, §1 eq. (1) and §2.2
 * eq. (9); readout §3 eq. (14); value ranges from Complex KDA, abstract):
 *
 *     S_t = (I - beta_t k_t k_t^T) diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = scale * S_t^T q_t        (the state after the update is read)
 *
 * per sequence and head, with a channel-wise gate alpha_t in [-1,1]^{d_k}
 * (negative and exactly-zero gates allowed; KDA's (0,1) is a special case), a
 * scalar beta_t in [0,2], and a d_k x d_v fp32 state carried across tokens.
 * The library does not clamp or check the ranges of alpha and beta; values
 * outside them are computed as given.
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers on the current CUDA device unless
 *    a parameter says "host". The caller owns every buffer, scratch included
 *    (ckda_fwd_workspace_bytes says how much); the library never allocates
 *    device memory and keeps no pointer after a call returns.
 *  - Layouts are dense, row-major (C order), last dimension contiguous:
 *      q, k     [T, H, d_k]     v, o      [T, H, d_v]
 *      alpha    [T, H, d_k] fp32          beta      [T, H]  fp32
 *      states   [N, H, d_k, d_v] fp32 (d_v contiguous)
 *    q, k, v and o share one element type (ckda_dtype); alpha, beta and the
 *    states are always fp32. Every pointer must be 16-byte aligned.
 *  - Supported sizes: d_k, d_v in {16, 32, 64, 128}; H >= 1. The chunked
 *    forward, the backward and the complex-phase forward take N and H up to
 *    65535 (CKDA_ERR_UNSUPPORTED beyond).
 *  - Calls are asynchronous on `stream` (0 = legacy default stream). Argument
 *    errors are detected on the host and returned before anything is
 *    launched. Launch failures return CKDA_ERR_CUDA. Errors found by a kernel
 *    (e.g. a malformed device-only cu_seqlens) are recorded in a per-device
 *    error word and reported by ckda_last_error().
 *  - Deterministic: no atomics in any reduction, so results are bitwise
 *    reproducible run to run on the same GPU and arguments.
 */
#ifndef CKDA_H
#define CKDA_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CKDA_OK = 0,
  CKDA_ERR_ARG = 1,          /* null/misaligned pointer, bad size, bad cu_seqlens */
  CKDA_ERR_UNSUPPORTED = 2,  /* d_k, d_v, chunk, dtype or N, H outside the supported set */
  CKDA_ERR_CUDA = 3,         /* a CUDA runtime call or kernel launch failed */
  CKDA_ERR_DEVICE = 4        /* a kernel flagged an error (see ckda_last_error) */
} ckda_status;

typedef enum {
  CKDA_BF16 = 0,             /* q, k, v, o are bfloat16 */
  CKDA_F32 = 1               /* q, k, v, o are float32 (fp32 check mode) */
} ckda_dtype;

/*
 * ckda_fwd_chunked: chunkwise-parallel forward (prefill) of the recurrence
 * over packed sequences.
 *
 * Chunking is an execution strategy only: inside each chunk of `chunk`
 * tokens the kernels build the chunk's WY / UT-transform factors (the
 * compact representation of the product of diagonal-plus-rank-one
 * transitions and its triangular solve, Semidirect Fourier Delta Attention
 * §2.2) and carry the state from chunk to chunk through the affine chunk
 * transfer (§1, contribution 4); the results equal the token recurrence up to
 * rounding ("chunkwise execution changes cost, never the numbers": Kimi Delta
 * Attention: a bounded case study, Exercise 2).
 *
 * q, k          [T_total, H, d_k] (dt)      token-major, packed sequences
 * v             [T_total, H, d_v] (dt)
 * alpha         [T_total, H, d_k] fp32      channel-wise gate
 * beta          [T_total, H]      fp32      delta coefficient
 * initial_state [N, H, d_k, d_v]  fp32 or NULL (NULL = zero state)
 * final_state   [N, H, d_k, d_v]  fp32 or NULL (NULL = not written); may be
 *               the same buffer as initial_state (read before written)
 * o             [T_total, H, d_v] (dt)      output; must not alias any input
 * cu_seqlens    device int32 [N+1] or NULL. NULL: N sequences of T tokens
 *               each (T_total = N*T). Otherwise sequence n owns tokens
 *               [cu[n], cu[n+1]), with cu[0]=0, non-decreasing, cu[N]=T and
 *               T = T_total. Zero-length sequences are allowed (their final
 *               state equals their initial state).
 * cu_seqlens_host optional host copy of cu_seqlens (may be NULL). When given
 *               it is validated on the host (CKDA_ERR_ARG if malformed).
 *               When NULL the kernels validate the device copy and record
 *               CKDA_ERR_DEVICE (skipping the bad sequence) instead.
 * N, T, H, d_k, d_v  sizes as above (N >= 0, T >= 0).
 * chunk         chunk length: 0 (default 64), 16, 32 or 64.
 * scale         multiplies every output (o_t = scale * S_t^T q_t).
 * dt            element type of q, k, v and o.
 * workspace     device scratch of at least workspace_bytes bytes, 16-byte
 *               aligned, owned by the caller, or NULL when
 *               ckda_fwd_workspace_bytes() returns 0 for these arguments.
 *               Its contents on entry are ignored; it must not overlap any
 *               other argument, and two calls running at the same time on
 *               the GPU must not share it.
 * workspace_bytes  size of workspace (CKDA_ERR_ARG if too small).
 */
ckda_status ckda_fwd_chunked(const void *q, const void *k, const void *v,
                             const float *alpha, const float *beta,
                             const float *initial_state, float *final_state,
                             void *o, const int32_t *cu_seqlens,
                             const int32_t *cu_seqlens_host, int32_t N,
                             int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                             int32_t chunk, float scale, ckda_dtype dt,
                             void *workspace, size_t workspace_bytes,
                             cudaStream_t stream);

/*
 * ckda_fwd_workspace_bytes: scratch that ckda_fwd_chunked needs for these
 * arguments (same meaning as there; varlen != 0 means cu_seqlens is given, so
 * T is the total token count). The tensor-core path (bf16, d_k = 128, chunk
 * 64, d_v in {32, 64, 128}) keeps each chunk's state-independent factors
 * there between its two kernels: about 160 KB per (chunk, head) for d_v = 128,
 * for floor(T_total / 64) + N chunk slots. Other arguments need none (0).
 */
size_t ckda_fwd_workspace_bytes(int32_t N, int32_t T, int32_t H, int32_t d_k,
                                int32_t d_v, int32_t chunk, int32_t varlen,
                                ckda_dtype dt);

/*
 * ckda_fwd_chunked_noalloc: ckda_fwd_chunked for callers that cannot give the
 * library any device memory. It has no counterpart in the paper; it exists
 * because some callers have no device allocator to draw a workspace from
 * (a plain C program) or must not call cudaMalloc while they run (a serving
 * loop, where cudaMalloc may synchronise the device and stall other work).
 *
 * Same arguments and results as ckda_fwd_chunked, without the workspace: the
 * scratch is one array of CKDA_NOALLOC_SCRATCH_BYTES bytes of device memory
 * inside the library, which every GPU that loads the library keeps until the
 * process exits. The function allocates nothing.
 *  - Limit: calls whose ckda_fwd_workspace_bytes() exceeds
 *    CKDA_NOALLOC_SCRATCH_BYTES return CKDA_ERR_UNSUPPORTED and launch
 *    nothing. With d_v = 128 the need is (floor(T_total / 64) + N) * H
 *    blocks of 164,864 bytes plus a small slot table: one sequence of 767
 *    tokens with 32 heads (12 x 32 blocks) fits, 768 tokens (13 x 32) do
 *    not. Calls that need no scratch run as in ckda_fwd_chunked.
 *  - The first call on each device looks up the array's device address (a
 *    cudaGetSymbolAddress on the current device); make that first call before
 *    any stream capture.
 *  - All calls on a device share the one array, which keeps what the last
 *    call left in it (nothing in it has to start at zero). Calls whose kernels
 *    overlap on the GPU (different streams, or different host threads) race on
 *    it: run them one after another.
 */
#define CKDA_NOALLOC_SCRATCH_BYTES (64u << 20)
ckda_status ckda_fwd_chunked_noalloc(const void *q, const void *k, const void *v,
                                     const float *alpha, const float *beta,
                                     const float *initial_state, float *final_state,
                                     void *o, const int32_t *cu_seqlens,
                                     const int32_t *cu_seqlens_host, int32_t N,
                                     int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                                     int32_t chunk, float scale, ckda_dtype dt,
                                     cudaStream_t stream);

/*
 * ckda_decode_step: one recurrent step for N sequences x H heads, one new
 * token each, updating the state in place (the recurrence above applied once;
 * Semidirect Fourier Delta Attention §1 eq. (1), readout §3 eq. (14)).
 *
 * q, k   [N, H, d_k] (dt)      v, o [N, H, d_v] (dt)
 * alpha  [N, H, d_k] fp32      beta [N, H] fp32
 * state  [N, H, d_k, d_v] fp32, read and written in place
 * o      must not alias state or any input.
 */
ckda_status ckda_decode_step(const void *q, const void *k, const void *v,
                             const float *alpha, const float *beta,
                             float *state, void *o, int32_t N, int32_t H,
                             int32_t d_k, int32_t d_v, float scale,
                             ckda_dtype dt, cudaStream_t stream);

/*
 * Fused input prologue: the gates and the key normalisation computed inside
 * the kernels from per-token logits, in the stable parameterisation of
 * Semidirect Fourier Delta Attention §3 eqs. (15), (17), (18):
 *
 *     alpha = alpha_min + (alpha_max - alpha_min) * sigmoid(a)   (per channel)
 *     beta  = beta_max * sigmoid(c)                              (per token)
 *     k     = k_raw / (||k_raw||_2 + k_eps)                      (per token)
 *
 * with sigmoid(x) = 1 / (1 + exp(-x)). alpha_min = -1, alpha_max = 1,
 * beta_max = 2 give the CKDA ranges (alpha = tanh(a / 2), exactly 0 at a = 0;
 * Complex KDA, abstract); alpha_min = 0, alpha_max = 1, beta_max = 1 give
 * KDA's. A key row whose ||k_raw|| + k_eps is 0 is taken as k = 0.
 * Requirements (CKDA_ERR_ARG otherwise): -1 <= alpha_min <= alpha_max <= 1,
 * 0 <= beta_max <= 2, k_eps >= 0, all finite.
 */
typedef struct {
  float alpha_min;
  float alpha_max;
  float beta_max;
  float k_eps;
} ckda_gate_params;

/*
 * ckda_fwd_chunked_gated: ckda_fwd_chunked with the fused input prologue.
 * Same arguments, results and workspace (ckda_fwd_workspace_bytes) as
 * ckda_fwd_chunked, except:
 *   k_raw    [T_total, H, d_k] (dt)   keys before normalisation
 *   a_logit  [T_total, H, d_k] (dt)   gate logits, in the I/O element type
 *                                     (half the bytes of fp32 gates in bf16)
 *   c_logit  [T_total, H]      fp32   delta-coefficient logits
 *   gp       the gate parameters above
 * q is used as given (the pages normalise only k).
 */
ckda_status ckda_fwd_chunked_gated(const void *q, const void *k_raw, const void *v,
                                   const void *a_logit, const float *c_logit,
                                   const float *initial_state, float *final_state,
                                   void *o, const int32_t *cu_seqlens,
                                   const int32_t *cu_seqlens_host, int32_t N,
                                   int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                                   int32_t chunk, float scale, ckda_dtype dt,
                                   ckda_gate_params gp, void *workspace,
                                   size_t workspace_bytes, cudaStream_t stream);

/*
 * ckda_decode_step_gated: ckda_decode_step with the fused input prologue
 * (k_raw [N, H, d_k] (dt), a_logit [N, H, d_k] (dt), c_logit [N, H] fp32 in
 * place of k, alpha, beta); otherwise as ckda_decode_step.
 */
ckda_status ckda_decode_step_gated(const void *q, const void *k_raw, const void *v,
                                   const void *a_logit, const float *c_logit,
                                   float *state, void *o, int32_t N, int32_t H,
                                   int32_t d_k, int32_t d_v, float scale,
                                   ckda_dtype dt, ckda_gate_params gp,
                                   cudaStream_t stream);

/*
 * ckda_bwd: gradients of ckda_fwd_chunked's outputs with respect to its
 * inputs, for a scalar loss L with dL/do = d_o and dL/d(final state) =
 * d_final_state. The pages state the forward recurrence only ("Semidirect
 * Fourier Delta Attention" §1 eq. (1), §3 eq. (14)); this is its adjoint, one
 * token at a time in reverse, with S_prev the state before token t:
 *   S' = diag(alpha_t) S_prev,  w = v_t - S'^T k_t,  S_t = S' + beta_t k_t w^T;
 *   G += scale q_t do_t^T;  dq_t = scale S_t do_t;  g = G^T k_t;
 *   dv_t = beta_t g;  dbeta_t = g . w;  dk_t = beta_t (G w - S' g);
 *   dS' = G - beta_t k_t g^T;  dalpha_t = rowsum(dS' * S_prev);  G <- diag(alpha_t) dS'
 * starting from G = d_final_state, ending with d_initial_state = G.
 *
 *   q, k, v, alpha, beta, initial_state, cu_seqlens, cu_seqlens_host, N, T,
 *               H, d_k, d_v, scale, dt: as for ckda_fwd_chunked (the same
 *               call's inputs; initial_state NULL = zero).
 *   d_o         [total_T, H, d_v], dtype dt: gradient of the output.
 *   d_final_state [N, H, d_k, d_v] fp32, or NULL (= zero).
 *   dq, dk      [total_T, H, d_k], dtype dt (outputs).
 *   dv          [total_T, H, d_v], dtype dt (output).
 *   dalpha      [total_T, H, d_k] fp32 (output).
 *   dbeta       [total_T, H] fp32 (output).
 *   d_initial_state [N, H, d_k, d_v] fp32 (output), or NULL (not written).
 *   workspace   device scratch of at least ckda_bwd_workspace_bytes() bytes,
 *               owned by the caller (state checkpoints every 16 tokens and a
 *               16-state buffer per (sequence, head)); required when N > 0.
 * Every pointer must be 16-byte aligned; no output may overlap an input,
 * another output or the workspace (CKDA_ERR_ARG). d_k, d_v in {16, 32, 64,
 * 128}, dt in {CKDA_BF16, CKDA_F32} (else CKDA_ERR_UNSUPPORTED). The call is
 * asynchronous on `stream`; device-side errors (malformed device cu_seqlens)
 * surface through ckda_last_error(). Results are deterministic (no atomics).
 * One CTA per (sequence, head) walks the tokens on CUDA cores.
 */
ckda_status ckda_bwd(const void *q, const void *k, const void *v, const float *alpha,
                     const float *beta, const float *initial_state, const void *d_o,
                     const float *d_final_state, void *dq, void *dk, void *dv,
                     float *dalpha, float *dbeta, float *d_initial_state,
                     const int32_t *cu_seqlens, const int32_t *cu_seqlens_host, int32_t N,
                     int32_t T, int32_t H, int32_t d_k, int32_t d_v, float scale,
                     ckda_dtype dt, void *workspace, size_t workspace_bytes,
                     cudaStream_t stream);

/*
 * ckda_bwd_chunked: the gradients of ckda_bwd (the same arguments, layouts,
 * errors and outputs) computed 16 tokens at a time in the chunk-WY form of the
 * forward ("Semidirect Fourier Delta Attention" §2.2 eqs. (9)-(10)) run in
 * reverse: per chunk, dU = scale M^T dO + Kbar dS_C, dR = T^T dU,
 * dv = diag(beta) dR, then dq, dk, dbeta from matrix products and the gated
 * Gram terms, and dalpha per channel as the gate product with the one factor
 * alpha_s left out (two running products, no logarithm and no division, so
 * zero and negative gates are exact). Only the d_k x d_v state gradient
 * dS = scale Qhat^T dO + diag(gamma) dS_C - Khat^T diag(beta) dR passes from
 * chunk to chunk. Four kernels: a prep over all chunks, a forward scan and a
 * reverse scan per (sequence, head, tile of up to 32 state columns) that
 * carry only the state products, and the gradients per (chunk, head), whose
 * column tiles are added in a fixed order. fp32 arithmetic on CUDA cores,
 * deterministic.
 *   workspace   device scratch of at least ckda_bwd_chunked_workspace_bytes()
 *               bytes, owned by the caller (one entry state and one exit-state
 *               gradient per 16-token chunk and the chunks' factors); required
 *               when N > 0.
 */
ckda_status ckda_bwd_chunked(const void *q, const void *k, const void *v, const float *alpha,
                             const float *beta, const float *initial_state, const void *d_o,
                             const float *d_final_state, void *dq, void *dk, void *dv,
                             float *dalpha, float *dbeta, float *d_initial_state,
                             const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                             int32_t N, int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                             float scale, ckda_dtype dt, void *workspace,
                             size_t workspace_bytes, cudaStream_t stream);

/*
 * ckda_fwd_complex: the complex-phase gate of "Semidirect Fourier Delta
 * Attention" §3, eqs. (13)-(14), with complex q, k, v and state:
 *   S_t = (I - beta_t k_t k_t^*) Lambda_t S_{t-1} + beta_t k_t v_t^*,
 *   Lambda_t = diag(alpha_t exp(i theta_t)),   o_t = scale S_t^* q_t
 * (^* the conjugate transpose; the page's real implementation of the gate is
 * a 2x2 rotation-decay block on each (real, imaginary) pair).
 *   q, k        [total_T, H, d_k] complex64 (interleaved real, imaginary fp32).
 *   v, o        [total_T, H, d_v] complex64 (o written).
 *   alpha, theta [total_T, H, d_k] fp32: decay and phase per channel.
 *   beta        [total_T, H] fp32.
 *   initial_state, final_state [N, H, d_k, d_v] complex64, or NULL (zero / not
 *               written); final_state may equal initial_state (in place).
 *   cu_seqlens, cu_seqlens_host, N, T, H, d_k, d_v, scale: as ckda_fwd_chunked.
 * Every pointer 16-byte aligned; o must not overlap an input; d_k, d_v in {16,
 * 32, 64, 128}. Token-serial on CUDA cores (one CTA per sequence, head and
 * 32-column tile), fp32 arithmetic, deterministic; no workspace. Asynchronous
 * on `stream`; device-side errors through ckda_last_error().
 */
ckda_status ckda_fwd_complex(const void *q, const void *k, const void *v, const float *alpha,
                             const float *theta, const float *beta, const void *initial_state,
                             void *final_state, void *o, const int32_t *cu_seqlens,
                             const int32_t *cu_seqlens_host, int32_t N, int32_t T, int32_t H,
                             int32_t d_k, int32_t d_v, float scale, cudaStream_t stream);

/*
 * ckda_fwd_complex_chunked: the outputs of ckda_fwd_complex (the same
 * arguments, layouts and errors, plus a workspace) computed 16 tokens at a
 * time in the chunk-WY form of "Semidirect Fourier Delta Attention" §2.2
 * eqs. (9)-(10) with complex gates lambda = alpha exp(i theta):
 *   A_ij = beta_i k_i^* G_ij k_j (j < i),  M_ij = q_i^* G_ij k_j (j <= i),
 *   T = (I + A)^-1,  U = T diag(beta) (conj(V) - Khat S),
 *   conj(O) = scale (Qhat S + M U),  S <- diag(gamma) S + Kbar^T U,
 * where G_ij is the product of the lambdas over (j, i], gamma and sigma the
 * chunk's prefix and suffix products, Khat = gamma conj(k), Qhat = gamma conj(q),
 * Kbar = sigma k. A prep kernel over all chunks forms T, W = T diag(beta) Khat,
 * T diag(beta) conj(V), Kbar, Qhat and M; a scan per (sequence, head, tile of
 * up to 32 complex columns) carries the state through U = T diag(beta) conj(V)
 * - W S and the update. fp32 arithmetic on CUDA cores, deterministic.
 *   workspace   device scratch of at least
 *               ckda_fwd_complex_chunked_workspace_bytes() bytes, owned by the
 *               caller; required when N > 0; must not overlap any tensor.
 */
ckda_status ckda_fwd_complex_chunked(const void *q, const void *k, const void *v,
                                     const float *alpha, const float *theta, const float *beta,
                                     const void *initial_state, void *final_state, void *o,
                                     const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                                     int32_t N, int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                                     float scale, void *workspace, size_t workspace_bytes,
                                     cudaStream_t stream);

/* Scratch that ckda_fwd_complex_chunked needs (arguments as ckda_bwd_workspace_bytes). */
size_t ckda_fwd_complex_chunked_workspace_bytes(int32_t N, int32_t T, int32_t H, int32_t d_k,
                                                int32_t d_v, int32_t varlen);

/*
 * ckda_bwd_workspace_bytes, ckda_bwd_chunked_workspace_bytes: scratch that
 * ckda_bwd and ckda_bwd_chunked need (T as in ckda_bwd; varlen nonzero when
 * cu_seqlens is given, so that T is total_T). 0 for unsupported or invalid
 * sizes.
 */
size_t ckda_bwd_workspace_bytes(int32_t N, int32_t T, int32_t H, int32_t d_k,
                                int32_t d_v, int32_t varlen);
size_t ckda_bwd_chunked_workspace_bytes(int32_t N, int32_t T, int32_t H, int32_t d_k,
                                        int32_t d_v, int32_t varlen);

/* Static description of a status code (never NULL). */
const char *ckda_status_string(ckda_status s);

/*
 * ckda_last_error: synchronises `stream`, then reads and clears the current
 * device's error word. Returns CKDA_OK if no kernel recorded an error since
 * the last call, CKDA_ERR_DEVICE if one did, CKDA_ERR_CUDA if the
 * synchronisation or the read failed.
 */
ckda_status ckda_last_error(cudaStream_t stream);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int32_t ckda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CKDA_H */
