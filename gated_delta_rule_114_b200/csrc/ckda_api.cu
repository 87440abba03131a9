// C ABI of the CKDA library: host-side validation, dispatch, error word.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "ckda.h"
#include "ckda_common.cuh"

namespace ckda {
// With g.on, `alpha` points to the gate logits a (I/O element type), `beta`
// to the fp32 logits c and `k` to the raw keys (the fused input prologue).
template <typename IOT>
cudaError_t launch_decode(int dk, int dv, const void *q, const void *k,
                          const void *v, const void *alpha, const float *beta,
                          float *state, void *o, int N, int H, float scale,
                          GateArgs g, cudaStream_t st);
template <typename IOT>
cudaError_t launch_fwd_simt(int dk, int dv, int chunk, const void *q,
                            const void *k, const void *v, const void *alpha,
                            const float *beta, const float *s0, float *sf,
                            void *o, const int32_t *cu, int N, int T,
                            int T_total, int H, float scale, GateArgs g,
                            unsigned int *err, cudaStream_t st);
size_t bwd_workspace_bytes(int N, int T_total, int H, int dk, int dv);
size_t complex_chunk_workspace_bytes(int N, int T_total, int H, int dk, int dv);
cudaError_t launch_fwd_complex_chunked(int dk, int dv, const void *q, const void *k,
                                       const void *v, const float *alpha, const float *theta,
                                       const float *beta, const void *s0, void *sf, void *o,
                                       const int32_t *cu, int N, int T, int T_total, int H,
                                       float scale, void *ws, unsigned int *err,
                                       cudaStream_t st);
cudaError_t launch_fwd_complex(int dk, int dv, const void *q, const void *k, const void *v,
                               const float *alpha, const float *theta, const float *beta,
                               const void *s0, void *sf, void *o, const int32_t *cu, int N,
                               int T, int T_total, int H, float scale, unsigned int *err,
                               cudaStream_t st);
template <typename IOT>
cudaError_t launch_bwd(int dk, int dv, const void *q, const void *k, const void *v,
                       const float *alpha, const float *beta, const float *s0,
                       const void *d_o, const float *dsf, void *dq, void *dk_, void *dv_,
                       float *dalpha, float *dbeta, float *ds0, const int32_t *cu, int N,
                       int T, int T_total, int H, float scale, void *ws,
                       unsigned int *err, cudaStream_t st);
size_t bwd_split_workspace_bytes(int N, int T_total, int H, int dk, int dv);
template <typename IOT>
cudaError_t launch_bwd_split(int dk, int dv, const void *q, const void *k, const void *v,
                             const float *alpha, const float *beta, const float *s0,
                             const void *d_o, const float *dsf, void *dq, void *dk_, void *dv_,
                             float *dalpha, float *dbeta, float *ds0, const int32_t *cu, int N,
                             int T, int T_total, int H, float scale, void *ws,
                             unsigned int *err, cudaStream_t st);
bool fwd_tc_supported(int dk, int dv, int chunk, ckda_dtype dt);
size_t fwd_tc_workspace_bytes(int N, int T_total, int H, int dv);
cudaError_t launch_fwd_tc(int dv, const void *q, const void *k, const void *v,
                          const void *alpha, const float *beta,
                          const float *s0, float *sf, void *o,
                          const int32_t *cu, int N, int T, int T_total, int H,
                          float scale, GateArgs g, void *ws, unsigned int *err,
                          cudaStream_t st);
}  // namespace ckda

// The per-device error word. Each device context gets its own instance.
__device__ unsigned int g_ckda_error_word = 0;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_err_mu;
unsigned int *g_err_addr[kMaxDevices] = {};

// Device address of the error word on the current device (cached).
unsigned int *error_word_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return nullptr;
  std::lock_guard<std::mutex> lk(g_err_mu);
  if (!g_err_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ckda_error_word) != cudaSuccess) return nullptr;
    g_err_addr[dev] = static_cast<unsigned int *>(p);
  }
  return g_err_addr[dev];
}

bool supported_dim(int32_t d) { return d == 16 || d == 32 || d == 64 || d == 128; }

// The sequence-parallel kernels put the sequence index, and the forward scan
// also the head, on grid.y or grid.z, which hold at most 65535 blocks.
constexpr int32_t kMaxGridYZ = 65535;
bool grid_fits(int32_t N, int32_t H) { return N <= kMaxGridYZ && H <= kMaxGridYZ; }

bool aligned16(const void *p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

// [a, a+na) and [b, b+nb) overlap (byte ranges; empty ranges never overlap)
bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a);
  const uintptr_t y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

size_t esize(ckda_dtype dt) { return dt == CKDA_F32 ? 4 : 2; }

bool finite(float x) { return x == x && x - x == 0.f; }

// Token rows of the packed [T_total, H, ...] tensors: N*T for fixed-length
// sequences, T for varlen (cu_seqlens given). A host copy of the offsets, when
// given, must start at 0, end at T and not decrease. False on any violation
// or a row count above INT32_MAX.
bool token_rows(const int32_t *cu_seqlens, const int32_t *cu_seqlens_host, int32_t N,
                int32_t T, int64_t &T_total) {
  if (cu_seqlens == nullptr) {
    if (cu_seqlens_host) return false;
    T_total = (int64_t)N * T;
  } else {
    T_total = T;
    if (cu_seqlens_host) {
      if (cu_seqlens_host[0] != 0 || cu_seqlens_host[N] != T) return false;
      for (int32_t n = 0; n < N; ++n)
        if (cu_seqlens_host[n + 1] < cu_seqlens_host[n]) return false;
    }
  }
  return T_total <= INT32_MAX;
}

// ckda_gate_params -> kernel arguments; false if outside the documented ranges
bool gate_args(const ckda_gate_params &gp, ckda::GateArgs &g) {
  if (!finite(gp.alpha_min) || !finite(gp.alpha_max) || !finite(gp.beta_max) ||
      !finite(gp.k_eps))
    return false;
  if (gp.alpha_min < -1.f || gp.alpha_max > 1.f || gp.alpha_min > gp.alpha_max) return false;
  if (gp.beta_max < 0.f || gp.beta_max > 2.f || gp.k_eps < 0.f) return false;
  g.on = 1;
  g.amin = gp.alpha_min;
  g.arange = gp.alpha_max - gp.alpha_min;
  g.bmax = gp.beta_max;
  g.keps = gp.k_eps;
  return true;
}

// The forward behind both entry points; with g.on, alpha is the logits a
// (element size es) and beta the logits c.
ckda_status fwd_impl(const void *q, const void *k, const void *v,
                     const void *alpha, const float *beta,
                     const float *initial_state, float *final_state, void *o,
                     const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                     int32_t N, int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                     int32_t chunk, float scale, ckda_dtype dt, ckda::GateArgs g,
                     void *workspace, size_t workspace_bytes, cudaStream_t stream);

ckda_status decode_impl(const void *q, const void *k, const void *v,
                        const void *alpha, const float *beta, float *state,
                        void *o, int32_t N, int32_t H, int32_t d_k, int32_t d_v,
                        float scale, ckda_dtype dt, ckda::GateArgs g,
                        cudaStream_t stream);

}  // namespace

extern "C" {

int32_t ckda_version(void) { return 100; }

const char *ckda_status_string(ckda_status s) {
  switch (s) {
    case CKDA_OK: return "CKDA_OK";
    case CKDA_ERR_ARG: return "CKDA_ERR_ARG: invalid argument";
    case CKDA_ERR_UNSUPPORTED: return "CKDA_ERR_UNSUPPORTED: unsupported size, chunk or dtype";
    case CKDA_ERR_CUDA: return "CKDA_ERR_CUDA: CUDA runtime or launch failure";
    case CKDA_ERR_DEVICE: return "CKDA_ERR_DEVICE: a kernel reported an error";
  }
  return "CKDA_UNKNOWN_STATUS";
}

ckda_status ckda_last_error(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return CKDA_ERR_CUDA;
  unsigned int w = 0;
  const unsigned int zero = 0;
  if (cudaMemcpyFromSymbol(&w, g_ckda_error_word, sizeof(w)) != cudaSuccess)
    return CKDA_ERR_CUDA;
  if (w != 0 &&
      cudaMemcpyToSymbol(g_ckda_error_word, &zero, sizeof(zero)) != cudaSuccess)
    return CKDA_ERR_CUDA;
  return w ? CKDA_ERR_DEVICE : CKDA_OK;
}

}  // extern "C"

namespace {

// ckda_fwd_complex (token-serial kernel, chunked = false) and
// ckda_fwd_complex_chunked: one validation, then the chosen launch.
ckda_status complex_impl(const void *q, const void *k, const void *v, const float *alpha,
                         const float *theta, const float *beta, const void *initial_state,
                         void *final_state, void *o, const int32_t *cu_seqlens,
                         const int32_t *cu_seqlens_host, int32_t N, int32_t T, int32_t H,
                         int32_t d_k, int32_t d_v, float scale, void *workspace,
                         size_t workspace_bytes, cudaStream_t stream, bool chunked) {
  if (!supported_dim(d_k) || !supported_dim(d_v)) return CKDA_ERR_UNSUPPORTED;
  if (N < 0 || T < 0 || H <= 0) return CKDA_ERR_ARG;
  if (!grid_fits(N, H)) return CKDA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !alpha || !theta || !beta || !o) return CKDA_ERR_ARG;
  const void *ptrs[] = {q, k, v, alpha, theta, beta, initial_state, final_state, o, cu_seqlens,
                        workspace};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return CKDA_ERR_ARG;
  int64_t T_total;
  if (!token_rows(cu_seqlens, cu_seqlens_host, N, T, T_total)) return CKDA_ERR_ARG;
  // complex64 = 8 bytes per element; no output may overlap an input, the other
  // output or the workspace
  const size_t th = (size_t)T_total * H;
  const size_t kb = th * d_k * 8, vb = th * d_v * 8, rb = th * d_k * sizeof(float);
  const size_t sb = (size_t)N * H * d_k * d_v * 8;
  const size_t need =
      chunked && N > 0 ? ckda::complex_chunk_workspace_bytes(N, (int)T_total, H, d_k, d_v) : 0;
  struct R { const void *p; size_t n; };
  const R ins[] = {{q, kb}, {k, kb}, {v, vb}, {alpha, rb}, {theta, rb}, {beta, th * sizeof(float)},
                   {initial_state, sb}};
  for (const R &x : ins)
    if (overlaps(o, vb, x.p, x.n)) return CKDA_ERR_ARG;
  for (size_t i = 0; i + 1 < sizeof(ins) / sizeof(ins[0]); ++i)  // final state: any input but s0
    if (overlaps(final_state, sb, ins[i].p, ins[i].n)) return CKDA_ERR_ARG;
  if (overlaps(final_state, sb, o, vb)) return CKDA_ERR_ARG;
  if (final_state && initial_state && final_state != initial_state &&
      overlaps(final_state, sb, initial_state, sb))
    return CKDA_ERR_ARG;
  if (chunked) {
    for (const R &x : ins)
      if (overlaps(workspace, need, x.p, x.n)) return CKDA_ERR_ARG;
    if (overlaps(workspace, need, o, vb) || overlaps(workspace, need, final_state, sb))
      return CKDA_ERR_ARG;
  }
  if (N == 0) return CKDA_OK;
  if (chunked && (!workspace || workspace_bytes < need)) return CKDA_ERR_ARG;
  const cudaError_t e =
      chunked ? ckda::launch_fwd_complex_chunked(d_k, d_v, q, k, v, alpha, theta, beta,
                                                 initial_state, final_state, o, cu_seqlens, N, T,
                                                 (int)T_total, H, scale, workspace,
                                                 error_word_ptr(), stream)
              : ckda::launch_fwd_complex(d_k, d_v, q, k, v, alpha, theta, beta, initial_state,
                                         final_state, o, cu_seqlens, N, T, (int)T_total, H,
                                         scale, error_word_ptr(), stream);
  return e == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
}

}  // namespace

extern "C" {

ckda_status ckda_fwd_complex(const void *q, const void *k, const void *v, const float *alpha,
                             const float *theta, const float *beta, const void *initial_state,
                             void *final_state, void *o, const int32_t *cu_seqlens,
                             const int32_t *cu_seqlens_host, int32_t N, int32_t T, int32_t H,
                             int32_t d_k, int32_t d_v, float scale, cudaStream_t stream) {
  return complex_impl(q, k, v, alpha, theta, beta, initial_state, final_state, o, cu_seqlens,
                      cu_seqlens_host, N, T, H, d_k, d_v, scale, nullptr, 0, stream, false);
}

ckda_status ckda_fwd_complex_chunked(const void *q, const void *k, const void *v,
                                     const float *alpha, const float *theta, const float *beta,
                                     const void *initial_state, void *final_state, void *o,
                                     const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                                     int32_t N, int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                                     float scale, void *workspace, size_t workspace_bytes,
                                     cudaStream_t stream) {
  return complex_impl(q, k, v, alpha, theta, beta, initial_state, final_state, o, cu_seqlens,
                      cu_seqlens_host, N, T, H, d_k, d_v, scale, workspace, workspace_bytes,
                      stream, true);
}

size_t ckda_fwd_complex_chunked_workspace_bytes(int32_t N, int32_t T, int32_t H, int32_t d_k,
                                                int32_t d_v, int32_t varlen) {
  if (N <= 0 || T < 0 || H <= 0 || !supported_dim(d_k) || !supported_dim(d_v)) return 0;
  const int64_t T_total = varlen ? (int64_t)T : (int64_t)N * T;
  if (T_total > INT32_MAX) return 0;
  return ckda::complex_chunk_workspace_bytes(N, (int)T_total, H, d_k, d_v);
}

size_t ckda_bwd_workspace_bytes(int32_t N, int32_t T, int32_t H, int32_t d_k,
                                int32_t d_v, int32_t varlen) {
  if (N <= 0 || T < 0 || H <= 0 || !supported_dim(d_k) || !supported_dim(d_v)) return 0;
  const int64_t T_total = varlen ? (int64_t)T : (int64_t)N * T;
  if (T_total > INT32_MAX) return 0;
  return ckda::bwd_workspace_bytes(N, (int)T_total, H, d_k, d_v);
}

size_t ckda_bwd_chunked_workspace_bytes(int32_t N, int32_t T, int32_t H, int32_t d_k,
                                        int32_t d_v, int32_t varlen) {
  if (N <= 0 || T < 0 || H <= 0 || !supported_dim(d_k) || !supported_dim(d_v)) return 0;
  const int64_t T_total = varlen ? (int64_t)T : (int64_t)N * T;
  if (T_total > INT32_MAX) return 0;
  return ckda::bwd_split_workspace_bytes(N, (int)T_total, H, d_k, d_v);
}

}  // extern "C"

namespace {

// ckda_bwd (token-serial kernel) and ckda_bwd_chunked (chunkwise kernel):
// one validation, then the chosen launch.
ckda_status bwd_impl(const void *q, const void *k, const void *v, const float *alpha,
                     const float *beta, const float *initial_state, const void *d_o,
                     const float *d_final_state, void *dq, void *dk, void *dv,
                     float *dalpha, float *dbeta, float *d_initial_state,
                     const int32_t *cu_seqlens, const int32_t *cu_seqlens_host, int32_t N,
                     int32_t T, int32_t H, int32_t d_k, int32_t d_v, float scale,
                     ckda_dtype dt, void *workspace, size_t workspace_bytes,
                     cudaStream_t stream, bool chunked) {
  if (dt != CKDA_BF16 && dt != CKDA_F32) return CKDA_ERR_UNSUPPORTED;
  if (!supported_dim(d_k) || !supported_dim(d_v)) return CKDA_ERR_UNSUPPORTED;
  if (N < 0 || T < 0 || H <= 0) return CKDA_ERR_ARG;
  if (!grid_fits(N, H)) return CKDA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !alpha || !beta || !d_o || !dq || !dk || !dv || !dalpha || !dbeta)
    return CKDA_ERR_ARG;
  const void *ptrs[] = {q, k, v, alpha, beta, initial_state, d_o, d_final_state, dq, dk,
                        dv, dalpha, dbeta, d_initial_state, cu_seqlens, workspace};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return CKDA_ERR_ARG;
  int64_t T_total;
  if (!token_rows(cu_seqlens, cu_seqlens_host, N, T, T_total)) return CKDA_ERR_ARG;
  // no output may overlap an input, another output or the workspace
  const size_t es = esize(dt), th = (size_t)T_total * H;
  const size_t kb = th * d_k * es, vb = th * d_v * es, ab = th * d_k * sizeof(float);
  const size_t bb = th * sizeof(float), sb = (size_t)N * H * d_k * d_v * sizeof(float);
  const size_t need = chunked
                          ? ckda_bwd_chunked_workspace_bytes(N, T, H, d_k, d_v, cu_seqlens != nullptr)
                          : ckda_bwd_workspace_bytes(N, T, H, d_k, d_v, cu_seqlens != nullptr);
  struct R { const void *p; size_t n; };
  const R ins[] = {{q, kb}, {k, kb}, {v, vb}, {alpha, ab}, {beta, bb}, {initial_state, sb},
                   {d_o, vb}, {d_final_state, sb},
                   {cu_seqlens, cu_seqlens ? (size_t)(N + 1) * sizeof(int32_t) : 0}};
  const R outs[] = {{dq, kb}, {dk, kb}, {dv, vb}, {dalpha, ab}, {dbeta, bb},
                    {d_initial_state, sb}, {workspace, need}};
  for (size_t i = 0; i < sizeof(outs) / sizeof(outs[0]); ++i) {
    for (const R &x : ins)
      if (overlaps(outs[i].p, outs[i].n, x.p, x.n)) return CKDA_ERR_ARG;
    for (size_t j = i + 1; j < sizeof(outs) / sizeof(outs[0]); ++j)
      if (overlaps(outs[i].p, outs[i].n, outs[j].p, outs[j].n)) return CKDA_ERR_ARG;
  }
  if (N == 0) return CKDA_OK;
  if (!workspace || workspace_bytes < need) return CKDA_ERR_ARG;
  unsigned int *err = error_word_ptr();
  auto launch = [&](auto io) {
    using IOT = decltype(io);
    return chunked ? ckda::launch_bwd_split<IOT>(d_k, d_v, q, k, v, alpha, beta, initial_state,
                                                 d_o, d_final_state, dq, dk, dv, dalpha, dbeta,
                                                 d_initial_state, cu_seqlens, N, T,
                                                 (int)T_total, H, scale, workspace, err, stream)
                   : ckda::launch_bwd<IOT>(d_k, d_v, q, k, v, alpha, beta, initial_state, d_o,
                                           d_final_state, dq, dk, dv, dalpha, dbeta,
                                           d_initial_state, cu_seqlens, N, T, (int)T_total, H,
                                           scale, workspace, err, stream);
  };
  const cudaError_t e = dt == CKDA_F32 ? launch(float{}) : launch(__nv_bfloat16{});
  return e == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
}

}  // namespace

extern "C" {

ckda_status ckda_bwd(const void *q, const void *k, const void *v, const float *alpha,
                     const float *beta, const float *initial_state, const void *d_o,
                     const float *d_final_state, void *dq, void *dk, void *dv,
                     float *dalpha, float *dbeta, float *d_initial_state,
                     const int32_t *cu_seqlens, const int32_t *cu_seqlens_host, int32_t N,
                     int32_t T, int32_t H, int32_t d_k, int32_t d_v, float scale,
                     ckda_dtype dt, void *workspace, size_t workspace_bytes,
                     cudaStream_t stream) {
  return bwd_impl(q, k, v, alpha, beta, initial_state, d_o, d_final_state, dq, dk, dv, dalpha,
                  dbeta, d_initial_state, cu_seqlens, cu_seqlens_host, N, T, H, d_k, d_v, scale,
                  dt, workspace, workspace_bytes, stream, false);
}

ckda_status ckda_bwd_chunked(const void *q, const void *k, const void *v, const float *alpha,
                             const float *beta, const float *initial_state, const void *d_o,
                             const float *d_final_state, void *dq, void *dk, void *dv,
                             float *dalpha, float *dbeta, float *d_initial_state,
                             const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                             int32_t N, int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                             float scale, ckda_dtype dt, void *workspace,
                             size_t workspace_bytes, cudaStream_t stream) {
  return bwd_impl(q, k, v, alpha, beta, initial_state, d_o, d_final_state, dq, dk, dv, dalpha,
                  dbeta, d_initial_state, cu_seqlens, cu_seqlens_host, N, T, H, d_k, d_v, scale,
                  dt, workspace, workspace_bytes, stream, true);
}

size_t ckda_fwd_workspace_bytes(int32_t N, int32_t T, int32_t H, int32_t d_k,
                                int32_t d_v, int32_t chunk, int32_t varlen,
                                ckda_dtype dt) {
  if (chunk == 0) chunk = 64;
  if (N <= 0 || T < 0 || H <= 0) return 0;
  if (!ckda::fwd_tc_supported(d_k, d_v, chunk, dt)) return 0;
  const int64_t T_total = varlen ? (int64_t)T : (int64_t)N * T;
  if (T_total > INT32_MAX) return 0;
  return ckda::fwd_tc_workspace_bytes(N, (int)T_total, H, d_v);
}

ckda_status ckda_fwd_chunked(const void *q, const void *k, const void *v,
                             const float *alpha, const float *beta,
                             const float *initial_state, float *final_state,
                             void *o, const int32_t *cu_seqlens,
                             const int32_t *cu_seqlens_host, int32_t N,
                             int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                             int32_t chunk, float scale, ckda_dtype dt,
                             void *workspace, size_t workspace_bytes,
                             cudaStream_t stream) {
  return fwd_impl(q, k, v, alpha, beta, initial_state, final_state, o, cu_seqlens,
                  cu_seqlens_host, N, T, H, d_k, d_v, chunk, scale, dt,
                  ckda::GateArgs{0, 0.f, 0.f, 0.f, 0.f}, workspace, workspace_bytes, stream);
}

ckda_status ckda_fwd_chunked_gated(const void *q, const void *k_raw, const void *v,
                                   const void *a_logit, const float *c_logit,
                                   const float *initial_state, float *final_state,
                                   void *o, const int32_t *cu_seqlens,
                                   const int32_t *cu_seqlens_host, int32_t N,
                                   int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                                   int32_t chunk, float scale, ckda_dtype dt,
                                   ckda_gate_params gp, void *workspace,
                                   size_t workspace_bytes, cudaStream_t stream) {
  ckda::GateArgs g;
  if (!gate_args(gp, g)) return CKDA_ERR_ARG;
  return fwd_impl(q, k_raw, v, a_logit, c_logit, initial_state, final_state, o,
                  cu_seqlens, cu_seqlens_host, N, T, H, d_k, d_v, chunk, scale, dt, g,
                  workspace, workspace_bytes, stream);
}

ckda_status ckda_decode_step(const void *q, const void *k, const void *v,
                             const float *alpha, const float *beta,
                             float *state, void *o, int32_t N, int32_t H,
                             int32_t d_k, int32_t d_v, float scale,
                             ckda_dtype dt, cudaStream_t stream) {
  return decode_impl(q, k, v, alpha, beta, state, o, N, H, d_k, d_v, scale, dt,
                     ckda::GateArgs{0, 0.f, 0.f, 0.f, 0.f}, stream);
}

ckda_status ckda_decode_step_gated(const void *q, const void *k_raw, const void *v,
                                   const void *a_logit, const float *c_logit,
                                   float *state, void *o, int32_t N, int32_t H,
                                   int32_t d_k, int32_t d_v, float scale,
                                   ckda_dtype dt, ckda_gate_params gp,
                                   cudaStream_t stream) {
  ckda::GateArgs g;
  if (!gate_args(gp, g)) return CKDA_ERR_ARG;
  return decode_impl(q, k_raw, v, a_logit, c_logit, state, o, N, H, d_k, d_v, scale,
                     dt, g, stream);
}

}  // extern "C"

namespace {

ckda_status fwd_impl(const void *q, const void *k, const void *v,
                     const void *alpha, const float *beta,
                     const float *initial_state, float *final_state, void *o,
                     const int32_t *cu_seqlens, const int32_t *cu_seqlens_host,
                     int32_t N, int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                     int32_t chunk, float scale, ckda_dtype dt, ckda::GateArgs g,
                     void *workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (dt != CKDA_BF16 && dt != CKDA_F32) return CKDA_ERR_UNSUPPORTED;
  if (!supported_dim(d_k) || !supported_dim(d_v)) return CKDA_ERR_UNSUPPORTED;
  if (chunk == 0) chunk = 64;
  if (chunk != 16 && chunk != 32 && chunk != 64) return CKDA_ERR_UNSUPPORTED;
  if (N < 0 || T < 0 || H <= 0) return CKDA_ERR_ARG;
  if (!grid_fits(N, H)) return CKDA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !alpha || !beta || !o) return CKDA_ERR_ARG;
  const void *ptrs[] = {q, k, v, alpha, beta, o, initial_state, final_state,
                        cu_seqlens, workspace};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return CKDA_ERR_ARG;

  int64_t T_total;
  if (!token_rows(cu_seqlens, cu_seqlens_host, N, T, T_total)) return CKDA_ERR_ARG;

  // the output must not overlap any input or state
  const size_t es = esize(dt);
  const size_t th = (size_t)T_total * H;
  const size_t ob = th * d_v * es;
  const size_t sb = (size_t)N * H * d_k * d_v * sizeof(float);
  const size_t ab = th * d_k * (g.on ? es : sizeof(float));  // alpha or its logits
  if (overlaps(o, ob, q, th * d_k * es) || overlaps(o, ob, k, th * d_k * es) ||
      overlaps(o, ob, v, th * d_v * es) ||
      overlaps(o, ob, alpha, ab) ||
      overlaps(o, ob, beta, th * sizeof(float)) ||
      overlaps(o, ob, initial_state, sb) || overlaps(o, ob, final_state, sb))
    return CKDA_ERR_ARG;
  if (final_state && initial_state && final_state != initial_state &&
      overlaps(final_state, sb, initial_state, sb))
    return CKDA_ERR_ARG;

  const size_t need = ckda_fwd_workspace_bytes(N, T, H, d_k, d_v, chunk,
                                               cu_seqlens != nullptr, dt);
  if (need > 0) {
    if (!workspace || workspace_bytes < need) return CKDA_ERR_ARG;
    const size_t ib = th * d_k * es;
    if (overlaps(workspace, need, q, ib) || overlaps(workspace, need, k, ib) ||
        overlaps(workspace, need, v, th * d_v * es) ||
        overlaps(workspace, need, alpha, ab) ||
        overlaps(workspace, need, beta, th * sizeof(float)) ||
        overlaps(workspace, need, o, ob) ||
        overlaps(workspace, need, initial_state, sb) ||
        overlaps(workspace, need, final_state, sb) ||
        overlaps(workspace, need, cu_seqlens, (size_t)(N + 1) * sizeof(int32_t)))
      return CKDA_ERR_ARG;
  }

  if (N == 0) return CKDA_OK;
  unsigned int *err = error_word_ptr();
  cudaError_t e;
  if (ckda::fwd_tc_supported(d_k, d_v, chunk, dt)) {
    e = ckda::launch_fwd_tc(d_v, q, k, v, alpha, beta, initial_state, final_state, o,
                            cu_seqlens, N, T, (int)T_total, H, scale, g, workspace,
                            err, stream);
  } else if (dt == CKDA_F32) {
    e = ckda::launch_fwd_simt<float>(d_k, d_v, chunk, q, k, v, alpha, beta,
                                     initial_state, final_state, o, cu_seqlens,
                                     N, T, (int)T_total, H, scale, g, err, stream);
  } else {
    e = ckda::launch_fwd_simt<__nv_bfloat16>(
        d_k, d_v, chunk, q, k, v, alpha, beta, initial_state, final_state, o,
        cu_seqlens, N, T, (int)T_total, H, scale, g, err, stream);
  }
  return e == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
}

ckda_status decode_impl(const void *q, const void *k, const void *v,
                        const void *alpha, const float *beta, float *state,
                        void *o, int32_t N, int32_t H, int32_t d_k, int32_t d_v,
                        float scale, ckda_dtype dt, ckda::GateArgs g,
                        cudaStream_t stream) {
  if (dt != CKDA_BF16 && dt != CKDA_F32) return CKDA_ERR_UNSUPPORTED;
  if (!supported_dim(d_k) || !supported_dim(d_v)) return CKDA_ERR_UNSUPPORTED;
  if (N < 0 || H <= 0) return CKDA_ERR_ARG;
  if (!q || !k || !v || !alpha || !beta || !state || !o) return CKDA_ERR_ARG;
  const void *ptrs[] = {q, k, v, alpha, beta, state, o};
  for (const void *p : ptrs)
    if (!aligned16(p)) return CKDA_ERR_ARG;
  const size_t es = esize(dt);
  const size_t nh = (size_t)N * H;
  const size_t ob = nh * d_v * es;
  if (overlaps(o, ob, state, nh * d_k * d_v * sizeof(float)) ||
      overlaps(o, ob, q, nh * d_k * es) || overlaps(o, ob, k, nh * d_k * es) ||
      overlaps(o, ob, v, nh * d_v * es) ||
      overlaps(o, ob, alpha, nh * d_k * (g.on ? es : sizeof(float))) ||
      overlaps(o, ob, beta, nh * sizeof(float)))
    return CKDA_ERR_ARG;
  if (nh > 0x7fffffffu) return CKDA_ERR_ARG;
  if (N == 0) return CKDA_OK;
  cudaError_t e =
      dt == CKDA_F32
          ? ckda::launch_decode<float>(d_k, d_v, q, k, v, alpha, beta, state, o,
                                       N, H, scale, g, stream)
          : ckda::launch_decode<__nv_bfloat16>(d_k, d_v, q, k, v, alpha, beta,
                                               state, o, N, H, scale, g, stream);
  return e == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
}

}  // namespace
