// Backward pass of the CKDA recurrence on CUDA cores (sm_100a).
//
// The forward, per (sequence, head) and token t, with S_prev the state before
// the step ("Semidirect Fourier Delta Attention" §1 eq. (1), readout §3 eq. (14)):
//   S' = diag(alpha_t) S_prev,  w = v_t - S'^T k_t,  S_t = S' + beta_t k_t w^T,
//   o_t = scale S_t^T q_t.
// Its adjoint, going backwards with G = dL/dS_t (d_final_state at the end):
//   G += scale q_t do_t^T;  dq_t = scale S_t do_t;  g = G^T k_t;
//   dv_t = beta_t g;  dbeta_t = g . w;  dk_t = beta_t (G w - S' g);
//   dS' = G - beta_t k_t g^T;  dalpha_t = rowsum(dS' * S_prev);
//   G <- diag(alpha_t) dS'   (and d_initial_state = G after the first token).
//
// The columns of S (and of G) evolve independently, so one CTA takes one
// (sequence, head, tile of DVT columns); thread (row r, column quarter cq)
// keeps DVT/4 columns of row r of the state (forward) or of G (backward) in
// registers. dv and the initial-state gradient are per column and written by
// the tile that owns them; dq, dk, dalpha and dbeta sum over all columns, so
// every tile writes fp32 partials and a second kernel adds the tiles in a
// fixed order. Pass 1 runs the forward and stores the state every CK = 16
// tokens (checkpoint slots in the workspace). Pass 2 walks the 16-token
// chunks backwards: it reloads the chunk's checkpoint, recomputes the
// chunk's pre-step states into a per-CTA buffer (w into shared memory), then
// runs the chunk's reverse steps. Every chunk's inputs are staged in shared
// memory once. The only reduction across rows (a column sum: p = S'^T k
// forward, g = G^T k backward) is a reduce-scatter over the 8 row lanes of a
// warp followed by a fixed-order sum across warps, so results are
// deterministic; sums across a row are shuffles among 4 lanes.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "ckda.h"
#include "ckda_common.cuh"
#include "ckda_rowcol.cuh"

namespace ckda {
namespace {

// first checkpoint slot of sequence n; chunk c of it sits at slot + c, which
// never collides and stays below floor(T_total / CK) + N
__device__ __forceinline__ int bwd_slot_base(const int32_t *cu, int n, int T) {
  const int b = cu ? __ldg(cu + n) : n * T;
  return b / CK + n;
}

// stage tokens [t0, t0 + L) of head h into shared memory as fp32
template <typename IOT, int DK, int DV>
__device__ __forceinline__ void stage_chunk(float *sm, const IOT *q, const IOT *k, const IOT *v,
                                            const float *alpha, const float *beta,
                                            const IOT *d_o, int t0, int L, int H, int h,
                                            int tid, int DVF, int c0) {
  using B = BwdShape<DK, DV>;  // DV: the tile width here; DVF: the full d_v
  for (int i = tid; i < L * DK; i += B::NT) {
    const int t = i / DK, r = i - t * DK;
    const size_t g = ((size_t)(t0 + t) * H + h) * DK + r;
    sm[B::OFF_Q + t * DK + r] = IO<IOT>::ld(q + g);
    sm[B::OFF_K + t * DK + r] = IO<IOT>::ld(k + g);
    sm[B::OFF_A + t * DK + r] = __ldg(alpha + g);
  }
  for (int i = tid; i < L * DV; i += B::NT) {
    const int t = i / DV, c = i - t * DV;
    const size_t g = ((size_t)(t0 + t) * H + h) * DVF + c0 + c;
    sm[B::OFF_V + t * B::DVP + B::pc(c)] = IO<IOT>::ld(v + g);
    sm[B::OFF_DO + t * B::DVP + B::pc(c)] = d_o ? IO<IOT>::ld(d_o + g) : 0.f;
  }
  for (int t = tid; t < L; t += B::NT) sm[B::OFF_B + t] = __ldg(beta + (size_t)(t0 + t) * H + h);
}

// one forward step on this thread's columns of row r; w (column values) is
// written to shared memory row tl by the row-0 threads
template <int DK, int DV>
__device__ __forceinline__ void fwd_step(float (&S)[DV / 4], float *sm, int tl, int r, int cq,
                                         int tid, bool store_w) {
  using B = BwdShape<DK, DV>;
  constexpr int CPT = B::CPT;
  const float kr = sm[B::OFF_K + tl * DK + r], ar = sm[B::OFF_A + tl * DK + r];
  const float bt = sm[B::OFF_B + tl];
  float x[CPT];
#pragma unroll
  for (int j = 0; j < CPT; ++j) x[j] = (ar * S[j]) * kr;
  col_sum<DK, DV>(x, sm + B::OFF_P, sm + B::OFF_CS, tid);  // p = S'^T k
  float vv[CPT];
  lds_vec<CPT>(vv, sm + B::OFF_V + tl * B::DVP + cq * (CPT + 4));
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    const float w = vv[j] - x[j];
    S[j] = ar * S[j] + kr * (bt * w);
    x[j] = w;
  }
  if (store_w && r == 0) {
    float *wd = sm + B::OFF_W + tl * B::DVP + cq * (CPT + 4);
#pragma unroll
    for (int j = 0; j < CPT; j += 4)
      *reinterpret_cast<float4 *>(wd + j) = make_float4(x[j], x[j + 1], x[j + 2], x[j + 3]);
  }
}

template <typename IOT, int DK, int DV>
__global__ void __launch_bounds__(4 * DK, 1)
ckda_bwd_kernel(const IOT *__restrict__ q, const IOT *__restrict__ k, const IOT *__restrict__ v,
                const float *__restrict__ alpha, const float *__restrict__ beta,
                const float *__restrict__ s0, const IOT *__restrict__ d_o,
                const float *__restrict__ dsf, IOT *__restrict__ dv,
                float *__restrict__ pq, float *__restrict__ pk, float *__restrict__ pa,
                float *__restrict__ pb, float *__restrict__ ds0,
                const int32_t *__restrict__ cu, int T, int T_total, int H, int DVF,
                float scale, float *__restrict__ ck, float *__restrict__ buf,
                unsigned int *err) {
  using B = BwdShape<DK, DV>;  // DV: the tile width; DVF: the full d_v
  constexpr int CPT = B::CPT;
  extern __shared__ float sm[];
  const int tid = threadIdx.x, r = tid >> 2, cq = tid & 3;
  const int h = blockIdx.x, n = blockIdx.y, tile = blockIdx.z, ntile = gridDim.z;
  const int c0 = tile * DV;
  const size_t TH = (size_t)T_total * H;
  int bos, eos;
  seq_bounds(cu, n, T, T_total, err, bos, eos);
  const int len = eos - bos, nck = (len + CK - 1) / CK;
  const int slot0 = bwd_slot_base(cu, n, T);
  const size_t row_off = (size_t)r * DVF + c0 + cq * CPT;  // within one DK x DVF state
  const size_t st_off = ((size_t)n * H + h) * DK * DVF + row_off;
  float *mybuf = buf + (((size_t)n * H + h) * ntile + tile) * CK * DK * DV;
  const size_t brow = (size_t)r * DV + cq * CPT;  // within one buffered DK x DV tile

  // ---- pass 1: forward, a checkpoint at the start of every chunk
  float S[CPT];
#pragma unroll
  for (int j = 0; j < CPT; ++j) S[j] = s0 ? s0[st_off + j] : 0.f;
  for (int i = 0; i < nck; ++i) {
    const int t0 = bos + CK * i, L = min(CK, eos - t0);
    float *cp = ck + ((size_t)(slot0 + i) * H + h) * DK * DVF + row_off;
#pragma unroll
    for (int j = 0; j < CPT; j += 4)
      *reinterpret_cast<float4 *>(cp + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    __syncthreads();  // the previous chunk's readers of the staged inputs are done
    stage_chunk<IOT, DK, DV>(sm, q, k, v, alpha, beta, nullptr, t0, L, H, h, tid, DVF, c0);
    __syncthreads();
    for (int tl = 0; tl < L; ++tl) fwd_step<DK, DV>(S, sm, tl, r, cq, tid, false);
  }

  // ---- pass 2: chunks in reverse; recompute the pre-step states, then the
  // reverse steps
  float G[CPT];
#pragma unroll
  for (int j = 0; j < CPT; ++j) G[j] = dsf ? dsf[st_off + j] : 0.f;
  for (int i = nck - 1; i >= 0; --i) {
    const int t0 = bos + CK * i, L = min(CK, eos - t0);
    const float *cp = ck + ((size_t)(slot0 + i) * H + h) * DK * DVF + row_off;
#pragma unroll
    for (int j = 0; j < CPT; j += 4) {
      const float4 x = *reinterpret_cast<const float4 *>(cp + j);
      S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
    }
    __syncthreads();
    stage_chunk<IOT, DK, DV>(sm, q, k, v, alpha, beta, d_o, t0, L, H, h, tid, DVF, c0);
    __syncthreads();
    for (int tl = 0; tl < L; ++tl) {
      float *bp = mybuf + (size_t)tl * DK * DV + brow;
#pragma unroll
      for (int j = 0; j < CPT; j += 4)
        *reinterpret_cast<float4 *>(bp + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
      fwd_step<DK, DV>(S, sm, tl, r, cq, tid, true);
    }
    __syncthreads();  // w rows in shared memory
    for (int tl = L - 1; tl >= 0; --tl) {
      const size_t tok = (size_t)(t0 + tl) * H + h;
      const float qr = sm[B::OFF_Q + tl * DK + r], kr = sm[B::OFF_K + tl * DK + r];
      const float ar = sm[B::OFF_A + tl * DK + r], bt = sm[B::OFF_B + tl];
      const float *wrow = sm + B::OFF_W + tl * B::DVP + cq * (CPT + 4);
      const float *bp = mybuf + (size_t)tl * DK * DV + brow;
      float sp[CPT];
#pragma unroll
      for (int j = 0; j < CPT; j += 4) {
        const float4 x = *reinterpret_cast<const float4 *>(bp + j);
        sp[j] = x.x; sp[j + 1] = x.y; sp[j + 2] = x.z; sp[j + 3] = x.w;
      }
      float dqp = 0.f;
      const float *dorow = sm + B::OFF_DO + tl * B::DVP + cq * (CPT + 4);
#pragma unroll
      for (int j = 0; j < CPT; j += 4) {
        float w4[4], d4[4];
        lds_vec<4>(w4, wrow + j);
        lds_vec<4>(d4, dorow + j);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          G[j + e] += scale * qr * d4[e];
          const float st = ar * sp[j + e] + kr * (bt * w4[e]);  // S_t
          dqp += st * d4[e];
        }
      }
      const float dqr = scale * row_sum4(dqp);
      float g[CPT];
#pragma unroll
      for (int j = 0; j < CPT; ++j) g[j] = G[j] * kr;
      col_sum<DK, DV>(g, sm + B::OFF_P, sm + B::OFF_CS, tid);  // g = G^T k
      float dkp = 0.f, dap = 0.f, dbp = 0.f;
#pragma unroll
      for (int j = 0; j < CPT; j += 4) {
        float w4[4];
        lds_vec<4>(w4, wrow + j);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float spj = ar * sp[j + e];  // S'
          dkp += G[j + e] * w4[e] - spj * g[j + e];
          const float dspj = G[j + e] - bt * kr * g[j + e];  // dS'
          dap += dspj * sp[j + e];
          G[j + e] = ar * dspj;
          dbp += g[j + e] * w4[e];
        }
      }
      const float dkr = bt * row_sum4(dkp), dar = row_sum4(dap), dbt = row_sum4(dbp);
      if (cq == 0) {  // this tile's share of the row sums
        const size_t pi = (tile * TH + tok) * DK + r;
        pq[pi] = dqr;
        pk[pi] = dkr;
        pa[pi] = dar;
      }
      if (r == 0) {
#pragma unroll
        for (int j = 0; j < CPT; ++j) IO<IOT>::st(dv + tok * DVF + c0 + cq * CPT + j, bt * g[j]);
        if (cq == 0) pb[tile * TH + tok] = dbt;
      }
    }
  }
  if (ds0) {
#pragma unroll
    for (int j = 0; j < CPT; j += 4)
      *reinterpret_cast<float4 *>(ds0 + st_off + j) = make_float4(G[j], G[j + 1], G[j + 2], G[j + 3]);
  }
}

// dq, dk, dalpha (n_tk = T_total H d_k entries) and dbeta (n_t = T_total H):
// the tiles' partials added in tile order
template <typename IOT>
__global__ void ckda_bwd_reduce_kernel(const float *__restrict__ pq, const float *__restrict__ pk,
                                       const float *__restrict__ pa, const float *__restrict__ pb,
                                       IOT *__restrict__ dq, IOT *__restrict__ dk,
                                       float *__restrict__ dalpha, float *__restrict__ dbeta,
                                       size_t n_tk, size_t n_t, int ntile) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_tk;
       i += (size_t)gridDim.x * blockDim.x) {
    float a = 0.f, b = 0.f, c = 0.f;
    for (int t = 0; t < ntile; ++t) {
      a += pq[t * n_tk + i];
      b += pk[t * n_tk + i];
      c += pa[t * n_tk + i];
    }
    IO<IOT>::st(dq + i, a);
    IO<IOT>::st(dk + i, b);
    dalpha[i] = c;
    if (i < n_t) {
      float e = 0.f;
      for (int t = 0; t < ntile; ++t) e += pb[t * n_t + i];
      dbeta[i] = e;
    }
  }
}

}  // namespace

template <typename IOT>
cudaError_t launch_bwd_reduce(const float *pq, const float *pk, const float *pa,
                              const float *pb, void *dq, void *dk, float *dalpha, float *dbeta,
                              size_t n_tk, size_t n_t, int ntile, cudaStream_t st);

namespace {

template <typename IOT, int DK, int DVT>
cudaError_t launch_bwd_dims(const void *q, const void *k, const void *v, const float *alpha,
                            const float *beta, const float *s0, const void *d_o,
                            const float *dsf, void *dq, void *dk, void *dv, float *dalpha,
                            float *dbeta, float *ds0, const int32_t *cu, int N, int T,
                            int T_total, int H, int DVF, float scale, float *ck, float *buf,
                            float *pq, float *pk, float *pa, float *pb, unsigned int *err,
                            cudaStream_t st) {
  using B = BwdShape<DK, DVT>;
  auto kern = ckda_bwd_kernel<IOT, DK, DVT>;
  const size_t smem = (size_t)B::FLOATS * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int ntile = DVF / DVT;
  kern<<<dim3(H, N, ntile), B::NT, smem, st>>>(
      static_cast<const IOT *>(q), static_cast<const IOT *>(k), static_cast<const IOT *>(v),
      alpha, beta, s0, static_cast<const IOT *>(d_o), dsf, static_cast<IOT *>(dv), pq, pk, pa,
      pb, ds0, cu, T, T_total, H, DVF, scale, ck, buf, err);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t n_t = (size_t)T_total * H;
  return launch_bwd_reduce<IOT>(pq, pk, pa, pb, dq, dk, dalpha, dbeta, n_t * DK, n_t, ntile, st);
}

}  // namespace

template <typename IOT>
cudaError_t launch_bwd_reduce(const float *pq, const float *pk, const float *pa,
                              const float *pb, void *dq, void *dk, float *dalpha, float *dbeta,
                              size_t n_tk, size_t n_t, int ntile, cudaStream_t st) {
  if (n_tk == 0) return cudaSuccess;
  const unsigned grid = (unsigned)std::min<size_t>((n_tk + 255) / 256, 148 * 16);
  ckda_bwd_reduce_kernel<IOT><<<grid, 256, 0, st>>>(pq, pk, pa, pb, static_cast<IOT *>(dq),
                                                   static_cast<IOT *>(dk), dalpha, dbeta, n_tk,
                                                   n_t, ntile);
  return cudaGetLastError();
}
template cudaError_t launch_bwd_reduce<float>(const float *, const float *, const float *,
                                              const float *, void *, void *, float *, float *,
                                              size_t, size_t, int, cudaStream_t);
template cudaError_t launch_bwd_reduce<__nv_bfloat16>(const float *, const float *,
                                                      const float *, const float *, void *,
                                                      void *, float *, float *, size_t, size_t,
                                                      int, cudaStream_t);

// columns per CTA
static int bwd_tile(int dv) { return dv < 32 ? dv : 32; }

size_t bwd_workspace_bytes(int N, int T_total, int H, int dk, int dv) {
  const size_t slots = (size_t)T_total / CK + (size_t)N;
  const size_t state = (size_t)dk * dv * sizeof(float);
  const size_t ntile = (size_t)(dv / bwd_tile(dv)), th = (size_t)T_total * H;
  return slots * H * state + (size_t)N * H * CK * state +
         ntile * th * (3 * (size_t)dk + 1) * sizeof(float);
}

template <typename IOT>
cudaError_t launch_bwd(int dk_, int dv_, const void *q, const void *k, const void *v,
                       const float *alpha, const float *beta, const float *s0,
                       const void *d_o, const float *dsf, void *dq, void *dk, void *dv,
                       float *dalpha, float *dbeta, float *ds0, const int32_t *cu, int N,
                       int T, int T_total, int H, float scale, void *ws,
                       unsigned int *err, cudaStream_t st) {
  // workspace: checkpoints | state buffers | partials dq, dk, dalpha [ntile][T_total H d_k],
  // dbeta [ntile][T_total H]
  float *ck = static_cast<float *>(ws);
  const size_t slots = (size_t)T_total / CK + (size_t)N;
  float *buf = ck + slots * H * (size_t)dk_ * dv_;
  const size_t ntile = (size_t)(dv_ / bwd_tile(dv_)), th = (size_t)T_total * H;
  float *pq = buf + (size_t)N * H * CK * dk_ * dv_;
  float *pk = pq + ntile * th * dk_;
  float *pa = pk + ntile * th * dk_;
  float *pb = pa + ntile * th * dk_;
#define CKDA_BWD_DK(X)                                                                          \
  if (dk_ == X) {                                                                               \
    if (dv_ == 16)                                                                              \
      return launch_bwd_dims<IOT, X, 16>(q, k, v, alpha, beta, s0, d_o, dsf, dq, dk, dv, dalpha, \
                                         dbeta, ds0, cu, N, T, T_total, H, dv_, scale, ck, buf, \
                                         pq, pk, pa, pb, err, st);                              \
    return launch_bwd_dims<IOT, X, 32>(q, k, v, alpha, beta, s0, d_o, dsf, dq, dk, dv, dalpha,   \
                                       dbeta, ds0, cu, N, T, T_total, H, dv_, scale, ck, buf,   \
                                       pq, pk, pa, pb, err, st);                                \
  }
  CKDA_BWD_DK(16) CKDA_BWD_DK(32) CKDA_BWD_DK(64) CKDA_BWD_DK(128)
#undef CKDA_BWD_DK
  return cudaErrorInvalidValue;
}

template cudaError_t launch_bwd<float>(int, int, const void *, const void *, const void *,
                                       const float *, const float *, const float *,
                                       const void *, const float *, void *, void *, void *,
                                       float *, float *, float *, const int32_t *, int, int,
                                       int, int, float, void *, unsigned int *, cudaStream_t);
template cudaError_t launch_bwd<__nv_bfloat16>(int, int, const void *, const void *,
                                               const void *, const float *, const float *,
                                               const float *, const void *, const float *,
                                               void *, void *, void *, float *, float *,
                                               float *, const int32_t *, int, int, int, int,
                                               float, void *, unsigned int *, cudaStream_t);

}  // namespace ckda
