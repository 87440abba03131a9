// Forward pass of the complex-phase gate on CUDA cores (sm_100a).
//
// "Semidirect Fourier Delta Attention" §3, eqs. (13)-(14), with complex q, k,
// v and state (complex64, interleaved real/imaginary fp32):
//   S' = Lambda_t S_{t-1},  Lambda_t = diag(alpha_t exp(i theta_t)),
//   p = k_t^* S',  S_t = S' + beta_t k_t (conj(v_t) - p)^T,  o_t = scale S_t^* q_t.
// One CTA per (sequence, head, tile of DVT complex columns); thread (row r,
// column quarter cq) keeps DVT/4 complex columns of row r of the state in
// registers. Tokens are staged in shared memory 16 at a time, with
// lambda = alpha (cos theta, sin theta) formed once per token and channel.
// Each token needs two column sums over the rows (p and o), each done on the
// real and imaginary parts together as one sum over 2 DVT "columns" (a warp
// reduce-scatter and a fixed-order sum across warps): deterministic. It is a
// token-serial first version of the complex path.
#include <cuda_runtime.h>

#include "ckda.h"
#include "ckda_common.cuh"
#include "ckda_rowcol.cuh"

namespace ckda {
namespace {

template <int DK, int DVT>
struct CplxShape {
  using B = BwdShape<DK, DVT>;       // per-column layout of the tile (padding, pc())
  using B2 = BwdShape<DK, 2 * DVT>;  // the column sums: real and imaginary parts
  static constexpr int NT = B::NT, CPT = B::CPT, DVP = B::DVP;
  // shared memory (floats): q, k, lambda [CK][DK][2]; v real, imaginary
  // [CK][DVP]; beta [CK]; column-sum partials [NW][DVP2] and sums [DVP2]
  static constexpr int OFF_Q = 0, OFF_K = OFF_Q + CK * DK * 2, OFF_L = OFF_K + CK * DK * 2;
  static constexpr int OFF_VR = OFF_L + CK * DK * 2, OFF_VI = OFF_VR + CK * DVP;
  static constexpr int OFF_B = OFF_VI + CK * DVP, OFF_P = OFF_B + CK;
  static constexpr int OFF_CS = OFF_P + B2::NW * B2::DVP;
  static constexpr int FLOATS = OFF_CS + B2::DVP;
};

template <int DK, int DVT>
__global__ void __launch_bounds__(4 * DK, 1)
ckda_fwd_complex_kernel(const float2 *__restrict__ q, const float2 *__restrict__ k,
                        const float2 *__restrict__ v, const float *__restrict__ alpha,
                        const float *__restrict__ theta, const float *__restrict__ beta,
                        const float2 *__restrict__ s0, float2 *__restrict__ sf,
                        float2 *__restrict__ o, const int32_t *__restrict__ cu, int T,
                        int T_total, int H, int DV, float scale, unsigned int *err) {
  using Sh = CplxShape<DK, DVT>;
  using B = typename Sh::B;
  constexpr int CPT = Sh::CPT;
  extern __shared__ float sm[];
  const int tid = threadIdx.x, r = tid >> 2, cq = tid & 3;
  const int h = blockIdx.x, n = blockIdx.y, c0 = blockIdx.z * DVT;
  int bos, eos;
  seq_bounds(cu, n, T, T_total, err, bos, eos);
  const size_t st_off = (((size_t)n * H + h) * DK + r) * DV + c0 + cq * CPT;
  float sr[CPT], si[CPT];
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    const float2 x = s0 ? s0[st_off + j] : make_float2(0.f, 0.f);
    sr[j] = x.x;
    si[j] = x.y;
  }
  for (int t0 = bos; t0 < eos; t0 += CK) {
    const int L = min(CK, eos - t0);
    __syncthreads();  // the previous chunk's readers of the staged inputs are done
    for (int i = tid; i < L * DK; i += Sh::NT) {
      const int t = i / DK, c = i - t * DK;
      const size_t g = ((size_t)(t0 + t) * H + h) * DK + c;
      const float2 qv = q[g], kv = k[g];
      float sn, cs;
      sincosf(__ldg(theta + g), &sn, &cs);
      const float a = __ldg(alpha + g);
      sm[Sh::OFF_Q + 2 * i] = qv.x; sm[Sh::OFF_Q + 2 * i + 1] = qv.y;
      sm[Sh::OFF_K + 2 * i] = kv.x; sm[Sh::OFF_K + 2 * i + 1] = kv.y;
      sm[Sh::OFF_L + 2 * i] = a * cs; sm[Sh::OFF_L + 2 * i + 1] = a * sn;
    }
    for (int i = tid; i < L * DVT; i += Sh::NT) {
      const int t = i / DVT, c = i - t * DVT;
      const float2 vv = v[((size_t)(t0 + t) * H + h) * DV + c0 + c];
      sm[Sh::OFF_VR + t * Sh::DVP + B::pc(c)] = vv.x;
      sm[Sh::OFF_VI + t * Sh::DVP + B::pc(c)] = vv.y;
    }
    for (int t = tid; t < L; t += Sh::NT) sm[Sh::OFF_B + t] = __ldg(beta + (size_t)(t0 + t) * H + h);
    __syncthreads();
    for (int tl = 0; tl < L; ++tl) {
      const int ri = 2 * (tl * DK + r);
      const float kr = sm[Sh::OFF_K + ri], ki = sm[Sh::OFF_K + ri + 1];
      const float lr = sm[Sh::OFF_L + ri], li = sm[Sh::OFF_L + ri + 1];
      const float qr = sm[Sh::OFF_Q + ri], qi = sm[Sh::OFF_Q + ri + 1];
      const float bt = sm[Sh::OFF_B + tl];
      float x[2 * CPT];
#pragma unroll
      for (int j = 0; j < CPT; ++j) {  // S' = lambda S; x = conj(k) S'
        const float a = sr[j], b = si[j];
        sr[j] = lr * a - li * b;
        si[j] = lr * b + li * a;
        x[j] = kr * sr[j] + ki * si[j];
        x[CPT + j] = kr * si[j] - ki * sr[j];
      }
      col_sum<DK, 2 * DVT>(x, sm + Sh::OFF_P, sm + Sh::OFF_CS, tid);  // p = k^* S'
      float vr[CPT], vi[CPT];
      lds_vec<CPT>(vr, sm + Sh::OFF_VR + tl * Sh::DVP + cq * (CPT + 4));
      lds_vec<CPT>(vi, sm + Sh::OFF_VI + tl * Sh::DVP + cq * (CPT + 4));
#pragma unroll
      for (int j = 0; j < CPT; ++j) {  // S = S' + beta k (conj(v) - p); x = conj(S) q
        const float ur = bt * (vr[j] - x[j]), ui = bt * (-vi[j] - x[CPT + j]);
        sr[j] += kr * ur - ki * ui;
        si[j] += kr * ui + ki * ur;
        x[j] = sr[j] * qr + si[j] * qi;
        x[CPT + j] = sr[j] * qi - si[j] * qr;
      }
      col_sum<DK, 2 * DVT>(x, sm + Sh::OFF_P, sm + Sh::OFF_CS, tid);  // o = S^* q
      if (r == 0) {
        float2 *dst = o + ((size_t)(t0 + tl) * H + h) * DV + c0 + cq * CPT;
#pragma unroll
        for (int j = 0; j < CPT; ++j) dst[j] = make_float2(scale * x[j], scale * x[CPT + j]);
      }
    }
  }
  if (sf) {
#pragma unroll
    for (int j = 0; j < CPT; ++j) sf[st_off + j] = make_float2(sr[j], si[j]);
  }
}

template <int DK, int DVT>
cudaError_t launch_complex_dims(const void *q, const void *k, const void *v, const float *alpha,
                                const float *theta, const float *beta, const void *s0, void *sf,
                                void *o, const int32_t *cu, int N, int T, int T_total, int H,
                                int DV, float scale, unsigned int *err, cudaStream_t st) {
  using Sh = CplxShape<DK, DVT>;
  auto kern = ckda_fwd_complex_kernel<DK, DVT>;
  const size_t smem = (size_t)Sh::FLOATS * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(H, N, DV / DVT), Sh::NT, smem, st>>>(
      static_cast<const float2 *>(q), static_cast<const float2 *>(k),
      static_cast<const float2 *>(v), alpha, theta, beta, static_cast<const float2 *>(s0),
      static_cast<float2 *>(sf), static_cast<float2 *>(o), cu, T, T_total, H, DV, scale, err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_complex(int dk, int dv, const void *q, const void *k, const void *v,
                               const float *alpha, const float *theta, const float *beta,
                               const void *s0, void *sf, void *o, const int32_t *cu, int N,
                               int T, int T_total, int H, float scale, unsigned int *err,
                               cudaStream_t st) {
#define CKDA_CPLX_DK(X)                                                                       \
  if (dk == X) {                                                                              \
    if (dv == 16)                                                                             \
      return launch_complex_dims<X, 16>(q, k, v, alpha, theta, beta, s0, sf, o, cu, N, T,     \
                                        T_total, H, dv, scale, err, st);                      \
    return launch_complex_dims<X, 32>(q, k, v, alpha, theta, beta, s0, sf, o, cu, N, T,       \
                                      T_total, H, dv, scale, err, st);                        \
  }
  CKDA_CPLX_DK(16) CKDA_CPLX_DK(32) CKDA_CPLX_DK(64) CKDA_CPLX_DK(128)
#undef CKDA_CPLX_DK
  return cudaErrorInvalidValue;
}

}  // namespace ckda
