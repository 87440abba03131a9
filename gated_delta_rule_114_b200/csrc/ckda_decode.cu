// Decode step: one token per (sequence, head), state updated in place.
//
// The recurrence applied once (Semidirect Fourier Delta Attention, §1
// eq. (1); readout of the updated state, §3 eq. (14)), rewritten so the state
// is read once and written once:
//
//     S' = diag(alpha) S            (gate)
//     p  = S'^T k,  r = S'^T q      (two reductions over d_k, one pass)
//     u  = beta (v - p)             (delta correction)
//     o  = scale (r + (k.q) u)      (= scale S_new^T q, since S_new = S' + k u^T)
//     S  = S' + k u^T               (written back)
//
// The step is bound by HBM: 2 * d_k * d_v * 4 bytes of state traffic against
// about 6 * d_k * d_v flops. Each CTA owns a slice of DVS state columns of one
// (sequence, head); thread (row group rg, column quad cg) keeps RPT rows x 4
// columns of the slice in registers, so the state is streamed with fully
// coalesced 16-byte loads and stores (evict-first: it never fits in L2).
#include "ckda_common.cuh"

namespace ckda {

template <int DK, int DVS>
struct DecodeShape {
  static constexpr int TPR = DVS / 4;                          // threads per row
  static constexpr int RG = (DK < 256 / TPR) ? DK : 256 / TPR; // row groups
  static constexpr int THREADS = TPR * RG;
  static constexpr int RPT = DK / RG;                          // rows per thread
  static_assert(DK % RG == 0, "row groups must tile d_k");
};

// GATED: the fused input prologue (GateArgs): alpha_in holds gate logits
// (IOT), beta logits, k raw keys; with rn = 1 / (||k|| + eps),
// p = rn S'^T k, k.q = rn (k.q) and the update adds (rn k) u^T.
template <int DK, int DV, int DVS, typename IOT, bool GATED>
__global__ void __launch_bounds__(DecodeShape<DK, DVS>::THREADS, 4)
decode_step_kernel(const IOT *__restrict__ q, const IOT *__restrict__ k,
                   const IOT *__restrict__ v, const void *__restrict__ alpha_in,
                   const float *__restrict__ beta, float *__restrict__ state,
                   IOT *__restrict__ o, float scale, GateArgs ga) {
  using Sh = DecodeShape<DK, DVS>;
  constexpr int TPR = Sh::TPR, RG = Sh::RG, RPT = Sh::RPT;
  __shared__ float4 red_p[RG][TPR];
  __shared__ float4 red_r[RG][TPR];
  __shared__ float red_kq[RG];
  __shared__ float red_kk[GATED ? RG : 1];
  const float *__restrict__ alpha = reinterpret_cast<const float *>(alpha_in);
  const IOT *__restrict__ alogit = reinterpret_cast<const IOT *>(alpha_in);

  const size_t nh = blockIdx.x;
  const int tid = threadIdx.x;
  const int cg = tid % TPR;
  const int rg = tid / TPR;
  const int col = blockIdx.y * DVS + cg * 4;
  float *S = state + nh * DK * DV;

  // Issue the state loads first: they carry almost all of the latency.
  float4 s[RPT];
#pragma unroll
  for (int m = 0; m < RPT; ++m) {
    const int r = rg + m * RG;
    s[m] = __ldcs(reinterpret_cast<const float4 *>(S + (size_t)r * DV + col));
  }
  float a[RPT], kk[RPT], qq[RPT];
#pragma unroll
  for (int m = 0; m < RPT; ++m) {
    const int r = rg + m * RG;
    if constexpr (GATED) a[m] = gate_alpha(ga, IO<IOT>::ld(alogit + nh * DK + r));
    else a[m] = __ldg(alpha + nh * DK + r);
    kk[m] = IO<IOT>::ld(k + nh * DK + r);
    qq[m] = IO<IOT>::ld(q + nh * DK + r);
  }

  float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 rq = p;
  float kq = 0.f, kk2 = 0.f;
#pragma unroll
  for (int m = 0; m < RPT; ++m) {
    if constexpr (GATED) kk2 += kk[m] * kk[m];
    s[m].x *= a[m];
    s[m].y *= a[m];
    s[m].z *= a[m];
    s[m].w *= a[m];
    p.x += kk[m] * s[m].x;
    p.y += kk[m] * s[m].y;
    p.z += kk[m] * s[m].z;
    p.w += kk[m] * s[m].w;
    rq.x += qq[m] * s[m].x;
    rq.y += qq[m] * s[m].y;
    rq.z += qq[m] * s[m].z;
    rq.w += qq[m] * s[m].w;
    kq += kk[m] * qq[m];
  }
  red_p[rg][cg] = p;
  red_r[rg][cg] = rq;
  if (cg == 0) {
    red_kq[rg] = kq;
    if constexpr (GATED) red_kk[rg] = kk2;
  }
  __syncthreads();
  p = make_float4(0.f, 0.f, 0.f, 0.f);
  rq = p;
  kq = 0.f;
  kk2 = 0.f;
#pragma unroll
  for (int g = 0; g < RG; ++g) {
    const float4 x = red_p[g][cg], y = red_r[g][cg];
    p.x += x.x;
    p.y += x.y;
    p.z += x.z;
    p.w += x.w;
    rq.x += y.x;
    rq.y += y.y;
    rq.z += y.z;
    rq.w += y.w;
    kq += red_kq[g];
    if constexpr (GATED) kk2 += red_kk[g];
  }
  if constexpr (GATED) {  // normalised key: scale what k entered
    const float rn = key_rnorm(ga, kk2);
    p.x *= rn; p.y *= rn; p.z *= rn; p.w *= rn;
    kq *= rn;
#pragma unroll
    for (int m = 0; m < RPT; ++m) kk[m] *= rn;
  }

  float b = __ldg(beta + nh);
  if constexpr (GATED) b = gate_beta(ga, b);
  const float4 vv = IO<IOT>::ld4(v + nh * DV + col);
  float4 u;
  u.x = b * (vv.x - p.x);
  u.y = b * (vv.y - p.y);
  u.z = b * (vv.z - p.z);
  u.w = b * (vv.w - p.w);
  if (rg == 0) {
    float4 out;
    out.x = scale * (rq.x + kq * u.x);
    out.y = scale * (rq.y + kq * u.y);
    out.z = scale * (rq.z + kq * u.z);
    out.w = scale * (rq.w + kq * u.w);
    IO<IOT>::st4(o + nh * DV + col, out);
  }
#pragma unroll
  for (int m = 0; m < RPT; ++m) {
    const int r = rg + m * RG;
    s[m].x += kk[m] * u.x;
    s[m].y += kk[m] * u.y;
    s[m].z += kk[m] * u.z;
    s[m].w += kk[m] * u.w;
    __stcs(reinterpret_cast<float4 *>(S + (size_t)r * DV + col), s[m]);
  }
}

template <int DK, int DV, typename IOT>
static cudaError_t launch_decode_dv(const void *q, const void *k, const void *v,
                                    const void *alpha, const float *beta,
                                    float *state, void *o, int N, int H,
                                    float scale, GateArgs g, cudaStream_t st) {
  constexpr int DVS = DV >= 64 ? 64 : DV;
  using Sh = DecodeShape<DK, DVS>;
  const dim3 grid((unsigned)((size_t)N * H), DV / DVS);
  if (g.on)
    decode_step_kernel<DK, DV, DVS, IOT, true><<<grid, Sh::THREADS, 0, st>>>(
        (const IOT *)q, (const IOT *)k, (const IOT *)v, alpha, beta, state,
        (IOT *)o, scale, g);
  else
    decode_step_kernel<DK, DV, DVS, IOT, false><<<grid, Sh::THREADS, 0, st>>>(
        (const IOT *)q, (const IOT *)k, (const IOT *)v, alpha, beta, state,
        (IOT *)o, scale, g);
  return cudaGetLastError();
}

template <int DK, typename IOT>
static cudaError_t launch_decode_dk(int dv, const void *q, const void *k,
                                    const void *v, const void *alpha,
                                    const float *beta, float *state, void *o,
                                    int N, int H, float scale, GateArgs g,
                                    cudaStream_t st) {
  switch (dv) {
    case 16: return launch_decode_dv<DK, 16, IOT>(q, k, v, alpha, beta, state, o, N, H, scale, g, st);
    case 32: return launch_decode_dv<DK, 32, IOT>(q, k, v, alpha, beta, state, o, N, H, scale, g, st);
    case 64: return launch_decode_dv<DK, 64, IOT>(q, k, v, alpha, beta, state, o, N, H, scale, g, st);
    case 128: return launch_decode_dv<DK, 128, IOT>(q, k, v, alpha, beta, state, o, N, H, scale, g, st);
  }
  return cudaErrorInvalidValue;
}

template <typename IOT>
cudaError_t launch_decode(int dk, int dv, const void *q, const void *k,
                          const void *v, const void *alpha, const float *beta,
                          float *state, void *o, int N, int H, float scale,
                          GateArgs g, cudaStream_t st) {
  switch (dk) {
    case 16: return launch_decode_dk<16, IOT>(dv, q, k, v, alpha, beta, state, o, N, H, scale, g, st);
    case 32: return launch_decode_dk<32, IOT>(dv, q, k, v, alpha, beta, state, o, N, H, scale, g, st);
    case 64: return launch_decode_dk<64, IOT>(dv, q, k, v, alpha, beta, state, o, N, H, scale, g, st);
    case 128: return launch_decode_dk<128, IOT>(dv, q, k, v, alpha, beta, state, o, N, H, scale, g, st);
  }
  return cudaErrorInvalidValue;
}

template cudaError_t launch_decode<float>(int, int, const void *, const void *,
                                          const void *, const void *,
                                          const float *, float *, void *, int,
                                          int, float, GateArgs, cudaStream_t);
template cudaError_t launch_decode<__nv_bfloat16>(
    int, int, const void *, const void *, const void *, const void *,
    const float *, float *, void *, int, int, float, GateArgs, cudaStream_t);

}  // namespace ckda
