// The chunkwise backward pass of the CKDA recurrence on CUDA cores (sm_100a).
//
// The per-CTA program is ckda_bwd_chunk.cuh (the chunk-WY reverse of
// "Semidirect Fourier Delta Attention" §2.2 eqs. (9)-(10), with the
// division-free gate gradient); here it runs with one CTA of 256 threads per
// (sequence, head, tile of DVT state columns), each phase a strided loop over
// the threads followed by __syncthreads. Its checkpoint slots and fp32
// partials use the token-serial backward's workspace layout, and the same
// reduce kernel adds the tiles' partials in tile order, so results are
// deterministic.
//
// Compared with the token-serial kernel, the only sequential dependence left
// is one d_k x DVT state gradient per 16-token chunk; everything inside a
// chunk is matrix products, triangular solves and per-channel running
// products over 16 tokens.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ckda.h"
#include "ckda_bwd_chunk.cuh"
#include "ckda_common.cuh"
#include "ckda_rowcol.cuh"

namespace ckda {

template <typename IOT>
cudaError_t launch_bwd_reduce(const float *pq, const float *pk, const float *pa,
                              const float *pb, void *dq, void *dk, float *dalpha, float *dbeta,
                              size_t n_tk, size_t n_t, int ntile, cudaStream_t st);

namespace {

static_assert(bwdc::C == CK, "checkpoint slots hold one state per CK tokens");

constexpr int kBwdChunkThreads = 256;

struct DeviceExec {
  template <class F>
  __device__ __forceinline__ void par(int n, F f) {
    for (int i = threadIdx.x; i < n; i += kBwdChunkThreads) f(i);
    __syncthreads();
  }
};

template <typename IOT, int DK, int DVT>
__global__ void __launch_bounds__(kBwdChunkThreads, 1)
ckda_bwd_chunk_kernel(bwdc::Args<IOT> a, const int32_t *__restrict__ cu, int T, int T_total,
                      unsigned int *err) {
  extern __shared__ float sm[];
  const int h = blockIdx.x, n = blockIdx.y, tile = blockIdx.z;
  int bos, eos;
  seq_bounds(cu, n, T, T_total, err, bos, eos);  // a malformed entry gives an empty range
  const int slot0 = bos / CK + n;                 // as the token-serial backward's slots
  DeviceExec x;
  bwdc::bwd_chunk_program<DeviceExec, IO<IOT>, IOT, DK, DVT>(x, a, sm, h, n, tile, bos, eos,
                                                             slot0);
}

template <typename IOT, int DK, int DVT>
cudaError_t launch_dims(const bwdc::Args<IOT> &a, const int32_t *cu, int N, int T, int T_total,
                        unsigned int *err, cudaStream_t st) {
  using Ly = bwdc::Layout<DK, DVT>;
  auto kern = ckda_bwd_chunk_kernel<IOT, DK, DVT>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Ly::BYTES);
  if (e != cudaSuccess) return e;
  kern<<<dim3(a.H, N, a.DVF / DVT), kBwdChunkThreads, Ly::BYTES, st>>>(a, cu, T, T_total, err);
  return cudaGetLastError();
}

}  // namespace

// Workspace of launch_bwd_chunk: checkpoint slots | partials dq, dk, dalpha
// [ntile][T_total H][d_k] | dbeta [ntile][T_total H]. At most the token-serial
// backward's (it needs no per-CTA state buffers).
size_t bwd_chunk_workspace_bytes(int N, int T_total, int H, int dk, int dv) {
  const size_t slots = (size_t)T_total / CK + (size_t)N;
  const size_t ntile = (size_t)(dv / (dv < 32 ? dv : 32)), th = (size_t)T_total * H;
  return slots * H * dk * dv * sizeof(float) + ntile * th * (3 * (size_t)dk + 1) * sizeof(float);
}

template <typename IOT>
cudaError_t launch_bwd_chunk(int dk_, int dv_, const void *q, const void *k, const void *v,
                             const float *alpha, const float *beta, const float *s0,
                             const void *d_o, const float *dsf, void *dq, void *dk, void *dv,
                             float *dalpha, float *dbeta, float *ds0, const int32_t *cu, int N,
                             int T, int T_total, int H, float scale, void *ws,
                             unsigned int *err, cudaStream_t st) {
  const int dvt = dv_ < 32 ? dv_ : 32;
  const size_t slots = (size_t)T_total / CK + (size_t)N, th = (size_t)T_total * H;
  const size_t ntile = (size_t)(dv_ / dvt);
  float *ck = static_cast<float *>(ws);
  float *pq = ck + slots * H * (size_t)dk_ * dv_;
  float *pk = pq + ntile * th * dk_;
  float *pa = pk + ntile * th * dk_;
  float *pb = pa + ntile * th * dk_;
  bwdc::Args<IOT> a{static_cast<const IOT *>(q), static_cast<const IOT *>(k),
                    static_cast<const IOT *>(v), alpha, beta, s0,
                    static_cast<const IOT *>(d_o), dsf, static_cast<IOT *>(dv), pq, pk, pa,
                    pb, ds0, ck, H, dv_, th, scale};
  cudaError_t e = cudaErrorInvalidValue;
#define CKDA_BWDC_DK(X)                                                  \
  if (dk_ == X)                                                          \
    e = dvt == 16 ? launch_dims<IOT, X, 16>(a, cu, N, T, T_total, err, st) \
                  : launch_dims<IOT, X, 32>(a, cu, N, T, T_total, err, st);
  CKDA_BWDC_DK(16) CKDA_BWDC_DK(32) CKDA_BWDC_DK(64) CKDA_BWDC_DK(128)
#undef CKDA_BWDC_DK
  if (e != cudaSuccess) return e;
  return launch_bwd_reduce<IOT>(pq, pk, pa, pb, dq, dk, dalpha, dbeta, th * dk_, th,
                                (int)ntile, st);
}

template cudaError_t launch_bwd_chunk<float>(int, int, const void *, const void *, const void *,
                                             const float *, const float *, const float *,
                                             const void *, const float *, void *, void *,
                                             void *, float *, float *, float *, const int32_t *,
                                             int, int, int, int, float, void *, unsigned int *,
                                             cudaStream_t);
template cudaError_t launch_bwd_chunk<__nv_bfloat16>(int, int, const void *, const void *,
                                                     const void *, const float *, const float *,
                                                     const float *, const void *, const float *,
                                                     void *, void *, void *, float *, float *,
                                                     float *, const int32_t *, int, int, int,
                                                     int, float, void *, unsigned int *,
                                                     cudaStream_t);

}  // namespace ckda
