// The complex-phase gate's chunked forward (ckda_complex_chunk.cuh) as two
// kernels on CUDA cores (sm_100a):
//   prep  grid (checkpoint slots, H)   256 threads, parallel over all chunks
//   scan  grid (H, N, d_v tiles)       256 threads, the chunks in order
// Slots are floor(cu[n] / 16) + n + chunk; a slot that starts no chunk exits
// at once, before any barrier, on every thread of its CTA.
#include <cuda_runtime.h>

#include "ckda.h"
#include "ckda_bwd_split.cuh"
#include "ckda_common.cuh"
#include "ckda_exec.cuh"
#include "ckda_complex_chunk.cuh"
#include "ckda_rowcol.cuh"

namespace ckda {
namespace {

// 512 threads per CTA: both programs' CTAs are few per SM (the scan's 176 KB
// of shared memory allow one, the prep's two), and their phases are chains of
// shared-memory loads and FMAs, so more warps per SM hide more of that latency.
constexpr int kThreads = 512;

using Exec = DeviceExec<kThreads>;  // one phase per barrier, kThreads threads

template <int DK, int DVT>
__global__ void __launch_bounds__(kThreads)
complex_prep_kernel(cplx::Args a, cplx::Ws w, const int32_t *__restrict__ cu, int N, int T,
                    int T_total, unsigned int *err) {
  extern __shared__ float sm[];
  int n, ci;
  if (!bwdc::slot_chunk(cu, N, T, (int)blockIdx.x, n, ci)) return;
  int bos, eos;
  seq_bounds(cu, n, T, T_total, err, bos, eos);
  if (ci >= (eos - bos + CK - 1) / CK) return;
  const int t0 = bos + CK * ci, L = eos - t0 < CK ? eos - t0 : CK;
  Exec x;
  cplx::prep_program<Exec, DK, DVT>(x, a, w, sm, blockIdx.y, t0, L, blockIdx.x);
}

template <int DK, int DVT>
__global__ void __launch_bounds__(kThreads)
complex_scan_kernel(cplx::Args a, cplx::Ws w, const int32_t *__restrict__ cu, int T, int T_total,
                    unsigned int *err) {
  extern __shared__ float sm[];
  const int h = blockIdx.x, n = blockIdx.y, tile = blockIdx.z;
  int bos, eos;
  seq_bounds(cu, n, T, T_total, err, bos, eos);
  Exec x;
  cplx::scan_program<Exec, DK, DVT>(x, a, w, sm, h, n, tile, bos, eos, bos / CK + n);
}

template <int DK, int DVT>
cudaError_t launch_dims(const cplx::Args &a, const cplx::Ws &w, const int32_t *cu, int N, int T,
                        int T_total, unsigned int *err, cudaStream_t st) {
  using PL = cplx::PrepLayout<DK, DVT>;
  using SL = cplx::ScanLayout<DK, DVT>;
  auto prep = complex_prep_kernel<DK, DVT>;
  auto scan = complex_scan_kernel<DK, DVT>;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)PL::BYTES)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(scan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)SL::BYTES)) != cudaSuccess)
    return e;
  const unsigned slots = (unsigned)(T_total / CK + N);
  prep<<<dim3(slots, a.H), kThreads, PL::BYTES, st>>>(a, w, cu, N, T, T_total, err);
  scan<<<dim3(a.H, N, a.DVF / DVT), kThreads, SL::BYTES, st>>>(a, w, cu, T, T_total, err);
  return cudaGetLastError();
}

// Workspace pieces (float counts): W, Kbar, Qhat | Utilde | M | gamma_{C-1}.
void piece_sizes(int N, int T_total, int H, int dk, int dv, size_t (&n)[6]) {
  const size_t slots = (size_t)T_total / CK + (size_t)N, th = (size_t)T_total * H;
  n[0] = n[1] = n[2] = 2 * th * dk;
  n[3] = 2 * th * dv;
  n[4] = 2 * slots * H * CK * CK;
  n[5] = 2 * slots * H * dk;
}

}  // namespace

size_t complex_chunk_workspace_bytes(int N, int T_total, int H, int dk, int dv) {
  size_t n[6], total = 0;
  piece_sizes(N, T_total, H, dk, dv, n);
  for (size_t x : n) total += x;
  return total * sizeof(float);
}

cudaError_t launch_fwd_complex_chunked(int dk, int dv, const void *q, const void *k,
                                       const void *v, const float *alpha, const float *theta,
                                       const float *beta, const void *s0, void *sf, void *o,
                                       const int32_t *cu, int N, int T, int T_total, int H,
                                       float scale, void *ws, unsigned int *err,
                                       cudaStream_t st) {
  size_t n[6];
  piece_sizes(N, T_total, H, dk, dv, n);
  float *p = static_cast<float *>(ws);
  float *piece[6];
  for (int i = 0; i < 6; ++i) {
    piece[i] = p;
    p += n[i];
  }
  const cplx::Ws w{piece[0], piece[1], piece[2], piece[3], piece[4], piece[5]};
  const cplx::Args a{static_cast<const float *>(q), static_cast<const float *>(k),
                     static_cast<const float *>(v), alpha, theta, beta,
                     static_cast<const float *>(s0), static_cast<float *>(sf),
                     static_cast<float *>(o), H, dv, scale};
#define CKDA_CPLXC_DK(X)                                                     \
  if (dk == X)                                                               \
    return dv == 16 ? launch_dims<X, 16>(a, w, cu, N, T, T_total, err, st)   \
                    : launch_dims<X, 32>(a, w, cu, N, T, T_total, err, st);
  CKDA_CPLXC_DK(16) CKDA_CPLXC_DK(32) CKDA_CPLXC_DK(64) CKDA_CPLXC_DK(128)
#undef CKDA_CPLXC_DK
  return cudaErrorInvalidValue;
}

}  // namespace ckda
