// The split chunkwise backward (ckda_bwd_split.cuh) as four kernels on CUDA
// cores (sm_100a):
//   prep   grid (checkpoint slots, H)   256 threads, parallel over chunks
//   scan1  grid (H, N, d_v / 16)        entry states and U, chunk by chunk
//   scan2  grid (H, N, d_v / 16)        exit-state gradients and dR, in reverse
//   grads  grid (checkpoint slots, H)   every gradient of a chunk, its columns
//                                       in 16-column tiles added in order
// A slot that starts no chunk (slots are floor(cu[n] / 16) + n + chunk) exits
// at once, before any barrier, on every thread of its CTA.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ckda.h"
#include "ckda_bwd_split.cuh"
#include "ckda_common.cuh"
#include "ckda_exec.cuh"
#include "ckda_rowcol.cuh"

namespace ckda {

namespace {

constexpr int kGradTile = 16;  // columns per tile of the gradient program
constexpr int kScanTile = 16;  // columns per CTA of the scans (and per tile of prep)

constexpr int kThreads = 256;
// the prep's CTAs (51 KB of shared memory, few registers) take 512 threads:
// four of them fill an SM's warp slots; so do the scans' (97 KB, two per SM,
// at most 64 registers a thread)
constexpr int kPrepThreads = 512;
constexpr int kScanThreads = 512;

using Exec = DeviceExec<kThreads>;  // one phase per barrier, kThreads threads
using PrepExec = DeviceExec<kPrepThreads>;
using ScanExec = DeviceExec<kScanThreads>;

// the chunk of slot blockIdx.x: token rows [t0, t0 + L); false if none
__device__ __forceinline__ bool slot_rows(const int32_t *cu, int N, int T, int T_total,
                                          unsigned int *err, int &t0, int &L) {
  int n, ci;
  if (!bwdc::slot_chunk(cu, N, T, (int)blockIdx.x, n, ci)) return false;
  int bos, eos;
  seq_bounds(cu, n, T, T_total, err, bos, eos);
  if (ci >= (eos - bos + bwdc::C - 1) / bwdc::C) return false;
  t0 = bos + bwdc::C * ci;
  L = eos - t0 < bwdc::C ? eos - t0 : bwdc::C;
  return true;
}

template <typename IOT, int DK, int DVT>
__global__ void __launch_bounds__(kPrepThreads)
bwd_prep_kernel(bwdc::Args<IOT> a, bwdc::SplitWs w, const int32_t *__restrict__ cu, int N,
                int T, int T_total, unsigned int *err) {
  extern __shared__ float sm[];
  int t0, L;
  if (!slot_rows(cu, N, T, T_total, err, t0, L)) return;
  PrepExec x;
  bwdc::prep_program<PrepExec, IO<IOT>, IOT, DK, DVT>(x, a, w, sm, blockIdx.y, t0, L,
                                                        blockIdx.x);
}

template <typename IOT, int DK, int DVT, bool REVERSE>
__global__ void __launch_bounds__(kScanThreads, 2)
bwd_scan_kernel(bwdc::Args<IOT> a, bwdc::SplitWs w, const int32_t *__restrict__ cu, int T,
                int T_total, unsigned int *err) {
  extern __shared__ float sm[];
  const int h = blockIdx.x, n = blockIdx.y, tile = blockIdx.z;
  int bos, eos;
  seq_bounds(cu, n, T, T_total, err, bos, eos);
  ScanExec x;
  if (REVERSE)
    bwdc::scan2_program<ScanExec, IO<IOT>, IOT, DK, DVT>(x, a, w, sm, h, n, tile, bos, eos,
                                                               bos / CK + n);
  else
    bwdc::scan1_program<ScanExec, IO<IOT>, IOT, DK, DVT>(x, a, w, sm, h, n, tile, bos, eos,
                                                               bos / CK + n);
}

template <typename IOT, int DK>
__global__ void __launch_bounds__(kThreads, 2)
bwd_grads_kernel(bwdc::Args<IOT> a, bwdc::SplitWs w, const int32_t *__restrict__ cu, int N,
                 int T, int T_total, unsigned int *err) {
  extern __shared__ float sm[];
  int t0, L;
  if (!slot_rows(cu, N, T, T_total, err, t0, L)) return;
  Exec x;
  bwdc::grads_program<Exec, IO<IOT>, IOT, DK, kGradTile>(x, a, w, sm, blockIdx.y, t0, L,
                                                               blockIdx.x);
}

template <class K>
cudaError_t set_smem(K kern, size_t bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <typename IOT, int DK, int DVT>
cudaError_t launch_dims(const bwdc::Args<IOT> &a, const bwdc::SplitWs &w, const int32_t *cu,
                        int N, int T, int T_total, unsigned int *err, cudaStream_t st) {
  const unsigned slots = (unsigned)(T_total / CK + N);
  const int ntile = a.DVF / DVT;
  using PL = bwdc::PrepLayout<DK, DVT>;
  using SL = bwdc::ScanLayout<DK, DVT>;
  using GL = bwdc::GradLayout<DK, kGradTile>;
  cudaError_t e;
  if ((e = set_smem(bwd_prep_kernel<IOT, DK, DVT>, PL::BYTES)) != cudaSuccess) return e;
  if ((e = set_smem(bwd_scan_kernel<IOT, DK, DVT, false>, SL::BYTES)) != cudaSuccess) return e;
  if ((e = set_smem(bwd_scan_kernel<IOT, DK, DVT, true>, SL::BYTES)) != cudaSuccess) return e;
  if ((e = set_smem(bwd_grads_kernel<IOT, DK>, GL::BYTES)) != cudaSuccess) return e;
  bwd_prep_kernel<IOT, DK, DVT><<<dim3(slots, a.H), kPrepThreads, PL::BYTES, st>>>(a, w, cu, N, T,
                                                                              T_total, err);
  bwd_scan_kernel<IOT, DK, DVT, false><<<dim3(a.H, N, ntile), kScanThreads, SL::BYTES, st>>>(
      a, w, cu, T, T_total, err);
  bwd_scan_kernel<IOT, DK, DVT, true><<<dim3(a.H, N, ntile), kScanThreads, SL::BYTES, st>>>(
      a, w, cu, T, T_total, err);
  bwd_grads_kernel<IOT, DK><<<dim3(slots, a.H), kThreads, GL::BYTES, st>>>(a, w, cu, N, T,
                                                                          T_total, err);
  return cudaGetLastError();
}

// Workspace pieces, in order: checkpoints S and dS | gamma_C | Abar | W, Kbar,
// Wb, Qs, BK | Utilde, X, U, dR (float counts).
constexpr int kPieces = 13;

void piece_sizes(int N, int T_total, int H, int dk, int dv, size_t (&n)[kPieces]) {
  const size_t slots = (size_t)T_total / CK + (size_t)N, th = (size_t)T_total * H;
  const size_t sizes[kPieces] = {slots * H * dk * dv, slots * H * dk * dv, slots * H * dk,
                                 slots * H * CK * CK, th * dk, th * dk, th * dk, th * dk,
                                 th * dk, th * dv, th * dv, th * dv, th * dv};
  for (int i = 0; i < kPieces; ++i) n[i] = sizes[i];
}

bwdc::SplitWs carve(float *base, int N, int T_total, int H, int dk, int dv) {
  size_t n[kPieces];
  piece_sizes(N, T_total, H, dk, dv, n);
  float *p[kPieces];
  for (int i = 0; i < kPieces; ++i) {
    p[i] = base;
    base += n[i];
  }
  return bwdc::SplitWs{p[0], p[1], p[2], p[3], p[4], p[5], p[6],
                       p[7], p[8], p[9], p[10], p[11], p[12]};
}

}  // namespace

size_t bwd_split_workspace_bytes(int N, int T_total, int H, int dk, int dv) {
  size_t n[kPieces], total = 0;
  piece_sizes(N, T_total, H, dk, dv, n);
  for (size_t x : n) total += x;
  return total * sizeof(float);
}

template <typename IOT>
cudaError_t launch_bwd_split(int dk_, int dv_, const void *q, const void *k, const void *v,
                             const float *alpha, const float *beta, const float *s0,
                             const void *d_o, const float *dsf, void *dq, void *dk, void *dv,
                             float *dalpha, float *dbeta, float *ds0, const int32_t *cu, int N,
                             int T, int T_total, int H, float scale, void *ws,
                             unsigned int *err, cudaStream_t st) {
  const bwdc::SplitWs w = carve(static_cast<float *>(ws), N, T_total, H, dk_, dv_);
  bwdc::Args<IOT> a{static_cast<const IOT *>(q),  static_cast<const IOT *>(k),
                    static_cast<const IOT *>(v),  alpha, beta, s0,
                    static_cast<const IOT *>(d_o), dsf,
                    static_cast<IOT *>(dq),       static_cast<IOT *>(dk),
                    static_cast<IOT *>(dv),       dalpha, dbeta, ds0, H, dv_, scale};
  // the scans take 16-column tiles: twice the CTAs of 32-column ones (d_v / 16
  // per sequence and head), each with half the work per chunk, up to three per SM
  switch (dk_) {
    case 16: return launch_dims<IOT, 16, kScanTile>(a, w, cu, N, T, T_total, err, st);
    case 32: return launch_dims<IOT, 32, kScanTile>(a, w, cu, N, T, T_total, err, st);
    case 64: return launch_dims<IOT, 64, kScanTile>(a, w, cu, N, T, T_total, err, st);
    case 128: return launch_dims<IOT, 128, kScanTile>(a, w, cu, N, T, T_total, err, st);
  }
  return cudaErrorInvalidValue;
}

template cudaError_t launch_bwd_split<float>(int, int, const void *, const void *, const void *,
                                             const float *, const float *, const float *,
                                             const void *, const float *, void *, void *,
                                             void *, float *, float *, float *, const int32_t *,
                                             int, int, int, int, float, void *, unsigned int *,
                                             cudaStream_t);
template cudaError_t launch_bwd_split<__nv_bfloat16>(int, int, const void *, const void *,
                                                     const void *, const float *, const float *,
                                                     const float *, const void *, const float *,
                                                     void *, void *, void *, float *, float *,
                                                     float *, const int32_t *, int, int, int,
                                                     int, float, void *, unsigned int *,
                                                     cudaStream_t);

}  // namespace ckda
