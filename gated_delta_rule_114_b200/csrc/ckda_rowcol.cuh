// Row/column helpers shared by the token-serial CUDA-core kernels (the
// backward pass and the complex-phase-gate forward): one CTA holds a d_k x DV
// state tile, thread (row r, column quarter cq) keeping DV/4 columns of row r
// in registers (4 d_k threads).
#pragma once

#include <cuda_runtime.h>

namespace ckda {
namespace {

constexpr int CK = 16;  // tokens staged per chunk (and between checkpoints)

template <int DK, int DV>
struct BwdShape {
  static constexpr int NT = 4 * DK;     // threads
  static constexpr int NW = NT / 32;    // warps
  static constexpr int CPT = DV / 4;    // columns per thread
  // Per-column vectors keep each column quarter 4 floats apart from the next
  // (column c at pc(c) = c + 4 (c / CPT), row length DVP): the four quarter
  // groups of a warp then read four different banks instead of one.
  static constexpr int DVP = DV + 16;
  // shared memory (floats): chunk inputs q, k, alpha [CK][DK]; v, do, w
  // [CK][DVP]; beta [CK]; column-sum partials [NW][DVP] and sums [DVP]
  static constexpr int OFF_Q = 0, OFF_K = OFF_Q + CK * DK, OFF_A = OFF_K + CK * DK;
  static constexpr int OFF_V = OFF_A + CK * DK, OFF_DO = OFF_V + CK * DVP;
  static constexpr int OFF_W = OFF_DO + CK * DVP, OFF_B = OFF_W + CK * DVP;
  static constexpr int OFF_P = OFF_B + CK, OFF_CS = OFF_P + NW * DVP;
  static constexpr int FLOATS = OFF_CS + DVP;
  static __device__ __forceinline__ int pc(int c) { return c + 4 * (c / CPT); }
};

// n (a multiple of 4) consecutive floats of shared memory into registers
template <int N>
__device__ __forceinline__ void lds_vec(float *dst, const float *src) {
#pragma unroll
  for (int j = 0; j < N; j += 4) {
    const float4 x = *reinterpret_cast<const float4 *>(src + j);
    dst[j] = x.x; dst[j + 1] = x.y; dst[j + 2] = x.z; dst[j + 3] = x.w;
  }
}

// Column sums of x (this thread's CPT columns of row r) over all DK rows;
// x is replaced by the sums of the same columns. Scratch in shared memory:
// part [NW][DVP], cs [DVP] (BwdShape<DK, DV>). Two CTA barriers.
template <int DK, int DV>
__device__ __forceinline__ void col_sum(float (&x)[DV / 4], float *part, float *cs, int tid) {
  using B = BwdShape<DK, DV>;
  constexpr int CPT = B::CPT;
  const int lane = tid & 31, warp = tid >> 5, cq = lane & 3;
  // reduce-scatter over lane bits 4, 3, 2 (the row lanes) while a lane holds
  // two values or more; all-reduce after that
  int off = 0;
  bool writer = true;
  constexpr int n1 = CPT, n2 = n1 >= 2 ? n1 / 2 : 1, n3 = n2 >= 2 ? n2 / 2 : 1;
  constexpr int nf = n3 >= 2 ? n3 / 2 : 1;
#pragma unroll
  for (int level = 0; level < 3; ++level) {
    const int m = 16 >> level;
    const int n = level == 0 ? n1 : (level == 1 ? n2 : n3);
    const bool up = (lane & m) != 0;
    if (n >= 2) {
      const int half = n / 2;
#pragma unroll
      for (int e = 0; e < CPT / 2; ++e) {
        if (e < half) {
          const float keep = up ? x[half + e] : x[e];
          const float send = up ? x[e] : x[half + e];
          x[e] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
      }
      off += up ? half : 0;
    } else {
      x[0] += __shfl_xor_sync(0xffffffffu, x[0], m);
      writer = writer && !up;
    }
  }
  if (writer) {
#pragma unroll
    for (int e = 0; e < nf; ++e) part[warp * B::DVP + cq * (CPT + 4) + off + e] = x[e];
  }
  __syncthreads();
  for (int c = tid; c < DV; c += B::NT) {
    float s = 0.f;
    const int cp = B::pc(c);
#pragma unroll
    for (int w = 0; w < B::NW; ++w) s += part[w * B::DVP + cp];
    cs[cp] = s;
  }
  __syncthreads();
  lds_vec<CPT>(x, cs + cq * (CPT + 4));
}

// sum over the 4 lanes of one row
__device__ __forceinline__ float row_sum4(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}

}  // namespace
}  // namespace ckda
