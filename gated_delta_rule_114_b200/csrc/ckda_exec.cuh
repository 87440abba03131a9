// The device executor of the chunked kernels' per-CTA programs (the programs
// and their executor contract are in ckda_bwd_chunk.cuh): one phase of N
// items is this thread's share of the items, threadIdx.x + r * NT for
// r = 0, 1, ..., fully unrolled (N is a compile-time count), then the CTA's
// barrier. Every thread of the CTA runs every phase.
#pragma once

#include <cuda_runtime.h>

namespace ckda {

template <int NT>
struct DeviceExec {
  template <int N, class F>
  __device__ __forceinline__ void run(F f) {
    constexpr int R = (N + NT - 1) / NT;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int i = threadIdx.x + r * NT;
      if (N % NT == 0 || i < N) f(i);
    }
    __syncthreads();
  }
};

}  // namespace ckda
