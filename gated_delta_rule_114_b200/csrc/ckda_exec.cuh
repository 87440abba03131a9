// The device executor of the chunked kernels' per-CTA programs (the programs
// and their executor contract are in ckda_bwd_chunk.cuh): one phase of N
// items is this thread's share of the items, threadIdx.x + r * NT for
// r = 0, 1, ..., fully unrolled (N is a compile-time count), then the CTA's
// barrier. Every thread of the CTA runs every phase. Asynchronous copies
// (acopy4) are grouped per thread by commit() and waited for by
// wait_copies<pending>().
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
  // Start copying the 4 bytes at global `src` to shared `dst` in the
  // background (cp.async); wait_copies makes the copy visible.
  __device__ __forceinline__ void acopy4(float *dst, const float *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(
                     static_cast<unsigned>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
  }
  // Close this thread's group of the copies started since the last commit
  // (possibly an empty group).
  __device__ __forceinline__ void commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
  // Wait until at most `pending` of this thread's most recent groups are
  // still in flight, then a barrier: every thread's copies of the older
  // groups are visible to the whole CTA.
  template <int pending>
  __device__ __forceinline__ void wait_copies() {
    asm volatile("cp.async.wait_group %0;" ::"n"(pending) : "memory");
    __syncthreads();
  }
};

}  // namespace ckda
