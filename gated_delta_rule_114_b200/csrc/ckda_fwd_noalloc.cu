// ckda_fwd_chunked_noalloc: the chunked forward for callers that cannot
// provide device scratch memory.
//
// Some callers have no way to hand the library a workspace: a plain C program
// with no device allocator of its own, or a serving loop that must not call
// cudaMalloc once it is running, because cudaMalloc may synchronise the whole
// device and stall every other stream. For them the tensor-core path takes its
// scratch from one fixed array in device memory that is part of this library
// and lives as long as the process (every GPU that loads the library keeps
// its own copy of the array until the process exits). Nothing here allocates:
// no cudaMalloc, no cudaFree, no allocating library routine.
#include <cuda_runtime.h>

#include <mutex>

#include "ckda.h"

// The scratch itself. Host code never dereferences this name: on the host it
// only stands for the symbol; its device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[CKDA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per
// device (on that device's first call) and cached. nullptr on failure.
void *scratch_address() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" {

ckda_status ckda_fwd_chunked_noalloc(const void *q, const void *k, const void *v,
                                     const float *alpha, const float *beta,
                                     const float *initial_state, float *final_state,
                                     void *o, const int32_t *cu_seqlens,
                                     const int32_t *cu_seqlens_host, int32_t N,
                                     int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                                     int32_t chunk, float scale, ckda_dtype dt,
                                     cudaStream_t stream) {
  const size_t need = ckda_fwd_workspace_bytes(N, T, H, d_k, d_v, chunk,
                                               cu_seqlens != nullptr, dt);
  if (need == 0)  // this configuration needs no scratch at all
    return ckda_fwd_chunked(q, k, v, alpha, beta, initial_state, final_state, o,
                            cu_seqlens, cu_seqlens_host, N, T, H, d_k, d_v, chunk,
                            scale, dt, nullptr, 0, stream);
  if (need > CKDA_NOALLOC_SCRATCH_BYTES) return CKDA_ERR_UNSUPPORTED;
  void *ws = scratch_address();
  if (!ws) return CKDA_ERR_CUDA;
  // Every byte of scratch that the kernels read is written earlier in the
  // same call, so nothing has to be cleared between calls.
  return ckda_fwd_chunked(q, k, v, alpha, beta, initial_state, final_state, o,
                          cu_seqlens, cu_seqlens_host, N, T, H, d_k, d_v, chunk,
                          scale, dt, ws, CKDA_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"
