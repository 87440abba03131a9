// Tensor-core (tcgen05 / TMEM) chunked forward: placeholder until the
// kernel lands; the dispatcher routes every call to the CUDA-core kernel.
#include "ckda.h"
#include "ckda_common.cuh"

namespace ckda {

bool fwd_tc_supported(int, int, int, ckda_dtype) { return false; }

cudaError_t launch_fwd_tc(const void *, const void *, const void *,
                          const float *, const float *, const float *, float *,
                          void *, const int32_t *, int, int, int, int, float,
                          unsigned int *, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace ckda
