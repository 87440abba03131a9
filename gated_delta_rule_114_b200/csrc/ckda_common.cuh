// Shared device helpers for the CKDA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ckda {

// Bits of the per-device error word (read and cleared by ckda_last_error).
enum : unsigned int {
  kErrBadSeqlens = 1u << 0,   // device cu_seqlens out of range / decreasing
  kErrMbarTimeout = 1u << 1,  // a bounded mbarrier wait gave up
  kErrTmemAlloc = 1u << 2,    // tensor-memory allocation returned garbage
};

// Kernels receive the device address of the per-device error word (defined
// in ckda_api.cu) as an argument; nullptr disables reporting.
__device__ __forceinline__ void flag_error(unsigned int *err, unsigned int bit) {
  if (err) atomicOr(err, bit);
}

// Fused input prologue (see ckda_gate_params in ckda.h). When `on`, the
// kernels read gate logits a (I/O element type) and c (fp32) in place of
// alpha and beta and raw keys in place of k, and form
//   alpha = amin + arange * sigmoid(a), beta = bmax * sigmoid(c),
//   k = k_raw * rn with rn = 1 / (||k_raw|| + keps) (0 when that sum is 0).
struct GateArgs {
  int on;
  float amin, arange, bmax, keps;
};
__device__ __forceinline__ float sigmoidf(float x) { return 1.f / (1.f + expf(-x)); }
__device__ __forceinline__ float gate_alpha(const GateArgs &g, float a) {
  return g.amin + g.arange * sigmoidf(a);
}
__device__ __forceinline__ float gate_beta(const GateArgs &g, float c) {
  return g.bmax * sigmoidf(c);
}
// The tensor-core path (tf32 products) takes the hardware exp2 and
// reciprocal approximations, a few ulp from the accurate forms above.
__device__ __forceinline__ float gate_alpha_fast(const GateArgs &g, float a) {
  return g.amin + g.arange * __fdividef(1.f, 1.f + __expf(-a));
}
__device__ __forceinline__ float key_rnorm(const GateArgs &g, float sumsq) {
  const float d = sqrtf(sumsq) + g.keps;
  return d > 0.f ? 1.f / d : 0.f;
}

// Element-type traits for q, k, v, o.
template <typename T> struct IO;
template <> struct IO<float> {
  static __device__ __forceinline__ float ld(const float *p) { return *p; }
  // read-only data (not written while the kernel runs)
  static __device__ __forceinline__ float ldg(const float *p) { return __ldg(p); }
  static __device__ __forceinline__ void st(float *p, float x) { *p = x; }
  // 4 consecutive elements (16-byte aligned for float)
  static __device__ __forceinline__ float4 ld4(const float *p) {
    return *reinterpret_cast<const float4 *>(p);
  }
  static __device__ __forceinline__ void st4(float *p, float4 x) {
    *reinterpret_cast<float4 *>(p) = x;
  }
};
template <> struct IO<__nv_bfloat16> {
  static __device__ __forceinline__ float ld(const __nv_bfloat16 *p) {
    return __bfloat162float(*p);
  }
  static __device__ __forceinline__ float ldg(const __nv_bfloat16 *p) {
    return __bfloat162float(__ldg(p));
  }
  static __device__ __forceinline__ void st(__nv_bfloat16 *p, float x) {
    *p = __float2bfloat16_rn(x);
  }
  // element `hi` (0 or 1) of a bf16 pair held in the 4 bytes of `pair`
  static __device__ __forceinline__ float pair_half(float pair, int hi) {
    const uint32_t b = __float_as_uint(pair);
    return __uint_as_float(hi ? (b & 0xffff0000u) : (b << 16));
  }
  // 4 consecutive elements (8-byte aligned)
  static __device__ __forceinline__ float4 ld4(const __nv_bfloat16 *p) {
    uint2 raw = *reinterpret_cast<const uint2 *>(p);
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&raw.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&raw.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
  }
  static __device__ __forceinline__ void st4(__nv_bfloat16 *p, float4 x) {
    __nv_bfloat162 a = __floats2bfloat162_rn(x.x, x.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(x.z, x.w);
    uint2 raw;
    raw.x = *reinterpret_cast<unsigned int *>(&a);
    raw.y = *reinterpret_cast<unsigned int *>(&b);
    *reinterpret_cast<uint2 *>(p) = raw;
  }
};

// Sequence bounds for sequence n: [bos, eos). With cu == nullptr every
// sequence has T tokens. A malformed device cu_seqlens entry flags an error
// and yields an empty range, so no kernel ever indexes outside [0, T_total).
__device__ __forceinline__ void seq_bounds(const int32_t *cu, int n, int T,
                                           int T_total, unsigned int *err,
                                           int &bos, int &eos) {
  if (cu == nullptr) {
    bos = n * T;
    eos = bos + T;
    return;
  }
  bos = __ldg(cu + n);
  eos = __ldg(cu + n + 1);
  if (bos < 0 || eos < bos || eos > T_total) {
    bos = 0;
    eos = 0;
    flag_error(err, kErrBadSeqlens);
  }
}

}  // namespace ckda
