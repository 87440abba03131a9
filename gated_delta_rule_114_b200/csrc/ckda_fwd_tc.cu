// Chunkwise CKDA forward with tcgen05 tensor cores (sm_100a): bf16 I/O,
// fp32 state, tf32 tensor-core operands with fp32 accumulation. d_k = 128,
// chunk 64, d_v tiled by 32.
//
// Operand precision: with bf16 operands the per-term rounding (2^-9) of the
// chunk products adds up to about 2-3% of rms(o) on the CKDA and KDA
// workloads (o is a difference of larger terms: Qhat S + M U), above the
// 1e-2 rms bound; tf32 operands (2^-11) keep it near 2e-3. Every MMA here is
// therefore kind::tf32, with operands rounded to tf32 when they are written.
//
// One CTA per (sequence, head, 32-column d_v tile), 256 threads. The CTA
// walks its sequence chunk by chunk; the state tile S (128 x 32) stays fp32 in
// the registers of warps 0-3 (thread = state row) and is mirrored in shared
// memory as an MMA operand.
//
// Per chunk (positions i, j in 0..63; chunk-WY derivation in
// ckda_fwd_simt.cu; Semidirect Fourier Delta Attention §2.2 and the affine
// chunk transfer of §1 contribution 4):
//
//   1. load q, k, alpha, beta, v-tile into shared memory
//   2. gate operands (bounded running products, exact for alpha <= 0):
//        Lk_I = k * F, Lq_I = q * F  (F = G_{i<-16I-1}, rows of sub-block I)
//        R^(I)_j = k_j * G_{16I-1<-j}  (j < 16 I)
//   3. Grams A (beta-scaled, strictly lower) and M (lower):
//        off-diagonal sub-blocks: one MMA  [Lk_1;Lq_1;..;Lq_3] x [R^(1);R^(2);R^(3)]^T
//        diagonal 16x16 sub-blocks: running products on CUDA cores
//   4. T = (I + A)^{-1} by blocked forward substitution (fp32), and M T;
//      [M T ; T] is written straight into tensor memory (A operand)
//   5. one MMA  [M T ; T] x [beta Khat | beta V]  gives  [M W | M Utilde ; W | Utilde]
//        (W = T diag(beta) Khat, Utilde = T diag(beta) V); Qtil = Qhat - M W is
//        formed in place in tensor memory: [Qtil ; W] is the next A operand
//   6. serial state step (two dependent MMAs, A operands in tensor memory):
//        D1 = [Qtil ; W] x S        -> O = scale (Qtil S + M Utilde)  (rows 0..63)
//                                   -> U = Utilde - W S              (rows 64..127)
//        D2 = Kbar^T x U            -> S <- diag(gamma_L) S + D2
//   Since O = Qhat S + M U = (Qhat - M W) S + M Utilde, the output needs no MMA
//   of its own on the serial chain.
#include <cuda_bf16.h>

#include "ckda.h"
#include "ckda_common.cuh"
#include "ckda_tc_ptx.cuh"

namespace ckda {
namespace {

using namespace tc;

constexpr int C = 64, DK = 128, DVT = 32, NT = 256;
constexpr int AL_S = 132;  // fp32 row stride of alpha / Qhat
constexpr int AS = 65;     // fp32 row stride of A, M, T

// shared-memory map (byte offsets from a 1024-aligned base); fp32 operands.
// MN-major tf32 operands use the 128B-swizzle / 32B-atom form (the only
// MN-major form tcgen05 accepts for 32-bit elements).
constexpr uint32_t OFF_GA = 0;        // 49152 Lk/Lq (96 rows x 128, K-major sw128)
                                      //       -> [beta Khat | beta V] (N160 x K64 MN-sw128b32)
constexpr uint32_t OFF_GB = 49152;    // 49152 R stack (96 rows x 128, K-major sw128)
                                      //       -> [M ; I] (128 x 64 K-major) + T operand
constexpr uint32_t OFF_A0 = OFF_GB;           // 32768 [M ; I], A of D0
constexpr uint32_t OFF_B0 = OFF_GB + 32768;   // 16384 T, B of D0 (K64 x N64 MN-sw128b32)
constexpr uint32_t OFF_SB = 98304;    // 16384 S, B of D1 (K128 x N32 MN-sw128b32)
constexpr uint32_t OFF_UB = 114688;   //  8192 U, B of D2 (K64 x N32 MN-sw128b32)
constexpr uint32_t OFF_Q = 122880;    // 16384 raw q bf16 [64][128] -> T fp32 [64][65]
constexpr uint32_t OFF_K = 139264;    // 16384 raw k bf16 [64][128]    (T spills in)
constexpr uint32_t OFF_XT = OFF_K + 4096;     //  3072 solve scratch (after raw k is dead)
constexpr uint32_t OFF_AL = 155648;   // 33792 alpha fp32 [64][132] -> Qhat fp32
constexpr uint32_t OFF_V = 189440;    //  4096 raw v bf16 [64][32]
constexpr uint32_t OFF_A = 193536;    // 16640 A fp32 [64][65]
constexpr uint32_t OFF_M = 210176;    // 16640 M fp32 [64][65]
constexpr uint32_t OFF_B = 226816;    //   256 beta
constexpr uint32_t OFF_GC = 227072;   //   512 gamma over the chunk
constexpr uint32_t OFF_BAR = 227584;  //    64 mbarriers [0..4] + TMEM address + flags
constexpr uint32_t SMEM_USED = 227648;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // alignment slack

// TMEM columns (512 allocated; one CTA per SM)
constexpr uint32_t TM_G = 0;      //  96 Gram accumulator
constexpr uint32_t TM_AD2 = 96;   //  64 Kbar^T (A of D2; lane = channel)
constexpr uint32_t TM_D5 = 160;   // 160 [M W | M Ut ; W | Ut] -> [Qtil ; W] (A of D1)
constexpr uint32_t TM_UT = 288;   //     (the M Ut / Ut columns of D5)
constexpr uint32_t TM_AD5 = 320;  //  64 [M T ; T] (A of D5)
constexpr uint32_t TM_D1 = 384;   //  32
constexpr uint32_t TM_D2 = 416;   //  32
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t ID_G = idesc_tf32(128, 96, 0, 0);
constexpr uint32_t ID_D0 = idesc_tf32(128, 64, 0, 1);
constexpr uint32_t ID_D5 = idesc_tf32(128, 160, 0, 1);
constexpr uint32_t ID_D1 = idesc_tf32(128, 32, 0, 1);
constexpr uint32_t ID_D2 = idesc_tf32(128, 32, 0, 1);

__device__ __forceinline__ float bf(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_f32(uint8_t *p, float x) {
  *reinterpret_cast<float *>(p) = to_tf32(x);
}
__device__ __forceinline__ void st4_f32(uint8_t *p, float a, float b, float c, float d) {
  *reinterpret_cast<float4 *>(p) = make_float4(to_tf32(a), to_tf32(b), to_tf32(c), to_tf32(d));
}

// Bounded wait of all threads on one mbarrier; false (and the abort flag set)
// if it timed out. Ends with every thread past a CTA barrier.
__device__ __forceinline__ bool wait_all(uint64_t *bar, uint32_t phase,
                                         volatile int *s_abort) {
  if (!mbar_wait(bar, phase)) *s_abort = 1;
  fence_after_sync();
  __syncthreads();
  return *s_abort == 0;
}

__global__ void __launch_bounds__(NT, 1)
fwd_tc_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
              const __nv_bfloat16 *__restrict__ v, const float *__restrict__ alpha,
              const float *__restrict__ beta, const float *__restrict__ s0,
              float *__restrict__ sfin, __nv_bfloat16 *__restrict__ o,
              const int32_t *__restrict__ cu, int T, int T_total, int H, int DV,
              float scale, unsigned int *err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  uint8_t *GA = sm + OFF_GA, *GB = sm + OFF_GB, *SB = sm + OFF_SB, *UB = sm + OFF_UB;
  const __nv_bfloat16 *sQr = reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_Q);
  const __nv_bfloat16 *sKr = reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_K);
  const __nv_bfloat16 *sVr = reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_V);
  float *sAl = reinterpret_cast<float *>(sm + OFF_AL);
  float *sA = reinterpret_cast<float *>(sm + OFF_A);
  float *sM = reinterpret_cast<float *>(sm + OFF_M);
  float *sT = reinterpret_cast<float *>(sm + OFF_Q);
  float *sXT = reinterpret_cast<float *>(sm + OFF_XT);
  float *sB = reinterpret_cast<float *>(sm + OFF_B);
  float *sGC = reinterpret_cast<float *>(sm + OFF_GC);
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_BAR);  // [0..4]
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 48);
  volatile int *s_abort = reinterpret_cast<volatile int *>(sm + OFF_BAR + 52);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int vt = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int c0 = vt * DVT;
  int bos, eos;
  seq_bounds(cu, n, T, T_total, err, bos, eos);
  const size_t st_base = ((size_t)n * H + h) * DK * DV;

  if (warp == 0) {
    tmem_alloc(s_tmem, TM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < 5; ++i) mbar_init(&bar[i], 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = *s_tmem;
  const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;

  // state rows in registers of warps 0..3 (thread = row r of the 128 x 32 tile)
  float S[DVT];
  if (warp < 4) {
    const int r = tid;
#pragma unroll
    for (int e = 0; e < DVT; e += 4) {
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (s0) x = *reinterpret_cast<const float4 *>(s0 + st_base + (size_t)r * DV + c0 + e);
      S[e] = x.x; S[e + 1] = x.y; S[e + 2] = x.z; S[e + 3] = x.w;
      st4_f32(SB + off_mn_sw128b32_f32(r, e, DK), x.x, x.y, x.z, x.w);
    }
  }
  float ut[DVT];  // rows of the D5 [M Ut ; Ut] columns (warps 0..3)
  uint32_t phase = 0;

  for (int t0 = bos; t0 < eos; t0 += C, phase ^= 1u) {
    const int L = min(C, eos - t0);
    // ---------------- 1. load the chunk: all global loads in flight at once
    {
      uint4 qv[4], kv[4], vv;
      float4 av[8];
      float bv = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {  // q, k: 64 rows x 16 pieces of 16 bytes
        const int idx = tid + u * NT, i = idx >> 4, ch = idx & 15;
        qv[u] = kv[u] = make_uint4(0, 0, 0, 0);
        if (i < L) {
          const size_t off = ((size_t)(t0 + i) * H + h) * DK + ch * 8;
          qv[u] = __ldg(reinterpret_cast<const uint4 *>(q + off));
          kv[u] = __ldg(reinterpret_cast<const uint4 *>(k + off));
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {  // alpha: 64 rows x 32 float4
        const int idx = tid + u * NT, i = idx >> 5, c4 = (idx & 31) * 4;
        av[u] = make_float4(1.f, 1.f, 1.f, 1.f);
        if (i < L)
          av[u] = __ldg(reinterpret_cast<const float4 *>(alpha + ((size_t)(t0 + i) * H + h) * DK + c4));
      }
      {  // v tile: 64 rows x 64 bytes
        const int i = tid >> 2, ch = tid & 3;
        vv = make_uint4(0, 0, 0, 0);
        if (i < L) vv = __ldg(reinterpret_cast<const uint4 *>(v + ((size_t)(t0 + i) * H + h) * DV + c0 + ch * 8));
      }
      if (tid < L) bv = __ldg(beta + (size_t)(t0 + tid) * H + h);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int idx = tid + u * NT, i = idx >> 4, ch = idx & 15;
        *reinterpret_cast<uint4 *>(sm + OFF_Q + i * 256 + ch * 16) = qv[u];
        *reinterpret_cast<uint4 *>(sm + OFF_K + i * 256 + ch * 16) = kv[u];
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int idx = tid + u * NT, i = idx >> 5, c4 = (idx & 31) * 4;
        *reinterpret_cast<float4 *>(sAl + i * AL_S + c4) = av[u];
      }
      *reinterpret_cast<uint4 *>(sm + OFF_V + (tid >> 2) * 64 + (tid & 3) * 16) = vv;
      if (tid < C) sB[tid] = bv;
    }
    if (tid < C && t0 + C + tid < eos) {  // next chunk's rows into L2
      const size_t th = (size_t)(t0 + C + tid) * H + h;
      prefetch_l2(q + th * DK, DK * 2);
      prefetch_l2(k + th * DK, DK * 2);
      prefetch_l2(alpha + th * DK, DK * 4);
      prefetch_l2(v + th * DV + c0, DVT * 2);
    }
    __syncthreads();

    // ---------------- 2. Gram operands (tf32, K-major 128B swizzle, 96 rows)
    // Each thread owns one channel; a sub-block's 16 rows are read into
    // registers before the running product walks them.
    if (tid < DK) {
      const int c = tid;
#pragma unroll 1
      for (int I = 1; I < 4; ++I) {
        float a[16], kk_[16], qq[16];
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) {
          const int i = 16 * I + ii;
          a[ii] = sAl[i * AL_S + c];
          kk_[ii] = bf(sKr + i * DK + c);
          qq[ii] = bf(sQr + i * DK + c);
        }
        float g = 1.f;
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) {
          g *= a[ii];
          st_f32(GA + off_k_sw128_f32((I - 1) * 32 + ii, c, 96), g * kk_[ii]);
          st_f32(GA + off_k_sw128_f32((I - 1) * 32 + 16 + ii, c, 96), g * qq[ii]);
        }
      }
    } else {
      // R^(I)_j = k_j G_{16I-1<-j}: one backward sweep over j = 47..0 carries
      // the three running products (each starts at its own 16I-1)
      const int c = tid - DK;
      float g1 = 1.f, g2 = 1.f, g3 = 1.f;
#pragma unroll 1
      for (int b = 2; b >= 0; --b) {
        float a[16], kk_[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int j = 16 * b + u;
          a[u] = sAl[j * AL_S + c];
          kk_[u] = bf(sKr + j * DK + c);
        }
#pragma unroll
        for (int u = 15; u >= 0; --u) {
          const int j = 16 * b + u;
          st_f32(GB + off_k_sw128_f32(48 + j, c, 96), g3 * kk_[u]);
          g3 *= a[u];
          if (b <= 1) {
            st_f32(GB + off_k_sw128_f32(16 + j, c, 96), g2 * kk_[u]);
            g2 *= a[u];
          }
          if (b == 0) {
            st_f32(GB + off_k_sw128_f32(j, c, 96), g1 * kk_[u]);
            g1 *= a[u];
          }
        }
      }
    }
    fence_async_smem();
    __syncthreads();

    // ---------------- 3. Grams: off-diagonal sub-blocks on tensor cores ...
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < DK / 8; ++kk)
        mma_tf32_ss(tm + TM_G, desc_k_sw128_f32(sb + OFF_GA, 96, kk),
                    desc_k_sw128_f32(sb + OFF_GB, 96, kk), ID_G, kk > 0);
      mma_commit(&bar[0]);
    }
    // ... diagonal 16x16 sub-blocks on CUDA cores, meanwhile: thread (column
    // j, lane sl) runs the gate product over channels 8 sl .. 8 sl + 7; the 16
    // lanes of a half-warp are then reduced with a reduce-scatter butterfly
    // that leaves entries 2 sl, 2 sl + 1 of [A column | M column] in lane sl.
    for (int I = 0; I < 4; ++I) {
      const int r0 = 16 * I;
      const int j = tid >> 4, sl = tid & 15, c8 = 8 * sl;
      float vv[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) vv[e] = 0.f;
      float kj[8], g[8];
      {
        const uint4 raw = *reinterpret_cast<const uint4 *>(sKr + (r0 + j) * DK + c8);
        const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(p2[e]);
          kj[2 * e] = f.x;
          kj[2 * e + 1] = f.y;
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) g[e] = 1.f;
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) {
        if (ii >= j) {
          const float4 a0 = *reinterpret_cast<const float4 *>(sAl + (r0 + ii) * AL_S + c8);
          const float4 a1 = *reinterpret_cast<const float4 *>(sAl + (r0 + ii) * AL_S + c8 + 4);
          const uint4 kr = *reinterpret_cast<const uint4 *>(sKr + (r0 + ii) * DK + c8);
          const uint4 qr = *reinterpret_cast<const uint4 *>(sQr + (r0 + ii) * DK + c8);
          const float al[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
          const __nv_bfloat162 *k2 = reinterpret_cast<const __nv_bfloat162 *>(&kr);
          const __nv_bfloat162 *q2 = reinterpret_cast<const __nv_bfloat162 *>(&qr);
          float sa = 0.f, sq = 0.f;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 kf = __bfloat1622float2(k2[e]), qf = __bfloat1622float2(q2[e]);
            if (ii > j) {
              g[2 * e] *= al[2 * e];
              g[2 * e + 1] *= al[2 * e + 1];
            }
            const float x0 = g[2 * e] * kj[2 * e], x1 = g[2 * e + 1] * kj[2 * e + 1];
            sa += kf.x * x0 + kf.y * x1;
            sq += qf.x * x0 + qf.y * x1;
          }
          vv[ii] += sa;
          vv[16 + ii] += sq;
        }
      }
      // reduce-scatter over the 16 lanes sharing column j
#pragma unroll
      for (int m = 8, n = 32; m > 0; m >>= 1, n >>= 1) {
        const bool up = (sl & m) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
          const float keep = up ? vv[n / 2 + i] : vv[i];
          const float send = up ? vv[i] : vv[n / 2 + i];
          vv[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int idx = 2 * sl + e, ii = idx & 15;
        if (idx >= 16) {
          if (ii >= j) sM[(r0 + ii) * AS + r0 + j] = vv[e];
        } else if (ii > j) {
          sA[(r0 + ii) * AS + r0 + j] = sB[r0 + ii] * vv[e];
        }
      }
    }
    if (!wait_all(&bar[0], phase, s_abort)) break;
    // off-diagonal blocks out of TMEM: warp quarter qw <-> sub-block row I = qw+1
    if (warp == 0 || warp == 1 || warp == 6) {
      const int qw = warp & 3, I = qw + 1, ii = lane & 15, isM = lane >> 4;
      const int i = 16 * I + ii, off = 8 * I * (I - 1), ncols = 16 * I;
      const uint32_t ta = tm + lane_base + TM_G + (uint32_t)off;
      for (int cb = 0; cb < ncols; cb += 16) {
        float x[16];
        tmem_ld16(ta + (uint32_t)cb, x);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          if (isM) sM[i * AS + cb + e] = x[e];
          else sA[i * AS + cb + e] = sB[i] * x[e];
        }
      }
    }
    fence_before_sync();
    __syncthreads();

    // ---------------- 2b. Kbar^T (into TMEM), beta Khat | beta V, Qhat, gamma
    if (tid < DK) {
      const int c = tid;  // = TMEM lane of this thread
      float kb0[32], kb1[32];
      float g = 1.f;
#pragma unroll
      for (int b = 3; b >= 0; --b) {  // sigma_j = prod_{s>j} alpha_s, j = 63..0
        float a[16], kk_[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          a[u] = sAl[(16 * b + u) * AL_S + c];
          kk_[u] = bf(sKr + (16 * b + u) * DK + c);
        }
#pragma unroll
        for (int u = 15; u >= 0; --u) {
          const int j = 16 * b + u;
          const float x = to_tf32(g * kk_[u]);
          if (j >= 32) kb1[j - 32] = x;
          else kb0[j] = x;
          g *= a[u];
        }
      }
      tmem_st32(tm + lane_base + TM_AD2, kb0);
      tmem_st32(tm + lane_base + TM_AD2 + 32, kb1);
      g = 1.f;
#pragma unroll 1
      for (int b = 0; b < 4; ++b) {       // gamma_i = prod_{s<=i} alpha_s
        float a[16], kk_[16], qq[16], bb[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int i = 16 * b + u;
          a[u] = sAl[i * AL_S + c];
          kk_[u] = bf(sKr + i * DK + c);
          qq[u] = bf(sQr + i * DK + c);
          bb[u] = sB[i];
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int i = 16 * b + u;
          g *= a[u];
          st_f32(GA + off_mn_sw128b32_f32(i, c, C), bb[u] * g * kk_[u]);
          sAl[i * AL_S + c] = g * qq[u];  // Qhat (fp32, in place)
        }
      }
      sGC[c] = g;
    } else {
      for (int task = tid - DK; task < C * 8; task += NT - DK) {  // beta V columns
        const int j = task >> 3, g4 = task & 7;
        const float b = sB[j];
        const __nv_bfloat16 *vr = sVr + j * DVT + 4 * g4;
        st4_f32(GA + off_mn_sw128b32_f32(j, DK + 4 * g4, C), b * bf(vr), b * bf(vr + 1),
                b * bf(vr + 2), b * bf(vr + 3));
      }
    }
    tmem_wait_st();
    fence_async_smem();
    fence_before_sync();
    __syncthreads();

    // ---------------- 4. T = (I + A)^{-1}; then [M T ; T] into TMEM
    if (tid < C) {
      const int b = tid >> 4, j = tid & 15, ob = b * 16;
      float t[16];
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) t[ii] = (ii == j) ? 1.f : 0.f;
#pragma unroll
      for (int ii = 1; ii < 16; ++ii) {
        if (ii > j) {
          float s = 0.f;
#pragma unroll
          for (int l = 0; l < ii; ++l)
            if (l >= j) s += sA[(ob + ii) * AS + ob + l] * t[l];
          t[ii] = -s;
        }
      }
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) sT[(ob + ii) * AS + ob + j] = t[ii];
    }
    __syncthreads();
    for (int d = 1; d < 4; ++d) {
      for (int idx = tid; idx < (4 - d) * 256; idx += NT) {
        const int p = idx >> 8, e = idx & 255, ii = e >> 4, jj = e & 15;
        const int I = d + p, J = p;
        float s = 0.f;
        for (int Lb = J; Lb < I; ++Lb)
#pragma unroll
          for (int l = 0; l < 16; ++l)
            s += sA[(I * 16 + ii) * AS + Lb * 16 + l] * sT[(Lb * 16 + l) * AS + J * 16 + jj];
        sXT[p * 256 + ii * 16 + jj] = s;
      }
      __syncthreads();
      for (int idx = tid; idx < (4 - d) * 256; idx += NT) {
        const int p = idx >> 8, e = idx & 255, ii = e >> 4, jj = e & 15;
        const int I = d + p, J = p;
        float s = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m)
          if (m <= ii) s += sT[(I * 16 + ii) * AS + I * 16 + m] * sXT[p * 256 + m * 16 + jj];
        sT[(I * 16 + ii) * AS + J * 16 + jj] = -s;
      }
      __syncthreads();
    }
    // [M T ; T] = [M ; I] x T on the tensor cores, straight into TMEM
    for (int task = tid; task < 128 * 16; task += NT) {  // A0 = [M ; I]
      const int row = task >> 4, k4 = (task & 15) * 4;
      float x[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int l = k4 + e;
        x[e] = (row < C) ? ((l <= row) ? sM[row * AS + l] : 0.f) : ((l == row - C) ? 1.f : 0.f);
      }
      st4_f32(sm + OFF_A0 + off_k_sw128_f32(row, k4, 128), x[0], x[1], x[2], x[3]);
    }
    for (int task = tid; task < C * 16; task += NT) {  // B0 = T (row l, columns j)
      const int l = task >> 4, j4 = (task & 15) * 4;
      float x[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) x[e] = (j4 + e <= l) ? sT[l * AS + j4 + e] : 0.f;
      st4_f32(sm + OFF_B0 + off_mn_sw128b32_f32(l, j4, C), x[0], x[1], x[2], x[3]);
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < C / 8; ++kk)
        mma_tf32_ss(tm + TM_AD5, desc_k_sw128_f32(sb + OFF_A0, 128, kk),
                    desc_mn_sw128b32_f32(sb + OFF_B0, C, kk), ID_D0, kk > 0);
      mma_commit(&bar[4]);
    }
    if (!wait_all(&bar[4], phase, s_abort)) break;
    if ((warp & 3) < 2) {  // rows of M T: round the fp32 accumulator to tf32
      const uint32_t ta = tm + lane_base + TM_AD5 + (uint32_t)(32 * (warp >> 2));
      float x[32];
      tmem_ld32(ta, x);
#pragma unroll
      for (int e = 0; e < 32; ++e) x[e] = to_tf32(x[e]);
      tmem_st32(ta, x);
    }
    tmem_wait_st();
    fence_before_sync();
    __syncthreads();

    // ---------------- 5. [M T ; T] x [beta Khat | beta V]
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < C / 8; ++kk)
        mma_tf32_ts(tm + TM_D5, tm + TM_AD5 + (uint32_t)(8 * kk),
                    desc_mn_sw128b32_f32(sb + OFF_GA, C, kk), ID_D5, kk > 0);
      mma_commit(&bar[1]);
    }
    if (!wait_all(&bar[1], phase, s_abort)) break;
    {  // [M W ; W] -> [Qtil ; W] in place (tf32); keep [M Ut ; Ut] rows
      const int qw = warp & 3, hf = warp >> 2, Lr = 32 * qw + lane;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int cb = 64 * hf + 32 * half;
        float x[32];
        tmem_ld32(tm + lane_base + TM_D5 + (uint32_t)cb, x);
        if (Lr < C) {
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] = to_tf32(sAl[Lr * AL_S + cb + e] - x[e]);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] = to_tf32(x[e]);
        }
        tmem_st32(tm + lane_base + TM_D5 + (uint32_t)cb, x);
      }
      if (hf == 0) tmem_ld32(tm + lane_base + TM_UT, ut);
    }
    tmem_wait_st();
    fence_before_sync();
    __syncthreads();

    // ---------------- 6. serial state step
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < DK / 8; ++kk)
        mma_tf32_ts(tm + TM_D1, tm + TM_D5 + (uint32_t)(8 * kk),
                    desc_mn_sw128b32_f32(sb + OFF_SB, DK, kk), ID_D1, kk > 0);
      mma_commit(&bar[2]);
    }
    if (!wait_all(&bar[2], phase, s_abort)) break;
    if (warp < 4) {
      float d1[32];
      tmem_ld32(tm + lane_base + TM_D1, d1);
      if (warp < 2) {  // output rows
        const int i = tid;
        if (i < L) {
          __nv_bfloat16 *dst = o + ((size_t)(t0 + i) * H + h) * DV + c0;
#pragma unroll
          for (int g8 = 0; g8 < 4; ++g8) {
            float y[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] = scale * (d1[8 * g8 + e] + ut[8 * g8 + e]);
            *reinterpret_cast<uint4 *>(dst + 8 * g8) = pack8_bf16(y);
          }
        }
      } else {  // U = Utilde - W S
        const int j = tid - C;
#pragma unroll
        for (int e = 0; e < DVT; e += 4)
          st4_f32(UB + off_mn_sw128b32_f32(j, e, C), ut[e] - d1[e], ut[e + 1] - d1[e + 1],
                  ut[e + 2] - d1[e + 2], ut[e + 3] - d1[e + 3]);
      }
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < C / 8; ++kk)
        mma_tf32_ts(tm + TM_D2, tm + TM_AD2 + (uint32_t)(8 * kk),
                    desc_mn_sw128b32_f32(sb + OFF_UB, C, kk), ID_D2, kk > 0);
      mma_commit(&bar[3]);
    }
    if (!wait_all(&bar[3], phase, s_abort)) break;
    if (warp < 4) {
      const int r = tid;
      float d2[32];
      tmem_ld32(tm + lane_base + TM_D2, d2);
      const float gc = sGC[r];
#pragma unroll
      for (int e = 0; e < DVT; ++e) S[e] = gc * S[e] + d2[e];
#pragma unroll
      for (int e = 0; e < DVT; e += 4)
        st4_f32(SB + off_mn_sw128b32_f32(r, e, DK), S[e], S[e + 1], S[e + 2], S[e + 3]);
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
  }

  if (*s_abort) {
    if (tid == 0) flag_error(err, kErrMbarTimeout);
    // give in-flight MMAs a bounded chance to drain before TMEM is released
    for (int i = 0; i < 5; ++i) (void)mbar_wait(&bar[i], phase, 100000000LL);
  } else if (sfin && warp < 4) {
    const int r = tid;
#pragma unroll
    for (int e = 0; e < DVT; e += 4)
      *reinterpret_cast<float4 *>(sfin + st_base + (size_t)r * DV + c0 + e) =
          make_float4(S[e], S[e + 1], S[e + 2], S[e + 3]);
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    fence_after_sync();
    tmem_dealloc(tm, TM_COLS);
  }
}

}  // namespace

bool fwd_tc_supported(int dk, int dv, int chunk, ckda_dtype dt) {
  return dt == CKDA_BF16 && dk == 128 && chunk == 64 && (dv % DVT) == 0;
}

cudaError_t launch_fwd_tc(int dv, const void *q, const void *k, const void *v,
                          const float *alpha, const float *beta,
                          const float *s0, float *sf, void *o,
                          const int32_t *cu, int N, int T, int T_total, int H,
                          float scale, unsigned int *err, cudaStream_t st) {
  if (dv % DVT != 0) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(
      fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const dim3 grid(dv / DVT, H, N);
  fwd_tc_kernel<<<grid, NT, SMEM_BYTES, st>>>(
      (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v,
      alpha, beta, s0, sf, (__nv_bfloat16 *)o, cu, T, T_total, H, dv, scale, err);
  return cudaGetLastError();
}

}  // namespace ckda
