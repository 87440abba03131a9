// Chunkwise CKDA forward with tcgen05 tensor cores (sm_100a): bf16 I/O,
// fp32 state, tf32 tensor-core operands with fp32 accumulation. d_k = 128,
// chunk 64, d_v in {32, 64, 128}.
//
// Two kernels, split where the work changes character:
//
//  * ckda_chunk_prep_kernel: one CTA per (chunk, head), all chunks of all
//    sequences in parallel. It builds everything about a chunk that does not
//    depend on the state entering it (the chunk-WY / UT-transform factors of
//    the product of diagonal-plus-rank-one transitions, Semidirect Fourier
//    Delta Attention §2.2, and the affine chunk transfer's write summary, §1
//    contribution 4), and stores the serial step's operands in a workspace:
//        [Qtil ; W]   = [Qhat - M W ; T diag(beta) Khat]       128 x d_k
//        Kbar^T                                                d_k x 64
//        [M Ut ; Ut]  = [M T ; T] diag(beta) V                 128 x d_v
//        gamma        = prod of the chunk's gates, per channel
//  * ckda_chunk_scan_kernel: one CTA per (sequence, head, 32-column d_v tile)
//    walks the chunks in order and only carries the state:
//        D1 = [Qtil ; W] S  ->  O = scale (Qtil S + M Ut)   (rows 0..63)
//                           ->  U = Ut - W S                (rows 64..127)
//        D2 = Kbar^T U      ->  S <- diag(gamma) S + D2
//    with the next chunk's operands bulk-copied into a second buffer while
//    the current one is used.
// O = Qhat S + M U with U = Ut - W S, so O = (Qhat - M W) S + M Ut: the output
// costs no MMA of its own on the serial chain.
//
// Chunk factors (positions i, j in 0..63; G_{i<-j} = prod_{s=j+1..i} alpha_s;
// gamma_i = G_{i<-0}; sigma_j = G_{63<-j}; see ckda_fwd_simt.cu):
//   A_ij = beta_i k_i^T G_{i<-j} k_j (j<i), M_ij = q_i^T G_{i<-j} k_j (j<=i),
//   T = (I + A)^{-1}, Khat_i = gamma_i k_i, Qhat_i = gamma_i q_i, Kbar_j = sigma_j k_j.
// Gate factors are bounded running products (exact for negative and zero
// gates; no logarithm, no division). Off-diagonal 16x16 sub-blocks of A and
// M factor through the sub-block boundary and run as one MMA; the diagonal
// sub-blocks use per-pair running products on CUDA cores.
//
// Operand precision: with bf16 operands the rounding of the chunk products
// adds up to about 2-3% of rms(o) on the CKDA and KDA workloads, above the
// 1e-2 rms bound; tf32 operands keep it near 2e-3. Every MMA is kind::tf32,
// operands rounded to tf32 when they are written.
#include <cuda_bf16.h>

#include "ckda.h"
#include "ckda_common.cuh"
#include "ckda_tc_ptx.cuh"

namespace ckda {
namespace {

using namespace tc;

constexpr int C = 64, DK = 128, DVT = 32;
constexpr int AL_S = 132;  // fp32 row stride of alpha / Qhat
constexpr int AS = 65;     // fp32 row stride of A, M, T

// ---------------------------------------------------------------- workspace
// One block per (chunk slot, head); chunk c of sequence n sits in slot
// floor(cu[n] / 64) + n + c, which never collides and is below
// floor(T_total / 64) + N.
constexpr uint32_t WS_A1 = 0;       // [Qtil ; W]: 128 x 128 tf32, K-major sw128 image
constexpr uint32_t WS_A2 = 65536;   // Kbar^T:     128 x 64 tf32, K-major sw128 image
constexpr uint32_t WS_OU = 98304;   // [M Ut ; Ut]: 128 rows x d_v fp32, row-major
__host__ __device__ constexpr uint32_t ws_gamma_off(int dv) { return WS_OU + 128u * dv * 4u; }
__host__ __device__ constexpr uint32_t ws_block_bytes(int dv) {
  return ws_gamma_off(dv) + 1024u;  // gamma: 128 fp32, block kept 1 KB aligned
}

// first slot of sequence n
__device__ __forceinline__ int slot_base(const int32_t *cu, int n, int T) {
  const int b = cu ? __ldg(cu + n) : n * T;
  return b / C + n;
}

// ---------------------------------------------------------------- prep kernel
// shared-memory map (byte offsets from a 1024-aligned base); fp32 operands.
// MN-major tf32 operands use the 128B-swizzle / 32B-atom form (the only
// MN-major form tcgen05 accepts for 32-bit elements).
constexpr int NTP = 256;
constexpr uint32_t P_GA = 0;          // 49152 Lk/Lq (96 rows x 128, K-major)
                                      //   -> [beta Khat | beta V] (K64 x N(128+dv) MN) 65536
constexpr uint32_t P_GB = 49152;      // 49152 R stack (96 rows x 128, K-major)
constexpr uint32_t P_A0 = 65536;      // 32768 [M ; I] (128 x 64 K-major), after the Grams
constexpr uint32_t P_B0 = 98304;      // 16384 T (K64 x N64 MN)
constexpr uint32_t P_Q = 114688;      // 16384 raw q bf16 [64][128] -> T fp32 [64][65]
constexpr uint32_t P_K = 131072;      // 16384 raw k bf16 [64][128]    (T spills in)
constexpr uint32_t P_XT = P_K + 4096; //  3072 solve scratch (after raw k is dead)
constexpr uint32_t P_AL = 147456;     // 33792 alpha fp32 [64][132] -> Qhat fp32
constexpr uint32_t P_A = 181248;      // 16640 A fp32 [64][65]
constexpr uint32_t P_M = 197888;      // 16640 M fp32 [64][65]
constexpr uint32_t P_B = 214528;      //   256 beta
constexpr uint32_t P_BAR = 214784;    //    64 mbarriers [0..2] + TMEM address + flag
constexpr uint32_t P_SMEM = 214848 + 1024;

// TMEM columns of the prep kernel (512 allocated; one CTA per SM)
constexpr uint32_t TP_G = 0;      //  96 Gram accumulator
constexpr uint32_t TP_AD5 = 96;   //  64 [M T ; T] (A of D5)
constexpr uint32_t TP_D5 = 160;   // 256 [M W | M Ut ; W | Ut]
constexpr uint32_t TP_COLS = 512;

constexpr uint32_t ID_G = idesc_tf32(128, 96, 0, 0);
constexpr uint32_t ID_D0 = idesc_tf32(128, 64, 0, 1);

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

__global__ void __launch_bounds__(NTP, 1)
ckda_chunk_prep_kernel(const __nv_bfloat16 *__restrict__ q,
                       const __nv_bfloat16 *__restrict__ k,
                       const __nv_bfloat16 *__restrict__ v,
                       const float *__restrict__ alpha,
                       const float *__restrict__ beta,
                       const int32_t *__restrict__ cu, int N, int T, int T_total,
                       int H, int DV, uint8_t *__restrict__ ws,
                       unsigned int *err) {
  // ---- which (sequence, chunk) this slot holds; empty slots leave at once
  const int slot = blockIdx.x, h = blockIdx.y;
  int n = 0;
  {
    int lo = 0, hi = N - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (slot_base(cu, mid, T) <= slot) lo = mid;
      else hi = mid - 1;
    }
    n = lo;
  }
  int bos, eos;
  seq_bounds(cu, n, T, T_total, err, bos, eos);
  const int cidx = slot - slot_base(cu, n, T);
  const int t0 = bos + C * cidx;
  if (cidx < 0 || t0 >= eos) return;
  const int L = min(C, eos - t0);

  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  uint8_t *GA = sm + P_GA, *GB = sm + P_GB;
  const __nv_bfloat16 *sQr = reinterpret_cast<const __nv_bfloat16 *>(sm + P_Q);
  const __nv_bfloat16 *sKr = reinterpret_cast<const __nv_bfloat16 *>(sm + P_K);
  float *sAl = reinterpret_cast<float *>(sm + P_AL);
  float *sA = reinterpret_cast<float *>(sm + P_A);
  float *sM = reinterpret_cast<float *>(sm + P_M);
  float *sT = reinterpret_cast<float *>(sm + P_Q);
  float *sXT = reinterpret_cast<float *>(sm + P_XT);
  float *sB = reinterpret_cast<float *>(sm + P_B);
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + P_BAR);  // [0..2]
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + P_BAR + 32);
  volatile int *s_abort = reinterpret_cast<volatile int *>(sm + P_BAR + 36);
  uint8_t *wsb = ws + ((size_t)slot * H + h) * ws_block_bytes(DV);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (warp == 0) {
    tmem_alloc(s_tmem, TP_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < 3; ++i) mbar_init(&bar[i], 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = *s_tmem;
  const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;

  do {  // one pass; `break` leaves on a timed-out wait
    // ---------------- 1. load the chunk: all global loads in flight at once
    {
      uint4 qv[4], kv[4];
      float4 av[8];
      float bv = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {  // q, k: 64 rows x 16 pieces of 16 bytes
        const int idx = tid + u * NTP, i = idx >> 4, ch = idx & 15;
        qv[u] = kv[u] = make_uint4(0, 0, 0, 0);
        if (i < L) {
          const size_t off = ((size_t)(t0 + i) * H + h) * DK + ch * 8;
          qv[u] = __ldg(reinterpret_cast<const uint4 *>(q + off));
          kv[u] = __ldg(reinterpret_cast<const uint4 *>(k + off));
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {  // alpha: 64 rows x 32 float4
        const int idx = tid + u * NTP, i = idx >> 5, c4 = (idx & 31) * 4;
        av[u] = make_float4(1.f, 1.f, 1.f, 1.f);
        if (i < L)
          av[u] = __ldg(reinterpret_cast<const float4 *>(alpha + ((size_t)(t0 + i) * H + h) * DK + c4));
      }
      if (tid < L) bv = __ldg(beta + (size_t)(t0 + tid) * H + h);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int idx = tid + u * NTP, i = idx >> 4, ch = idx & 15;
        *reinterpret_cast<uint4 *>(sm + P_Q + i * 256 + ch * 16) = qv[u];
        *reinterpret_cast<uint4 *>(sm + P_K + i * 256 + ch * 16) = kv[u];
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int idx = tid + u * NTP, i = idx >> 5, c4 = (idx & 31) * 4;
        *reinterpret_cast<float4 *>(sAl + i * AL_S + c4) = av[u];
      }
      if (tid < C) sB[tid] = bv;
    }
    __syncthreads();

    // ---------------- 2. Gram operands (tf32, K-major 128B swizzle, 96 rows)
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
        mma_tf32_ss(tm + TP_G, desc_k_sw128_f32(sb + P_GA, 96, kk),
                    desc_k_sw128_f32(sb + P_GB, 96, kk), ID_G, kk > 0);
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
#pragma unroll
      for (int m = 8, nn = 32; m > 0; m >>= 1, nn >>= 1) {
        const bool up = (sl & m) != 0;
#pragma unroll
        for (int i = 0; i < nn / 2; ++i) {
          const float keep = up ? vv[nn / 2 + i] : vv[i];
          const float send = up ? vv[i] : vv[nn / 2 + i];
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
    if (!wait_all(&bar[0], 0, s_abort)) break;
    // off-diagonal blocks out of TMEM: warp quarter qw <-> sub-block row I = qw+1
    if (warp == 0 || warp == 1 || warp == 6) {
      const int qw = warp & 3, I = qw + 1, ii = lane & 15, isM = lane >> 4;
      const int i = 16 * I + ii, off = 8 * I * (I - 1), ncols = 16 * I;
      const uint32_t ta = tm + lane_base + TP_G + (uint32_t)off;
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

    // ---------------- 4. Kbar^T (to the workspace), beta Khat | beta V, Qhat, gamma
    if (tid < DK) {
      const int c = tid;
      float kb[C];
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
          kb[16 * b + u] = to_tf32(g * kk_[u]);
          g *= a[u];
        }
      }
#pragma unroll
      for (int j = 0; j < C; j += 4)  // row c of Kbar^T (K-major sw128 image)
        *reinterpret_cast<float4 *>(wsb + WS_A2 + off_k_sw128_f32(c, j, DK)) =
            make_float4(kb[j], kb[j + 1], kb[j + 2], kb[j + 3]);
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
      reinterpret_cast<float *>(wsb + ws_gamma_off(DV))[c] = g;
    } else {
      // beta V columns 128 .. 128+DV of the D5 B operand, straight from global
      const int nq = DV / 4;  // 4-column groups per row
      for (int task0 = tid - DK; task0 < C * nq; task0 += 16 * (NTP - DK)) {
        uint2 raw[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int task = task0 + u * (NTP - DK), j = task / nq, g4 = task % nq;
          raw[u] = make_uint2(0, 0);
          if (task < C * nq && j < L)
            raw[u] = __ldg(reinterpret_cast<const uint2 *>(v + ((size_t)(t0 + j) * H + h) * DV + 4 * g4));
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int task = task0 + u * (NTP - DK), j = task / nq, g4 = task % nq;
          if (task < C * nq) {
            const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&raw[u]);
            const float2 x = __bfloat1622float2(p2[0]), y = __bfloat1622float2(p2[1]);
            const float b = sB[j];
            st4_f32(GA + off_mn_sw128b32_f32(j, DK + 4 * g4, C), b * x.x, b * x.y, b * y.x, b * y.y);
          }
        }
      }
    }
    __syncthreads();

    // ---------------- 5. T = (I + A)^{-1} by blocked forward substitution
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
      for (int idx = tid; idx < (4 - d) * 256; idx += NTP) {
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
      for (int idx = tid; idx < (4 - d) * 256; idx += NTP) {
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

    // ---------------- 6. [M T ; T] = [M ; I] x T on the tensor cores, into TMEM
    for (int task = tid; task < 128 * 16; task += NTP) {  // A0 = [M ; I]
      const int row = task >> 4, k4 = (task & 15) * 4;
      float x[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int l = k4 + e;
        x[e] = (row < C) ? ((l <= row) ? sM[row * AS + l] : 0.f) : ((l == row - C) ? 1.f : 0.f);
      }
      st4_f32(sm + P_A0 + off_k_sw128_f32(row, k4, 128), x[0], x[1], x[2], x[3]);
    }
    for (int task = tid; task < C * 16; task += NTP) {  // B0 = T (row l, columns j)
      const int l = task >> 4, j4 = (task & 15) * 4;
      float x[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) x[e] = (j4 + e <= l) ? sT[l * AS + j4 + e] : 0.f;
      st4_f32(sm + P_B0 + off_mn_sw128b32_f32(l, j4, C), x[0], x[1], x[2], x[3]);
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < C / 8; ++kk)
        mma_tf32_ss(tm + TP_AD5, desc_k_sw128_f32(sb + P_A0, 128, kk),
                    desc_mn_sw128b32_f32(sb + P_B0, C, kk), ID_D0, kk > 0);
      mma_commit(&bar[1]);
    }
    if (!wait_all(&bar[1], 0, s_abort)) break;
    if ((warp & 3) < 2) {  // rows of M T: round the fp32 accumulator to tf32
      const uint32_t ta = tm + lane_base + TP_AD5 + (uint32_t)(32 * (warp >> 2));
      float x[32];
      tmem_ld32(ta, x);
#pragma unroll
      for (int e = 0; e < 32; ++e) x[e] = to_tf32(x[e]);
      tmem_st32(ta, x);
    }
    tmem_wait_st();
    fence_before_sync();
    __syncthreads();

    // ---------------- 7. [M T ; T] x [beta Khat | beta V] -> workspace
    if (tid == 0) {
      fence_after_sync();
      const uint32_t id5 = idesc_tf32(128, DK + DV, 0, 1);
#pragma unroll
      for (int kk = 0; kk < C / 8; ++kk)
        mma_tf32_ts(tm + TP_D5, tm + TP_AD5 + (uint32_t)(8 * kk),
                    desc_mn_sw128b32_f32(sb + P_GA, C, kk), id5, kk > 0);
      mma_commit(&bar[2]);
    }
    if (!wait_all(&bar[2], 0, s_abort)) break;
    {
      const int qw = warp & 3, hw = warp >> 2, row = 32 * qw + lane;
      if (hw == 0) {  // [Qtil ; W] rows, tf32, K-major sw128 image
        for (int cb = 0; cb < DK; cb += 32) {
          float x[32];
          tmem_ld32(tm + lane_base + TP_D5 + (uint32_t)cb, x);
          if (row < C) {
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = sAl[row * AL_S + cb + e] - x[e];
          }
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4 *>(wsb + WS_A1 + off_k_sw128_f32(row, cb + e, DK)) =
                make_float4(to_tf32(x[e]), to_tf32(x[e + 1]), to_tf32(x[e + 2]), to_tf32(x[e + 3]));
        }
      } else {  // [M Ut ; Ut] rows, fp32 row-major
        float *dst = reinterpret_cast<float *>(wsb + WS_OU) + (size_t)row * DV;
        for (int cb = 0; cb < DV; cb += 32) {
          float x[32];
          tmem_ld32(tm + lane_base + TP_D5 + (uint32_t)(DK + cb), x);
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4 *>(dst + cb + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
        }
      }
    }
  } while (0);

  if (*s_abort && tid == 0) flag_error(err, kErrMbarTimeout);
  fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    fence_after_sync();
    tmem_dealloc(tm, TP_COLS);
  }
}

// ---------------------------------------------------------------- scan kernel
constexpr int NTS = 128;
constexpr uint32_t S_A1 = 0;          // 2 x 65536 [Qtil ; W] buffers
constexpr uint32_t S_A2 = 131072;     // 2 x 32768 Kbar^T buffers
constexpr uint32_t S_S = 196608;      // 16384 S, B of D1 (K128 x N32 MN)
constexpr uint32_t S_U = 212992;      //  8192 U, B of D2 (K64 x N32 MN)
constexpr uint32_t S_BAR = 221184;    //    64 mbarriers [0..2] + TMEM address + flag
constexpr uint32_t S_SMEM = 221248 + 1024;
constexpr uint32_t TS_D1 = 0, TS_D2 = 32, TS_COLS = 64;
constexpr uint32_t ID_D1 = idesc_tf32(128, 32, 0, 1);
constexpr uint32_t ID_D2 = idesc_tf32(128, 32, 0, 1);
constexpr uint32_t LOAD_BYTES = 65536 + 32768;

__global__ void __launch_bounds__(NTS, 1)
ckda_chunk_scan_kernel(const float *__restrict__ s0, float *__restrict__ sfin,
                       __nv_bfloat16 *__restrict__ o, const int32_t *__restrict__ cu,
                       int T, int T_total, int H, int DV, float scale,
                       const uint8_t *__restrict__ ws, unsigned int *err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + S_BAR);  // [0..1] loads, [2] MMAs
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + S_BAR + 32);
  volatile int *s_abort = reinterpret_cast<volatile int *>(sm + S_BAR + 36);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int vt = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int c0 = vt * DVT;
  int bos, eos;
  seq_bounds(cu, n, T, T_total, err, bos, eos);
  const int nch = (eos - bos + C - 1) / C;
  const int base = slot_base(cu, n, T);
  const size_t st_base = ((size_t)n * H + h) * DK * DV;
  const uint32_t wsz = ws_block_bytes(DV);

  if (warp == 0) {
    tmem_alloc(s_tmem, TS_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < 3; ++i) mbar_init(&bar[i], 1);
    *s_abort = 0;
    fence_mbar_init();
    if (nch > 0) {  // chunk 0 into buffer 0
      const uint8_t *blk = ws + ((size_t)base * H + h) * wsz;
      mbar_arrive_expect_tx(&bar[0], LOAD_BYTES);
      bulk_g2s(sm + S_A1, blk + WS_A1, 65536, &bar[0]);
      bulk_g2s(sm + S_A2, blk + WS_A2, 32768, &bar[0]);
    }
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = *s_tmem;
  const uint32_t lane_base = (uint32_t)(32 * warp) << 16;

  // state row r = tid of the 128 x 32 tile, fp32 in registers
  float S[DVT];
  {
    const int r = tid;
#pragma unroll
    for (int e = 0; e < DVT; e += 4) {
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (s0) x = *reinterpret_cast<const float4 *>(s0 + st_base + (size_t)r * DV + c0 + e);
      S[e] = x.x; S[e + 1] = x.y; S[e + 2] = x.z; S[e + 3] = x.w;
      st4_f32(sm + S_S + off_mn_sw128b32_f32(r, e, DK), x.x, x.y, x.z, x.w);
    }
  }
  fence_async_smem();
  __syncthreads();

  // this thread's row of [M Ut ; Ut] (d_v tile) and gamma of its state row,
  // read one chunk ahead so the loads overlap the previous chunk's MMAs
  float ou_next[DVT], gc_next = 0.f;
  auto load_rows = [&](int c) {
    const uint8_t *blk = ws + ((size_t)(base + c) * H + h) * wsz;
    const float *src = reinterpret_cast<const float *>(blk + WS_OU) + (size_t)tid * DV + c0;
#pragma unroll
    for (int e = 0; e < DVT; e += 4) {
      const float4 x = __ldg(reinterpret_cast<const float4 *>(src + e));
      ou_next[e] = x.x; ou_next[e + 1] = x.y; ou_next[e + 2] = x.z; ou_next[e + 3] = x.w;
    }
    gc_next = __ldg(reinterpret_cast<const float *>(blk + ws_gamma_off(DV)) + tid);
  };
  if (nch > 0) load_rows(0);

  for (int c = 0; c < nch; ++c) {
    const int buf = c & 1;
    const int t0 = bos + C * c, L = min(C, eos - t0);
    // next chunk's operands into the other buffer (free: chunk c-1 is done)
    if (tid == 0 && c + 1 < nch) {
      const uint8_t *nb = ws + ((size_t)(base + c + 1) * H + h) * wsz;
      mbar_arrive_expect_tx(&bar[buf ^ 1], LOAD_BYTES);
      bulk_g2s(sm + S_A1 + (buf ^ 1) * 65536, nb + WS_A1, 65536, &bar[buf ^ 1]);
      bulk_g2s(sm + S_A2 + (buf ^ 1) * 32768, nb + WS_A2, 32768, &bar[buf ^ 1]);
    }
    float ou[DVT];
#pragma unroll
    for (int e = 0; e < DVT; ++e) ou[e] = ou_next[e];
    const float gc = gc_next;
    if (c + 1 < nch) load_rows(c + 1);
    if (!mbar_wait(&bar[buf], (uint32_t)(c >> 1) & 1u)) *s_abort = 1;
    __syncthreads();
    if (*s_abort) break;

    // D1 = [Qtil ; W] x S
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < DK / 8; ++kk)
        mma_tf32_ss(tm + TS_D1, desc_k_sw128_f32(sb + S_A1 + buf * 65536, 128, kk),
                    desc_mn_sw128b32_f32(sb + S_S, DK, kk), ID_D1, kk > 0);
      mma_commit(&bar[2]);
    }
    if (!wait_all(&bar[2], 0, s_abort)) break;
    {
      float d1[32];
      tmem_ld32(tm + lane_base + TS_D1, d1);
      if (tid < C) {  // output rows
        const int i = tid;
        if (i < L) {
          __nv_bfloat16 *dst = o + ((size_t)(t0 + i) * H + h) * DV + c0;
#pragma unroll
          for (int g8 = 0; g8 < 4; ++g8) {
            float y[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] = scale * (d1[8 * g8 + e] + ou[8 * g8 + e]);
            *reinterpret_cast<uint4 *>(dst + 8 * g8) = pack8_bf16(y);
          }
        }
      } else {  // U = Ut - W S
        const int j = tid - C;
#pragma unroll
        for (int e = 0; e < DVT; e += 4)
          st4_f32(sm + S_U + off_mn_sw128b32_f32(j, e, C), ou[e] - d1[e], ou[e + 1] - d1[e + 1],
                  ou[e + 2] - d1[e + 2], ou[e + 3] - d1[e + 3]);
      }
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    // D2 = Kbar^T x U
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < C / 8; ++kk)
        mma_tf32_ss(tm + TS_D2, desc_k_sw128_f32(sb + S_A2 + buf * 32768, 128, kk),
                    desc_mn_sw128b32_f32(sb + S_U, C, kk), ID_D2, kk > 0);
      mma_commit(&bar[2]);
    }
    if (!wait_all(&bar[2], 1, s_abort)) break;
    {
      float d2[32];
      tmem_ld32(tm + lane_base + TS_D2, d2);
#pragma unroll
      for (int e = 0; e < DVT; ++e) S[e] = gc * S[e] + d2[e];
#pragma unroll
      for (int e = 0; e < DVT; e += 4)
        st4_f32(sm + S_S + off_mn_sw128b32_f32(tid, e, DK), S[e], S[e + 1], S[e + 2], S[e + 3]);
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
  }

  if (*s_abort) {
    if (tid == 0) flag_error(err, kErrMbarTimeout);
    // let in-flight copies and MMAs drain (bounded) before shared memory and
    // tensor memory are released
    for (int i = 0; i < 3; ++i) {
      (void)mbar_wait(&bar[i], 0, 100000000LL);
      (void)mbar_wait(&bar[i], 1, 100000000LL);
    }
  } else if (sfin) {
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
    tmem_dealloc(tm, TS_COLS);
  }
}

}  // namespace

bool fwd_tc_supported(int dk, int dv, int chunk, ckda_dtype dt) {
  return dt == CKDA_BF16 && dk == 128 && chunk == 64 &&
         (dv == 32 || dv == 64 || dv == 128);
}

size_t fwd_tc_workspace_bytes(int N, int T_total, int H, int dv) {
  const size_t slots = (size_t)T_total / C + (size_t)N;
  return slots * (size_t)H * ws_block_bytes(dv);
}

cudaError_t launch_fwd_tc(int dv, const void *q, const void *k, const void *v,
                          const float *alpha, const float *beta,
                          const float *s0, float *sf, void *o,
                          const int32_t *cu, int N, int T, int T_total, int H,
                          float scale, void *ws, unsigned int *err,
                          cudaStream_t st) {
  if (!fwd_tc_supported(DK, dv, C, CKDA_BF16)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(
      ckda_chunk_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P_SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(ckda_chunk_scan_kernel,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S_SMEM);
  if (e != cudaSuccess) return e;
  const int slots = T_total / C + N;
  if (slots > 0 && T_total > 0) {
    ckda_chunk_prep_kernel<<<dim3(slots, H), NTP, P_SMEM, st>>>(
        (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v,
        alpha, beta, cu, N, T, T_total, H, dv, (uint8_t *)ws, err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  ckda_chunk_scan_kernel<<<dim3(dv / DVT, H, N), NTS, S_SMEM, st>>>(
      s0, sf, (__nv_bfloat16 *)o, cu, T, T_total, H, dv, scale, (const uint8_t *)ws, err);
  return cudaGetLastError();
}

}  // namespace ckda
