// Chunkwise CKDA forward on CUDA cores, fp32 throughout (the fp32 check mode,
// and the path for shapes the tensor-core kernel does not take).
//
// One CTA per (sequence, head, d_v tile of DVT columns); it walks the
// sequence chunk by chunk with the state tile resident in shared memory.
// Columns of the state evolve independently (each column is its own
// recurrence driven by the same k, q, alpha, beta), so d_v tiles need no
// communication.
//
// Per chunk of L <= C tokens with entry state S (positions i, j in 0..L-1;
// G_{i<-j} = prod_{s=j+1..i} diag(alpha_s); gamma_i = prod_{s<=i} alpha_s;
// sigma_j = prod_{s>j} alpha_s), the chunk-WY / UT-transform form of the
// product of diagonal-plus-rank-one transitions (Semidirect Fourier Delta
// Attention §2.2, and the affine chunk transfer of §1 contribution 4):
//
//   A_ij = beta_i k_i^T G_{i<-j} k_j  (j < i)    M_ij = q_i^T G_{i<-j} k_j (j <= i)
//   T    = (I + A)^{-1}                           (unit lower triangular)
//   U    = T diag(beta) (V - Khat S)              Khat_i = gamma_i * k_i
//   O    = scale (Qhat S + M U)                   Qhat_i = gamma_i * q_i
//   S   <- diag(gamma_L) S + Kbar^T U             Kbar_j = sigma_j * k_j
//
// Gate cumulant, exact for negative and zero gates: every gate factor is a
// running product of alpha inside a 16-token sub-block or across whole
// sub-blocks, always over an index range (j, i] with j <= i, so every factor
// has magnitude <= 1 and carries its sign (the parity of negative gates) and
// its zeros (a zero gate in range makes it exactly 0) with no logarithm and no
// division. For sub-block rows I (positions 16I..16I+15) and r = 16I - 1:
//   off-diagonal pairs (j <= r < i):  G_{i<-j} = G_{i<-r} G_{r<-j}, so
//     A_ij = beta_i (k_i * F_i) . (k_j * R_j)  with F_i = G_{i<-r}, R_j = G_{r<-j};
//   diagonal sub-block pairs: running products per column j.
// Padded rows (i >= L) get k = q = v = 0, beta = 0 and alpha = 1, which makes
// them inert (zero rows of A, M, U; gamma_L = gamma_{C-1}).
#include "ckda_common.cuh"

namespace ckda {

template <int DK, int DVT, int C>
struct SimtShape {
  static constexpr int NT = 256;
  static constexpr int KS = DK + 4;      // row stride of C x DK arrays (floats)
  static constexpr int VS = DVT + 4;     // row stride of C x DVT / DK x DVT
  static constexpr int AS = C + 1;       // row stride of C x C arrays
  static constexpr int NB = C / 16;      // sub-blocks per chunk
  static constexpr int YROWS_T = (C * AS + KS - 1) / KS;
  static constexpr int YROWS = YROWS_T > 32 ? YROWS_T : 32;
  // output micro-tiles for the C x DVT and DK x DVT products
  // two columns per thread when the resulting row-thread count still fits
  static constexpr int TR2 = NT / (DVT / 2);
  static constexpr int CPT = (TR2 <= C && TR2 <= DK) ? 2 : 1;  // cols/thread
  static constexpr int TC = DVT / CPT;                 // column threads
  static constexpr int TR = NT / TC;                   // row threads
  static constexpr int RPT = C / TR;                   // chunk rows per thread
  static constexpr int SRPT = DK / TR;                 // state rows per thread
  static constexpr size_t FLOATS =
      (size_t)4 * C * KS + (size_t)YROWS * KS + (size_t)C * VS + C + DK +
      (size_t)2 * C * AS + (size_t)DK * VS;
  static constexpr size_t BYTES = FLOATS * sizeof(float);
  static_assert(C % 16 == 0 && C <= 64, "chunk must be 16, 32 or 64");
  static_assert(DK % 16 == 0 && DK <= 128, "d_k must be 16..128");
  static_assert(DK + C <= NT, "factor and solve threads must fit the CTA");
  static_assert(RPT >= 1 && SRPT >= 1, "micro-tile must cover the tile");
  static_assert(TC * CPT == DVT && TR * TC == NT, "thread grid");
};

template <int DK, int DVT, int C, typename IOT>
__global__ void __launch_bounds__(256, 1)
fwd_simt_kernel(const IOT *__restrict__ q, const IOT *__restrict__ k,
                const IOT *__restrict__ v, const void *__restrict__ alpha_in,
                const float *__restrict__ beta, const float *__restrict__ s0,
                float *__restrict__ sfin, IOT *__restrict__ o,
                const int32_t *__restrict__ cu, int T, int T_total, int H,
                int DV, float scale, GateArgs ga, unsigned int *err) {
  // ga.on: alpha_in holds gate logits (IOT), beta logits, k raw keys (the
  // fused input prologue); the keys are normalised in shared memory
  const float *__restrict__ alpha = reinterpret_cast<const float *>(alpha_in);
  const IOT *__restrict__ alogit = reinterpret_cast<const IOT *>(alpha_in);
  using Sh = SimtShape<DK, DVT, C>;
  constexpr int KS = Sh::KS, VS = Sh::VS, AS = Sh::AS, NB = Sh::NB;
  constexpr int CPT = Sh::CPT, TC = Sh::TC, TR = Sh::TR, RPT = Sh::RPT,
                SRPT = Sh::SRPT;
  extern __shared__ float4 smem4[];
  float *sK = reinterpret_cast<float *>(smem4);  // k  -> (free after factors)
  float *sQ = sK + C * KS;                       // q  -> Qhat
  float *sAl = sQ + C * KS;                      // alpha -> Khat
  float *sX = sAl + C * KS;                      // R rows -> Kbar
  float *sY = sX + C * KS;                       // F*k, F*q rows -> T
  float *sV = sY + Sh::YROWS * KS;               // v -> R -> U
  float *sB = sV + C * VS;                       // beta
  float *sGC = sB + C;                           // gamma of the whole chunk
  float *sA = sGC + DK;                          // A (strictly lower)
  float *sM = sA + C * AS;                       // M (lower)
  float *sS = sM + C * AS;                       // state tile, fp32 master
  float *sT = sY;

  const int tid = threadIdx.x;
  const int vt = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int c0 = vt * DVT;
  int bos, eos;
  seq_bounds(cu, n, T, T_total, err, bos, eos);
  const size_t st_base = ((size_t)n * H + h) * DK * DV;

  for (int idx = tid; idx < DK * DVT; idx += Sh::NT) {
    const int r = idx / DVT, c = idx % DVT;
    sS[r * VS + c] = s0 ? s0[st_base + (size_t)r * DV + c0 + c] : 0.f;
  }

  const int tc = tid % TC, tr = tid / TC;

  for (int t0 = bos; t0 < eos; t0 += C) {
    const int L = min(C, eos - t0);
    __syncthreads();
    // ---- 1. load the chunk (fp32 in shared memory; pad rows inert)
    for (int idx = tid; idx < C * (DK / 4); idx += Sh::NT) {
      const int i = idx / (DK / 4), c4 = (idx % (DK / 4)) * 4;
      float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), qv = kv;
      float4 av = make_float4(1.f, 1.f, 1.f, 1.f);
      if (i < L) {
        const size_t off = ((size_t)(t0 + i) * H + h) * DK + c4;
        kv = IO<IOT>::ld4(k + off);
        qv = IO<IOT>::ld4(q + off);
        if (ga.on) {
          const float4 x = IO<IOT>::ld4(alogit + off);
          av = make_float4(gate_alpha(ga, x.x), gate_alpha(ga, x.y), gate_alpha(ga, x.z),
                           gate_alpha(ga, x.w));
        } else {
          av = *reinterpret_cast<const float4 *>(alpha + off);
        }
      }
      *reinterpret_cast<float4 *>(sK + i * KS + c4) = kv;
      *reinterpret_cast<float4 *>(sQ + i * KS + c4) = qv;
      *reinterpret_cast<float4 *>(sAl + i * KS + c4) = av;
    }
    for (int idx = tid; idx < C * (DVT / 4); idx += Sh::NT) {
      const int i = idx / (DVT / 4), c4 = (idx % (DVT / 4)) * 4;
      float4 vv = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < L) vv = IO<IOT>::ld4(v + ((size_t)(t0 + i) * H + h) * DV + c0 + c4);
      *reinterpret_cast<float4 *>(sV + i * VS + c4) = vv;
    }
    for (int i = tid; i < C; i += Sh::NT) {
      float b = (i < L) ? beta[(size_t)(t0 + i) * H + h] : 0.f;
      if (ga.on && i < L) b = gate_beta(ga, b);
      sB[i] = b;
    }
    __syncthreads();
    if (ga.on) {  // k_i <- k_i / (||k_i|| + eps), a warp per row
      for (int i = tid >> 5; i < C; i += Sh::NT / 32) {
        float ss = 0.f;
        for (int c = tid & 31; c < DK; c += 32) ss += sK[i * KS + c] * sK[i * KS + c];
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
        const float rn = key_rnorm(ga, ss);
        for (int c = tid & 31; c < DK; c += 32) sK[i * KS + c] *= rn;
      }
      __syncthreads();
    }

    // ---- 2. gated Grams A and M, one 16-row sub-block at a time
    for (int I = 0; I < NB; ++I) {
      const int r0 = I * 16;
      if (tid < DK) {
        // F_i = G_{i <- r0-1}: forward running product inside sub-block I
        const int c = tid;
        float g = 1.f;
        for (int ii = 0; ii < 16; ++ii) {
          const int i = r0 + ii;
          g *= sAl[i * KS + c];
          sY[ii * KS + c] = sK[i * KS + c] * g;
          sY[(16 + ii) * KS + c] = sQ[i * KS + c] * g;
        }
      } else if (tid < 2 * DK && r0 > 0) {
        // R_j = G_{r0-1 <- j}: backward running product from r0-1 down to 0
        const int c = tid - DK;
        float g = 1.f;
        for (int j = r0 - 1; j >= 0; --j) {
          sX[j * KS + c] = sK[j * KS + c] * g;
          g *= sAl[j * KS + c];
        }
      }
      __syncthreads();
      // off-diagonal sub-blocks: rows of block I against all earlier columns
      for (int idx = tid; idx < 16 * r0; idx += Sh::NT) {
        const int ii = idx / r0, j = idx % r0;
        float a = 0.f, m = 0.f;
#pragma unroll 8
        for (int c = 0; c < DK; c += 4) {
          const float4 lk = *reinterpret_cast<const float4 *>(sY + ii * KS + c);
          const float4 lq = *reinterpret_cast<const float4 *>(sY + (16 + ii) * KS + c);
          const float4 rr = *reinterpret_cast<const float4 *>(sX + j * KS + c);
          a += lk.x * rr.x + lk.y * rr.y + lk.z * rr.z + lk.w * rr.w;
          m += lq.x * rr.x + lq.y * rr.y + lq.z * rr.z + lq.w * rr.w;
        }
        sA[(r0 + ii) * AS + j] = sB[r0 + ii] * a;
        sM[(r0 + ii) * AS + j] = m;
      }
      // diagonal sub-block: thread = (column j, channel lane sl); channels
      // sl, sl+16, ... ; reduced over the 16 lanes of a half-warp
      {
        const int j = tid / 16, sl = tid % 16;
        float accA[16], accM[16];
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) accA[ii] = accM[ii] = 0.f;
        for (int c = sl; c < DK; c += 16) {
          const float kj = sK[(r0 + j) * KS + c];
          float g = 1.f;
#pragma unroll
          for (int ii = 0; ii < 16; ++ii) {
            if (ii >= j) {
              if (ii > j) g *= sAl[(r0 + ii) * KS + c];
              const float x = g * kj;
              accA[ii] += sK[(r0 + ii) * KS + c] * x;
              accM[ii] += sQ[(r0 + ii) * KS + c] * x;
            }
          }
        }
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) {
#pragma unroll
          for (int off = 8; off > 0; off >>= 1) {
            accA[ii] += __shfl_xor_sync(0xffffffffu, accA[ii], off);
            accM[ii] += __shfl_xor_sync(0xffffffffu, accM[ii], off);
          }
        }
        if (sl == 0) {
#pragma unroll
          for (int ii = 0; ii < 16; ++ii) {
            if (ii > j) sA[(r0 + ii) * AS + r0 + j] = sB[r0 + ii] * accA[ii];
            if (ii >= j) sM[(r0 + ii) * AS + r0 + j] = accM[ii];
          }
        }
      }
      __syncthreads();
    }

    // ---- 3. factors (Kbar, Khat, Qhat, gamma_L) and the diagonal solves
    if (tid < DK) {
      const int c = tid;
      float g = 1.f;
      for (int j = C - 1; j >= 0; --j) {  // sigma_j = prod_{s>j} alpha_s
        sX[j * KS + c] = g * sK[j * KS + c];
        g *= sAl[j * KS + c];
      }
      g = 1.f;
      for (int i = 0; i < C; ++i) {       // gamma_i = prod_{s<=i} alpha_s
        g *= sAl[i * KS + c];
        sAl[i * KS + c] = g * sK[i * KS + c];
        sQ[i * KS + c] *= g;
      }
      sGC[c] = g;
    } else if (tid < DK + C) {
      // T_II = (I + A_II)^{-1}: thread owns column j of sub-block b
      const int b = (tid - DK) / 16, j = (tid - DK) % 16, ob = b * 16;
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
    // off-diagonal blocks of T, by distance d from the diagonal:
    //   T_IJ = -T_II * sum_{L=J}^{I-1} A_IL T_LJ   (J = I - d)
    for (int d = 1; d < NB; ++d) {
      float *sXT = sK;  // free now
      for (int idx = tid; idx < (NB - d) * 256; idx += Sh::NT) {
        const int p = idx / 256, e = idx % 256, ii = e / 16, jj = e % 16;
        const int I = d + p, J = p;
        float s = 0.f;
        for (int Lb = J; Lb < I; ++Lb)
#pragma unroll
          for (int l = 0; l < 16; ++l)
            s += sA[(I * 16 + ii) * AS + Lb * 16 + l] *
                 sT[(Lb * 16 + l) * AS + J * 16 + jj];
        sXT[p * 256 + ii * 16 + jj] = s;
      }
      __syncthreads();
      for (int idx = tid; idx < (NB - d) * 256; idx += Sh::NT) {
        const int p = idx / 256, e = idx % 256, ii = e / 16, jj = e % 16;
        const int I = d + p, J = p;
        float s = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m)
          if (m <= ii) s += sT[(I * 16 + ii) * AS + I * 16 + m] * sXT[p * 256 + m * 16 + jj];
        sT[(I * 16 + ii) * AS + J * 16 + jj] = -s;
      }
      __syncthreads();
    }

    // ---- 4. R = diag(beta)(V - Khat S) into sV; O1 = Qhat S kept in registers
    float o1[RPT][CPT];
    {
      float ks[RPT][CPT];
#pragma unroll
      for (int a = 0; a < RPT; ++a)
#pragma unroll
        for (int b = 0; b < CPT; ++b) ks[a][b] = o1[a][b] = 0.f;
      for (int r = 0; r < DK; r += 4) {
        float s4[4][CPT];
#pragma unroll
        for (int b = 0; b < CPT; ++b)
#pragma unroll
          for (int u = 0; u < 4; ++u) s4[u][b] = sS[(r + u) * VS + tc + b * TC];
#pragma unroll
        for (int a = 0; a < RPT; ++a) {
          const int i = tr + a * TR;
          const float4 kh = *reinterpret_cast<const float4 *>(sAl + i * KS + r);
          const float4 qh = *reinterpret_cast<const float4 *>(sQ + i * KS + r);
#pragma unroll
          for (int b = 0; b < CPT; ++b) {
            ks[a][b] += kh.x * s4[0][b] + kh.y * s4[1][b] + kh.z * s4[2][b] + kh.w * s4[3][b];
            o1[a][b] += qh.x * s4[0][b] + qh.y * s4[1][b] + qh.z * s4[2][b] + qh.w * s4[3][b];
          }
        }
      }
#pragma unroll
      for (int a = 0; a < RPT; ++a) {
        const int i = tr + a * TR;
#pragma unroll
        for (int b = 0; b < CPT; ++b) {
          const int c = tc + b * TC;
          sV[i * VS + c] = sB[i] * (sV[i * VS + c] - ks[a][b]);
        }
      }
    }
    __syncthreads();
    // ---- 5. U = T R (rows depend on earlier rows: compute all, then write)
    {
      float u[RPT][CPT];
#pragma unroll
      for (int a = 0; a < RPT; ++a) {
        const int i = tr + a * TR;
#pragma unroll
        for (int b = 0; b < CPT; ++b) u[a][b] = 0.f;
        for (int j = 0; j <= i; ++j) {
          const float tij = sT[i * AS + j];
#pragma unroll
          for (int b = 0; b < CPT; ++b) u[a][b] += tij * sV[j * VS + tc + b * TC];
        }
      }
      __syncthreads();
#pragma unroll
      for (int a = 0; a < RPT; ++a)
#pragma unroll
        for (int b = 0; b < CPT; ++b) sV[(tr + a * TR) * VS + tc + b * TC] = u[a][b];
    }
    __syncthreads();
    // ---- 6. O = scale (Qhat S + M U) for the valid rows
#pragma unroll
    for (int a = 0; a < RPT; ++a) {
      const int i = tr + a * TR;
      float acc[CPT];
#pragma unroll
      for (int b = 0; b < CPT; ++b) acc[b] = o1[a][b];
      for (int j = 0; j <= i; ++j) {
        const float mij = sM[i * AS + j];
#pragma unroll
        for (int b = 0; b < CPT; ++b) acc[b] += mij * sV[j * VS + tc + b * TC];
      }
      if (i < L) {
#pragma unroll
        for (int b = 0; b < CPT; ++b)
          IO<IOT>::st(o + ((size_t)(t0 + i) * H + h) * DV + c0 + tc + b * TC,
                      scale * acc[b]);
      }
    }
    // ---- 7. S <- diag(gamma_L) S + Kbar^T U (rows r = tr*SRPT .. +SRPT-1)
    {
      float acc[SRPT][CPT];
#pragma unroll
      for (int a = 0; a < SRPT; ++a) {
        const int r = tr * SRPT + a;
#pragma unroll
        for (int b = 0; b < CPT; ++b) acc[a][b] = sGC[r] * sS[r * VS + tc + b * TC];
      }
      for (int j = 0; j < C; ++j) {
        float uj[CPT];
#pragma unroll
        for (int b = 0; b < CPT; ++b) uj[b] = sV[j * VS + tc + b * TC];
#pragma unroll
        for (int a = 0; a < SRPT; ++a) {
          const float kb = sX[j * KS + tr * SRPT + a];
#pragma unroll
          for (int b = 0; b < CPT; ++b) acc[a][b] += kb * uj[b];
        }
      }
#pragma unroll
      for (int a = 0; a < SRPT; ++a)
#pragma unroll
        for (int b = 0; b < CPT; ++b) sS[(tr * SRPT + a) * VS + tc + b * TC] = acc[a][b];
    }
  }
  __syncthreads();
  if (sfin) {
    for (int idx = tid; idx < DK * DVT; idx += Sh::NT) {
      const int r = idx / DVT, c = idx % DVT;
      sfin[st_base + (size_t)r * DV + c0 + c] = sS[r * VS + c];
    }
  }
}

template <int DK, int DVT, int C, typename IOT>
static cudaError_t launch_simt_cfg(const void *q, const void *k, const void *v,
                                   const void *alpha, const float *beta,
                                   const float *s0, float *sf, void *o,
                                   const int32_t *cu, int N, int T, int T_total,
                                   int H, int DV, float scale, GateArgs g,
                                   unsigned int *err, cudaStream_t st) {
  using Sh = SimtShape<DK, DVT, C>;
  auto kern = fwd_simt_kernel<DK, DVT, C, IOT>;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Sh::BYTES);
  if (e != cudaSuccess) return e;
  const dim3 grid(DV / DVT, H, N);
  kern<<<grid, Sh::NT, Sh::BYTES, st>>>((const IOT *)q, (const IOT *)k,
                                        (const IOT *)v, alpha, beta, s0, sf,
                                        (IOT *)o, cu, T, T_total, H, DV, scale,
                                        g, err);
  return cudaGetLastError();
}

template <int DK, int DVT, typename IOT>
static cudaError_t launch_simt_chunk(int chunk, const void *q, const void *k,
                                     const void *v, const void *alpha,
                                     const float *beta, const float *s0,
                                     float *sf, void *o, const int32_t *cu,
                                     int N, int T, int T_total, int H, int DV,
                                     float scale, GateArgs g, unsigned int *err,
                                     cudaStream_t st) {
  switch (chunk) {
    case 16: return launch_simt_cfg<DK, DVT, 16, IOT>(q, k, v, alpha, beta, s0, sf, o, cu, N, T, T_total, H, DV, scale, g, err, st);
    case 32: return launch_simt_cfg<DK, DVT, 32, IOT>(q, k, v, alpha, beta, s0, sf, o, cu, N, T, T_total, H, DV, scale, g, err, st);
    case 64: return launch_simt_cfg<DK, DVT, 64, IOT>(q, k, v, alpha, beta, s0, sf, o, cu, N, T, T_total, H, DV, scale, g, err, st);
  }
  return cudaErrorInvalidValue;
}

// d_v is tiled by DVT = min(d_v, 32) columns per CTA.
template <typename IOT>
cudaError_t launch_fwd_simt(int dk, int dv, int chunk, const void *q,
                            const void *k, const void *v, const void *alpha,
                            const float *beta, const float *s0, float *sf,
                            void *o, const int32_t *cu, int N, int T,
                            int T_total, int H, float scale, GateArgs g,
                            unsigned int *err, cudaStream_t st) {
#define CKDA_SIMT_DK(DKV)                                                       \
  case DKV:                                                                     \
    if (dv == 16)                                                               \
      return launch_simt_chunk<DKV, 16, IOT>(chunk, q, k, v, alpha, beta, s0,   \
                                             sf, o, cu, N, T, T_total, H, dv,   \
                                             scale, g, err, st);                \
    return launch_simt_chunk<DKV, 32, IOT>(chunk, q, k, v, alpha, beta, s0, sf, \
                                           o, cu, N, T, T_total, H, dv, scale,  \
                                           g, err, st);
  switch (dk) {
    CKDA_SIMT_DK(16)
    CKDA_SIMT_DK(32)
    CKDA_SIMT_DK(64)
    CKDA_SIMT_DK(128)
  }
#undef CKDA_SIMT_DK
  return cudaErrorInvalidValue;
}

template cudaError_t launch_fwd_simt<float>(int, int, int, const void *,
                                            const void *, const void *,
                                            const void *, const float *,
                                            const float *, float *, void *,
                                            const int32_t *, int, int, int, int,
                                            float, GateArgs, unsigned int *,
                                            cudaStream_t);
template cudaError_t launch_fwd_simt<__nv_bfloat16>(
    int, int, int, const void *, const void *, const void *, const void *,
    const float *, const float *, float *, void *, const int32_t *, int, int,
    int, int, float, GateArgs, unsigned int *, cudaStream_t);

}  // namespace ckda
