// Chunkwise CKDA forward with tcgen05 tensor cores (sm_100a): bf16 I/O,
// fp32 state, tf32 tensor-core operands with fp32 accumulation. d_k = 128,
// chunk 64, d_v in {32, 64, 128}.
//
// Two kernels, split where the work changes character:
//
//  * ckda_chunk_prep_kernel: persistent, one CTA per SM, walking the (chunk,
//    head) items of all sequences (a small kernel first tabulates which
//    chunk each slot holds); q, k, v and alpha come in by tensor-map copies.
//    For each item it builds everything that does not depend on the state
//    entering it (the chunk-WY / UT-transform factors of the product of
//    diagonal-plus-rank-one transitions, Semidirect Fourier Delta Attention
//    §2.2, and the affine chunk transfer's write summary, §1 contribution 4),
//    and stores the serial step's operands in a workspace:
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
#include <cuda.h>  // CUtensorMap (the encoder is reached through the runtime)
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "ckda.h"
#include "ckda_common.cuh"
#include "ckda_tc_ptx.cuh"

namespace ckda {
namespace {

using namespace tc;

constexpr int C = 64, DK = 128, DVT = 32;
constexpr int AL_S = 132;  // fp32 row stride of alpha / Qhat

// Float offset of (row i, channel c) in the alpha / Qhat buffer: rows of 128
// channels padded to 132 floats (the tensor-map copy of alpha fills the
// padding with zeros), so that 16-byte reads of one channel block by the
// threads of 32 consecutive rows fall into different banks.
__device__ __forceinline__ int al_off(int i, int c) { return i * AL_S + c; }

// ---------------------------------------------------------------- workspace
// One block per (chunk slot, head); chunk c of sequence n sits in slot
// floor(cu[n] / 64) + n + c, which never collides and is below
// floor(T_total / 64) + N.
constexpr uint32_t WS_A1 = 0;       // [Qtil ; W]: 128 x 128 tf32, K-major sw128 image
constexpr uint32_t WS_A2 = 65536;   // Kbar^T:     128 x 64 tf32, K-major sw128 image
constexpr uint32_t WS_OU = 98304;   // [M Ut ; Ut]: 128 rows x d_v fp32, 16-byte pieces swizzled by row
__host__ __device__ constexpr uint32_t ws_gamma_off(int dv) { return WS_OU + 128u * dv * 4u; }
__host__ __device__ constexpr uint32_t ws_block_bytes(int dv) {
  return ws_gamma_off(dv) + 1024u;  // gamma: 128 fp32, block kept 1 KB aligned
}

// first slot of sequence n
__device__ __forceinline__ int slot_base(const int32_t *cu, int n, int T) {
  const int b = cu ? __ldg(cu + n) : n * T;
  return b / C + n;
}

// Slot table (after the blocks): per slot, {first token, tokens} of the chunk
// it holds ({0, 0} for an empty slot).
__host__ __device__ constexpr size_t slot_table_off(size_t slots, size_t H, int dv) {
  return slots * H * ws_block_bytes(dv);
}
__host__ __device__ constexpr size_t slot_table_bytes(size_t slots) {
  return (slots * sizeof(int2) + 1023) & ~size_t(1023);
}

// One thread per slot: which (sequence, chunk) the slot holds. Every slot is
// written, and a malformed device cu_seqlens only ever yields token ranges
// inside [0, T_total) (seq_bounds flags it).
__global__ void ckda_slot_table_kernel(const int32_t *__restrict__ cu, int N, int T,
                                       int T_total, int slots, int2 *__restrict__ tab,
                                       unsigned int *err) {
  const int slot = blockIdx.x * blockDim.x + threadIdx.x;
  if (slot >= slots) return;
  int lo = 0, hi = N - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (slot_base(cu, mid, T) <= slot) lo = mid;
    else hi = mid - 1;
  }
  int bos, eos;
  seq_bounds(cu, lo, T, T_total, err, bos, eos);
  const int cidx = slot - slot_base(cu, lo, T);
  const long long t0 = (long long)bos + (long long)C * cidx;
  int2 e = make_int2(0, 0);
  if (cidx >= 0 && t0 < eos) e = make_int2((int)t0, min(C, eos - (int)t0));
  tab[slot] = e;
}

// ---------------------------------------------------------------- prep kernel
// shared-memory map (byte offsets from a 1024-aligned base); fp32 operands.
// MN-major tf32 operands use the 128B-swizzle / 32B-atom form (the only
// MN-major form tcgen05 accepts for 32-bit elements).
constexpr int NTP = 512;
constexpr int RS = 68;                // fp32 row stride of A, M, T (16-byte aligned rows)
constexpr uint32_t P_GA = 0;          // 65536 Lk/Lq (M128 x K128, MN-major; rows 96.. unused)
                                      //   -> [beta Khat | beta V] (N(128+dv) x K64, K-major)
                                      //   -> staged [Qtil ; W] image (epilogue)
constexpr uint32_t P_GB = 49152;      // 49152 R stack (N96 x K128, MN-major)
constexpr uint32_t P_T = 65536;       // 17408 T fp32 [64][68] (after the Grams)
constexpr uint32_t P_XT = P_T + 17408; //  3072 solve scratch
constexpr uint32_t P_OU = 65536;      // <=32768 staged M Ut rows (epilogue; Ut rows at P_A)
constexpr uint32_t P_V = 98304;       // 16384 raw v bf16 [64][dv] (until beta V is built)
constexpr uint32_t P_B0 = 98304;      // 16384 T (K64 x N64 MN)
constexpr uint32_t P_Q = 114688;      // 16384 raw q bf16 [64][128]
constexpr uint32_t P_K = 131072;      // 16384 raw k bf16 [64][128]
constexpr uint32_t P_A0 = 114688;     // 32768 [M ; I] (128 x 64 K-major), over raw q and k
constexpr uint32_t P_AL = 147456;     // 33792 alpha fp32 [64][132] -> Qhat fp32
constexpr uint32_t P_AL_LOGIT = 17408; // fused prologue: the bf16 gate logits [64][128] land here in alpha's buffer
constexpr uint32_t P_A = 181248;      // 17408 A fp32 [64][68] (with P_M: staged Ut rows, epilogue)
constexpr uint32_t P_M = 198656;      // 17408 M fp32 [64][68]
constexpr uint32_t P_B = 216064;      //   256 beta
constexpr uint32_t P_BAR = 216320;    //    64 mbarriers [0..3], TMEM address, flag, input mbarriers [2]
constexpr uint32_t P_P = 216384;      //  2048 gate products of whole sub-blocks [4][128]
constexpr uint32_t P_RN = 218432;     //   256 key row inverse norms (fused prologue)
constexpr uint32_t P_SMEM = 218688 + 1024;

// TMEM columns of the prep kernel (512 allocated; one CTA per SM)
constexpr uint32_t TP_G = 0;      //  96 Gram accumulator
constexpr uint32_t TP_G4 = 96;    //  96 Gram inside the 16-token sub-blocks
constexpr uint32_t TP_QH = 0;     // 128 Qhat (lanes 0..63), once both Grams are read
constexpr uint32_t TP_AD5 = 192;  //  64 [M T ; T] (A of D5)
constexpr uint32_t TP_D5 = 256;   // 256 [M W | M Ut ; W | Ut]
constexpr uint32_t TP_COLS = 512;

constexpr uint32_t ID_G = idesc_tf32(128, 96, 1, 1);
constexpr uint32_t ID_D0 = idesc_tf32(128, 64, 0, 1);

__device__ __forceinline__ float bf(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st4_f32(uint8_t *p, float a, float b, float c, float d) {
  *reinterpret_cast<float4 *>(p) = make_float4(to_tf32(a), to_tf32(b), to_tf32(c), to_tf32(d));
}

// Two 16-byte stores of one channel into an MN-major image, rows mn0 and
// mn0 + 4 (the two 16-byte halves of one 32-byte swizzle chunk). `swap`
// (lane bit 2, independent of the channel's swizzle chunk k mod 4) reverses
// their order in half of the lanes, so that each store instruction of a warp
// (32 consecutive channels) covers all 32 banks instead of half of them.
__device__ __forceinline__ void st4x2_mn(uint8_t *base, int k, int mn0, int ktot,
                                         const float *v0, const float *v1, bool swap) {
  const uint32_t o0 = off_mn_sw128b32_f32(k, mn0, ktot), o1 = off_mn_sw128b32_f32(k, mn0 + 4, ktot);
  float a[4], b[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    a[e] = swap ? v1[e] : v0[e];
    b[e] = swap ? v0[e] : v1[e];
  }
  st4_f32(base + (swap ? o1 : o0), a[0], a[1], a[2], a[3]);
  st4_f32(base + (swap ? o0 : o1), b[0], b[1], b[2], b[3]);
}

// Row r of [M Ut ; Ut] keeps its 16-byte piece p at p ^ (r mod 8), in the
// workspace as in shared memory, so that the row-per-thread writes of the
// prep epilogue hit distinct banks.
__device__ __forceinline__ int ou_piece(int row, int piece) { return piece ^ (row & 7); }

// Bounded wait of all threads on one mbarrier; false (and the abort flag set)
// if it timed out. Ends with every thread past a CTA barrier.
__device__ __forceinline__ bool wait_all(uint64_t *bar, uint32_t phase,
                                         volatile int *s_abort) {
  if (!mbar_wait(bar, phase)) *s_abort = 1;
  fence_after_sync();
  __syncthreads();
  return *s_abort == 0;
}

// GATED: the fused input prologue (GateArgs): the alpha tensor map is over
// bf16 gate logits, `beta` holds fp32 logits and `k` raw keys; the key row
// inverse norms rn are applied to every product k enters (Gram rows, R, Kbar,
// beta Khat and the diagonal sub-blocks), which is the same as using the
// normalised keys.
template <bool GATED>
__global__ void __launch_bounds__(NTP, 1)
ckda_chunk_prep_kernel(const float *__restrict__ beta,
                       const int2 *__restrict__ slot_tab, int n_items,
                       int H, int DV, GateArgs ga, uint8_t *__restrict__ ws,
                       unsigned int *err, const __grid_constant__ CUtensorMap map_q,
                       const __grid_constant__ CUtensorMap map_k,
                       const __grid_constant__ CUtensorMap map_v,
                       const __grid_constant__ CUtensorMap map_a) {
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
  float *sT = reinterpret_cast<float *>(sm + P_T);
  float *sXT = reinterpret_cast<float *>(sm + P_XT);
  float *sB = reinterpret_cast<float *>(sm + P_B);
  float *sP = reinterpret_cast<float *>(sm + P_P);
  float *sRN = reinterpret_cast<float *>(sm + P_RN);
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + P_BAR);  // [0..3]
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + P_BAR + 32);
  volatile int *s_abort = reinterpret_cast<volatile int *>(sm + P_BAR + 36);
  uint64_t *bin = reinterpret_cast<uint64_t *>(sm + P_BAR + 40);  // input copies: [0] q, k, v; [1] alpha (or its logits)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (warp == 0) {
    tmem_alloc(s_tmem, TP_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(&bar[i], 1);
    for (int i = 0; i < 2; ++i) mbar_init(&bin[i], 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = *s_tmem;
  const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;

  // An item's q, k and v rows and alpha (with the fused prologue, alpha's bf16
  // logits, into the upper half of alpha's buffer) arrive by tensor-map copies
  // (one box of 64 token rows per input, issued by thread 0, counted on
  // mbarrier bin[0] or bin[1]); beta (or its logits) by per-thread copies
  // (cp.async). They are issued during the previous item
  // once each buffer's last reader is done: alpha and beta when the [M ; I]
  // and T operands are built (Qhat has moved to tensor memory, and gamma and
  // beta were last read by the WY operand build), q, k, v while D5 runs
  // ([M ; I] x T was their last reader). An item whose copies were not issued
  // ahead (the first, or one after empty slots) issues them at its start. Box
  // rows past the chunk's end hold the next sequence's tokens (zeros past the
  // last token) until the item's start overwrites them (q, k, v: 0, alpha: 1);
  // beta rows past the end are written as 0.
  const int nvp = DV / 8, lnv = __ffs(nvp) - 1;  // 16-byte pieces of a v row (a power of 2)
  auto issue_qkv = [&](int t0r, int hr) {
    if (tid == 0) {
      mbar_arrive_expect_tx(&bin[0], (uint32_t)C * (2 * DK + DV) * 2u);
      tma_load_3d(sm + P_Q, &map_q, 0, hr, t0r, &bin[0]);
      tma_load_3d(sm + P_K, &map_k, 0, hr, t0r, &bin[0]);
      tma_load_3d(sm + P_V, &map_v, 0, hr, t0r, &bin[0]);
    }
  };
  // Beta is copied by threads BT .. BT + 63, not by thread 0: thread 0
  // commits the workspace's bulk stores, and its cp.async wait was measured
  // to last until those stores had finished.
  constexpr int BT = 64;
  auto issue_gates = [&](int t0r, int Lr, int hr) {  // alpha (or its logits), beta
    if (tid == 0) {
      if constexpr (GATED) {
        mbar_arrive_expect_tx(&bin[1], (uint32_t)C * DK * 2u);
        tma_load_3d(sm + P_AL + P_AL_LOGIT, &map_a, 0, hr, t0r, &bin[1]);
      } else {
        mbar_arrive_expect_tx(&bin[1], (uint32_t)C * AL_S * 4u);
        tma_load_3d(sAl, &map_a, 0, hr, t0r, &bin[1]);
      }
    }
    if (tid >= BT && tid < BT + C) {  // beta: threads BT .. BT + 63
      const int j = tid - BT;
      if (j < Lr) cp_async4(sB + j, beta + (size_t)(t0r + j) * H + hr);
      else sB[j] = 0.f;
      cp_async_commit();
    }
  };
  auto wait_in = [&](int b, uint32_t parity) {  // all threads
    if (!mbar_wait(&bin[b], parity)) *s_abort = 1;
  };
  // copy groups issued for the next item and not yet waited for (bit 0: q, k,
  // v; bit 1: alpha); looked at only when an abort ends the loop
  int ahead = 0;
  int raw_for = -1;  // item whose row copies were issued ahead (CTA-uniform)

  // Persistent: items (slot, head) = it / H, it % H, strided by the grid.
  // Each mbarrier completes once per non-empty item: parity `ph`.
  uint32_t ph = 0;
  int2 cur = make_int2(0, 0);
  if ((int)blockIdx.x < n_items) cur = __ldg(slot_tab + blockIdx.x / H);
  for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
  const int slot = it / H, h = it - slot * H;
  const int t0 = cur.x, L = cur.y;
  const int nit = it + gridDim.x;
  int2 nxt = make_int2(0, 0);
  if (nit < n_items) nxt = __ldg(slot_tab + nit / H);
  if (L <= 0) {  // empty slot (CTA-uniform)
    cur = nxt;
    continue;
  }
  uint8_t *wsb = ws + ((size_t)slot * H + h) * ws_block_bytes(DV);

  do {  // one pass; `break` leaves on a timed-out wait
    // ---------------- 1. load the chunk: q, k, v, alpha (or its logits) and
    // beta have been copied in asynchronously
    if (raw_for != it) {
      issue_qkv(t0, h);
      issue_gates(t0, L, h);
    }
    raw_for = -1;
    {
      wait_in(0, ph);
      wait_in(1, ph);
      ahead = 0;
      uint4 al[2];  // GATED: 64 rows x 16 pieces of 8 bf16 logits, read before alpha overwrites them
      (void)al;
      if constexpr (GATED) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int idx = tid + u * NTP, i = idx >> 4, ch = idx & 15;
          al[u] = make_uint4(0, 0, 0, 0);
          if (i < L) al[u] = *reinterpret_cast<const uint4 *>(sm + P_AL + P_AL_LOGIT + i * 256 + ch * 16);
        }
      }
      if (tid >= BT && tid < BT + C) cp_async_wait_all();
      if constexpr (GATED) {
        __syncthreads();  // every thread's logits are read (alpha goes over them)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int idx = tid + u * NTP, i = idx >> 4, ch = idx & 15;
          // alpha from the logits (1 on padded rows)
          float x[8];
          const uint32_t w[4] = {al[u].x, al[u].y, al[u].z, al[u].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            x[2 * e] = __uint_as_float(w[e] << 16);
            x[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = (i < L) ? gate_alpha_fast(ga, x[e]) : 1.f;
          *reinterpret_cast<float4 *>(sAl + al_off(i, 8 * ch)) = make_float4(x[0], x[1], x[2], x[3]);
          *reinterpret_cast<float4 *>(sAl + al_off(i, 8 * ch + 4)) = make_float4(x[4], x[5], x[6], x[7]);
          // key row inverse norm: 16 lanes hold row i's 128 channels
          uint4 kq = make_uint4(0, 0, 0, 0);
          if (i < L) kq = *reinterpret_cast<const uint4 *>(sm + P_K + i * 256 + ch * 16);
          const uint32_t kw[4] = {kq.x, kq.y, kq.z, kq.w};
          float ss = 0.f;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float lo = __uint_as_float(kw[e] << 16), hi = __uint_as_float(kw[e] & 0xffff0000u);
            ss += lo * lo + hi * hi;
          }
#pragma unroll
          for (int m = 8; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
          if (ch == 0) sRN[i] = (i < L) ? key_rnorm(ga, ss) : 0.f;
        }
        if (tid < L) sB[tid] = gate_beta(ga, sB[tid]);  // beta from its logit
      }
      // rows past the chunk's end: q, k, v zero, alpha one (the fused
      // prologue has set its alpha rows and reads no k row past the end)
      if (L < C) {
        const int nr = C - L;
        for (int idx = tid; idx < nr * 16; idx += NTP) {
          const int i = L + (idx >> 4), w = idx & 15;
          *reinterpret_cast<uint4 *>(sm + P_Q + i * 256 + w * 16) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4 *>(sm + P_K + i * 256 + w * 16) = make_uint4(0, 0, 0, 0);
        }
        for (int idx = tid; idx < nr * nvp; idx += NTP) {
          const int i = L + (idx >> lnv), w = idx & (nvp - 1);
          *reinterpret_cast<uint4 *>(sm + P_V + i * DV * 2 + w * 16) = make_uint4(0, 0, 0, 0);
        }
        if constexpr (!GATED) {
          for (int idx = tid; idx < nr * 32; idx += NTP) {
            const int i = L + (idx >> 5), c4 = (idx & 31) * 4;
            *reinterpret_cast<float4 *>(sAl + al_off(i, c4)) = make_float4(1.f, 1.f, 1.f, 1.f);
          }
        }
      }
      // The previous item's workspace stores read their staging in three
      // groups, committed in the order this item writes over them. The gate
      // pass's Gram rows go over group 1 ([Qtil ; W] columns 0..95).
      if (tid == 0) bulk_wait_read<2>();
    }
    __syncthreads();

    // ---------------- 2. gate pass: thread (16-token sub-block g, channel c)
    // forms the sub-block prefix products p_u = prod_{s=16g..16g+u} alpha_s
    // and suffix products prod_{s=16g+u+1..16g+15} alpha_s, and the product
    // P_g of the whole sub-block; with the P of the other sub-blocks
    //   Lk_i = k_i G_{i<-16g-1} = k_i p_u, Lq_i = q_i p_u      (Gram rows, g >= 1)
    //   R^(I)_j = k_j G_{16I-1<-j} = (k_j suffix_u) P_{g+1} .. P_{I-1}   (I > g)
    //   Kbar_j = k_j sigma_j = (k_j suffix_u) P_{g+1} .. P_3
    const int gq = tid >> 7, gc = tid & 127;
    {
      float pre = 1.f;
      float a[16], kr[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        a[u] = sAl[al_off(16 * gq + u, gc)];
        kr[u] = bf(sKr + (16 * gq + u) * DK + gc);
        if constexpr (GATED) kr[u] *= sRN[16 * gq + u];
      }
      // Gram rows, MN-major (rows contiguous): a thread's 16 rows of one
      // channel are four 16-byte stores per operand
      if (gq >= 1) {
        float lk[16], lq[16], pu = 1.f;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          pu *= a[u];
          lk[u] = pu * kr[u];
          lq[u] = pu * bf(sQr + (16 * gq + u) * DK + gc);
        }
#pragma unroll
        for (int u = 0; u < 16; u += 8) {
          st4x2_mn(GA, gc, (gq - 1) * 32 + u, DK, lk + u, lk + u + 4, (lane >> 2) & 1);
          st4x2_mn(GA, gc, (gq - 1) * 32 + 16 + u, DK, lq + u, lq + u + 4, (lane >> 2) & 1);
        }
      }
      float p = 1.f;
#pragma unroll
      for (int u = 0; u < 16; ++u) p *= a[u];
      float sfx = 1.f;
#pragma unroll
      for (int u = 15; u >= 0; --u) {
        kr[u] *= sfx;  // k_j times the suffix product of its sub-block
        sfx *= a[u];
      }
      sP[gq * DK + gc] = p;
      if (tid == 0) bulk_wait_read<1>();  // the R stack goes over group 2
      __syncthreads();
      float P[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) P[b] = sP[b * DK + gc];
      float suf = 1.f;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        if (b < gq) pre *= P[b];
        if (b > gq) suf *= P[b];
      }
      float f = 1.f;
#pragma unroll
      for (int I = 1; I < 4; ++I) {
        if (I > gq) {
          if (I > gq + 1) f *= P[I - 1];
#pragma unroll
          for (int u = 0; u < 16; u += 8) {
            const float r0[4] = {f * kr[u], f * kr[u + 1], f * kr[u + 2], f * kr[u + 3]};
            const float r1[4] = {f * kr[u + 4], f * kr[u + 5], f * kr[u + 6], f * kr[u + 7]};
            st4x2_mn(GB, gc, 8 * I * (I - 1) + 16 * gq + u, DK, r0, r1, (lane >> 2) & 1);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 16; u += 4)  // row c of Kbar^T (K-major sw128 image)
        *reinterpret_cast<float4 *>(wsb + WS_A2 + off_k_sw128_f32(gc, 16 * gq + u, DK)) =
            make_float4(to_tf32(suf * kr[u]), to_tf32(suf * kr[u + 1]),
                        to_tf32(suf * kr[u + 2]), to_tf32(suf * kr[u + 3]));
      if (gq == 3) reinterpret_cast<float *>(wsb + ws_gamma_off(DV))[gc] = pre * p;
    }
    if (tid == 0) bulk_wait_read<0>();  // the sweep's A and M go over group 3
    fence_async_smem();
    __syncthreads();

    // ---------------- 3. Grams: off-diagonal sub-blocks on tensor cores ...
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < DK / 8; ++kk)
        mma_tf32_ss(tm + TP_G, desc_mn_sw128b32_f32(sb + P_GA, DK, kk),
                    desc_mn_sw128b32_f32(sb + P_GB, DK, kk), ID_G, kk > 0);
      mma_commit(&bar[0]);
    }
    // ... and, meanwhile on CUDA cores, the pairs inside each 4-token group
    // (j <= i, same group). A half-warp owns row i (lane sl: channels
    // 4 sl .. 4 sl + 3 and 64 + 4 sl .. 64 + 4 sl + 3, so that the 8 lanes
    // of each 16-byte access phase read 128 consecutive bytes of a row) and
    // walks j = i, i-1, ... down the group carrying
    // G_{i<-j} (paired fp32); a reduce-scatter butterfly over the 16 lanes
    // then leaves entry sl / 2 of [A row | M row] (4 + 4 entries) in lanes
    // sl. Warp w takes group 2 (w / 2) + half and its rows {0, 3} (w even) or
    // {1, 2} (w odd), so every half-warp walks 5 steps.
    {
      const int sl = lane & 15, c4 = 4 * sl;
      auto ld8 = [&](const __nv_bfloat16 *row) {  // this lane's 8 channels of a bf16 row
        const uint2 lo = *reinterpret_cast<const uint2 *>(row + c4);
        const uint2 hi = *reinterpret_cast<const uint2 *>(row + 64 + c4);
        return make_uint4(lo.x, lo.y, hi.x, hi.y);
      };
      const int r0 = 4 * (2 * (warp >> 1) + (lane >> 4));
#pragma unroll 1
      for (int pass = 0; pass < 2; ++pass) {
        const int ii = (warp & 1) ? 1 + pass : 3 * pass, i = r0 + ii;
        uint64_t ki[4], qi[4], g[4];
        {
          const uint4 kr = ld8(sKr + i * DK);
          const uint4 qr = ld8(sQr + i * DK);
          ki[0] = bf2_to_f2(kr.x); ki[1] = bf2_to_f2(kr.y);
          ki[2] = bf2_to_f2(kr.z); ki[3] = bf2_to_f2(kr.w);
          qi[0] = bf2_to_f2(qr.x); qi[1] = bf2_to_f2(qr.y);
          qi[2] = bf2_to_f2(qr.z); qi[3] = bf2_to_f2(qr.w);
          if constexpr (GATED) {
            const uint64_t rn2 = f2pack(sRN[i], sRN[i]);
#pragma unroll
            for (int e = 0; e < 4; ++e) ki[e] = f2mul(ki[e], rn2);
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) g[e] = f2pack(1.f, 1.f);
        float vv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) vv[e] = 0.f;
#pragma unroll
        for (int jj = 3; jj >= 0; --jj) {
          if (jj <= ii) {
            const int j = r0 + jj;
            const uint4 kr = ld8(sKr + j * DK);
            const float4 a0 = *reinterpret_cast<const float4 *>(sAl + al_off(j, c4));
            const float4 a1 = *reinterpret_cast<const float4 *>(sAl + al_off(j, 64 + c4));
            const uint64_t x0 = f2mul(g[0], bf2_to_f2(kr.x)), x1 = f2mul(g[1], bf2_to_f2(kr.y));
            const uint64_t x2 = f2mul(g[2], bf2_to_f2(kr.z)), x3 = f2mul(g[3], bf2_to_f2(kr.w));
            uint64_t sa = f2mul(ki[0], x0), sq = f2mul(qi[0], x0);
            sa = f2fma(ki[1], x1, sa); sq = f2fma(qi[1], x1, sq);
            sa = f2fma(ki[2], x2, sa); sq = f2fma(qi[2], x2, sq);
            sa = f2fma(ki[3], x3, sa); sq = f2fma(qi[3], x3, sq);
            const float2 fa = f2unpack(sa), fq = f2unpack(sq);
            vv[jj] = fa.x + fa.y;
            vv[4 + jj] = fq.x + fq.y;
            g[0] = f2mul(g[0], f2pack(a0.x, a0.y));
            g[1] = f2mul(g[1], f2pack(a0.z, a0.w));
            g[2] = f2mul(g[2], f2pack(a1.x, a1.y));
            g[3] = f2mul(g[3], f2pack(a1.z, a1.w));
          }
        }
#pragma unroll
        for (int m = 8, nn = 8; m > 1; m >>= 1, nn >>= 1) {
          const bool up = (sl & m) != 0;
#pragma unroll
          for (int e = 0; e < nn / 2; ++e) {
            const float keep = up ? vv[nn / 2 + e] : vv[e];
            const float send = up ? vv[e] : vv[nn / 2 + e];
            vv[e] = keep + __shfl_xor_sync(0xffffffffu, send, m);
          }
        }
        vv[0] += __shfl_xor_sync(0xffffffffu, vv[0], 1);
        if ((sl & 1) == 0) {
          const int idx = sl >> 1, jj = idx & 3;
          const float rj = GATED ? sRN[r0 + jj] : 1.f;  // column j's key norm
          if (idx >= 4) {
            if (jj <= ii) sM[i * RS + r0 + jj] = rj * vv[0];
          } else if (jj < ii) {
            sA[i * RS + r0 + jj] = sB[i] * rj * vv[0];
          }
        }
      }
    }
    if (!wait_all(&bar[0], ph, s_abort)) break;  // the first Gram has read its operands

    // ---------------- 3b. inside each 16-token sub-block b, a pair of
    // different 4-token groups factors at the boundary before i's group m:
    //   G_{i<-j} = G_{i<-4m-1} G_{4m-1<-j}          (token indices local to b)
    // with both factors bounded products, so the rows
    //   Lk4_i = k_i G_{i<-4m-1},  Lq4_i = q_i G_{i<-4m-1}           (m >= 1)
    // and the columns R4^(m)_j = k_j G_{4m-1<-j} (j < 4m) give all of them
    // as one more tensor-core product, in the buffers of the first: row
    // 32 (m - 1) + 8 b + 4 kind + u (kind 0: Lk4, 1: Lq4; u = i - 4m),
    // column off_m + 4 m b + j with off_m = 0, 16, 48. Thread (b = gq,
    // channel gc), which also writes gamma_i over its own alpha column.
    {
      float a[16], kr[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        a[u] = sAl[al_off(16 * gq + u, gc)];
        kr[u] = bf(sKr + (16 * gq + u) * DK + gc);
        if constexpr (GATED) kr[u] *= sRN[16 * gq + u];
      }
#pragma unroll
      for (int m = 1; m < 4; ++m) {
        float lk[4], lq[4], p = 1.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = 4 * m + u;
          p *= a[i];
          lk[u] = p * kr[i];
          lq[u] = p * bf(sQr + (16 * gq + i) * DK + gc);
        }
        st4x2_mn(GA, gc, 32 * (m - 1) + 8 * gq, DK, lk, lq, (lane >> 2) & 1);
      }
#pragma unroll
      for (int m = 1; m < 4; ++m) {
        float r[12], sfx = 1.f;
#pragma unroll
        for (int j = 4 * m - 1; j >= 0; --j) {
          r[j] = sfx * kr[j];
          sfx *= a[j];
        }
        const int col = (m == 1 ? 0 : (m == 2 ? 16 : 48)) + 4 * m * gq;
        if (m == 1) st4_f32(GB + off_mn_sw128b32_f32(gc, col, DK), r[0], r[1], r[2], r[3]);
        else st4x2_mn(GB, gc, col, DK, r, r + 4, (lane >> 2) & 1);
        if (m == 3) st4_f32(GB + off_mn_sw128b32_f32(gc, col + 8, DK), r[8], r[9], r[10], r[11]);
      }
      float gam = 1.f;  // gamma_i = prod_{s <= i} alpha_s, over alpha (read only here from now on)
      for (int b = 0; b < gq; ++b) gam *= sP[b * DK + gc];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        gam *= a[u];
        sAl[al_off(16 * gq + u, gc)] = gam;
      }
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < DK / 8; ++kk)
        mma_tf32_ss(tm + TP_G4, desc_mn_sw128b32_f32(sb + P_GA, DK, kk),
                    desc_mn_sw128b32_f32(sb + P_GB, DK, kk), ID_G, kk > 0);
      mma_commit(&bar[3]);
    }

    // ---------------- 4. Gram blocks out of TMEM: first the pairs of
    // different 16-token sub-blocks (while the second product runs) ...
    {
      // sub-block row I = qw + 1 sits in lane quarter qw (lanes 0-15 Lk rows,
      // 16-31 Lq rows); warp part takes columns 16 part .. 16 part + 15
      const int qw = warp & 3, part = warp >> 2;
      if (qw < 3 && part <= qw) {
        const int I = qw + 1, ii = lane & 15, i = 16 * I + ii;
        const int cb = 16 * part;
        float x[16];
        tmem_ld16(tm + lane_base + TP_G + (uint32_t)(8 * I * (I - 1) + cb), x);
        const float b = (lane >> 4) ? 1.f : sB[i];
        float *dst = ((lane >> 4) ? sM : sA) + i * RS + cb;
#pragma unroll
        for (int e = 0; e < 16; e += 4)
          *reinterpret_cast<float4 *>(dst + e) =
              make_float4(b * x[e], b * x[e + 1], b * x[e + 2], b * x[e + 3]);
      }
    }
    if (!wait_all(&bar[3], ph, s_abort)) break;
    // ... then those of different 4-token groups of one sub-block: warp
    // (lane quarter m - 1, sub-block b = warp / 4) reads the 4 m columns of
    // R4^(m) of block b; its lanes 8 b .. 8 b + 7 hold rows (kind, u).
    {
      const int qw = warp & 3, b = warp >> 2;
      if (qw < 3) {
        const int m = qw + 1;
        const uint32_t ta = tm + lane_base + TP_G4 + (uint32_t)((m == 1 ? 0 : (m == 2 ? 16 : 48)) + 4 * m * b);
        float x[12];
#pragma unroll
        for (int e = 0; e < 12; ++e) x[e] = 0.f;
        if (m == 1) {
          tmem_ld4(ta, x);
        } else {
          tmem_ld8(ta, x);
          if (m == 3) tmem_ld4(ta + 8, x + 8);
        }
        if ((lane >> 3) == b) {
          const int kind = (lane >> 2) & 1, u = lane & 3, i = 16 * b + 4 * m + u;
          const float sc = kind ? 1.f : sB[i];
          float *dst = (kind ? sM : sA) + i * RS + 16 * b;
#pragma unroll
          for (int e = 0; e < 12; e += 4)
            if (e < 4 * m)
              *reinterpret_cast<float4 *>(dst + e) =
                  make_float4(sc * x[e], sc * x[e + 1], sc * x[e + 2], sc * x[e + 3]);
        }
      }
    }
    fence_before_sync();
    __syncthreads();

    if (warp < NTP / 64) {  // warps 0..7 invert; named barrier 1 among them
      // ---------------- 5. T = (I + A)^{-1} by blocked forward substitution
      // diagonal 16x16 blocks T_II in two levels of 8: first the 8x8 diagonal
      // sub-blocks by forward substitution, thread (block b, half h, column
      // j), with row ii + 1 loaded while row ii is solved ...
      if (tid < C) {
        const int b = tid >> 4, h = (tid >> 3) & 1, j = tid & 7, o8 = 16 * b + 8 * h;
        const float *Ab = sA + o8 * RS + o8;
        float t[8], ar[8];
#pragma unroll
        for (int ii = 0; ii < 8; ++ii) t[ii] = (ii == j) ? 1.f : 0.f;
        {
          const float4 v = *reinterpret_cast<const float4 *>(Ab + RS);
          ar[0] = v.x; ar[1] = v.y; ar[2] = v.z; ar[3] = v.w;
        }
#pragma unroll
        for (int ii = 1; ii < 8; ++ii) {
          float cur[8];
#pragma unroll
          for (int l = 0; l < ii; ++l) cur[l] = ar[l];
          if (ii + 1 < 8) {
#pragma unroll
            for (int q4 = 0; q4 < (ii + 4) / 4; ++q4) {  // columns 0 .. ii of row ii + 1
              const float4 v = *reinterpret_cast<const float4 *>(Ab + (ii + 1) * RS + 4 * q4);
              ar[4 * q4] = v.x; ar[4 * q4 + 1] = v.y; ar[4 * q4 + 2] = v.z; ar[4 * q4 + 3] = v.w;
            }
          }
          if (ii > j) {
            float s = 0.f;
#pragma unroll
            for (int l = 0; l < ii; ++l)
              if (l >= j) s += cur[l] * t[l];
            t[ii] = -s;
          }
        }
#pragma unroll
        for (int ii = 0; ii < 8; ++ii) sT[(o8 + ii) * RS + o8 + j] = t[ii];
      }
      named_bar_sync(1, NTP / 2);
      // ... then the lower-left 8x8 block T21 = -T22 (A21 T11), thread
      // (block b, row r, column c); the upper-right block is zero
      {
        const int b = tid >> 6, r = (tid >> 3) & 7, c = tid & 7, ob = 16 * b;
        float x = 0.f;
#pragma unroll
        for (int m = 0; m < 8; ++m)
          if (m >= c) x += sA[(ob + 8 + r) * RS + ob + m] * sT[(ob + m) * RS + ob + c];
        sXT[b * 64 + r * 8 + c] = x;
        named_bar_sync(1, NTP / 2);
        float y = 0.f;
#pragma unroll
        for (int m = 0; m < 8; ++m)
          if (m <= r) y += sT[(ob + 8 + r) * RS + ob + 8 + m] * sXT[b * 64 + m * 8 + c];
        sT[(ob + 8 + r) * RS + ob + c] = -y;
        sT[(ob + r) * RS + ob + 8 + c] = 0.f;
      }
      named_bar_sync(1, NTP / 2);
      // off-diagonal blocks by doubling. Level 1 (16 -> 32): T_10 =
      // -T_11 (A_10 T_00) and T_32 = -T_33 (A_32 T_22), thread (block pair q,
      // row r, column pair cp); the upper-right blocks T_01, T_23 are zero.
      {
        const int q = tid >> 7, r = (tid >> 3) & 15, cp = tid & 7;
        const int J = 2 * q, I = 2 * q + 1, c = 16 * J + 2 * cp;
        float a[16];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const float4 u = *reinterpret_cast<const float4 *>(sA + (16 * I + r) * RS + 16 * J + 4 * q4);
          a[4 * q4] = u.x; a[4 * q4 + 1] = u.y; a[4 * q4 + 2] = u.z; a[4 * q4 + 3] = u.w;
        }
        float x0 = 0.f, x1 = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const float2 tv = *reinterpret_cast<const float2 *>(sT + (16 * J + m) * RS + c);
          x0 += a[m] * tv.x; x1 += a[m] * tv.y;
        }
        *reinterpret_cast<float2 *>(sXT + q * 256 + r * 16 + 2 * cp) = make_float2(x0, x1);
        named_bar_sync(1, NTP / 2);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {  // row r of T_II (zero above its diagonal)
          const float4 u = *reinterpret_cast<const float4 *>(sT + (16 * I + r) * RS + 16 * I + 4 * q4);
          a[4 * q4] = u.x; a[4 * q4 + 1] = u.y; a[4 * q4 + 2] = u.z; a[4 * q4 + 3] = u.w;
        }
        float y0 = 0.f, y1 = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const float2 xv = *reinterpret_cast<const float2 *>(sXT + q * 256 + m * 16 + 2 * cp);
          y0 += a[m] * xv.x; y1 += a[m] * xv.y;
        }
        *reinterpret_cast<float2 *>(sT + (16 * I + r) * RS + c) = make_float2(-y0, -y1);
        *reinterpret_cast<float2 *>(sT + (16 * J + r) * RS + 16 * I + 2 * cp) = make_float2(0.f, 0.f);
      }
      named_bar_sync(1, NTP / 2);
      // Level 2 (32 -> 64): T_hl = -T_hi (A_hl T_lo) over 32x32 blocks (rows
      // 32 .. 63, columns 0 .. 31). X = A_hl T_lo is kept in the unused
      // upper-right 32x32 block of T (rows 0 .. 31, columns 32 .. 63).
      // Thread = 2x2 tile; the zero block of T_lo (rows < 16, columns >= 16)
      // and that of T_hi (rows < 16, columns >= 16) are skipped.
      {
        const int ch = tid >> 7, tr = (tid >> 3) & 15, tc = tid & 7;
        const int r = 2 * tr, c = 16 * ch + 2 * tc;
        float x00 = 0.f, x01 = 0.f, x10 = 0.f, x11 = 0.f;
        for (int Lb = ch; Lb < 2; ++Lb) {
          float ra[16], rb[16];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const float4 u0 = *reinterpret_cast<const float4 *>(sA + (32 + r) * RS + 16 * Lb + 4 * q4);
            const float4 u1 = *reinterpret_cast<const float4 *>(sA + (33 + r) * RS + 16 * Lb + 4 * q4);
            ra[4 * q4] = u0.x; ra[4 * q4 + 1] = u0.y; ra[4 * q4 + 2] = u0.z; ra[4 * q4 + 3] = u0.w;
            rb[4 * q4] = u1.x; rb[4 * q4 + 1] = u1.y; rb[4 * q4 + 2] = u1.z; rb[4 * q4 + 3] = u1.w;
          }
#pragma unroll
          for (int l = 0; l < 16; ++l) {
            const float2 tv = *reinterpret_cast<const float2 *>(sT + (16 * Lb + l) * RS + c);
            x00 += ra[l] * tv.x; x01 += ra[l] * tv.y;
            x10 += rb[l] * tv.x; x11 += rb[l] * tv.y;
          }
        }
        *reinterpret_cast<float2 *>(sT + r * RS + 32 + c) = make_float2(x00, x01);
        *reinterpret_cast<float2 *>(sT + (r + 1) * RS + 32 + c) = make_float2(x10, x11);
      }
      named_bar_sync(1, NTP / 2);
      {
        const int rh = tid >> 7, tr = (tid >> 4) & 7, tc = tid & 15;
        const int r = 16 * rh + 2 * tr, c = 2 * tc;
        float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
        for (int Lb = 0; Lb <= rh; ++Lb) {
          float ta[16], tb[16];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const float4 u0 = *reinterpret_cast<const float4 *>(sT + (32 + r) * RS + 32 + 16 * Lb + 4 * q4);
            const float4 u1 = *reinterpret_cast<const float4 *>(sT + (33 + r) * RS + 32 + 16 * Lb + 4 * q4);
            ta[4 * q4] = u0.x; ta[4 * q4 + 1] = u0.y; ta[4 * q4 + 2] = u0.z; ta[4 * q4 + 3] = u0.w;
            tb[4 * q4] = u1.x; tb[4 * q4 + 1] = u1.y; tb[4 * q4 + 2] = u1.z; tb[4 * q4 + 3] = u1.w;
          }
#pragma unroll
          for (int l = 0; l < 16; ++l) {
            const float2 xv = *reinterpret_cast<const float2 *>(sT + (16 * Lb + l) * RS + 32 + c);
            y00 += ta[l] * xv.x; y01 += ta[l] * xv.y;
            y10 += tb[l] * xv.x; y11 += tb[l] * xv.y;
          }
        }
        *reinterpret_cast<float2 *>(sT + (32 + r) * RS + c) = make_float2(-y00, -y01);
        *reinterpret_cast<float2 *>(sT + (33 + r) * RS + c) = make_float2(-y10, -y11);
      }
      named_bar_sync(1, NTP / 2);
    } else {
      // ---------------- 5'. meanwhile (warps 8..15): the last MMA's B operand
      // [beta Khat | beta V], K-major (row n = output column, 4 tokens per
      // 16-byte store, 128 + DV rows), and Qhat over gamma
      // thread (channel pair cp, 16-token quarter), 8 tokens at a time, every
      // load ahead of the stores; the two rows' stores alternate on lane bit 2
      const int t = tid - NTP / 2;
      const bool sw = (lane >> 2) & 1;
      {
        const int c = 2 * (t & 63), j0 = 16 * (t >> 6);
#pragma unroll
        for (int h8 = 0; h8 < 16; h8 += 8) {
          float g0[8], g1[8], k0[8], k1[8], q0[8], q1[8], bb[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int i = j0 + h8 + e;
            const float2 gm = *reinterpret_cast<const float2 *>(sAl + al_off(i, c));
            const uint32_t kw = *reinterpret_cast<const uint32_t *>(sKr + i * DK + c);
            const uint32_t qw = *reinterpret_cast<const uint32_t *>(sQr + i * DK + c);
            g0[e] = gm.x; g1[e] = gm.y;
            k0[e] = __uint_as_float(kw << 16); k1[e] = __uint_as_float(kw & 0xffff0000u);
            q0[e] = __uint_as_float(qw << 16); q1[e] = __uint_as_float(qw & 0xffff0000u);
          }
#pragma unroll
          for (int e = 0; e < 8; e += 4) {
            const float4 b4 = *reinterpret_cast<const float4 *>(sB + j0 + h8 + e);
            bb[e] = b4.x; bb[e + 1] = b4.y; bb[e + 2] = b4.z; bb[e + 3] = b4.w;
          }
#pragma unroll
          for (int e = 0; e < 8; ++e)  // Qhat (fp32, in place)
            *reinterpret_cast<float2 *>(sAl + al_off(j0 + h8 + e, c)) = make_float2(g0[e] * q0[e], g1[e] * q1[e]);
#pragma unroll
          for (int g = 0; g < 8; g += 4) {
            float x0[4], x1[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float b0 = bb[g + e] * g0[g + e] * k0[g + e], b1 = bb[g + e] * g1[g + e] * k1[g + e];
              if constexpr (GATED) {
                b0 *= sRN[j0 + h8 + g + e];
                b1 *= sRN[j0 + h8 + g + e];
              }
              x0[e] = sw ? b1 : b0;
              x1[e] = sw ? b0 : b1;
            }
            st4_f32(GA + off_k_sw128_f32(c + (sw ? 1 : 0), j0 + h8 + g, DK + DV), x0[0], x0[1], x0[2], x0[3]);
            st4_f32(GA + off_k_sw128_f32(c + (sw ? 0 : 1), j0 + h8 + g, DK + DV), x1[0], x1[1], x1[2], x1[3]);
          }
        }
      }
      // beta V rows 128 .. 128 + DV: thread (channel pair cp, 16-token quarter);
      // the two rows' stores alternate their order on lane bit 2 (rows 2 cp
      // and 2 cp + 1 then cover all eight 16-byte slots of a swizzle line)
      const __nv_bfloat16 *sV = reinterpret_cast<const __nv_bfloat16 *>(sm + P_V);
      const int npair = DV / 2;
      if (t < 4 * npair) {
        const int cv = 2 * (t % npair), j0 = 16 * (t / npair);
        float lo[16], hi[16], bb[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const uint32_t w = *reinterpret_cast<const uint32_t *>(sV + (j0 + e) * DV + cv);
          lo[e] = __uint_as_float(w << 16);
          hi[e] = __uint_as_float(w & 0xffff0000u);
        }
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          const float4 b4 = *reinterpret_cast<const float4 *>(sB + j0 + e);
          bb[e] = b4.x; bb[e + 1] = b4.y; bb[e + 2] = b4.z; bb[e + 3] = b4.w;
        }
#pragma unroll
        for (int g = 0; g < 16; g += 4) {
          float x0[4], x1[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            x0[e] = bb[g + e] * (sw ? hi[g + e] : lo[g + e]);
            x1[e] = bb[g + e] * (sw ? lo[g + e] : hi[g + e]);
          }
          st4_f32(GA + off_k_sw128_f32(DK + cv + (sw ? 1 : 0), j0 + g, DK + DV), x0[0], x0[1], x0[2], x0[3]);
          st4_f32(GA + off_k_sw128_f32(DK + cv + (sw ? 0 : 1), j0 + g, DK + DV), x1[0], x1[1], x1[2], x1[3]);
        }
      }
      // Qhat rows 0..63 into tensor memory (lanes 0..63, columns TP_QH ..
      // TP_QH + 127), so that alpha's buffer is free from here on: warps 8, 9
      // take columns 0..63 and warps 12, 13 columns 64..127, a row per lane
      named_bar_sync(2, NTP / 2);  // every Qhat value of this phase is in place
      if ((warp & 3) < 2) {
        const int row = 32 * (warp & 3) + lane, c0 = 64 * ((warp >> 2) & 1);
#pragma unroll
        for (int hh = 0; hh < 64; hh += 32) {
          float x[32];
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 qv = *reinterpret_cast<const float4 *>(sAl + al_off(row, c0 + hh + e));
            x[e] = qv.x; x[e + 1] = qv.y; x[e + 2] = qv.z; x[e + 3] = qv.w;
          }
          tmem_st32(tm + lane_base + TP_QH + (uint32_t)(c0 + hh), x);
        }
        tmem_wait_st();
      }
      fence_before_sync();
    }
    __syncthreads();

    // ---------------- 6. [M T ; T] = [M ; I] x T on the tensor cores, into TMEM
    for (int task = tid; task < 128 * 16; task += NTP) {  // A0 = [M ; I]
      const int row = task >> 4, k4 = (task & 15) * 4;
      float x[4];
      if (row < C) {
        const float4 mv = *reinterpret_cast<const float4 *>(sM + row * RS + k4);
        x[0] = mv.x; x[1] = mv.y; x[2] = mv.z; x[3] = mv.w;
#pragma unroll
        for (int e = 0; e < 4; ++e) if (k4 + e > row) x[e] = 0.f;
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = (k4 + e == row - C) ? 1.f : 0.f;
      }
      st4_f32(sm + P_A0 + off_k_sw128_f32(row, k4, 128), x[0], x[1], x[2], x[3]);
    }
    for (int task = tid; task < C * 16; task += NTP) {  // B0 = T (row l, columns j)
      const int l = task >> 4, j4 = (task & 15) * 4;
      const float4 tv = *reinterpret_cast<const float4 *>(sT + l * RS + j4);
      float x[4] = {tv.x, tv.y, tv.z, tv.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) if (j4 + e > l) x[e] = 0.f;
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
    // gamma, Qhat (now in tensor memory) and beta have had their last reads:
    // the next item's alpha and beta may come in
    if (nxt.y > 0) {
      issue_gates(nxt.x, nxt.y, nit % H);
      raw_for = nit;
      ahead |= 2;
    }
    if (!wait_all(&bar[1], ph, s_abort)) break;
    if ((warp & 3) < 2) {  // rows of M T: round the fp32 accumulator to tf32
      const uint32_t ta = tm + lane_base + TP_AD5 + (uint32_t)(16 * (warp >> 2));
      float x[16];
      tmem_ld16(ta, x);
#pragma unroll
      for (int e = 0; e < 16; ++e) x[e] = to_tf32(x[e]);
      tmem_st16(ta, x);
    }
    tmem_wait_st();
    fence_before_sync();
    __syncthreads();

    // ---------------- 7. [M T ; T] x [beta Khat | beta V], staged, -> workspace
    if (tid == 0) {
      fence_after_sync();
      const uint32_t id5 = idesc_tf32(128, DK + DV, 0, 0);
#pragma unroll
      for (int kk = 0; kk < C / 8; ++kk)
        mma_tf32_ts(tm + TP_D5, tm + TP_AD5 + (uint32_t)(8 * kk),
                    desc_k_sw128_f32(sb + P_GA, DK + DV, kk), id5, kk > 0);
      mma_commit(&bar[2]);
    }
    // while D5 runs: the q, k, v buffers' last reader ([M ; I] x T) is done,
    // so the next item's rows may come in
    if (nxt.y > 0) {
      issue_qkv(nxt.x, nit % H);
      ahead |= 1;
    }
    if (!wait_all(&bar[2], ph, s_abort)) break;
    {
      const int qw = warp & 3, cg = warp >> 2, row = 32 * qw + lane;
      {  // [Qtil ; W] columns 32 cg .. 32 cg + 31, tf32, K-major sw128 image
        const int cb = 32 * cg;
        float x[32];
        tmem_ld32(tm + lane_base + TP_D5 + (uint32_t)cb, x);
        if (row < C) {  // warp-uniform (lane quarters 0, 1)
          float qh[32];
          tmem_ld32(tm + lane_base + TP_QH + (uint32_t)cb, qh);
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] = qh[e] - x[e];
        }
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          st4_f32(sm + P_GA + off_k_sw128_f32(row, cb + e, DK), x[e], x[e + 1], x[e + 2], x[e + 3]);
      }
      // The workspace stores go in three groups, in the order the next item
      // writes over their sources: [Qtil ; W] columns 0..95 (the Gram rows'
      // buffer); its columns 96..127 and the M Ut rows (the R stack's); the Ut
      // rows (over A and M). The [Qtil ; W] image is complete here, so its
      // stores start while the [M Ut ; Ut] rows are staged.
      fence_async_smem();
      __syncthreads();
      if (tid == 0) {
        bulk_s2g(wsb + WS_A1, sm + P_GA, 49152);
        bulk_commit();
        bulk_s2g(wsb + WS_A1 + 49152, sm + P_GA + 49152, 16384);
      }
      // [M Ut ; Ut] rows, fp32, pieces swizzled by row (Ut rows over A, M)
      for (int cb = 32 * cg + DK; cb < DK + DV; cb += 128) {
        float x[32];
        tmem_ld32(tm + lane_base + TP_D5 + (uint32_t)cb, x);
        uint8_t *dst = row < C ? sm + P_OU + (size_t)row * DV * 4 : sm + P_A + (size_t)(row - C) * DV * 4;
        const int pc0 = (cb - DK) >> 2;
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4 *>(dst + 16 * ou_piece(row, pc0 + (e >> 2))) =
              make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
      }
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      bulk_s2g(wsb + WS_OU, sm + P_OU, 64u * DV * 4u);
      bulk_commit();
      bulk_s2g(wsb + WS_OU + 64u * DV * 4u, sm + P_A, 64u * DV * 4u);
      bulk_commit();
    }
  } while (0);
  if (*s_abort) break;  // CTA-uniform: read after a barrier
  ph ^= 1u;
  cur = nxt;
  }  // item loop

  // After an abort, copies still in flight land before shared memory is
  // released: those issued for the next item complete phase ph ^ 1; an
  // item's own, if waiting for them is what timed out, phase ph (an already
  // completed phase is not waited for).
  if (*s_abort) {
    for (int b = 0; b < 2; ++b) wait_in(b, ((ahead >> b) & 1) ? ph ^ 1u : ph);
  }
  cp_async_wait_all();  // copies issued ahead land before shared memory is released
  if (tid == 0) {
    if (*s_abort) flag_error(err, kErrMbarTimeout);
    bulk_wait_read0();  // shared memory stays valid until the stores read it
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    fence_after_sync();
    tmem_dealloc(tm, TP_COLS);
  }
}

// ---------------------------------------------------------------- scan kernel
// 4 consumer warps (thread r = state row r of the 128 x 32 tile) and one
// producer warp. The producer bulk-copies each chunk's [Qtil ; W] and Kbar^T
// images into a shared-memory landing buffer two chunks ahead and moves them
// into tensor memory (tcgen05.cp, 128 lanes x 8 columns per K-step), so both
// MMAs of the state chain take their A operand from tensor memory and read
// only the small B operand (S or U) from shared memory. Each product is
// issued by two threads in different warps, each taking half of the K-steps
// into its own accumulator (the chain is bound by how fast MMAs are issued,
// not by the tensor pipe); readers add the two halves.
constexpr int NTS = 160, NCONS = 128;
constexpr uint32_t S_A1 = 0;          // 2 x 65536 [Qtil ; W] landing buffers
constexpr uint32_t S_A2 = 131072;     // 2 x 32768 Kbar^T landing buffers
constexpr uint32_t S_S = 196608;      // 16384 S, B of D1 (K128 x N32 MN)
constexpr uint32_t S_U = 212992;      //  8192 U, B of D2 (K64 x N32 MN)
constexpr uint32_t S_BAR = 221184;    //   128 mbarriers [0..9] + TMEM address + flag
constexpr uint32_t S_SMEM = 221312 + 1024;
// mbarriers: landed[2] (bulk copy into landing buffer b), ready[2] (buffer b
// in tensor memory), free[2] (the MMAs that read tensor-memory buffer b are
// done), D1, D2. Each completes once per use of its buffer or chunk (free,
// D1 and D2 after one commit from each of the two issuers), and no waiter
// can be two completions behind, so parity waits are exact.
enum { B_LANDED = 0, B_READY = 2, B_FREE = 4, B_D1 = 6, B_D2 = 7, NBAR = 8 };
// tensor memory: D1, D2 accumulators (first issuer's halves); [Qtil ; W] and
// Kbar^T, two buffers each; the second issuer's D1, D2 halves
constexpr uint32_t TS_D1 = 0, TS_D2 = 32, TS_A1 = 64, TS_A2 = 320, TS_D1B = 448, TS_D2B = 480;
constexpr uint32_t TS_COLS = 512;
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
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + S_BAR);
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + S_BAR + 8 * NBAR);
  volatile int *s_abort = reinterpret_cast<volatile int *>(sm + S_BAR + 8 * NBAR + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int vt = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int c0 = vt * DVT;
  int bos, eos;
  seq_bounds(cu, n, T, T_total, err, bos, eos);
  const int nch = (eos - bos + C - 1) / C;
  const int base = slot_base(cu, n, T);
  const size_t st_base = ((size_t)n * H + h) * DK * DV;
  const uint32_t wsz = ws_block_bytes(DV);
  // Consumer threads ISS and ISS2 (lane 0 of the two U-half warps) issue the
  // MMAs, K-steps 0 .. K/2-1 and K/2 .. K-1 respectively.
  constexpr int ISS = C, ISS2 = C + 32;
  constexpr int PROD = NCONS;  // producer thread (lane 0 of warp 4)

  if (warp == 0) {
    tmem_alloc(s_tmem, TS_COLS);
    tmem_relinquish();
  }
  if (tid == PROD) {
    for (int i = 0; i < NBAR; ++i) mbar_init(&bar[i], i >= B_FREE ? 2 : 1);  // free, D1, D2: two issuers
    fence_mbar_init();
  }
  if (tid == 0) *s_abort = 0;
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = *s_tmem;

  if (warp == NCONS / 32) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      auto load = [&](int c) {
        const int b = c & 1;
        const uint8_t *blk = ws + ((size_t)(base + c) * H + h) * wsz;
        mbar_arrive_expect_tx(&bar[B_LANDED + b], LOAD_BYTES);
        bulk_g2s(sm + S_A1 + b * 65536, blk + WS_A1, 65536, &bar[B_LANDED + b]);
        bulk_g2s(sm + S_A2 + b * 32768, blk + WS_A2, 32768, &bar[B_LANDED + b]);
      };
      if (nch > 0) load(0);
      if (nch > 1) load(1);
      for (int c = 0; c < nch; ++c) {
        const int b = c & 1;
        const uint32_t use = (uint32_t)(c >> 1);  // how often buffer b was used before
        bool ok = mbar_wait(&bar[B_LANDED + b], use & 1u);
        if (ok && c >= 2) ok = mbar_wait(&bar[B_FREE + b], (use - 1) & 1u);
        if (!ok) {
          *s_abort = 1;
          break;
        }
        fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < DK / 8; ++kk)
          tmem_cp_128x256b(tm + TS_A1 + b * 128 + 8 * kk,
                           desc_k_sw128_f32(sb + S_A1 + b * 65536, 128, kk));
#pragma unroll
        for (int kk = 0; kk < C / 8; ++kk)
          tmem_cp_128x256b(tm + TS_A2 + b * 64 + 8 * kk,
                           desc_k_sw128_f32(sb + S_A2 + b * 32768, 128, kk));
        mma_commit(&bar[B_READY + b]);
        if (c + 2 < nch) {  // landing buffer b again, once the copies have read it
          if (!mbar_wait(&bar[B_READY + b], use & 1u)) {
            *s_abort = 1;
            break;
          }
          load(c + 2);
        }
        if (*s_abort) break;
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
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
      }
#pragma unroll
      for (int e = 0; e < DVT; e += 8) st4x2_mn(sm + S_S, r, e, DK, S + e, S + e + 4, (lane >> 2) & 1);
    }
    fence_async_smem();
    named_bar_sync(2, NCONS);

    // this thread's row of [M Ut ; Ut] (d_v tile) and gamma of its state row,
    // read one chunk ahead so the loads overlap the previous chunk's MMAs
    float ou_next[DVT], gc_next = 0.f;
    auto load_rows = [&](int c) {
      const uint8_t *blk = ws + ((size_t)(base + c) * H + h) * wsz;
      const float *src = reinterpret_cast<const float *>(blk + WS_OU) + (size_t)tid * DV;
#pragma unroll
      for (int e = 0; e < DVT; e += 4) {
        const float4 x = __ldg(reinterpret_cast<const float4 *>(src + 4 * ou_piece(tid, (c0 + e) >> 2)));
        ou_next[e] = x.x; ou_next[e + 1] = x.y; ou_next[e + 2] = x.z; ou_next[e + 3] = x.w;
      }
      gc_next = __ldg(reinterpret_cast<const float *>(blk + ws_gamma_off(DV)) + tid);
    };
    if (nch > 0) load_rows(0);

    // Per chunk one barrier of the consumers (the state tile is complete in
    // shared memory); the U half hands D2 over through named barrier 1 while
    // the output half stores O. A timed-out wait only sets the abort flag,
    // read after the chunk's barrier.
    for (int c = 0; c < nch; ++c) {
      const int b = c & 1;
      const int t0 = bos + C * c, L = min(C, eos - t0);
      if (tid == ISS || tid == ISS2) {  // D1 = [Qtil ; W] x S, K split over two issuers
        const int h2 = tid == ISS2;
        if (!mbar_wait(&bar[B_READY + b], (uint32_t)(c >> 1) & 1u)) *s_abort = 1;
        fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk)
          mma_tf32_ts(tm + (h2 ? TS_D1B : TS_D1), tm + TS_A1 + b * 128 + 8 * (kk + 8 * h2),
                      desc_mn_sw128b32_f32(sb + S_S, DK, kk + 8 * h2), ID_D1, kk > 0);
        mma_commit(&bar[B_D1]);
      }
      // this chunk's rows (loaded one chunk ahead) and the next chunk's loads
      // come after the MMA issue, so that the issuing threads reach it first
      float ou[DVT];
#pragma unroll
      for (int e = 0; e < DVT; ++e) ou[e] = ou_next[e];
      const float gc = gc_next;
      if (c + 1 < nch) load_rows(c + 1);
      if (!mbar_wait(&bar[B_D1], (uint32_t)c & 1u)) *s_abort = 1;
      fence_after_sync();
      float d1[32];
      {
        float d1b[32];
        tmem_ld32(tm + lane_base + TS_D1, d1);
        tmem_ld32(tm + lane_base + TS_D1B, d1b);
#pragma unroll
        for (int e = 0; e < 32; ++e) d1[e] += d1b[e];
      }
      if (tid >= C) {  // U = Ut - W S, then D2 = Kbar^T x U
        const int j = tid - C;
        float u[DVT];
#pragma unroll
        for (int e = 0; e < DVT; ++e) u[e] = ou[e] - d1[e];
#pragma unroll
        for (int e = 0; e < DVT; e += 8) st4x2_mn(sm + S_U, j, e, C, u + e, u + e + 4, (lane >> 2) & 1);
        fence_async_smem();
        named_bar_sync(1, NCONS - C);
        if (tid == ISS || tid == ISS2) {
          const int h2 = tid == ISS2;
          fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < C / 16; ++kk)
            mma_tf32_ts(tm + (h2 ? TS_D2B : TS_D2), tm + TS_A2 + b * 64 + 8 * (kk + 4 * h2),
                        desc_mn_sw128b32_f32(sb + S_U, C, kk + 4 * h2), ID_D2, kk > 0);
          mma_commit(&bar[B_D2]);
          mma_commit(&bar[B_FREE + b]);  // tensor-memory buffer b may be refilled
        }
      } else {  // output rows, while D2 runs
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
      }
      if (!mbar_wait(&bar[B_D2], (uint32_t)c & 1u)) *s_abort = 1;
      fence_after_sync();
      {
        float d2[32];
        {
          float d2b[32];
          tmem_ld32(tm + lane_base + TS_D2, d2);
          tmem_ld32(tm + lane_base + TS_D2B, d2b);
#pragma unroll
          for (int e = 0; e < 32; ++e) d2[e] += d2b[e];
        }
#pragma unroll
        for (int e = 0; e < DVT; ++e) S[e] = gc * S[e] + d2[e];
#pragma unroll
        for (int e = 0; e < DVT; e += 8) st4x2_mn(sm + S_S, tid, e, DK, S + e, S + e + 4, (lane >> 2) & 1);
      }
      fence_async_smem();
      fence_before_sync();
      named_bar_sync(2, NCONS);
      if (*s_abort) break;
    }
    // the last two buffer-free commits are never waited for by the producer:
    // let their arrivals land before shared memory is released
    if (tid == ISS && !*s_abort) {
      for (int c = max(nch - 2, 0); c < nch; ++c)
        if (!mbar_wait(&bar[B_FREE + (c & 1)], (uint32_t)(c >> 1) & 1u)) *s_abort = 1;
    }
    if (!*s_abort && sfin) {
      const int r = tid;
#pragma unroll
      for (int e = 0; e < DVT; e += 4)
        *reinterpret_cast<float4 *>(sfin + st_base + (size_t)r * DV + c0 + e) =
            make_float4(S[e], S[e + 1], S[e + 2], S[e + 3]);
    }
  }

  fence_before_sync();
  __syncthreads();
  if (*s_abort) {
    if (tid == 0) flag_error(err, kErrMbarTimeout);
    // let in-flight copies and MMAs drain (bounded) before shared memory and
    // tensor memory are released
    if (tid == PROD)
      for (int i = 0; i < NBAR; ++i) {
        (void)mbar_wait(&bar[i], 0, 100000000LL);
        (void)mbar_wait(&bar[i], 1, 100000000LL);
      }
    __syncthreads();
  }
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
  return slot_table_off(slots, (size_t)H, dv) + slot_table_bytes(slots);
}

// SM count of the current device (looked up once per device).
static int sm_count() {
  static std::mutex mu;
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lk(mu);
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

// cuTensorMapEncodeTiled, reached through the runtime (no link against the
// driver library).
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Tensor map over a [T_total, H, d] row-major tensor (dims d, H, T_total,
// innermost first) whose box is `box0` elements of one head's row by 64
// tokens, laid out densely in shared memory. box0 may exceed d: those
// elements are filled with zeros.
static bool encode_rows(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int esize,
                        int d, int H, int T_total, int box0) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T_total};
  const cuuint64_t strides[2] = {(cuuint64_t)d * esize, (cuuint64_t)H * d * esize};
  const cuuint32_t box[3] = {(cuuint32_t)box0, 1u, (cuuint32_t)C};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_fwd_tc(int dv, const void *q, const void *k, const void *v,
                          const void *alpha, const float *beta,
                          const float *s0, float *sf, void *o,
                          const int32_t *cu, int N, int T, int T_total, int H,
                          float scale, GateArgs g, void *ws, unsigned int *err,
                          cudaStream_t st) {
  if (!fwd_tc_supported(DK, dv, C, CKDA_BF16)) return cudaErrorInvalidValue;
  auto prep = g.on ? ckda_chunk_prep_kernel<true> : ckda_chunk_prep_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(
      prep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P_SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(ckda_chunk_scan_kernel,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S_SMEM);
  if (e != cudaSuccess) return e;
  const int slots = T_total / C + N;
  if (slots > 0 && T_total > 0) {
    int2 *tab = reinterpret_cast<int2 *>((uint8_t *)ws + slot_table_off(slots, H, dv));
    ckda_slot_table_kernel<<<(slots + 255) / 256, 256, 0, st>>>(cu, N, T, T_total, slots,
                                                               tab, err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const long long items = (long long)slots * H;
    if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
    const int grid = (int)std::min<long long>(items, (long long)sm_count());
    // input boxes: q, k (128 channels), v (d_v), and alpha (128 channels padded
    // to the 132-float shared row) or, with the fused prologue, its bf16 logits
    CUtensorMap mq, mk, mv, ma;
    const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (!encode_rows(&mq, q, bf, 2, DK, H, T_total, DK) ||
        !encode_rows(&mk, k, bf, 2, DK, H, T_total, DK) ||
        !encode_rows(&mv, v, bf, 2, dv, H, T_total, dv) ||
        !(g.on ? encode_rows(&ma, alpha, bf, 2, DK, H, T_total, DK)
               : encode_rows(&ma, alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, DK, H, T_total, AL_S)))
      return cudaErrorInvalidValue;
    prep<<<grid, NTP, P_SMEM, st>>>(beta, tab, (int)items, H, dv, g, (uint8_t *)ws, err,
                                     mq, mk, mv, ma);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  ckda_chunk_scan_kernel<<<dim3(dv / DVT, H, N), NTS, S_SMEM, st>>>(
      s0, sf, (__nv_bfloat16 *)o, cu, T, T_total, H, dv, scale, (const uint8_t *)ws, err);
  return cudaGetLastError();
}

}  // namespace ckda
