// Thin wrappers over the sm_100a PTX used by the tensor-core kernels:
// tcgen05 (TMEM allocation, MMA, commit, TMEM loads), mbarriers with bounded
// waits, proxy fences, and the shared-memory operand layouts / descriptors of
// the UMMA canonical forms (K-major and MN-major, 128-byte swizzle or none).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "ckda_common.cuh"

namespace ckda {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------ operand layouts
// Byte offsets inside an operand tile whose base is 1024-byte aligned.
// bf16 elements; a "row" of the K-major form is one M (or N) index.

// K-major, 128B swizzle: atoms of 8 rows x 64 K-elements (1024 B); K atoms
// are ROWS*128 bytes apart. Both row-parallel and K-parallel 16-byte (or
// 2-byte) accesses are bank-conflict free.
__device__ __forceinline__ uint32_t off_k_sw128(int row, int k, int rows) {
  return (uint32_t)((k >> 6) * (rows * 128) + (row >> 3) * 1024 + (row & 7) * 128 +
                    ((((k & 63) >> 3) ^ (row & 7)) << 4) + ((k & 7) << 1));
}
// MN-major, 128B swizzle: atoms of 8 K-rows x 64 MN-elements; MN atoms are
// ktot*128 bytes apart (LBO), 8-row K groups 1024 bytes apart (SBO).
__device__ __forceinline__ uint32_t off_mn_sw128(int k, int mn, int ktot) {
  return (uint32_t)((mn >> 6) * (ktot * 128) + (k >> 3) * 1024 + (k & 7) * 128 +
                    ((((mn & 63) >> 3) ^ (k & 7)) << 4) + ((mn & 7) << 1));
}
// MN-major, no swizzle: core matrices of 8 K-rows x 8 MN-elements (128 B);
// K groups 128 bytes apart (LBO), MN groups ktot*16 bytes apart (SBO).
__device__ __forceinline__ uint32_t off_mn_none(int k, int mn, int ktot) {
  return (uint32_t)((mn >> 3) * (ktot * 16) + (k >> 3) * 128 + (k & 7) * 16 +
                    ((mn & 7) << 1));
}

// Shared-memory matrix descriptor (tcgen05 format: version 1 at bits 46-47).
__device__ __forceinline__ uint64_t make_desc(uint32_t saddr, uint32_t lbo,
                                              uint32_t sbo, uint32_t layout) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) |
         ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) |
         ((uint64_t)(layout & 7u) << 61);
}
constexpr uint32_t kLayoutNone = 0, kLayoutSw128B32 = 1, kLayoutSw128 = 2;

// descriptor of K-step kk (16 elements) for each layout
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t base, int rows, int kk) {
  return make_desc(base + (uint32_t)((kk >> 2) * rows * 128 + (kk & 3) * 32), 16,
                   1024, kLayoutSw128);
}
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t base, int ktot, int kk) {
  return make_desc(base + (uint32_t)(kk * 2048), (uint32_t)(ktot * 128), 1024,
                   kLayoutSw128);
}
__device__ __forceinline__ uint64_t desc_mn_none(uint32_t base, int ktot, int kk) {
  return make_desc(base + (uint32_t)(kk * 256), 128, (uint32_t)(ktot * 16),
                   kLayoutNone);
}

// 32-bit (tf32) element variants: a 128-byte swizzle row holds 32 elements.
// K-major: atoms of 8 rows x 32 K-elements; K atoms are rows*128 bytes apart.
__device__ __forceinline__ uint32_t off_k_sw128_f32(int row, int k, int rows) {
  return (uint32_t)((k >> 5) * (rows * 128) + (row >> 3) * 1024 + (row & 7) * 128 +
                    ((((k & 31) >> 2) ^ (row & 7)) << 4) + ((k & 3) << 2));
}
// MN-major tf32 operands take only the "128B swizzle with 32B atomicity" form:
// atoms of 4 K-rows x 32 MN-elements (512 B), 32-byte chunks XOR-ed with the
// row index (mod 4); 4-row K groups 512 bytes apart (SBO), MN atoms
// ktot*128 bytes apart (LBO).
__device__ __forceinline__ uint32_t off_mn_sw128b32_f32(int k, int mn, int ktot) {
  return (uint32_t)((mn >> 5) * (ktot * 128) + (k >> 2) * 512 + (k & 3) * 128 +
                    ((((mn & 31) >> 3) ^ (k & 3)) << 5) + ((mn & 7) << 2));
}
// descriptors of K-step kk (8 tf32 elements = 32 bytes)
__device__ __forceinline__ uint64_t desc_k_sw128_f32(uint32_t base, int rows, int kk) {
  return make_desc(base + (uint32_t)((kk >> 2) * rows * 128 + (kk & 3) * 32), 16,
                   1024, kLayoutSw128);
}
__device__ __forceinline__ uint64_t desc_mn_sw128b32_f32(uint32_t base, int ktot, int kk) {
  return make_desc(base + (uint32_t)(kk * 1024), (uint32_t)(ktot * 128), 512,
                   kLayoutSw128B32);
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) |
         ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Instruction descriptor, kind::tf32: tf32 A and B, fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)a_mn << 15) |
         ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// fp32 -> tf32 (round to nearest, ties away), kept in a 32-bit container.
__device__ __forceinline__ float to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// ------------------------------------------------------------ tcgen05
// D (TMEM) (+)= A (smem) x B (smem), tf32 inputs.
__device__ __forceinline__ void mma_tf32_ss(uint32_t d_tmem, uint64_t a, uint64_t b,
                                            uint32_t idesc, uint32_t accumulate) {
  const uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t"
      "}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(m0), "r"(m1), "r"(m2),
      "r"(m3));
}
// D (TMEM) (+)= A (TMEM, K-major: lane = row, column = k) x B (smem), tf32.
__device__ __forceinline__ void mma_tf32_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                            uint32_t idesc, uint32_t accumulate) {
  const uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t"
      "}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate), "r"(m0), "r"(m1), "r"(m2),
      "r"(m3));
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b,
                                         uint32_t idesc, uint32_t accumulate) {
  const uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t"
      "}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(m0), "r"(m1), "r"(m2),
      "r"(m3));
}

// Copy a 128-row x 256-bit (8 x 32-bit) matrix from shared memory, described
// like an MMA operand, into 128 lanes x 8 columns of tensor memory (lane =
// row). Completion is tracked by tcgen05.commit like an MMA.
__device__ __forceinline__ void tmem_cp_128x256b(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.128x256b [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// Arrive on an mbarrier when every MMA (or tensor-memory copy) issued so far
// by this thread is done.
__device__ __forceinline__ void mma_commit(uint64_t *mbar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(mbar))
      : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 consecutive 32-bit columns; thread t gets lane (base+t).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
        "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
        "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]),
        "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// 32 lanes x 8 (x4) consecutive columns, into v[0..7] (v[0..3]).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float *v) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
        "=r"(r[6]), "=r"(r[7])
      : "r"(taddr));
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, float *v) {
  uint32_t r[4];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}
// 32 lanes x 16 consecutive columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
        "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
        "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// 32 lanes x 32 consecutive columns from registers; thread t writes lane (base+t).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

// 32 lanes x 16 consecutive columns from registers.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}

// ------------------------------------------------------------ mbarriers
__device__ __forceinline__ void mbar_init(uint64_t *mbar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(mbar)),
               "r"(count)
               : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *mbar, uint32_t phase) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(mbar)), "r"(phase)
      : "memory");
  return done != 0;
}
// Bounded wait: gives up after ~limit_cycles SM clocks and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t *mbar, uint32_t phase,
                                          long long limit_cycles = 4000000000LL) {
  if (mbar_try_wait(mbar, phase)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(mbar, phase)) {
    if (clock64() - t0 > limit_cycles) return false;
  }
  return true;
}

// Plain arrival of this thread on an mbarrier.
__device__ __forceinline__ void mbar_arrive(uint64_t *mbar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(mbar)) : "memory");
}
// Barrier among the `count` threads (a multiple of 32) that use named barrier `id`.
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Expect `bytes` of asynchronous transactions on an mbarrier (one arrival).
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *mbar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(mbar)),
               "r"(bytes)
               : "memory");
}
// Bulk copy global -> shared (this CTA), completion counted on an mbarrier.
// Both addresses 16-byte aligned, bytes % 16 == 0. No multicast.
__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src, uint32_t bytes,
                                         uint64_t *mbar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst_smem)),
      "l"(src), "r"(bytes), "r"(smem_u32(mbar))
      : "memory");
}

// Tiled 3-D tensor copy global -> shared (this CTA, no multicast) through a
// tensor map `map` (a __grid_constant__ kernel parameter), box origin
// (x, y, z) in elements, innermost first; x * element size must be a multiple
// of 16 bytes. Elements outside the tensor are written as zero. Completion:
// the whole box's bytes are counted on the mbarrier.
__device__ __forceinline__ void tma_load_3d(void *dst_smem, const void *map, int x, int y, int z,
                                            uint64_t *mbar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst_smem)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(mbar))
      : "memory");
}

// Bulk copy shared (this CTA) -> global, tracked in this thread's bulk
// async-group. Both addresses 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_s2g(void *dst, const void *src_smem, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_u32(src_smem)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until every bulk store this thread committed has finished reading its
// shared-memory source (the source may then be overwritten).
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until at most N of this thread's most recently committed bulk groups
// are still reading their shared-memory sources (groups complete in commit
// order, so every older group has finished reading).
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Per-thread asynchronous copy of one 4-byte element global -> shared
// (cp.async, no registers in between; both addresses 4-byte aligned).
// Completion: cp_async_commit() groups this thread's copies,
// cp_async_wait_all() waits for all of them.
__device__ __forceinline__ void cp_async4(void *dst_smem, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst_smem)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Prefetch the cache line holding p into L2 (no data returned).
__device__ __forceinline__ void prefetch_line_l2(const void *p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Generic-proxy shared-memory writes -> visible to the async proxy (MMA).
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------ packed fp32 pairs
// Two fp32 values in one 64-bit register pair, for the sm_100 paired fp32
// instructions (each rounds like its scalar form).
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 f2unpack(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t f2mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
// a bf16 pair (element 0 in the low half) -> the fp32 pair (exact)
__device__ __forceinline__ uint64_t bf2_to_f2(uint32_t w) {
  return f2pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// 8 floats -> 8 bf16 packed in 16 bytes.
__device__ __forceinline__ uint4 pack8_bf16(const float *x) {
  uint4 r;
  __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]);
  __nv_bfloat162 b = __floats2bfloat162_rn(x[2], x[3]);
  __nv_bfloat162 c = __floats2bfloat162_rn(x[4], x[5]);
  __nv_bfloat162 d = __floats2bfloat162_rn(x[6], x[7]);
  r.x = *reinterpret_cast<uint32_t *>(&a);
  r.y = *reinterpret_cast<uint32_t *>(&b);
  r.z = *reinterpret_cast<uint32_t *>(&c);
  r.w = *reinterpret_cast<uint32_t *>(&d);
  return r;
}

}  // namespace tc
}  // namespace ckda
