// umma.cuh -- the sm_100a tensor-core path: tcgen05 MMAs reading bf16
// operands from shared memory and accumulating f32 in tensor memory (TMEM).
//
// Operand layout (no swizzle, "core matrices" of 8 rows x 16 bytes): a tile
// of R rows by K bf16 columns, K-major, keeps element (r, k) at byte
//   (r / 8) * (K * 16) + (k / 8) * 128 + (r % 8) * 16 + (k % 8) * 2.
// One MMA takes 16 columns of K (two core matrices), so successive K-steps
// advance the descriptor start by 256 bytes; LBO = 128 B separates the two K
// halves and SBO = K * 16 B the 8-row groups.  The same bytes read with rows
// as the K dimension form an MN-major operand: SBO = 128 B between 8-wide MN
// groups, LBO = MN * 16 B between 8-deep K groups, a K-step then advancing by
// 2 * LBO.
//
// f32 values enter as three bf16 parts, v = v0 + v1 + v2 (each part the bf16
// rounding of what the previous parts leave), about 24 bits in all; a product
// takes the six part products whose order is above 2^-24 (a0b0, a0b1, a1b0,
// a0b2, a1b1, a2b0), added smallest first, so it is accurate to f32 rounding.
// Exact bf16 operands (the inputs) go as one part.
//
// Accumulators with M = 64 rows occupy TMEM lanes 16 w .. 16 w + 15 of each
// 32-lane quarter w (row 16 w + i at lane 32 w + i); warp w of a CTA reads its
// quarter w % 4 with tcgen05.ld.32x32b, lanes 0..15 of the warp receiving
// rows 16 (w % 4) + lane.
//
// Every wait on an mbarrier is bounded; a wait that runs out reports failure
// and the caller turns its outputs into NaN rather than hang.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace msc {
namespace umma {

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// byte offset of (r, k) in a K-major bf16 tile with K columns
__device__ __forceinline__ int koff(int r, int k, int K) {
  return (r >> 3) * (K * 16) + (k >> 3) * 128 + (r & 7) * 16 + (k & 7) * 2;
}

__device__ __forceinline__ uint64_t desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version of sm_100
  return d;              // base offset 0, no swizzle
}

// instruction descriptor: bf16 x bf16 -> f32, M = 64, N columns; A K-major,
// B K-major (kBMN = false) or MN-major (kBMN = true)
template <int N, bool kBMN>
__device__ __forceinline__ uint32_t idesc_bf16() {
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "N");
  return (1u << 4) | (1u << 7) | (1u << 10) | ((kBMN ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         ((64u >> 4) << 24);
}

__device__ __forceinline__ void mma(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                    bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate ? 1u : 0u));
}

__device__ __forceinline__ void commit(uint32_t mbar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
      : "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t mbar) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mbar));
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// wait for the given phase parity; false if the bound ran out
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity) {
  uint32_t done = 0;
  for (int it = 0; it < (1 << 22) && !done; ++it) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(mbar), "r"(parity)
        : "memory");
  }
  return done != 0;
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// TMEM allocation by one whole warp; the address lands in *slot
__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_addr(slot)),
               "r"(ncols));
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}

// 8 consecutive f32 columns of this warp's TMEM quarter: thread i gets lane
// (32 (warp % 4) + i), columns col .. col + 7
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// the three bf16 parts of v
__device__ __forceinline__ void split3(float v, __nv_bfloat16 (&p)[3]) {
  p[0] = __float2bfloat16_rn(v);
  float r = v - __bfloat162float(p[0]);
  p[1] = __float2bfloat16_rn(r);
  r -= __bfloat162float(p[1]);
  p[2] = __float2bfloat16_rn(r);
}

}  // namespace umma
}  // namespace msc
