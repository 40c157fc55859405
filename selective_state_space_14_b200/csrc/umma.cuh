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
// 32-lane quarter w (row 16 w + i at lane 32 w + i).  Warp w of a CTA reads
// the 16 rows of its quarter w % 4 with tcgen05.ld.16x256b, which spreads
// them over all 32 threads: per block of 8 columns, thread i receives rows
// i / 4 and 8 + i / 4 (of the 16), columns 2 (i % 4) and 2 (i % 4) + 1.
// Each load and its tcgen05.wait::ld sit in one asm statement, so that no use
// of the registers can be scheduled ahead of the wait.
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

// instruction descriptor: bf16 x bf16 -> f32, M = 64, N columns; A K-major
// (kAMN = false) or MN-major (bit 15), B K-major (kBMN = false) or MN-major
// (bit 16)
template <int N, bool kBMN, bool kAMN = false>
__device__ __forceinline__ uint32_t idesc_bf16() {
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "N");
  return (1u << 4) | (1u << 7) | (1u << 10) | ((kAMN ? 1u : 0u) << 15) | ((kBMN ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((64u >> 4) << 24);
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

// 16 TMEM lanes x 8 R columns from the lane and column in taddr (tcgen05.ld
// .16x256b.xR), waited for: per block c of 8 columns, thread i gets v[4 c],
// v[4 c + 1] = (lane i / 4, columns 8 c + 2 (i % 4) + 0, 1) and v[4 c + 2],
// v[4 c + 3] = (lane 8 + i / 4, the same columns).
template <int R>
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *v);
// two such loads (ta into va, tb into vb) in flight together
template <int R>
__device__ __forceinline__ void tmem_ld16_pair(uint32_t ta, uint32_t tb, float *va, float *vb);

template <>
__device__ __forceinline__ void tmem_ld16<1>(uint32_t taddr, float *v) {
  uint32_t r[4];
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x1.b32 {%0,%1,%2,%3}, [%4];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}
template <>
__device__ __forceinline__ void tmem_ld16_pair<1>(uint32_t ta, uint32_t tb, float *va, float *vb) {
  uint32_t a[4], b[4];
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x1.b32 {%0,%1,%2,%3}, [%8];\n\t"
      "tcgen05.ld.sync.aligned.16x256b.x1.b32 {%4,%5,%6,%7}, [%9];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]),
        "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3])
      : "r"(ta), "r"(tb)
      : "memory");
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    va[i] = __uint_as_float(a[i]);
    vb[i] = __uint_as_float(b[i]);
  }
}

template <>
__device__ __forceinline__ void tmem_ld16<2>(uint32_t taddr, float *v) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
template <>
__device__ __forceinline__ void tmem_ld16_pair<2>(uint32_t ta, uint32_t tb, float *va, float *vb) {
  uint32_t a[8], b[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%16];\n\t"
      "tcgen05.ld.sync.aligned.16x256b.x2.b32 {%8,%9,%10,%11,%12,%13,%14,%15}, [%17];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]),
        "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3]), "=r"(b[4]), "=r"(b[5]), "=r"(b[6]), "=r"(b[7])
      : "r"(ta), "r"(tb)
      : "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    va[i] = __uint_as_float(a[i]);
    vb[i] = __uint_as_float(b[i]);
  }
}

template <>
__device__ __forceinline__ void tmem_ld16<4>(uint32_t taddr, float *v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
template <>
__device__ __forceinline__ void tmem_ld16_pair<4>(uint32_t ta, uint32_t tb, float *va, float *vb) {
  uint32_t a[16], b[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%32];\n\t"
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%33];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]), "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15]),
        "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3]), "=r"(b[4]), "=r"(b[5]), "=r"(b[6]), "=r"(b[7]), "=r"(b[8]), "=r"(b[9]), "=r"(b[10]), "=r"(b[11]), "=r"(b[12]), "=r"(b[13]), "=r"(b[14]), "=r"(b[15])
      : "r"(ta), "r"(tb)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    va[i] = __uint_as_float(a[i]);
    vb[i] = __uint_as_float(b[i]);
  }
}

// the three bf16 parts of v0 and v1, packed per part: w[q] holds part q of
// v0 in its low half and of v1 in its high half (the memory order of two
// consecutive bf16)
__device__ __forceinline__ void split3x2(float v0, float v1, uint32_t (&w)[3]) {
  const __nv_bfloat162 p0 = __floats2bfloat162_rn(v0, v1);
  const float2 f0 = __bfloat1622float2(p0);
  const float r0 = v0 - f0.x, r1 = v1 - f0.y;
  const __nv_bfloat162 p1 = __floats2bfloat162_rn(r0, r1);
  const float2 f1 = __bfloat1622float2(p1);
  const __nv_bfloat162 p2 = __floats2bfloat162_rn(r0 - f1.x, r1 - f1.y);
  w[0] = *reinterpret_cast<const uint32_t *>(&p0);
  w[1] = *reinterpret_cast<const uint32_t *>(&p1);
  w[2] = *reinterpret_cast<const uint32_t *>(&p2);
}

}  // namespace umma
}  // namespace msc
