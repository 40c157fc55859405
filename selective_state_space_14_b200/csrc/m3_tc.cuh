// m3_tc.cuh -- tensor-core pieces of the bf16 Mamba-3 SISO scan kernels.
//
// The chunk contractions (64-step chunks, m3_common.cuh) run as warp-level
// m16n8k8 tf32 MMAs with f32 accumulation.  Operands that are not exact in
// tf32 (rotated B and C, W, the state) are split when their fragments are
// loaded, v = hi + lo with hi = tf32(v) and lo = tf32(v - hi), and a product
// takes hi*hi + hi*lo + lo*hi (the lo*lo term is below f32 rounding): the
// error is that of an f32 product rather than the 2^-11 of one tf32 rounding.
// bf16 inputs (x) are exact in tf32 and go unsplit.
//
// Work split of an M x N product over the 8 warps of a CTA: the 16 x 8 output
// tiles are numbered tt = rb + (M/16) cb (row block rb, column block cb) and
// warp w owns tiles tt = w + 8 i.  Since M/16 divides 8, a warp's tiles share
// one row block, so its A fragment is loaded once per k-step.
//
// Fragment layout of m16n8k8 (g = lane / 4, q = lane % 4):
//   A (16 x 8, row): a0 (g, q)  a1 (g+8, q)  a2 (g, q+4)  a3 (g+8, q+4)
//   B (8 x 8, col):  b0 (k=q, n=g)  b1 (k=q+4, n=g)
//   C (16 x 8):      c0 (g, 2q)  c1 (g, 2q+1)  c2 (g+8, 2q)  c3 (g+8, 2q+1)
#pragma once

#include "m3_common.cuh"

namespace msc {
namespace m3 {

constexpr int kTcWarps = kThreads / 32;  // 8

__device__ __forceinline__ float tf32r(float v) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(v));
  return __uint_as_float(r);
}

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int M, int N>
struct TileSplit {
  static_assert(M % 16 == 0 && N % 8 == 0 && 8 % (M / 16) == 0, "tile split");
  static constexpr int kRB = M / 16;
  static constexpr int kTiles = kRB * (N / 8);
  static constexpr int kPerWarp = (kTiles + kTcWarps - 1) / kTcWarps;
  // tile i of warp w: valid when w + 8 i < kTiles
  __device__ static bool valid(int w, int i) { return w + kTcWarps * i < kTiles; }
  __device__ static int rb(int w) { return w % kRB; }
  __device__ static int cb(int w, int i) { return (w + kTcWarps * i) / kRB; }
};

template <int M, int N>
__device__ __forceinline__ void zero_acc(float (&acc)[TileSplit<M, N>::kPerWarp][4]) {
#pragma unroll
  for (int i = 0; i < TileSplit<M, N>::kPerWarp; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
}

// acc (+)= A B over k < K for the warp's tiles.  fa(m, k) and fb(k, n) return
// the f32 operand values (from shared memory); kSplitA / kSplitB say whether
// that operand is split into tf32 hi + lo parts or is already exact in tf32.
template <int M, int N, int K, bool kSplitA, bool kSplitB, typename FA, typename FB>
__device__ __forceinline__ void mma_tiles(float (&acc)[TileSplit<M, N>::kPerWarp][4], FA fa,
                                          FB fb) {
  using TS = TileSplit<M, N>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  if (!TS::valid(warp, 0)) return;
  const int m0 = TS::rb(warp) * 16;
#pragma unroll 2
  for (int k0 = 0; k0 < K; k0 += 8) {
    const float av[4] = {fa(m0 + g, k0 + q), fa(m0 + g + 8, k0 + q), fa(m0 + g, k0 + q + 4),
                         fa(m0 + g + 8, k0 + q + 4)};
    uint32_t ah[4], al[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      if (kSplitA) {
        const float hi = tf32r(av[r]);
        ah[r] = __float_as_uint(hi);
        al[r] = __float_as_uint(tf32r(av[r] - hi));
      } else {
        ah[r] = __float_as_uint(av[r]);
      }
    }
#pragma unroll
    for (int i = 0; i < TS::kPerWarp; ++i) {
      if (TS::valid(warp, i)) {
        const int n0 = TS::cb(warp, i) * 8;
        const float b0 = fb(k0 + q, n0 + g), b1 = fb(k0 + q + 4, n0 + g);
        if (kSplitB) {
          const float h0 = tf32r(b0), h1 = tf32r(b1);
          mma_tf32(acc[i], ah, __float_as_uint(tf32r(b0 - h0)), __float_as_uint(tf32r(b1 - h1)));
          if (kSplitA) mma_tf32(acc[i], al, __float_as_uint(h0), __float_as_uint(h1));
          mma_tf32(acc[i], ah, __float_as_uint(h0), __float_as_uint(h1));
        } else {
          if (kSplitA) mma_tf32(acc[i], al, __float_as_uint(b0), __float_as_uint(b1));
          mma_tf32(acc[i], ah, __float_as_uint(b0), __float_as_uint(b1));
        }
      }
    }
  }
}

// Visit the warp's accumulator entries: f(i, j, m, n) for entry j of tile i at
// output position (m, n).
template <int M, int N, typename F>
__device__ __forceinline__ void for_acc(F f) {
  using TS = TileSplit<M, N>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
#pragma unroll
  for (int i = 0; i < TS::kPerWarp; ++i) {
    if (!TS::valid(warp, i)) continue;
    const int m0 = TS::rb(warp) * 16, n0 = TS::cb(warp, i) * 8;
#pragma unroll
    for (int j = 0; j < 4; ++j) f(i, j, m0 + g + (j >> 1) * 8, n0 + 2 * q + (j & 1));
  }
}

}  // namespace m3
}  // namespace msc

namespace msc {
namespace m3 {

// Drop-in for mm() of m3_common.cuh on the tensor cores:
//   C[m][n] (+)= rowscale[m] * sum_k kscale[k] * A(m, k) * B(k, n)
// with the same operand conventions; operands that are exact in tf32 may be
// declared unsplit.  Executed by all threads of the CTA; callers separate it
// from producers and consumers of its operands with block barriers.
template <int M, int N, int K, bool kAT, bool kBT, bool kSplitA = true, bool kSplitB = true>
__device__ __forceinline__ void mmt(float *C, int ldc, const float *A, int lda, const float *B,
                                    int ldb, const float *rowscale, const float *kscale,
                                    bool accumulate) {
  float acc[TileSplit<M, N>::kPerWarp][4];
  zero_acc<M, N>(acc);
  auto fa = [&](int m, int k) {
    const float v = kAT ? A[k * lda + m] : A[m * lda + k];
    return kscale ? v * kscale[k] : v;
  };
  auto fb = [&](int k, int n) { return kBT ? B[n * ldb + k] : B[k * ldb + n]; };
  if (kscale) {
    mma_tiles<M, N, K, true, kSplitB>(acc, fa, fb);
  } else {
    mma_tiles<M, N, K, kSplitA, kSplitB>(acc, fa, fb);
  }
  for_acc<M, N>([&](int i, int j, int m, int n) {
    float v = acc[i][j];
    if (rowscale) v *= rowscale[m];
    float *dst = C + m * ldc + n;
    *dst = accumulate ? *dst + v : v;
  });
}

}  // namespace m3
}  // namespace msc
