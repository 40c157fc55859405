// m3_common.cuh -- pieces shared by the Mamba-3 SISO scan kernels.
//
// The chunked form.  Within a chunk of Q steps (indices t, s in [0, Q), the
// state entering the chunk S_in, the last key of the previous chunk
// K_prev = x_prev (outer) Bt_prev), with d(t, s) = prod_{r=s+1..t} alpha_r
// (d(t, t) = 1, d(t, -1) = prod_{r=0..t} alpha_r) the trapezoidal recurrence
//   S_t = alpha_t S_{t-1} + beta_t K_{t-1} + gamma_t K_t,  K_t = x_t (outer) Bt_t
// unrolls to
//   S_t = d(t,-1) S_in + beta_0 d(t,0) K_prev + sum_{s<=t} c(t,s) K_s,
//   c(t,t) = gamma_t,   c(t,s) = d(t,s+1) (alpha_{s+1} gamma_s + beta_{s+1})  (s < t),
// so that, with W = c o (Ct Bt^T) (masked to s <= t),
//   Y = W X + diag(d(.,-1)) Ct S_in^T + beta_0 diag(d(.,0)) (Ct Bt_prev) x_prev^T + D X,
//   S_out = d(Q-1,-1) S_in + beta_0 d(Q-1,0) K_prev + X^T diag(c(Q-1,.)) Bt.
// The contractions are 64 x 64 x 64 tile products on shared memory.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace msc {
namespace m3 {

constexpr int kQ = MSC_M3_CHUNK_STEPS;   // steps per chunk
constexpr int kThreads = 256;

// C[m][n] (+)= rowscale[m] * sum_k kscale[k] * A(m, k) * B(k, n), with
//   A(m, k) = kAT ? A[k * lda + m] : A[m * lda + k]
//   B(k, n) = kBT ? B[n * ldb + k] : B[k * ldb + n]
// C is [M][N] with row stride ldc.  M, N, K are multiples of 4; each thread
// owns a 4 x 4 block of C and walks K four at a time with 16-byte loads.
// Executed by all kThreads threads of the CTA, each on its own output blocks
// (the same blocks on every call with the same M, N); callers separate it
// from producers and consumers of its operands with block barriers.
template <int M, int N, int K, bool kAT, bool kBT>
__device__ __forceinline__ void mm(float *C, int ldc, const float *A, int lda, const float *B,
                                   int ldb, const float *rowscale, const float *kscale,
                                   bool accumulate) {
  constexpr int kTiles = (M / 4) * (N / 4);
  for (int tile = threadIdx.x; tile < kTiles; tile += kThreads) {
    const int m0 = (tile / (N / 4)) * 4;
    const int n0 = (tile % (N / 4)) * 4;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) acc[i][jj] = 0.f;
#pragma unroll 2
    for (int k0 = 0; k0 < K; k0 += 4) {
      float a[4][4], bv[4][4];  // a[m][k], bv[k][n] of this 4 x 4 x 4 step
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float4 v = kAT ? *reinterpret_cast<const float4 *>(A + (k0 + r) * lda + m0)
                             : *reinterpret_cast<const float4 *>(A + (m0 + r) * lda + k0);
        const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (kAT) a[q][r] = e[q];
          else a[r][q] = e[q];
        }
        const float4 w = kBT ? *reinterpret_cast<const float4 *>(B + (n0 + r) * ldb + k0)
                             : *reinterpret_cast<const float4 *>(B + (k0 + r) * ldb + n0);
        const float f[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (kBT) bv[q][r] = f[q];
          else bv[r][q] = f[q];
        }
      }
      if (kscale) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float ks = kscale[k0 + q];
#pragma unroll
          for (int r = 0; r < 4; ++r) a[r][q] *= ks;
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) acc[i][jj] = fmaf(a[i][q], bv[q][jj], acc[i][jj]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float rs = rowscale ? rowscale[m0 + i] : 1.f;
      float4 *dst = reinterpret_cast<float4 *>(C + (m0 + i) * ldc + n0);
      float4 v = make_float4(rs * acc[i][0], rs * acc[i][1], rs * acc[i][2], rs * acc[i][3]);
      if (accumulate) {
        const float4 o = *dst;
        v.x += o.x; v.y += o.y; v.z += o.z; v.w += o.w;
      }
      *dst = v;
    }
  }
}

template <typename T>
__device__ __forceinline__ float ldv(const void *base, int64_t i) {
  return to_f32(static_cast<const T *>(base)[i]);
}

}  // namespace m3
}  // namespace msc
