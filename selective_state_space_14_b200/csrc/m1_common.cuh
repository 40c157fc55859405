// m1_common.cuh -- work layout shared by the Mamba-1 scan kernels.
//
// One thread owns one (batch b, channel c) sequence restricted to one pair of
// state indices (n, n+1) = (2p, 2p+1), and walks time sequentially: the pair
// of states lives in registers for the whole sequence, and the recurrence
// runs on packed f32x2 arithmetic with no scan and no recomputation.
// d_state is padded to kN (16, 32 or 64): the kP = kN/2 lanes of one channel
// are consecutive lanes of a warp, so a warp holds 32/kP channels.  Padded
// state indices get A = 0 and B = C = 0 and stay at zero.
//
// Time runs in chunks of kT = 64 steps.  For each chunk a CTA stages in
// shared memory, once for all its channels:
//   * per (channel, step): a float4 of per-token values (for the forward:
//     delta, delta*x, D*x, silu(z));
//   * per (step, pair): a float4 (B[2p], B[2p+1], C[2p], C[2p+1]) of the
//     batch row's B and C, converted to f32 -- the lanes of every channel read
//     the same 8..32 float4 of a step (broadcast across channels, no bank
//     conflicts).
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace msc {
namespace m1 {

constexpr int kT = 64;  // forward steps per chunk
static_assert(kT % kM1SaveInterval == 0, "chunk must hold whole saved-state intervals");

__host__ __device__ constexpr int pad_n(int64_t n) { return n <= 16 ? 16 : (n <= 32 ? 32 : 64); }

template <int kN, int kWarps>
struct Layout {
  static constexpr int kP = kN / 2;                    // lanes (state pairs) per channel
  static constexpr int kChPerWarp = 32 / kP;           // 4, 2 or 1
  static constexpr int kCh = kWarps * kChPerWarp;      // channels per CTA
  static constexpr int kThreads = kWarps * 32;
};

// Stage B and C of the chunk starting at tc (rows n < N, steps t < L; zero
// elsewhere) into bc[t][p] = (B[2p], B[2p+1], C[2p], C[2p+1]).
template <typename T, int kN, int kSteps>
__device__ __forceinline__ void stage_bc(float4 *bc, const T *Bg, const T *Cg, int64_t N,
                                         int64_t L, int64_t tc, bool vec, int tid, int nthreads) {
  constexpr int kP = kN / 2;
  constexpr int kUnits = kP * (kSteps / 8);  // (pair, 8-step segment)
  for (int u = tid; u < kUnits; u += nthreads) {
    const int p = u % kP;
    const int seg = u / kP;
    const int64_t t = tc + seg * 8;
    float r[4][8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t n = 2 * p + (k & 1);
      const T *src = (k < 2 ? Bg : Cg) + n * L;
      if (n < N) {
        load_run<8, Cache::kKeep>(src, t, L, vec, r[k], 0.f);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) r[k][i] = 0.f;
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
      bc[(seg * 8 + i) * kP + p] = make_float4(r[0][i], r[1][i], r[2][i], r[3][i]);
  }
}

}  // namespace m1
}  // namespace msc
