// m3_disc_common.cuh -- the per-(token, head) coefficients of the Mamba-3
// discretisation (stage B6 of Mamba3Scratch, mamba-rs 0.4.2
// src/mamba3_siso/cpu/scratch.rs, read as the exponential-trapezoid rule of
// the Mamba-3 paper), shared by the discretisation kernels and the decode
// step that fuses them, so that both evaluate the same expressions:
//   dt = softplus(dd_dt + dt_bias),  A = min(-softplus(dd_a), -A_floor)
//   alpha = exp(dt A),  lam = sigmoid(trap),  beta = (1 - lam) dt alpha,
//   gamma = lam dt
#pragma once

#include "common.cuh"

namespace msc {

struct DiscCoef {
  float dt, sig_u, A, dA_dda, alpha, lam;
};

__device__ __forceinline__ DiscCoef disc_coef(float dd_dt, float bias, float dd_a, float trap,
                                              float A_floor) {
  DiscCoef c;
  const float u = dd_dt + bias;
  c.dt = softplus(u);
  c.sig_u = sigmoid(u);
  const float sa = softplus(dd_a);
  const bool clamped = -sa > -A_floor;  // A held at -A_floor: no gradient to dd_a
  c.A = clamped ? -A_floor : -sa;
  c.dA_dda = clamped ? 0.f : -sigmoid(dd_a);
  c.alpha = __expf(c.dt * c.A);
  c.lam = sigmoid(trap);
  return c;
}

__device__ __forceinline__ float disc_beta(const DiscCoef &c) {
  return (1.f - c.lam) * c.dt * c.alpha;
}
__device__ __forceinline__ float disc_gamma(const DiscCoef &c) { return c.lam * c.dt; }

// Lanes per B or C row in the 16-byte path: a row of N = 8 S elements (S a
// power of two <= 32) is served by S lanes; 0 where rows take the scalar path.
__host__ __device__ constexpr int disc_row_lanes(int N) {
  return (N % 8 == 0 && N / 8 <= 32 && ((N / 8) & (N / 8 - 1)) == 0) ? N / 8 : 0;
}

}  // namespace msc
