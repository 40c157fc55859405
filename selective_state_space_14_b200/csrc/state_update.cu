// state_update.cu -- single-token recurrent state update for decoding (sm_100a).
//
// One step of the Mamba-1 recurrence applied to a stored state, for every
// (batch b, channel c) (mamba_step / GpuMambaBackbone::step, mamba-rs 0.7.0
// README, "Quick start"):
//   state[n] <- exp(delta A[c,n]) state[n] + delta B[n] x,
//   out       = (sum_n C[n] state[n] + D[c] x) silu(z).
// The arithmetic is the scan kernel's step, operation for operation
// (exp as 2^(delta * (A log2 e)), the input term as (delta x) B, fused
// multiply-adds in the same places, y summed over n in ascending order), so a
// decode step reproduces the forward scan's bits for the same inputs.
//
// One thread owns one (b, c) row of the state: it reads the row's N floats
// with 16-byte loads, updates them and writes them back.  The kernel is bound
// by HBM traffic: 8 N bytes of state plus four io elements per (b, c).
#include "common.cuh"
#include "kernels.h"

namespace msc {
namespace {

template <typename T, bool kVec4>
__global__ void __launch_bounds__(256) state_update_kernel(const SUParams p) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t D = p.D, N = p.N;
  if (i >= p.B * D) return;
  const int64_t b = i / D, c = i % D, g = c / (D / p.G);
  const float x = to_f32(static_cast<const T *>(p.x)[i]);
  const float v = to_f32(static_cast<const T *>(p.delta)[i]) + (p.bias ? p.bias[c] : 0.f);
  const float d = p.softplus ? softplus(v) : v;
  const float dtx = d * x;
  float y = (p.Dp ? p.Dp[c] : 0.f) * x;
  const T *Bp = static_cast<const T *>(p.Bm) + (b * p.G + g) * N;
  const T *Cp = static_cast<const T *>(p.Cm) + (b * p.G + g) * N;
  const float *Ap = p.A + c * N;
  float *st = p.state + i * N;
  if constexpr (kVec4) {
    for (int64_t n = 0; n < N; n += 4) {
      float4 h = *reinterpret_cast<const float4 *>(st + n);
      const float4 A4 = __ldg(reinterpret_cast<const float4 *>(Ap + n));
      float hv[4] = {h.x, h.y, h.z, h.w};
      const float Av[4] = {A4.x, A4.y, A4.z, A4.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float a = ex2(d * (Av[k] * kLog2e));
        hv[k] = fmaf(a, hv[k], dtx * to_f32(Bp[n + k]));
        y = fmaf(to_f32(Cp[n + k]), hv[k], y);
      }
      *reinterpret_cast<float4 *>(st + n) = make_float4(hv[0], hv[1], hv[2], hv[3]);
    }
  } else {
    for (int64_t n = 0; n < N; ++n) {
      const float a = ex2(d * (Ap[n] * kLog2e));
      const float h = fmaf(a, st[n], dtx * to_f32(Bp[n]));
      st[n] = h;
      y = fmaf(to_f32(Cp[n]), h, y);
    }
  }
  if (p.z) y *= silu(to_f32(static_cast<const T *>(p.z)[i]));
  static_cast<T *>(p.out)[i] = from_f32<T>(y);
}

template <typename T>
cudaError_t launch_t(const SUParams &p, cudaStream_t s) {
  const int64_t rows = p.B * p.D;
  const unsigned blocks = (unsigned)((rows + 255) / 256);
  if (p.N % 4 == 0)
    state_update_kernel<T, true><<<blocks, 256, 0, s>>>(p);
  else
    state_update_kernel<T, false><<<blocks, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_state_update(const SUParams &p, cudaStream_t s) {
  return p.io_bf16 ? launch_t<bf16>(p, s) : launch_t<float>(p, s);
}

}  // namespace msc
