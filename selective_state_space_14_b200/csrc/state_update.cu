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

template <typename T>
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
  if (N % 8 == 0) {
    // B and C in 16-byte runs (8 io elements) next to the state's 16-byte pieces
    for (int64_t n = 0; n < N; n += 8) {
      float bv[8], cv[8];
      load_run<8, Cache::kKeep>(Bp, n, N, true, bv, 0.f);
      load_run<8, Cache::kKeep>(Cp, n, N, true, cv, 0.f);
#pragma unroll
      for (int q = 0; q < 8; q += 4) {
        const float4 h4 = *reinterpret_cast<const float4 *>(st + n + q);
        const float4 A4 = __ldg(reinterpret_cast<const float4 *>(Ap + n + q));
        float2 h01 = make_float2(h4.x, h4.y), h23 = make_float2(h4.z, h4.w);
        const float2 a01 = ex2_2(mul2(splat2(d), mul2(make_float2(A4.x, A4.y), splat2(kLog2e))));
        const float2 a23 = ex2_2(mul2(splat2(d), mul2(make_float2(A4.z, A4.w), splat2(kLog2e))));
        h01 = fma2(a01, h01, mul2(splat2(dtx), make_float2(bv[q], bv[q + 1])));
        h23 = fma2(a23, h23, mul2(splat2(dtx), make_float2(bv[q + 2], bv[q + 3])));
        y = fmaf(cv[q], h01.x, y);
        y = fmaf(cv[q + 1], h01.y, y);
        y = fmaf(cv[q + 2], h23.x, y);
        y = fmaf(cv[q + 3], h23.y, y);
        *reinterpret_cast<float4 *>(st + n + q) = make_float4(h01.x, h01.y, h23.x, h23.y);
      }
    }
  } else if (N % 4 == 0) {
    for (int64_t n = 0; n < N; n += 4) {
      const float4 h4 = *reinterpret_cast<const float4 *>(st + n);
      const float4 A4 = __ldg(reinterpret_cast<const float4 *>(Ap + n));
      float2 h01 = make_float2(h4.x, h4.y), h23 = make_float2(h4.z, h4.w);
      const float2 a01 = ex2_2(mul2(splat2(d), mul2(make_float2(A4.x, A4.y), splat2(kLog2e))));
      const float2 a23 = ex2_2(mul2(splat2(d), mul2(make_float2(A4.z, A4.w), splat2(kLog2e))));
      h01 = fma2(a01, h01, mul2(splat2(dtx), make_float2(to_f32(Bp[n]), to_f32(Bp[n + 1]))));
      h23 = fma2(a23, h23, mul2(splat2(dtx), make_float2(to_f32(Bp[n + 2]), to_f32(Bp[n + 3]))));
      y = fmaf(to_f32(Cp[n]), h01.x, y);
      y = fmaf(to_f32(Cp[n + 1]), h01.y, y);
      y = fmaf(to_f32(Cp[n + 2]), h23.x, y);
      y = fmaf(to_f32(Cp[n + 3]), h23.y, y);
      *reinterpret_cast<float4 *>(st + n) = make_float4(h01.x, h01.y, h23.x, h23.y);
    }
  } else {
    for (int64_t n = 0; n < N; n += 2) {
      const bool two = n + 1 < N;
      float2 h = make_float2(st[n], two ? st[n + 1] : 0.f);
      const float2 A2 = mul2(make_float2(Ap[n], two ? Ap[n + 1] : 0.f), splat2(kLog2e));
      const float2 a = ex2_2(mul2(splat2(d), A2));
      const float2 Bv = make_float2(to_f32(Bp[n]), two ? to_f32(Bp[n + 1]) : 0.f);
      const float2 Cv = make_float2(to_f32(Cp[n]), two ? to_f32(Cp[n + 1]) : 0.f);
      h = fma2(a, h, mul2(splat2(dtx), Bv));
      y = fmaf(Cv.y, h.y, fmaf(Cv.x, h.x, y));
      st[n] = h.x;
      if (two) st[n + 1] = h.y;
    }
  }
  if (p.z) y *= silu(to_f32(static_cast<const T *>(p.z)[i]));
  static_cast<T *>(p.out)[i] = from_f32<T>(y);
}

// The same step for a compile-time N (16): every load of the row (its
// state, B, C and A pieces) is issued before the first store, so a thread has
// all of them in flight at once instead of one 8-state group at a time.  The
// arithmetic is the kernel above's, operation for operation.
template <typename T, int kN>
__global__ void __launch_bounds__(256) state_update_fixed_kernel(const SUParams p) {
  static_assert(kN % 8 == 0, "rows of 8-element runs");
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t D = p.D;
  if (i >= p.B * D) return;
  const int64_t b = i / D, c = i % D, g = c / (D / p.G);
  const T *Bp = static_cast<const T *>(p.Bm) + (b * p.G + g) * kN;
  const T *Cp = static_cast<const T *>(p.Cm) + (b * p.G + g) * kN;
  const float4 *Ap = reinterpret_cast<const float4 *>(p.A + c * kN);
  float4 *st = reinterpret_cast<float4 *>(p.state + i * kN);
  float4 h4[kN / 4], A4[kN / 4];
  float bv[kN / 8][8], cv[kN / 8][8];
#pragma unroll
  for (int k = 0; k < kN / 4; ++k) h4[k] = st[k];
#pragma unroll
  for (int k = 0; k < kN / 8; ++k) {
    load_run<8, Cache::kKeep>(Bp, 8 * k, kN, true, bv[k], 0.f);
    load_run<8, Cache::kKeep>(Cp, 8 * k, kN, true, cv[k], 0.f);
  }
#pragma unroll
  for (int k = 0; k < kN / 4; ++k) A4[k] = __ldg(Ap + k);
  const float x = to_f32(static_cast<const T *>(p.x)[i]);
  const float v = to_f32(static_cast<const T *>(p.delta)[i]) + (p.bias ? p.bias[c] : 0.f);
  const float zv = p.z ? to_f32(static_cast<const T *>(p.z)[i]) : 0.f;
  const float d = p.softplus ? softplus(v) : v;
  const float dtx = d * x;
  float y = (p.Dp ? p.Dp[c] : 0.f) * x;
#pragma unroll
  for (int k = 0; k < kN / 4; ++k) {
    const float *bq = &bv[k / 2][(k & 1) * 4];
    const float *cq = &cv[k / 2][(k & 1) * 4];
    float2 h01 = make_float2(h4[k].x, h4[k].y), h23 = make_float2(h4[k].z, h4[k].w);
    const float2 a01 = ex2_2(mul2(splat2(d), mul2(make_float2(A4[k].x, A4[k].y), splat2(kLog2e))));
    const float2 a23 = ex2_2(mul2(splat2(d), mul2(make_float2(A4[k].z, A4[k].w), splat2(kLog2e))));
    h01 = fma2(a01, h01, mul2(splat2(dtx), make_float2(bq[0], bq[1])));
    h23 = fma2(a23, h23, mul2(splat2(dtx), make_float2(bq[2], bq[3])));
    y = fmaf(cq[0], h01.x, y);
    y = fmaf(cq[1], h01.y, y);
    y = fmaf(cq[2], h23.x, y);
    y = fmaf(cq[3], h23.y, y);
    st[k] = make_float4(h01.x, h01.y, h23.x, h23.y);
  }
  if (p.z) y *= silu(zv);
  static_cast<T *>(p.out)[i] = from_f32<T>(y);
}

template <typename T>
cudaError_t launch_t(const SUParams &p, cudaStream_t s) {
  const int64_t rows = p.B * p.D;
  const unsigned blocks = (unsigned)((rows + 255) / 256);
  if (p.N == 16)  // (at 32 states the row in registers would halve the occupancy)
    state_update_fixed_kernel<T, 16><<<blocks, 256, 0, s>>>(p);
  else
    state_update_kernel<T><<<blocks, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_state_update(const SUParams &p, cudaStream_t s) {
  switch (p.io) {
    case 1: return launch_t<bf16>(p, s);
    case 2: return launch_t<f16>(p, s);
    default: return launch_t<float>(p, s);
  }
}

}  // namespace msc
