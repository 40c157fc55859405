// conv1d.cu -- causal depthwise conv1d + SiLU ahead of the Mamba-1 scan
// (sm_100a): the Mamba block's local convolution of width d_conv (the Mamba
// README, "Usage / Mamba Block"; its causal-conv1d extra), u = silu(bias +
// sum_k w[k] x[t-(W-1)+k]) per channel, and its backward.
//
// Both directions are bound by HBM traffic (an io element in and out per
// token-channel, plus du and dx in the backward).  A thread owns a run of
// kRun consecutive steps of one (b, c) row: it reads the run and the W-1
// inputs before it (or after it, in the backward) with plain loads that the
// neighbouring threads' runs share through L1, keeps the W weights in
// registers, and writes the run back in 16-byte pieces when the row allows.
// The backward's dw and dbias are per-row sums written to a workspace and
// added over the batch in ascending order by a second kernel (no atomics).
#include "common.cuh"
#include "kernels.h"

namespace msc {
namespace {

constexpr int kConvThreads = 256;
constexpr int kRun = 8;  // steps per thread

template <typename T>
__device__ __forceinline__ float ld_io(const void *p, int64_t i) {
  return to_f32(static_cast<const T *>(p)[i]);
}

// x at step t of row r (t may be negative: the conv state, or 0)
template <typename T>
__device__ __forceinline__ float x_at(const ConvParams &p, int64_t r, int64_t t) {
  if (t >= 0) return ld_io<T>(p.x, r * p.L + t);
  return p.xs_in ? p.xs_in[r * (p.W - 1) + (p.W - 1) + t] : 0.f;
}

template <typename T, int W>
__global__ void __launch_bounds__(kConvThreads) conv1d_fwd_kernel(const ConvParams p) {
  const int64_t runs = (p.L + kRun - 1) / kRun;
  const int64_t i = (int64_t)blockIdx.x * kConvThreads + threadIdx.x;
  if (i >= p.B * p.D * runs) return;
  const int64_t r = i / runs, t0 = (i % runs) * kRun;
  const int64_t c = r % p.D;
  float w[W];
#pragma unroll
  for (int k = 0; k < W; ++k) w[k] = p.w[c * W + k];
  const float bias = p.bias ? p.bias[c] : 0.f;
  float xs[kRun + W - 1];  // x at t0-(W-1) .. t0+kRun-1
#pragma unroll
  for (int j = 0; j < W - 1; ++j) xs[j] = x_at<T>(p, r, t0 - (W - 1) + j);
  float run[kRun];
  load_run<kRun, Cache::kStream>(static_cast<const T *>(p.x) + r * p.L, t0, p.L, p.vec, run, 0.f);
#pragma unroll
  for (int j = 0; j < kRun; ++j) xs[W - 1 + j] = run[j];
  float u[kRun];
#pragma unroll
  for (int j = 0; j < kRun; ++j) {
    float v = bias;
#pragma unroll
    for (int k = 0; k < W; ++k) v = fmaf(w[k], xs[j + k], v);
    u[j] = silu(v);
  }
  store_run<kRun>(static_cast<T *>(p.u) + r * p.L, t0, p.L, p.vec, u);
  // the last W-1 inputs: the conv state of the next call
  if (p.xs_out && t0 + kRun >= p.L) {
#pragma unroll
    for (int j = 0; j < W - 1; ++j) p.xs_out[r * (W - 1) + j] = x_at<T>(p, r, p.L - (W - 1) + j);
  }
}

// Backward: a thread owns steps t0 .. t0+kRun-1 of row r.  dx needs dv at
// t .. t+W-1; dv at s needs v at s, so the thread recomputes v over
// t0 .. t0+kRun+W-2 from x at t0-(W-1) .. t0+kRun+W-2.
template <typename T, int W>
__global__ void __launch_bounds__(kConvThreads) conv1d_bwd_kernel(const ConvParams p) {
  const int64_t runs = (p.L + kRun - 1) / kRun;
  const int64_t i = (int64_t)blockIdx.x * kConvThreads + threadIdx.x;
  if (i >= p.B * p.D * runs) return;
  const int64_t r = i / runs, run_i = i % runs, t0 = run_i * kRun;
  const int64_t c = r % p.D, L = p.L;
  float w[W];
#pragma unroll
  for (int k = 0; k < W; ++k) w[k] = p.w[c * W + k];
  const float bias = p.bias ? p.bias[c] : 0.f;
  constexpr int kX = kRun + 2 * (W - 1);  // x at t0-(W-1) .. t0+kRun+W-2
  float xs[kX];
#pragma unroll
  for (int j = 0; j < kX; ++j) {
    const int64_t t = t0 - (W - 1) + j;
    xs[j] = t < L ? x_at<T>(p, r, t) : 0.f;
  }
  constexpr int kV = kRun + W - 1;  // dv at t0 .. t0+kRun+W-2
  float dv[kV];
#pragma unroll
  for (int j = 0; j < kV; ++j) {
    const int64_t t = t0 + j;
    float v = bias;
#pragma unroll
    for (int k = 0; k < W; ++k) v = fmaf(w[k], xs[j + k], v);
    dv[j] = t < L ? ld_io<T>(p.du, r * L + t) * dsilu(v) : 0.f;
  }
  float dx[kRun];
#pragma unroll
  for (int j = 0; j < kRun; ++j) {
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < W; ++k) s = fmaf(w[k], dv[j + (W - 1) - k], s);
    dx[j] = s;
  }
  store_run<kRun>(static_cast<T *>(p.dx) + r * L, t0, L, p.vec, dx);
  // this run's share of dw and dbias (its own steps t0 .. t0+kRun-1), and of
  // the conv state's gradient (the first run of a row)
  float dw[W], db = 0.f;
#pragma unroll
  for (int k = 0; k < W; ++k) dw[k] = 0.f;
#pragma unroll
  for (int j = 0; j < kRun; ++j) {
    db += dv[j];
#pragma unroll
    for (int k = 0; k < W; ++k) dw[k] = fmaf(dv[j], xs[j + k], dw[k]);
  }
  float *part = p.ws + i * (W + 1);
#pragma unroll
  for (int k = 0; k < W; ++k) part[k] = dw[k];
  part[W] = db;
  if (p.dxs_in && run_i == 0) {
#pragma unroll
    for (int j = 0; j < W - 1; ++j) {  // conv-state entry j: x at time j-(W-1)
      float s = 0.f;
#pragma unroll
      for (int k = 0; k < W; ++k) {
        const int idx = j - (W - 1) + (W - 1) - k;  // dv index of time tau+(W-1)-k
        if (idx >= 0 && idx < kV) s = fmaf(w[k], dv[idx], s);
      }
      p.dxs_in[r * (W - 1) + j] = s;
    }
  }
}

// dw[c,k], dbias[c]: the runs of every (b, c) row in ascending order, then
// the batch in ascending order
__global__ void conv1d_reduce_kernel(const ConvParams p) {
  const int64_t runs = (p.L + kRun - 1) / kRun;
  const int W = (int)p.W;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < p.D * (W + 1);
       j += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = j / (W + 1), k = j % (W + 1);
    float s = 0.f;
    for (int64_t b = 0; b < p.B; ++b) {
      const float *row = p.ws + ((b * p.D + c) * runs) * (W + 1) + k;
      float sr = 0.f;
      for (int64_t q = 0; q < runs; ++q) sr += row[q * (W + 1)];
      s += sr;
    }
    if (k < W) p.dw[c * W + k] = s;
    else if (p.dbias) p.dbias[c] = s;
  }
}

template <typename T, int W>
cudaError_t launch_w(const ConvParams &p, cudaStream_t s, bool bwd) {
  const int64_t runs = (p.L + kRun - 1) / kRun;
  const int64_t n = p.B * p.D * runs;
  const unsigned blocks = (unsigned)((n + kConvThreads - 1) / kConvThreads);
  if (!bwd) {
    conv1d_fwd_kernel<T, W><<<blocks, kConvThreads, 0, s>>>(p);
    return cudaGetLastError();
  }
  conv1d_bwd_kernel<T, W><<<blocks, kConvThreads, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t m = p.D * (W + 1);
  int64_t rb = (m + 255) / 256;
  if (rb > 148 * 8) rb = 148 * 8;
  conv1d_reduce_kernel<<<(unsigned)rb, 256, 0, s>>>(p);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const ConvParams &p, cudaStream_t s, bool bwd) {
  switch (p.W) {
    case 1: return launch_w<T, 1>(p, s, bwd);
    case 2: return launch_w<T, 2>(p, s, bwd);
    case 3: return launch_w<T, 3>(p, s, bwd);
    default: return launch_w<T, 4>(p, s, bwd);
  }
}

cudaError_t launch(const ConvParams &p, cudaStream_t s, bool bwd) {
  switch (p.io) {
    case 1: return launch_t<bf16>(p, s, bwd);
    case 2: return launch_t<f16>(p, s, bwd);
    default: return launch_t<float>(p, s, bwd);
  }
}

}  // namespace

cudaError_t launch_conv1d_fwd(const ConvParams &p, cudaStream_t s) { return launch(p, s, false); }
cudaError_t launch_conv1d_bwd(const ConvParams &p, cudaStream_t s) { return launch(p, s, true); }
size_t conv1d_bwd_workspace_bytes(int64_t B, int64_t D, int64_t L, int64_t W) {
  const int64_t runs = (L + kRun - 1) / kRun;
  return sizeof(float) * (size_t)(B * D * runs * (W + 1));
}

}  // namespace msc
