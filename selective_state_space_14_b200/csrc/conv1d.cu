// conv1d.cu -- causal depthwise conv1d + SiLU ahead of the Mamba-1 scan
// (sm_100a): the Mamba block's local convolution of width d_conv (the Mamba
// README, "Usage / Mamba Block"; its causal-conv1d extra), u = silu(bias +
// sum_k w[k] x[t-(W-1)+k]) per channel, and its backward.
//
// Both directions are bound by HBM traffic (an io element in and out per
// token-channel, plus du and dx in the backward).  A CTA owns one (b, c) row
// (and, for long rows, every gridDim.y-th segment of it); a thread owns a run
// of kRun consecutive steps, read and written in 16-byte pieces.  The W-1
// inputs before a run (and, in the backward, the inputs and gradients after
// it) come from the neighbouring lane by a shuffle; only the lanes at a warp's
// edge load them.  The backward's dw and dbias are summed over a CTA's runs in
// a fixed tree, one partial per (segment slot, row) goes to a workspace, and a
// second kernel adds the partials over the slots and the batch in ascending
// order (no atomics: the sums do not depend on scheduling).
#include "common.cuh"
#include "kernels.h"

namespace msc {
namespace {

constexpr int kConvMaxThreads = 256;
constexpr int kRun = 16;        // steps per thread
constexpr int kMaxSlots = 64;   // segment slots per row (gridDim.y)
constexpr unsigned kFull = 0xffffffffu;

// CTA size and segment slots for a row of L steps: a CTA covers up to 256
// runs; rows longer than 64 CTAs' worth loop over their segments
struct ConvGrid {
  int threads;
  int64_t slots;
};
inline ConvGrid conv_grid(int64_t L) {
  const int64_t runs = (L + kRun - 1) / kRun;
  int t = 32;
  while (t < kConvMaxThreads && t < runs) t *= 2;
  const int64_t segs = (runs + t - 1) / t;
  return {t, segs < kMaxSlots ? segs : kMaxSlots};
}

template <typename T>
__device__ __forceinline__ float ld_io(const void *p, int64_t i) {
  return to_f32(static_cast<const T *>(p)[i]);
}

// x at step t of row r: the conv state (or 0) before the row, 0 after it
template <typename T>
__device__ __forceinline__ float x_at(const ConvParams &p, int64_t r, int64_t t) {
  if (t >= p.L) return 0.f;
  if (t >= 0) return ld_io<T>(p.x, r * p.L + t);
  return p.xs_in ? p.xs_in[r * (p.W - 1) + (p.W - 1) + t] : 0.f;
}

template <typename T, int W>
__global__ void __launch_bounds__(kConvMaxThreads) conv1d_fwd_kernel(const ConvParams p) {
  const int64_t r = blockIdx.x, c = r % p.D, L = p.L;
  const int lane = threadIdx.x & 31;
  const int64_t span = (int64_t)blockDim.x * kRun;
  float w[W];
#pragma unroll
  for (int k = 0; k < W; ++k) w[k] = p.w[c * W + k];
  const float bias = p.bias ? p.bias[c] : 0.f;
  const T *xr = static_cast<const T *>(p.x) + r * L;
  T *ur = static_cast<T *>(p.u) + r * L;
  // the loop bound is uniform over the CTA: every lane takes part in the shuffles
  for (int64_t s0 = blockIdx.y * span; s0 < L; s0 += gridDim.y * span) {
    const int64_t t0 = s0 + threadIdx.x * kRun;
    float run[kRun];
    load_run<kRun, Cache::kStream>(xr, t0, L, p.vec, run, 0.f);
    float xs[kRun + W - 1];  // x at t0-(W-1) .. t0+kRun-1
#pragma unroll
    for (int j = 0; j < W - 1; ++j) {
      const float v = __shfl_up_sync(kFull, run[kRun - (W - 1) + j], 1);
      xs[j] = lane == 0 ? x_at<T>(p, r, t0 - (W - 1) + j) : v;
    }
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
    store_run<kRun>(ur, t0, L, p.vec, u);
    // the last W-1 inputs: the conv state of the next call
    if (p.xs_out && t0 < L && t0 + kRun >= L) {
#pragma unroll
      for (int j = 0; j < W - 1; ++j) p.xs_out[r * (W - 1) + j] = x_at<T>(p, r, L - (W - 1) + j);
    }
  }
}

// Backward: a thread owns steps t0 .. t0+kRun-1 of row r.  dx needs dv at
// t .. t+W-1; dv at s needs v at s, so the thread recomputes v over
// t0 .. t0+kRun+W-2 from x at t0-(W-1) .. t0+kRun+W-2.
template <typename T, int W>
__global__ void __launch_bounds__(kConvMaxThreads) conv1d_bwd_kernel(const ConvParams p) {
  const int64_t r = blockIdx.x, c = r % p.D, L = p.L;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t span = (int64_t)blockDim.x * kRun;
  float w[W];
#pragma unroll
  for (int k = 0; k < W; ++k) w[k] = p.w[c * W + k];
  const float bias = p.bias ? p.bias[c] : 0.f;
  const T *xr = static_cast<const T *>(p.x) + r * L;
  const T *gr = static_cast<const T *>(p.du) + r * L;
  float dw[W], db = 0.f;  // this thread's share over its runs
#pragma unroll
  for (int k = 0; k < W; ++k) dw[k] = 0.f;
  for (int64_t s0 = blockIdx.y * span; s0 < L; s0 += gridDim.y * span) {
    const int64_t t0 = s0 + threadIdx.x * kRun;
    float xrun[kRun], grun[kRun];
    load_run<kRun, Cache::kStream>(xr, t0, L, p.vec, xrun, 0.f);
    load_run<kRun, Cache::kStream>(gr, t0, L, p.vec, grun, 0.f);
    constexpr int kX = kRun + 2 * (W - 1);  // x at t0-(W-1) .. t0+kRun+W-2
    constexpr int kV = kRun + W - 1;        // dv at t0 .. t0+kRun+W-2
    float xs[kX], gs[kV];
#pragma unroll
    for (int j = 0; j < W - 1; ++j) {
      const float before = __shfl_up_sync(kFull, xrun[kRun - (W - 1) + j], 1);
      xs[j] = lane == 0 ? x_at<T>(p, r, t0 - (W - 1) + j) : before;
      const float xa = __shfl_down_sync(kFull, xrun[j], 1);
      const float ga = __shfl_down_sync(kFull, grun[j], 1);
      const int64_t ta = t0 + kRun + j;
      xs[W - 1 + kRun + j] = lane == 31 ? x_at<T>(p, r, ta) : xa;
      gs[kRun + j] = lane == 31 ? (ta < L ? ld_io<T>(p.du, r * L + ta) : 0.f) : ga;
    }
#pragma unroll
    for (int j = 0; j < kRun; ++j) {
      xs[W - 1 + j] = xrun[j];
      gs[j] = grun[j];
    }
    float dv[kV];
#pragma unroll
    for (int j = 0; j < kV; ++j) {
      float v = bias;
#pragma unroll
      for (int k = 0; k < W; ++k) v = fmaf(w[k], xs[j + k], v);
      dv[j] = t0 + j < L ? gs[j] * dsilu(v) : 0.f;
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
#pragma unroll
    for (int j = 0; j < kRun; ++j) {
      db += dv[j];
#pragma unroll
      for (int k = 0; k < W; ++k) dw[k] = fmaf(dv[j], xs[j + k], dw[k]);
    }
    // the conv state's gradient: entry j (x at time j-(W-1)) meets dv at j-k
    if (p.dxs_in && t0 == 0) {
#pragma unroll
      for (int j = 0; j < W - 1; ++j) {
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < W; ++k)
          if (j - k >= 0) s = fmaf(w[k], dv[j - k], s);
        p.dxs_in[r * (W - 1) + j] = s;
      }
    }
  }
  // the CTA's sums in a fixed tree: within each warp, then the warps in order
  __shared__ float red[kConvMaxThreads / 32][W + 1];
  float v[W + 1];
#pragma unroll
  for (int k = 0; k < W; ++k) v[k] = dw[k];
  v[W] = db;
#pragma unroll
  for (int k = 0; k <= W; ++k) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v[k] += __shfl_down_sync(kFull, v[k], off);
    if (lane == 0) red[warp][k] = v[k];
  }
  __syncthreads();
  if (threadIdx.x <= W) {
    float s = 0.f;
    for (int q = 0; q < (int)(blockDim.x >> 5); ++q) s += red[q][threadIdx.x];
    p.ws[((int64_t)blockIdx.y * p.B * p.D + r) * (W + 1) + threadIdx.x] = s;
  }
}

// dw[c,k], dbias[c]: per (b, c) the segment slots in ascending order, then the
// batch in ascending order
__global__ void conv1d_reduce_kernel(const ConvParams p, int64_t slots) {
  const int W1 = (int)p.W + 1;
  const int64_t m = p.D * W1;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < m;
       j += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int64_t b = 0; b < p.B; ++b) {
      float sr = 0.f;
      for (int64_t y = 0; y < slots; ++y) sr += p.ws[(y * p.B + b) * m + j];
      s += sr;
    }
    const int64_t c = j / W1, k = j % W1;
    if (k < p.W) p.dw[c * p.W + k] = s;
    else if (p.dbias) p.dbias[c] = s;
  }
}

template <typename T, int W>
cudaError_t launch_w(const ConvParams &p, cudaStream_t s, bool bwd) {
  const ConvGrid g = conv_grid(p.L);
  const dim3 grid((unsigned)(p.B * p.D), (unsigned)g.slots);
  if (!bwd) {
    conv1d_fwd_kernel<T, W><<<grid, g.threads, 0, s>>>(p);
    return cudaGetLastError();
  }
  conv1d_bwd_kernel<T, W><<<grid, g.threads, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t m = p.D * (W + 1);
  int64_t rb = (m + 255) / 256;
  if (rb > 148 * 8) rb = 148 * 8;
  conv1d_reduce_kernel<<<(unsigned)rb, 256, 0, s>>>(p, g.slots);
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
  return sizeof(float) * (size_t)(conv_grid(L).slots * B * D * (W + 1));
}

}  // namespace msc
