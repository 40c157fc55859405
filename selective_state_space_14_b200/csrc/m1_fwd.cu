// m1_fwd.cu -- Mamba-1 selective scan, forward (sm_100a).
//
// Computes, per (batch b, channel c) and t = 0..L-1 (the selective SSM layer,
// state-spaces/mamba README "Usage / Selective SSM"; mamba-rs 0.7.0 README
// "Features"):
//   delta_t = softplus(delta_raw + bias[c])
//   h_t[n]  = exp(delta_t A[c,n]) h_{t-1}[n] + delta_t B_t[n] x_t
//   out_t   = (sum_n C_t[n] h_t[n] + D[c] x_t) * silu(z_t)
//
// Work decomposition.  One warp owns one (b, c) sequence; its 32 lanes split a
// chunk of 32*kItems consecutive time steps, kItems per lane, and the warp
// walks the chunks of L in order.  Within a chunk, for every state index n:
//   1. each lane forms its steps' (a_i, b_i) = (2^(delta_i A2[n]), delta_i x_i B_i[n])
//      and folds them into one local pair (prod a, h with zero carry-in);
//   2. a 5-level warp-shuffle scan of those pairs under
//      (p, h) o (p', h') = (p p', p' h + h') gives each lane the state that
//      enters its first step, given the state carried in from the previous
//      chunk (one value per n per warp, kept in shared memory);
//   3. each lane re-runs its kItems steps from that state (the a_i, b_i are
//      still in registers, so every exponential is computed once) and
//      accumulates C_i[n] h_i into its outputs.
// The running state never goes to HBM; B and C rows are read through L1 (all
// warps of a CTA share one batch row), x/delta/z/out stream once from HBM
// with 16-byte accesses.  States at multiples of the save interval go to
// `saved` for the backward pass.
#include "common.cuh"
#include "kernels.h"

namespace msc {
namespace {

constexpr int kFwdItems = 16;  // time steps per lane per chunk
constexpr int kFwdWarps = 4;   // channels per CTA

template <typename T>
__global__ void __launch_bounds__(kFwdWarps * 32)
m1_fwd_kernel(const M1Params p) {
  // per-warp state carried across chunks, and A[c, :] * log2(e)
  __shared__ float s_carry[kFwdWarps][MSC_MAX_N];
  __shared__ float s_A2[kFwdWarps][MSC_MAX_N];
  constexpr int kT = 32 * kFwdItems;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t b = blockIdx.y;
  const int64_t c = (int64_t)blockIdx.x * kFwdWarps + warp;
  if (c >= p.D) return;  // no block-level synchronisation in this kernel
  const int64_t D = p.D, L = p.L, N = p.N;
  const int64_t g = c / (D / p.G);
  const int64_t row = (b * D + c) * L;
  const T *u = static_cast<const T *>(p.u) + row;
  const T *dl = static_cast<const T *>(p.delta) + row;
  const T *zr = p.z ? static_cast<const T *>(p.z) + row : nullptr;
  T *out = static_cast<T *>(p.out) + row;
  const T *Bg = static_cast<const T *>(p.Bm) + (b * p.G + g) * N * L;
  const T *Cg = static_cast<const T *>(p.Cm) + (b * p.G + g) * N * L;
  const float Dc = p.Dp ? p.Dp[c] : 0.f;
  const float bias = p.bias ? p.bias[c] : 0.f;
  const int64_t n_save = (L + kM1SaveInterval - 1) / kM1SaveInterval;

  float *carry = s_carry[warp];
  float *A2 = s_A2[warp];
  for (int n = lane; n < N; n += 32) {
    A2[n] = p.A[c * N + n] * kLog2e;
    carry[n] = p.h0 ? p.h0[(b * D + c) * N + n] : 0.f;
  }
  __syncwarp();

  const int64_t n_chunks = (L + kT - 1) / kT;
  for (int64_t ch = 0; ch < n_chunks; ++ch) {
    const int64_t t0 = ch * kT + (int64_t)lane * kFwdItems;
    float dt[kFwdItems], dtx[kFwdItems], y[kFwdItems];
    load_run<kFwdItems>(u, t0, L, p.vec, dtx, 0.f);
    load_run<kFwdItems>(dl, t0, L, p.vec, dt, 0.f);
#pragma unroll
    for (int i = 0; i < kFwdItems; ++i) {
      const float v = dt[i] + bias;
      float d = p.softplus ? softplus(v) : v;
      if (t0 + i >= L) d = 0.f;  // identity step past the end
      const float x = dtx[i];
      y[i] = Dc * x;
      dt[i] = d;
      dtx[i] = d * x;
    }
    const bool saver = (t0 < L) && (t0 % kM1SaveInterval == 0);

#pragma unroll 2
    for (int n = 0; n < N; ++n) {
      float Bv[kFwdItems], Cv[kFwdItems];
      load_run<kFwdItems, Cache::kKeep>(Bg + n * L, t0, L, p.vec, Bv, 0.f);
      load_run<kFwdItems, Cache::kKeep>(Cg + n * L, t0, L, p.vec, Cv, 0.f);
      float a[kFwdItems], bb[kFwdItems];
      float pl = 1.f, hl = 0.f;
#pragma unroll
      for (int i = 0; i < kFwdItems; ++i) {
        a[i] = ex2(dt[i] * A2[n]);
        bb[i] = dtx[i] * Bv[i];
        hl = fmaf(a[i], hl, bb[i]);
        pl = pl * a[i];
      }
      float pe, he;
      warp_scan_fwd(pl, hl, pe, he);
      float h = fmaf(pe, carry[n], he);
      if (saver && p.saved)
        p.saved[((b * D + c) * n_save + t0 / kM1SaveInterval) * N + n] = h;
#pragma unroll
      for (int i = 0; i < kFwdItems; ++i) {
        h = fmaf(a[i], h, bb[i]);
        y[i] = fmaf(Cv[i], h, y[i]);
      }
      h = __shfl_sync(0xffffffffu, h, 31);
      __syncwarp();
      if (lane == 0) carry[n] = h;
    }
    __syncwarp();

    if (zr) {
      float zv[kFwdItems];
      load_run<kFwdItems>(zr, t0, L, p.vec, zv, 0.f);
#pragma unroll
      for (int i = 0; i < kFwdItems; ++i) y[i] *= silu(zv[i]);
    }
    store_run<kFwdItems>(out, t0, L, p.vec, y);
  }

  if (p.final_state)
    for (int n = lane; n < N; n += 32) p.final_state[(b * D + c) * N + n] = carry[n];
}

template <typename T>
cudaError_t launch_t(const M1Params &p, cudaStream_t s) {
  dim3 grid((unsigned)((p.D + kFwdWarps - 1) / kFwdWarps), (unsigned)p.B);
  m1_fwd_kernel<T><<<grid, kFwdWarps * 32, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_m1_fwd(const M1Params &p, cudaStream_t s) {
  return p.io_bf16 ? launch_t<bf16>(p, s) : launch_t<float>(p, s);
}

}  // namespace msc
