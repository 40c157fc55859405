// m3_disc.cu -- Mamba-3 SISO discretisation and BCNorm ahead of the scan
// (sm_100a), and their backward.
//
// Stage B6 "discretization" of Mamba3Scratch (mamba-rs 0.4.2
// src/mamba3_siso/cpu/scratch.rs: d_dd_dt, d_dd_a, d_trap [T * nheads],
// d_angles [T * n_angles]) read as the exponential-trapezoid discretisation of
// the Mamba-3 paper, and stage B5 "BCNorm" (d_b_raw, d_c_raw):
//   dt = softplus(dd_dt + dt_bias[h]),  A = min(-softplus(dd_a), -A_floor)
//   alpha = exp(dt A),  lam = sigmoid(trap)
//   beta = (1 - lam) dt alpha,  gamma = lam dt,  theta[k] = dt angles[k]
//   B = B_raw / sqrt(mean_n B_raw^2 + eps)   (C likewise)
//
// Both directions are elementwise per token apart from two sums: a token's
// B and C rows are normalised over d_state (and the backward needs two dot
// products per row), and the backward's dangles and ddt_bias sum over heads
// and over tokens.  A warp owns one token at a time: its lanes walk the
// heads, the (head, angle) entries of theta (contiguous per token), and the
// d_state entries of each B and C row, with shuffle sums in a fixed butterfly
// order.  The per-head dt and the angles of the token are kept in shared
// memory for the theta and dangles passes; the backward also stages the
// token's dtheta rows there (16-byte loads).  B and C rows whose length is 8
// times a power of two move in 16-byte pieces, several rows per warp pass.
// ddt_bias is a second, fixed-order pass over ddd_dt (one CTA per head).
// Bound: HBM (the theta write dominates the forward, the dtheta read the
// backward).
#include "kernels.h"
#include "m3_disc_common.cuh"

namespace msc {
namespace {

constexpr int kDiscWarps = 8;
constexpr unsigned kFullMask = 0xffffffffu;

template <typename T>
__device__ __forceinline__ float ldv(const void *p, int64_t i) {
  return to_f32(static_cast<const T *>(p)[i]);
}

// the same sum in every lane (xor butterfly: partners add the same two values)
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(kFullMask, v, m);
  return v;
}

template <typename T>
__device__ __forceinline__ DiscCoef head_coef(const M3DiscParams &p, int64_t i, int h) {
  return disc_coef(ldv<T>(p.dd_dt, i), p.dt_bias ? p.dt_bias[h] : 0.f, ldv<T>(p.dd_a, i),
                   ldv<T>(p.trap, i), p.A_floor);
}

// Row pieces of 8 elements: a B or C row of N = 8 S elements (S a power of
// two <= 32) is served by S lanes, 32 / S rows per pass, 16-byte accesses.
__device__ __forceinline__ int row_lanes(int N) { return disc_row_lanes(N); }

// the same sum in every lane of each aligned group of `seg` lanes
__device__ __forceinline__ float seg_sum(float v, int seg) {
#pragma unroll
  for (int m = 1; m < 32; m <<= 1)
    if (m < seg) v += __shfl_xor_sync(kFullMask, v, m);
  return v;
}

template <typename T>
__device__ __forceinline__ void load8(const void *p, int64_t i, float (&v)[8]) {
  if constexpr (sizeof(T) == 2) {
    const uint4 w = *reinterpret_cast<const uint4 *>(static_cast<const T *>(p) + i);
    unpack2<T>(w.x, v[0], v[1]);
    unpack2<T>(w.y, v[2], v[3]);
    unpack2<T>(w.z, v[4], v[5]);
    unpack2<T>(w.w, v[6], v[7]);
  } else {
    const float4 a = *reinterpret_cast<const float4 *>(static_cast<const float *>(p) + i);
    const float4 b = *reinterpret_cast<const float4 *>(static_cast<const float *>(p) + i + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

template <typename T>
__device__ __forceinline__ void store8(void *p, int64_t i, const float (&v)[8]) {
  if constexpr (sizeof(T) == 2) {
    *reinterpret_cast<uint4 *>(static_cast<T *>(p) + i) =
        make_uint4(pack2<T>(v[0], v[1]), pack2<T>(v[2], v[3]), pack2<T>(v[4], v[5]),
                   pack2<T>(v[6], v[7]));
  } else {
    float *q = static_cast<float *>(p) + i;
    *reinterpret_cast<float4 *>(q) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4 *>(q + 4) = make_float4(v[4], v[5], v[6], v[7]);
  }
}

__device__ __forceinline__ void load8f(const float *p, int64_t i, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4 *>(p + i);
  const float4 b = *reinterpret_cast<const float4 *>(p + i + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// shared floats per warp: dt [H], angles [K], and (backward) the token's
// dtheta rows [H][K + 1] (padded: the per-head pass reads down a column)
__host__ __device__ __forceinline__ int64_t disc_warp_floats(int64_t H, int64_t K, bool bwd) {
  return H + K + (bwd ? H * (K + 1) : 0);
}

template <typename T>
__global__ void __launch_bounds__(kDiscWarps * 32) m3_disc_fwd_kernel(const M3DiscParams p) {
  extern __shared__ float sm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = (int)p.H, K = (int)p.K, N = (int)p.N, G = (int)p.G;
  float *sdt = sm + warp * disc_warp_floats(H, K, false);
  float *sang = sdt + H;
  const int seg = row_lanes(N);
  const bool vec_theta = K % 8 == 0;
  const int64_t ntok = p.B * p.L;
  for (int64_t tok = (int64_t)blockIdx.x * kDiscWarps + warp; tok < ntok;
       tok += (int64_t)gridDim.x * kDiscWarps) {
    for (int h = lane; h < H && !p.bc_only; h += 32) {
      const int64_t i = tok * H + h;
      const DiscCoef c = head_coef<T>(p, i, h);
      static_cast<T *>(p.alpha)[i] = from_f32<T>(c.alpha);
      static_cast<T *>(p.beta)[i] = from_f32<T>(disc_beta(c));
      static_cast<T *>(p.gamma)[i] = from_f32<T>(disc_gamma(c));
      sdt[h] = c.dt;
    }
    const int Kd = p.bc_only ? 0 : K;  // BCNorm alone: no theta
    for (int k = lane; k < Kd; k += 32) sang[k] = ldv<T>(p.angles, tok * K + k);
    __syncwarp();
    if (vec_theta) {  // 8 angles of one head per lane, one 16-byte store (f32: two)
      for (int j = 8 * lane; j < H * Kd; j += 256) {
        const int h = j / K, k = j - h * K;
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = sdt[h] * sang[k + e];
        store8<T>(p.theta, tok * H * K + j, v);
      }
    } else {
      for (int j = lane; j < H * Kd; j += 32) {
        const int h = j / K, k = j - h * K;
        static_cast<T *>(p.theta)[tok * H * K + j] = from_f32<T>(sdt[h] * sang[k]);
      }
    }
    if (seg > 0) {
      // rows 0 .. G-1 are B's groups, G .. 2G-1 C's; seg lanes per row
      const int per = 32 / seg;
      for (int r0 = 0; r0 < 2 * G; r0 += per) {
        const int r = r0 + lane / seg, pc = lane % seg;
        const bool act = r < 2 * G;
        const void *raw = r < G ? p.B_raw : p.C_raw;
        void *out = r < G ? p.Bm : p.Cm;
        const int64_t off = (tok * G + (r < G ? r : r - G)) * N + pc * 8;
        float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (act) load8<T>(raw, off, v);
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(v[e], v[e], ss);
        const float rn = rsqrtf(seg_sum(ss, seg) / (float)N + p.eps);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] *= rn;
        if (act) store8<T>(out, off, v);
      }
    } else {
      for (int q = 0; q < 2 * G; ++q) {
        const void *raw = q < G ? p.B_raw : p.C_raw;
        T *out = static_cast<T *>(q < G ? p.Bm : p.Cm);
        const int64_t row = (tok * G + (q < G ? q : q - G)) * N;
        float ss = 0.f;
        for (int n = lane; n < N; n += 32) {
          const float v = ldv<T>(raw, row + n);
          ss = fmaf(v, v, ss);
        }
        const float rn = rsqrtf(warp_sum(ss) / (float)N + p.eps);
        for (int n = lane; n < N; n += 32) out[row + n] = from_f32<T>(ldv<T>(raw, row + n) * rn);
      }
    }
    __syncwarp();  // the shared rows are rewritten for the next token
  }
}

template <typename T>
__global__ void __launch_bounds__(kDiscWarps * 32) m3_disc_bwd_kernel(const M3DiscParams p) {
  extern __shared__ float sm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = (int)p.H, K = (int)p.K, N = (int)p.N, G = (int)p.G;
  float *sdt = sm + warp * disc_warp_floats(H, K, true);
  float *sang = sdt + H;
  float *sth = sang + K;  // [H][K + 1]
  const int seg = row_lanes(N);
  const int64_t ntok = p.B * p.L;
  for (int64_t tok = (int64_t)blockIdx.x * kDiscWarps + warp; tok < ntok;
       tok += (int64_t)gridDim.x * kDiscWarps) {
    for (int h = lane; h < H; h += 32)
      sdt[h] = softplus(ldv<T>(p.dd_dt, tok * H + h) + (p.dt_bias ? p.dt_bias[h] : 0.f));
    for (int k = lane; k < K; k += 32) sang[k] = ldv<T>(p.angles, tok * K + k);
    // the token's dtheta [H][K], contiguous: 16-byte loads when rows allow
    const float *dth = p.dtheta + tok * H * K;
    if ((H * K) % 4 == 0) {
      for (int j = 4 * lane; j < H * K; j += 128) {
        const float4 v = *reinterpret_cast<const float4 *>(dth + j);
        const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int h = (j + q) / K, k = j + q - h * K;
          sth[h * (K + 1) + k] = e[q];
        }
      }
    } else {
      for (int j = lane; j < H * K; j += 32) {
        const int h = j / K, k = j - h * K;
        sth[h * (K + 1) + k] = dth[j];
      }
    }
    __syncwarp();
    // dangles[k] = sum_h dtheta[h, k] dt[h], heads in ascending order
    for (int k = lane; k < K; k += 32) {
      float s = 0.f;
      for (int h = 0; h < H; ++h) s = fmaf(sth[h * (K + 1) + k], sdt[h], s);
      p.dangles[tok * K + k] = s;
    }
    for (int h = lane; h < H; h += 32) {
      const int64_t i = tok * H + h;
      const DiscCoef c = head_coef<T>(p, i, h);
      float gth = 0.f;  // sum_k dtheta[h, k] angles[k]
      for (int k = 0; k < K; ++k) gth = fmaf(sth[h * (K + 1) + k], sang[k], gth);
      const float ga = p.dalpha[i], gb = p.dbeta[i], gg = p.dgamma[i];
      const float g_alpha = fmaf(gb * (1.f - c.lam), c.dt, ga);  // alpha directly and via beta
      const float d_dt = g_alpha * c.alpha * c.A + gb * (1.f - c.lam) * c.alpha + gg * c.lam + gth;
      const float d_A = g_alpha * c.alpha * c.dt;
      const float d_lam = (gg - gb * c.alpha) * c.dt;
      p.ddd_dt[i] = d_dt * c.sig_u;
      p.ddd_a[i] = d_A * c.dA_dda;
      p.dtrap[i] = d_lam * c.lam * (1.f - c.lam);
    }
    // RMS-norm backward per row: dx = r (g - xh mean(g xh)), xh = x r
    if (seg > 0) {
      const int per = 32 / seg;
      for (int r0 = 0; r0 < 2 * G; r0 += per) {
        const int r = r0 + lane / seg, pc = lane % seg;
        const bool act = r < 2 * G;
        const void *raw = r < G ? p.B_raw : p.C_raw;
        const float *g = r < G ? p.dB : p.dC;
        float *dout = r < G ? p.dB_raw : p.dC_raw;
        const int64_t off = (tok * G + (r < G ? r : r - G)) * N + pc * 8;
        float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, gv[8] = {0.f, 0.f, 0.f, 0.f,
                                                                        0.f, 0.f, 0.f, 0.f};
        if (act) {
          load8<T>(raw, off, v);
          load8f(g, off, gv);
        }
        float ss = 0.f, gx = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          ss = fmaf(v[e], v[e], ss);
          gx = fmaf(gv[e], v[e], gx);
        }
        const float rn = rsqrtf(seg_sum(ss, seg) / (float)N + p.eps);
        const float m = seg_sum(gx, seg) * rn * rn / (float)N;  // mean(g xh) / r
        float d[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) d[e] = rn * (gv[e] - v[e] * m);
        if (act) store8<float>(dout, off, d);
      }
    } else {
      for (int q = 0; q < 2 * G; ++q) {
        const void *raw = q < G ? p.B_raw : p.C_raw;
        const float *g = q < G ? p.dB : p.dC;
        float *dout = q < G ? p.dB_raw : p.dC_raw;
        const int64_t row = (tok * G + (q < G ? q : q - G)) * N;
        float ss = 0.f, gx = 0.f;
        for (int n = lane; n < N; n += 32) {
          const float v = ldv<T>(raw, row + n);
          ss = fmaf(v, v, ss);
          gx = fmaf(g[row + n], v, gx);
        }
        const float rn = rsqrtf(warp_sum(ss) / (float)N + p.eps);
        const float m = warp_sum(gx) * rn * rn / (float)N;
        for (int n = lane; n < N; n += 32)
          dout[row + n] = rn * (g[row + n] - ldv<T>(raw, row + n) * m);
      }
    }
    __syncwarp();
  }
}

// ddt_bias[h] = sum over tokens of ddd_dt[., h]: per-thread sums over a fixed
// stride of tokens, then a fixed tree over the CTA
__global__ void __launch_bounds__(256) m3_disc_bias_kernel(const M3DiscParams p) {
  __shared__ float red[8];
  const int64_t h = blockIdx.x, ntok = p.B * p.L;
  float s = 0.f;
  for (int64_t t = threadIdx.x; t < ntok; t += 256) s += p.ddd_dt[t * p.H + h];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_down_sync(kFullMask, s, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
    for (int w = 0; w < 8; ++w) tot += red[w];
    p.ddt_bias[h] = tot;
  }
}

template <typename T>
cudaError_t launch_t(const M3DiscParams &p, cudaStream_t s, bool bwd) {
  const int64_t ntok = p.B * p.L;
  int64_t blocks = (ntok + kDiscWarps - 1) / kDiscWarps;
  if (blocks > 148 * 8) blocks = 148 * 8;
  const size_t smem = sizeof(float) * kDiscWarps * (size_t)disc_warp_floats(p.H, p.K, bwd);
  if (!bwd) {
    cudaError_t e = cudaFuncSetAttribute(m3_disc_fwd_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    m3_disc_fwd_kernel<T><<<(unsigned)blocks, kDiscWarps * 32, smem, s>>>(p);
    return cudaGetLastError();
  }
  cudaError_t e = cudaFuncSetAttribute(m3_disc_bwd_kernel<T>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  m3_disc_bwd_kernel<T><<<(unsigned)blocks, kDiscWarps * 32, smem, s>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess || !p.ddt_bias) return e;
  m3_disc_bias_kernel<<<(unsigned)p.H, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch(const M3DiscParams &p, cudaStream_t s, bool bwd) {
  switch (p.io) {
    case 1: return launch_t<bf16>(p, s, bwd);
    case 2: return launch_t<f16>(p, s, bwd);
    default: return launch_t<float>(p, s, bwd);
  }
}

}  // namespace

cudaError_t launch_m3_disc_fwd(const M3DiscParams &p, cudaStream_t s) { return launch(p, s, false); }
cudaError_t launch_m3_disc_bwd(const M3DiscParams &p, cudaStream_t s) { return launch(p, s, true); }

}  // namespace msc
