// m3_state_update.cu -- Mamba-3 SISO single-token state update (decode).
//
// One step of the Mamba-3 SISO recurrence (mamba-rs 0.7.0 README, "Features";
// the step mamba3_step applies to a Mamba3State, the same README, "Quick
// start (CPU)") for every (b, h), on a carried state S [P][N], the last
// input x_prev [P], the last rotated key bt_prev [N] and the cumulative
// angles phi [K]:
//   phi <- phi + theta;  Bt = R(phi) B;  Ct = R(phi) C
//   S   <- alpha S + beta x_prev (outer) bt_prev + gamma x (outer) Bt
//   out  = (S Ct + D x) silu(z);   x_prev <- x;  bt_prev <- Bt
//
// The step is bound by HBM: S is read and written once (2 P N 4 bytes per
// head), everything else is a few hundred bytes per head.  A head is served
// by P N / 16 threads, N / 16 per row of S, each holding 16 state entries as
// four 16-byte pieces interleaved with its row neighbours' (so that the
// threads of a row read and write one contiguous run per instruction).  A
// CTA of 256 threads serves 256 / (P N / 16) heads.  Per head, the first N/2
// threads rotate one pair of B and C each into shared memory (sin and cos by
// Cody and Waite's reduction and the SFU, common.cuh); y sums a row's
// partials over its N / 16 threads with shuffles in a fixed order.  Wider
// states (128, 192, 256) are walked in slabs of 64 states with the 64-state
// layout, y carried across the slabs in registers.
//
// kRaw fuses the discretisation and BCNorm ahead (m3_disc_common.cuh): the
// first lanes of a head (its first warp, or half-warp when a warp holds two
// heads) derive dt, alpha, beta, gamma from dd_dt, dd_a, trap and the RMS
// scales of the head's raw B and C rows, and the rotating threads take
// theta = dt angles.  Up to 64 states the rotating lanes hold the whole row,
// so everything comes from one round of loads and shuffles; wider states
// take a pass over the raw rows first.  Every derived value is rounded to
// the io type and the row sums follow the discretisation kernel's order, so
// the fused step gives the same bits as the discretisation kernel followed
// by the plain step.
#include "kernels.h"
#include "m3_disc_common.cuh"

namespace msc {
namespace {

constexpr int kSUThreads = 256;

template <typename T>
__device__ __forceinline__ float ldf(const void *base, int64_t i) {
  return to_f32(static_cast<const T *>(base)[i]);
}

// The RMS scale 1/sqrt(mean(v^2) + eps) of the raw row at `row` (N entries),
// its square sum taken in the discretisation kernel's order: in the 16-byte
// path lane l < S sums its 8 entries in order and the S lanes add with xor
// shuffles at distances 1, 2, ...; otherwise lane l sums entries l, l + 32, ...
// and the warp adds at distances 16, 8, ....  Every lane of the warp calls it;
// lane l of each aligned group of kLW lanes takes the role of lane l there,
// and the group's lane 0 holds the result.
template <typename T, int N, int kLW>
__device__ __forceinline__ float raw_rms_scale(const void *raw, int64_t row, bool live, int lg,
                                               float eps) {
  constexpr int kS = disc_row_lanes(N);
  float ss = 0.f;
  if constexpr (kS > 0) {
    static_assert(kS <= kLW, "a row's lanes sit in one group");
    if (live && lg < kS) {
      const T *src = static_cast<const T *>(raw) + row + lg * 8;
      float v[8];
      if constexpr (sizeof(T) == 2) {
        const uint4 w = *reinterpret_cast<const uint4 *>(src);
        unpack2<T>(w.x, v[0], v[1]);
        unpack2<T>(w.y, v[2], v[3]);
        unpack2<T>(w.z, v[4], v[5]);
        unpack2<T>(w.w, v[6], v[7]);
      } else {
        const float4 a = reinterpret_cast<const float4 *>(src)[0];
        const float4 b = reinterpret_cast<const float4 *>(src)[1];
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(v[e], v[e], ss);
    }
#pragma unroll
    for (int m = 1; m < kS; m <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
  } else {
    static_assert(kLW == 32, "the scalar path uses whole warps");
    if (live)
      for (int n = lg; n < N; n += 32) {
        const float v = ldf<T>(raw, row + n);
        ss = fmaf(v, v, ss);
      }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
  }
  return rsqrtf(ss / (float)N + eps);
}

// The same scale when the row (N = 16, 32 or 64) is held in registers, two
// consecutive entries (e0, e1) per lane j < N / 2 of a group of kLW lanes:
// the discretisation kernel's lane l (8 entries) is lanes 4 l .. 4 l + 3 here,
// so its running sum is passed along those four lanes, and its xor tree over
// l becomes one over lane distances 4, 8, 16.  Lane 3 of the group ends with
// the sum and broadcasts the scale.  Every lane of the warp calls it.
template <int N, int kLW>
__device__ __forceinline__ float pair_rms_scale(float e0, float e1, int j, float eps) {
  constexpr int kS = disc_row_lanes(N);
  static_assert(kS > 0 && 4 * kS <= kLW && N <= 64, "the row sits in one lane group");
  float s = fmaf(e1, e1, __fmul_rn(e0, e0));
#pragma unroll
  for (int r = 1; r < 4; ++r) {
    const float prev = __shfl_up_sync(0xffffffffu, s, 1);
    if ((j & 3) == r) s = fmaf(e1, e1, fmaf(e0, e0, prev));
  }
#pragma unroll
  for (int m = 1; m < kS; m <<= 1) s += __shfl_xor_sync(0xffffffffu, s, 4 * m);
  s = __shfl_sync(0xffffffffu, s, 3, kLW);
  return rsqrtf(s / (float)N + eps);
}

template <typename T, int P, int N, bool kRaw>
__global__ void __launch_bounds__(kSUThreads) m3_state_update_kernel(const M3SUParams p) {
  constexpr int kSN = N < 64 ? N : 64;     // states per slab (wider states: slabs of 64 in turn)
  constexpr int kNS = N / kSN;             // slabs
  constexpr int kTPR = kSN / 16;           // threads per row of a slab
  constexpr int kTPH = P * kTPR;           // threads per head
  constexpr int kHPC = kSUThreads / kTPH;  // heads per CTA
  constexpr int kLW = kTPH < 32 ? kTPH : 32;  // lanes of a head in its first warp
  // shared floats per head: Bt, Ct, bt_prev (a slab), x_prev; (kRaw) alpha, beta, gamma
  constexpr int kPer = 3 * kSN + P + (kRaw ? 4 : 0);
  __shared__ __align__(16) float sm[kHPC * kPer];

  const int tid = threadIdx.x;
  const int hl = tid / kTPH, j = tid % kTPH;
  const int64_t BH = p.B * p.H;
  const int64_t bh = (int64_t)blockIdx.x * kHPC + hl;
  const bool live = bh < BH;
  const int64_t b = bh / p.H, h = bh % p.H;
  const int64_t g = h / (p.H / p.G);
  const int K = (int)p.K;
  float *sBt = sm + hl * kPer, *sCt = sBt + kSN, *sBp = sCt + kSN, *sXp = sBp + kSN;
  const int row = j / kTPR, q = j % kTPR;
  float4 *srow = reinterpret_cast<float4 *>(p.state + (bh * P + row) * N);

  float al = 0.f, be = 0.f, ga = 0.f, xv = 0.f;
  float dt = 0.f, rB = 0.f, rC = 0.f;  // kRaw: the head's dt and B, C scales (rotating lanes)
  if constexpr (kRaw) {
    if (live) {
      xv = ldf<T>(p.x, bh * P + row);
      for (int i = j; i < P; i += kTPH) sXp[i] = p.x_prev[bh * P + i];
    }
  } else if (live) {
    al = ldf<T>(p.alpha, bh);
    be = ldf<T>(p.beta, bh);
    ga = ldf<T>(p.gamma, bh);
    xv = ldf<T>(p.x, bh * P + row);
    for (int i = j; i < P; i += kTPH) sXp[i] = p.x_prev[bh * P + i];
  }
  float y = 0.f;
#pragma unroll
  for (int sl = 0; sl < kNS; ++sl) {
    const int n0 = sl * kSN;
    // this thread's state entries of the slab and the slab's rotated B and
    // C; the carried bt_prev of the slab
    float4 st[4];
    if (live) {
#pragma unroll
      for (int i = 0; i < 4; ++i) st[i] = srow[n0 / 4 + i * kTPR + q];
    }
    if constexpr (kRaw && kNS > 1) {
      // (wide states; first slab, after the state loads are under way) the
      // head's dt, alpha, beta, gamma and the scales of its raw B and C rows
      if (sl == 0 && j < kLW) {  // the head's first lanes; every lane of their warp is here
        float *sCoef = sXp + P;
        if (live) {
          const DiscCoef c = disc_coef(ldf<T>(p.dd_dt, bh), p.dt_bias ? p.dt_bias[h] : 0.f,
                                       ldf<T>(p.dd_a, bh), ldf<T>(p.trap, bh), p.A_floor);
          dt = c.dt;
          if (j == 0) {
            sCoef[0] = to_f32(from_f32<T>(c.alpha));
            sCoef[1] = to_f32(from_f32<T>(disc_beta(c)));
            sCoef[2] = to_f32(from_f32<T>(disc_gamma(c)));
          }
        }
        const int64_t brow = (b * p.G + g) * N;
        rB = __shfl_sync(0xffffffffu, raw_rms_scale<T, N, kLW>(p.B_raw, brow, live, j, p.eps),
                         0, kLW);
        rC = __shfl_sync(0xffffffffu, raw_rms_scale<T, N, kLW>(p.C_raw, brow, live, j, p.eps),
                         0, kLW);
      }
    }
    if constexpr (kRaw && kNS == 1) {
      // the whole row in one slab: the rotating lanes load their raw pairs,
      // the angle and the head's raw scalars together, derive the coefficients
      // and the row scales in registers, and rotate
      if (j < kLW) {  // every lane of the warp is here
        const bool rot = live && j < kSN / 2;
        const int64_t o = (b * p.G + g) * N + 2 * j;
        float e0 = 0.f, e1 = 0.f, f0 = 0.f, f1 = 0.f, ang = 0.f;
        if (rot) {
          e0 = ldf<T>(p.B_raw, o); e1 = ldf<T>(p.B_raw, o + 1);
          f0 = ldf<T>(p.C_raw, o); f1 = ldf<T>(p.C_raw, o + 1);
          if (j < K) ang = ldf<T>(p.angles, b * K + j);
        }
        if (live) {
          const DiscCoef c = disc_coef(ldf<T>(p.dd_dt, bh), p.dt_bias ? p.dt_bias[h] : 0.f,
                                       ldf<T>(p.dd_a, bh), ldf<T>(p.trap, bh), p.A_floor);
          dt = c.dt;
          if (j == 0) {
            float *sCoef = sXp + P;
            sCoef[0] = to_f32(from_f32<T>(c.alpha));
            sCoef[1] = to_f32(from_f32<T>(disc_beta(c)));
            sCoef[2] = to_f32(from_f32<T>(disc_gamma(c)));
          }
        }
        rB = pair_rms_scale<N, kLW>(e0, e1, j, p.eps);
        rC = pair_rms_scale<N, kLW>(f0, f1, j, p.eps);
        if (rot) {
          float b0 = to_f32(from_f32<T>(__fmul_rn(e0, rB)));
          float b1 = to_f32(from_f32<T>(__fmul_rn(e1, rB)));
          float c0 = to_f32(from_f32<T>(__fmul_rn(f0, rC)));
          float c1 = to_f32(from_f32<T>(__fmul_rn(f1, rC)));
          if (j < K) {
            const float th = to_f32(from_f32<T>(__fmul_rn(dt, ang)));
            const float phi = p.phi[bh * K + j] + th;
            p.phi[bh * K + j] = phi;
            float sn, cs;
            sincos_reduced(phi, sn, cs);
            const float rb0 = cs * b0 - sn * b1, rb1 = sn * b0 + cs * b1;
            const float rc0 = cs * c0 - sn * c1, rc1 = sn * c0 + cs * c1;
            b0 = rb0; b1 = rb1; c0 = rc0; c1 = rc1;
          }
          sBt[2 * j] = b0; sBt[2 * j + 1] = b1;
          sCt[2 * j] = c0; sCt[2 * j + 1] = c1;
        }
      }
      if (live)
        for (int i = j; i < kSN; i += kTPH) sBp[i] = p.bt_prev[bh * N + n0 + i];
    } else if (live) {
      if (j < kSN / 2) {
        const int ka = n0 / 2 + j;  // global angle pair
        const int64_t o = (b * p.G + g) * N + n0 + 2 * j;
        float b0, b1, c0, c1;
        // (kRaw) products in __fmul_rn: with f32 io nothing rounds between them
        // and their next use, and a contraction into an FMA would change the bits
        if constexpr (kRaw) {  // normalised as the discretisation kernel stores them
          b0 = to_f32(from_f32<T>(__fmul_rn(ldf<T>(p.B_raw, o), rB)));
          b1 = to_f32(from_f32<T>(__fmul_rn(ldf<T>(p.B_raw, o + 1), rB)));
          c0 = to_f32(from_f32<T>(__fmul_rn(ldf<T>(p.C_raw, o), rC)));
          c1 = to_f32(from_f32<T>(__fmul_rn(ldf<T>(p.C_raw, o + 1), rC)));
        } else {
          b0 = ldf<T>(p.Bm, o); b1 = ldf<T>(p.Bm, o + 1);
          c0 = ldf<T>(p.Cm, o); c1 = ldf<T>(p.Cm, o + 1);
        }
        if (ka < K) {
          const float th = kRaw ? to_f32(from_f32<T>(__fmul_rn(dt, ldf<T>(p.angles, b * K + ka))))
                                : ldf<T>(p.theta, bh * K + ka);
          const float phi = p.phi[bh * K + ka] + th;
          p.phi[bh * K + ka] = phi;
          float sn, cs;
          sincos_reduced(phi, sn, cs);
          const float rb0 = cs * b0 - sn * b1, rb1 = sn * b0 + cs * b1;
          const float rc0 = cs * c0 - sn * c1, rc1 = sn * c0 + cs * c1;
          b0 = rb0; b1 = rb1; c0 = rc0; c1 = rc1;
        }
        sBt[2 * j] = b0; sBt[2 * j + 1] = b1;
        sCt[2 * j] = c0; sCt[2 * j + 1] = c1;
      }
      for (int i = j; i < kSN; i += kTPH) sBp[i] = p.bt_prev[bh * N + n0 + i];
    }
    __syncthreads();
    if constexpr (kRaw) {
      if (sl == 0) {
        const float *sCoef = sXp + P;
        al = sCoef[0]; be = sCoef[1]; ga = sCoef[2];
      }
    }
    if (live) {
      // the carried key of the next step (every read of the old one is done)
      for (int i = j; i < kSN; i += kTPH) p.bt_prev[bh * N + n0 + i] = sBt[i];
      const float bxq = be * sXp[row], gx = ga * xv;
      const float4 *vBt = reinterpret_cast<const float4 *>(sBt);
      const float4 *vCt = reinterpret_cast<const float4 *>(sCt);
      const float4 *vBp = reinterpret_cast<const float4 *>(sBp);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int v = i * kTPR + q;
        const float4 bt = vBt[v], ct = vCt[v], bp = vBp[v];
        st[i].x = fmaf(al, st[i].x, fmaf(bxq, bp.x, gx * bt.x));
        st[i].y = fmaf(al, st[i].y, fmaf(bxq, bp.y, gx * bt.y));
        st[i].z = fmaf(al, st[i].z, fmaf(bxq, bp.z, gx * bt.z));
        st[i].w = fmaf(al, st[i].w, fmaf(bxq, bp.w, gx * bt.w));
        y = fmaf(ct.x, st[i].x, y);
        y = fmaf(ct.y, st[i].y, y);
        y = fmaf(ct.z, st[i].z, y);
        y = fmaf(ct.w, st[i].w, y);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) srow[n0 / 4 + i * kTPR + q] = st[i];
    }
    if (kNS > 1) __syncthreads();  // the slab's tables are free for the next slab
  }
  if (!live) return;
  for (int i = j; i < P; i += kTPH) p.x_prev[bh * P + i] = ldf<T>(p.x, bh * P + i);
  // (kTPR > 1 only for N >= 32, where a warp holds threads of one head only,
  // so no lane of a shuffling warp has returned above)
#pragma unroll
  for (int off = 1; off < kTPR; off <<= 1) y += __shfl_xor_sync(0xffffffffu, y, off, kTPR);
  if (q == 0) {
    if (p.Dp) y = fmaf(p.Dp[h], xv, y);
    if (p.z) y *= silu(ldf<T>(p.z, bh * P + row));
    static_cast<T *>(p.out)[bh * P + row] = from_f32<T>(y);
  }
}

template <typename T, int P, int N>
cudaError_t launch_pn(const M3SUParams &p, cudaStream_t s) {
  constexpr int kHPC = kSUThreads / (P * (N < 64 ? N : 64) / 16);
  const int64_t blocks = (p.B * p.H + kHPC - 1) / kHPC;
  if (p.raw)
    m3_state_update_kernel<T, P, N, true><<<(unsigned)blocks, kSUThreads, 0, s>>>(p);
  else
    m3_state_update_kernel<T, P, N, false><<<(unsigned)blocks, kSUThreads, 0, s>>>(p);
  return cudaGetLastError();
}

template <typename T, int P>
cudaError_t launch_p(const M3SUParams &p, cudaStream_t s) {
  switch (p.N) {
    case 16: return launch_pn<T, P, 16>(p, s);
    case 32: return launch_pn<T, P, 32>(p, s);
    case 64: return launch_pn<T, P, 64>(p, s);
    case 128: return launch_pn<T, P, 128>(p, s);
    case 192: return launch_pn<T, P, 192>(p, s);
    default: return launch_pn<T, P, 256>(p, s);
  }
}

template <typename T>
cudaError_t launch_t(const M3SUParams &p, cudaStream_t s) {
  switch (p.P) {
    case 16: return launch_p<T, 16>(p, s);
    case 32: return launch_p<T, 32>(p, s);
    default: return launch_p<T, 64>(p, s);
  }
}

}  // namespace

cudaError_t launch_m3_state_update(const M3SUParams &p, cudaStream_t s) {
  switch (p.io) {
    case 1: return launch_t<bf16>(p, s);
    case 2: return launch_t<f16>(p, s);
    default: return launch_t<float>(p, s);
  }
}

}  // namespace msc
