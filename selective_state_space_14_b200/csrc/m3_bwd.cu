// m3_bwd.cu -- Mamba-3 SISO scan, backward for f32 and f16 io (sm_100a, CUDA
// cores): backward stages B2 (output gating), B3 (BPTT through the
// trapezoidal state) and B4 (RoPE) of Mamba3Scratch in mamba-rs 0.4.2
// src/mamba3_siso/cpu/scratch.rs.  bf16 io runs the chunk-parallel
// tensor-core backward of m3_bwd_umma.cu, which uses the same chunk algebra.
//
// Chunk-local notation as in m3_common.cuh (t, s, tau in [0, Q); g_t the
// gradient of y_t, i.e. dout_t silu(z_t)).  The state adjoint
// Lambda_t = dL/dS_t is never formed step by step: with U the adjoint of the
// first state of the next chunk (its alpha, beta written alpha_Q, beta_Q),
//   Lambda_t = sum_{tau>=t} d(tau,t) g_tau (outer) Ct_tau + d(Q-1,t) alpha_Q U,
// and every gradient is a contraction of chunk tiles:
//   dK_t   = sum_tau c(tau,t) g_tau (outer) Ct_tau + wU_t U,
//            wU_t = alpha_Q c(Q-1,t) + [t = Q-1] beta_Q
//   dX     = W^T G + diag(wU) Bt U^T + D G                       (W = c o Ct Bt^T)
//   dBt    = (c o G X^T)^T Ct + diag(wU) X U
//   dCt    = diag(d(.,-1)) G S_in + (c o G X^T) Bt + beta_0 diag(d(.,0)) (G x_prev) Bt_prev^T
//   U_prev = G^T diag(d(.,0)) Ct + d(Q-1,0) alpha_Q U             (adjoint of the chunk's S_0)
//   dgamma_s = sum_{tau>=s} d(tau,s) (Ct_tau.Bt_s)(g_tau.x_s) + alpha_Q d(Q-1,s) v_s
//   dbeta_s  = sum_{tau>=s} d(tau,s) (Ct_tau.Bt_{s-1})(g_tau.x_{s-1}) + alpha_Q d(Q-1,s) v_{s-1}
//     (v_s = x_s^T U Bt_s; index -1 is the previous chunk's last step)
//   dalpha_s = <Lambda_s, S_{s-1}>, taken without any subtraction: every term of it
//     carries alpha_s, so with the U row written as tau = Q (d(Q,.) = alpha_Q d(Q-1,.),
//     c(Q,.) = alpha_Q c(Q-1,.), its "a" = <U, S_in>, "e" = v_{-1}, "M" = v) and
//     M(tau,j) = (Ct_tau.Bt_j)(g_tau.x_j), a_tau = g_tau^T S_in Ct_tau,
//     e_tau = (Ct_tau.Bt_prev)(g_tau.x_prev):
//   dalpha_s = (1/alpha_s) sum_{tau=s..Q} [d(tau,-1) a_tau + beta_0 d(tau,0) e_tau
//                                          + sum_{j<=s-2} c(tau,j) M(tau,j)]
//              + gamma_{s-1} dbeta_s                                   (s >= 1)
//   dalpha_0 = sum_{tau=0..Q} d(tau,0) a_tau
// The RoPE backward rotates dBt, dCt back (R^T) per head, forms dphi and
// the reverse cumulative sum dtheta; the per-head dB, dC go to the workspace
// and a second kernel adds the heads of each group in ascending order.
// One CTA per (b, h) walks the chunks from last to first; the chunk-start
// states come from the forward's saved states, the chunk-start angles from a
// sequential sum per angle identical to the forward's.  The contractions are
// f32 on the CUDA cores (mm in m3_common.cuh).
#include "m3_common.cuh"

namespace msc {
namespace {

using namespace m3;

// 8 consecutive io elements from global memory at index j (16-byte aligned
// for bf16), or zeros when !valid
template <typename T>
__device__ __forceinline__ void ld8(const void *base, int64_t j, bool valid, float (&v)[8]) {
  if (!valid) {
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = 0.f;
    return;
  }
  if constexpr (sizeof(T) == 2) {
    const uint4 r = __ldg(reinterpret_cast<const uint4 *>(static_cast<const T *>(base) + j));
    unpack2<T>(r.x, v[0], v[1]);
    unpack2<T>(r.y, v[2], v[3]);
    unpack2<T>(r.z, v[4], v[5]);
    unpack2<T>(r.w, v[6], v[7]);
  } else {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(base) + j));
    const float4 c = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(base) + j + 4));
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = c.x; v[5] = c.y; v[6] = c.z; v[7] = c.w;
  }
}

// Sum over the CTA's kThreads threads in a fixed order (warp butterflies, then
// the warp sums in warp order); every thread gets the sum.  Contains block
// barriers: call from uniform control flow.
__device__ __forceinline__ float block_sum(float v, float *sRed) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  if ((threadIdx.x & 31) == 0) sRed[threadIdx.x >> 5] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) s += sRed[w];
  __syncthreads();
  return s;
}

template <int P, int N>
struct BwdSmem {
  static constexpr int kK = N / 2;
  static constexpr int kMx = (P > N ? P : N) > kQ ? (P > N ? P : N) : kQ;  // widest row
  // row strides, padded by 4 floats so that the tensor-core fragment loads
  // (8 rows x 4 columns per instruction) spread over the banks
  static constexpr int lP = P + 4, lN = N + 4, lQ = kQ + 4, lMx = kMx + 4;
  static constexpr int X = 0;                          // [Q][lP]
  static constexpr int Gm = X + kQ * lP;               // [Q][lP]  g = dout silu(z)
  static constexpr int Bt = Gm + kQ * lP;              // [Q][lN]
  static constexpr int Ct = Bt + kQ * lN;              // [Q][lN]
  static constexpr int Sin = Ct + kQ * lN;             // [P][lN]
  static constexpr int U = Sin + P * lN;               // [P][lN]
  static constexpr int CB = U + P * lN;                // [Q][lQ]  Ct Bt^T, later c o G X^T
  static constexpr int W = CB + kQ * lQ;               // [Q][lQ]  c o Ct Bt^T, later dBt [Q][lN]
  static constexpr int T1 = W + kQ * lQ;               // [Q][lMx] Y, dX, dCt
  static constexpr int T2 = T1 + kQ * lMx;             // [Q][lMx] G X^T, X U
  static constexpr int T3 = T2 + kQ * lMx;             // [kMx][lMx] G S_in, U_prev
  static constexpr int Dm = T3 + kMx * lMx;            // [Q][Q+1]
  static constexpr int Phi = Dm + kQ * (kQ + 1);       // [Q][kK] angles, later dphi
  static constexpr int vec = Phi + kQ * kK;
  static constexpr int al = vec, be = al + kQ, ga = be + kQ, d1 = ga + kQ, d0 = d1 + kQ,
                       crow = d0 + kQ, wu = crow + kQ, cbp = wu + kQ, gxp = cbp + kQ,
                       vv = gxp + kQ /* v_{-1..Q-1}: Q + 1 */, dgam = vv + kQ + 4,
                       dbet = dgam + kQ, rowe = dbet + kQ, cole = rowe + kQ, xprev = cole + kQ,
                       bprev = xprev + P, phist = bprev + N, dth = phist + kK,
                       red = dth + kK /* kThreads */;
  static constexpr int total = red + kThreads;
};

// kSlab: one slab of a wider d_state (runtime row length and offsets);
// otherwise the whole d_state with compile-time strides
template <typename T, int P, int N, bool kSlab>
__global__ void __launch_bounds__(kThreads, 1) m3_bwd_kernel(const M3Params p, float *ws_dB,
                                                             float *ws_dC, float *ws_dD) {
  using S = BwdSmem<P, N>;
  constexpr int kK = S::kK;
  constexpr int lP = S::lP, lN = S::lN, lQ = S::lQ, lMx = S::lMx;
  extern __shared__ float4 smem4[];
  float *sm = reinterpret_cast<float *>(smem4);
  float *sX = sm + S::X, *sG = sm + S::Gm, *sBt = sm + S::Bt, *sCt = sm + S::Ct;
  float *sSin = sm + S::Sin, *sU = sm + S::U, *sCB = sm + S::CB, *sW = sm + S::W;
  float *sT1 = sm + S::T1, *sT2 = sm + S::T2, *sT3 = sm + S::T3, *sDm = sm + S::Dm;
  float *sPhi = sm + S::Phi;
  float *sAl = sm + S::al, *sBe = sm + S::be, *sGa = sm + S::ga, *sD1 = sm + S::d1;
  float *sD0 = sm + S::d0, *sCrow = sm + S::crow, *sWu = sm + S::wu, *sCbp = sm + S::cbp;
  float *sGxp = sm + S::gxp, *sV = sm + S::vv + 1 /* sV[-1] valid */, *sDgam = sm + S::dgam;
  float *sDbet = sm + S::dbet, *sRowE = sm + S::rowe, *sColE = sm + S::cole;
  float *sXprev = sm + S::xprev, *sBprev = sm + S::bprev, *sPhiSt = sm + S::phist;
  float *sDth = sm + S::dth, *sRed = sm + S::red;

  const int tid = threadIdx.x;
  const int64_t h = blockIdx.x, b = blockIdx.y;
  const int64_t L = p.L, H = p.H, G = p.G;
  // this slab's states n0 .. n0 + N - 1 of ldN; its angle pairs k0 .. k0 + K - 1 of Kt
  const int64_t ldN = kSlab ? p.ldN : N, n0 = kSlab ? p.n0 : 0, Kt = p.K, k0 = n0 / 2;
  const int64_t K = Kt - k0 < 0 ? 0 : (Kt - k0 > kK ? kK : Kt - k0);
  const int slab = kSlab ? p.slab : kSlabWhole;
  const bool finish = slab == kSlabWhole || slab == kSlabLast;
  const int64_t g = h / (H / G);
  const float Dh = (p.Dp && finish) ? p.Dp[h] : 0.f;  // the D terms join once
  const int64_t n_chunks = (L + kQ - 1) / kQ;
  // chunk-start angles, as the forward accumulated them (after the states)
  const float *phi_start =
      p.saved_in + p.B * H * n_chunks * P * ldN + (b * H + h) * n_chunks * (ldN / 2) + k0;

  for (int i = tid; i < P * lN; i += kThreads) sU[i] = 0.f;
  for (int i = tid; i < kK; i += kThreads) sDth[i] = 0.f;
  float alQ = 1.f, beQ = 0.f;  // alpha, beta of the next chunk's first step
  float dD_l = 0.f;

  for (int64_t ch = n_chunks - 1; ch >= 0; --ch) {
    const int64_t t0 = ch * kQ;
    const int Qc = (int)((L - t0) < kQ ? (L - t0) : kQ);
    // ---- A. stage the chunk ---------------------------------------------------
    // the chunk's starting state by cp.async, straight into its padded rows
    {
      const float *src = p.saved_in + ((b * H + h) * n_chunks + ch) * P * ldN + n0;
      for (int u = tid; u < P * (N / 4); u += kThreads) {
        const int r = u / (N / 4), pc = u % (N / 4);
        cp_async16(sSin + r * lN + pc * 4, src + r * ldN + pc * 4, 16);
      }
      cp_async_commit();
    }
    // x, dout, z: runs of 8 along p, all loads of a thread issued first
    for (int u0 = tid; u0 < kQ * (P / 8); u0 += 2 * kThreads) {
      float xv[2][8], dv[2][8], zv[2][8];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int u = u0 + r * kThreads;
        const int t = u / (P / 8), pc = u % (P / 8);
        const bool in = u < kQ * (P / 8) && t < Qc;
        const int64_t j = ((b * L + t0 + t) * H + h) * P + pc * 8;
        ld8<T>(p.x, j, in, xv[r]);
        ld8<T>(p.dout, j, in, dv[r]);
        ld8<T>(p.z, j, in && p.z, zv[r]);
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int u = u0 + r * kThreads;
        if (u >= kQ * (P / 8)) continue;
        const int t = u / (P / 8), pc = u % (P / 8);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float gv = p.z ? dv[r][e] * silu(zv[r][e]) : dv[r][e];
          sX[t * lP + pc * 8 + e] = xv[r][e];
          sG[t * lP + pc * 8 + e] = gv;
          dD_l = fmaf(gv, xv[r][e], dD_l);
        }
      }
    }
    // B and C rows: runs of 8 along n
    for (int u = tid; u < kQ * (N / 8); u += kThreads) {
      const int t = u / (N / 8), pc = u % (N / 8);
      const bool in = t < Qc;
      const int64_t j = ((b * L + t0 + t) * G + g) * ldN + n0 + pc * 8;
      float bv[8], cv[8];
      ld8<T>(p.Bm, j, in, bv);
      ld8<T>(p.Cm, j, in, cv);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        sBt[t * lN + pc * 8 + e] = bv[e];
        sCt[t * lN + pc * 8 + e] = cv[e];
      }
    }
    for (int t = tid; t < kQ; t += kThreads) {
      const bool in = t < Qc;
      const int64_t j = (b * L + t0 + t) * H + h;
      sAl[t] = in ? ldv<T>(p.alpha, j) : 1.f;
      sBe[t] = in ? ldv<T>(p.beta, j) : 0.f;
      sGa[t] = in ? ldv<T>(p.gamma, j) : 0.f;
    }
    for (int i = tid; i < kQ * K; i += kThreads) {
      const int t = i / (int)K, k = i % (int)K;
      sPhi[t * kK + k] = t < Qc ? ldv<T>(p.theta, ((b * L + t0 + t) * H + h) * Kt + k0 + k) : 0.f;
    }
    for (int i = tid; i < kK; i += kThreads) sPhiSt[i] = i < K ? phi_start[ch * (ldN / 2) + i] : 0.f;
    for (int i = tid; i < P; i += kThreads)
      sXprev[i] = t0 > 0 ? ldv<T>(p.x, ((b * L + t0 - 1) * H + h) * P + i) : 0.f;
    for (int i = tid; i < N; i += kThreads)
      sBprev[i] = t0 > 0 ? ldv<T>(p.Bm, ((b * L + t0 - 1) * G + g) * ldN + n0 + i) : 0.f;
    // the previous chunk's rows into L2 while this one computes
    if (ch > 0) {
      const int64_t tp = t0 - kQ;
      for (int u = tid; u < 4 * kQ; u += kThreads) {
        const int k = u / kQ, t = u % kQ;
        const void *ptr;
        if (k < 3) {
          const void *base = k == 0 ? p.x : (k == 1 ? p.dout : p.z);
          if (!base) continue;
          ptr = static_cast<const T *>(base) + ((b * L + tp + t) * H + h) * P;
        } else {
          ptr = static_cast<const T *>(p.Bm) + ((b * L + tp + t) * G + g) * ldN + n0;
        }
        asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
      }
      const float *sv = p.saved_in + ((b * H + h) * n_chunks + ch - 1) * P * ldN + n0;
      constexpr int kLines = (N + 31) / 32;  // 128-byte lines per row
      for (int u = tid; u < P * kLines; u += kThreads)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(sv + (u / kLines) * ldN + (u % kLines) * 32));
    }
    cp_async_wait<0>();
    __syncthreads();
    // ---- B. angles, decays, rotations -----------------------------------------
    if (tid < K) {
      float acc = sPhiSt[tid];
      for (int t = 0; t < kQ; ++t) {
        acc += sPhi[t * kK + tid];
        sPhi[t * kK + tid] = acc;
      }
    }
    for (int col = tid; col <= kQ; col += kThreads) {
      const int s = col - 1;
      float v = 1.f;
      if (s >= 0) sDm[s * (kQ + 1) + col] = 1.f;
      for (int t = s + 1; t < kQ; ++t) {
        v *= sAl[t];
        sDm[t * (kQ + 1) + col] = v;
      }
    }
    __syncthreads();
    for (int i = tid; i < (kQ + 1) * (N / 2); i += kThreads) {
      // rows 0..Q-1: the chunk's B and C; row Q: the previous step's B
      const int t = i / (N / 2), k = i % (N / 2);
      float *bb = t < kQ ? sBt + t * lN : sBprev;
      const float b0 = bb[2 * k], b1 = bb[2 * k + 1];
      float c0 = 0.f, c1 = 0.f;
      if (t < kQ) { c0 = sCt[t * lN + 2 * k]; c1 = sCt[t * lN + 2 * k + 1]; }
      if (k < K) {
        float sn, cs;
        sincosf(t < kQ ? sPhi[t * kK + k] : sPhiSt[k], &sn, &cs);
        bb[2 * k] = cs * b0 - sn * b1;
        bb[2 * k + 1] = sn * b0 + cs * b1;
        if (t < kQ) {
          sCt[t * lN + 2 * k] = cs * c0 - sn * c1;
          sCt[t * lN + 2 * k + 1] = sn * c0 + cs * c1;
        }
      }
    }
    __syncthreads();
    // ---- C. Ct Bt^T, per-step vectors, W ---------------------------------------
    mm<kQ, kQ, N, false, true>(sCB, lQ, sCt, lN, sBt, lN, nullptr, nullptr, false);
    for (int t = tid; t < kQ; t += kThreads) {
      sD1[t] = sDm[t * (kQ + 1)];
      sD0[t] = sDm[t * (kQ + 1) + 1];
      sCrow[t] = (t == kQ - 1) ? sGa[t]
                               : sDm[(kQ - 1) * (kQ + 1) + t + 2] * (sAl[t + 1] * sGa[t] + sBe[t + 1]);
      float cb = 0.f, gx = 0.f;
      for (int n = 0; n < N; ++n) cb = fmaf(sCt[t * lN + n], sBprev[n], cb);
      for (int q = 0; q < P; ++q) gx = fmaf(sG[t * lP + q], sXprev[q], gx);
      sCbp[t] = cb;
      sGxp[t] = gx;
    }
    __syncthreads();
    for (int t = tid; t < kQ; t += kThreads) sWu[t] = alQ * sCrow[t] + (t == kQ - 1 ? beQ : 0.f);
    for (int i = tid; i < kQ * kQ; i += kThreads) {
      const int t = i / kQ, s = i % kQ;
      float w = 0.f;
      if (s == t) w = sGa[t] * sCB[t * lQ + s];
      else if (s < t)
        w = sDm[t * (kQ + 1) + s + 2] * (sAl[s + 1] * sGa[s] + sBe[s + 1]) * sCB[t * lQ + s];
      sW[t * lQ + s] = w;
    }
    __syncthreads();
    // ---- D. y (for dz) -----------------------------------------------------------
    mm<kQ, P, kQ, false, false>(sT1, lMx, sW, lQ, sX, lP, nullptr, nullptr, false);
    mm<kQ, P, N, false, true>(sT1, lMx, sCt, lN, sSin, lN, sD1, nullptr, true);
    __syncthreads();
    if (p.dz) {
      for (int i = tid; i < kQ * P; i += kThreads) {
        const int t = i / P, pp = i % P;
        if (t < Qc) {
          float y =
              sT1[t * lMx + pp] + sBe[0] * sD0[t] * sCbp[t] * sXprev[pp] + Dh * sX[t * lP + pp];
          const int64_t j = ((b * L + t0 + t) * H + h) * P + pp;
          if (slab != kSlabWhole) {  // y sums over the states: across the slabs
            if (slab != kSlabFirst) y = p.tok_y[j] + y;
            if (!finish) {
              p.tok_y[j] = y;
              continue;
            }
          }
          const float dy = ldv<T>(p.dout, j);
          static_cast<T *>(p.dz)[j] = from_f32<T>(y * dy * dsilu(ldv<T>(p.z, j)));
        }
      }
    }
    // ---- E. G X^T, G S_in; first scalar pass -----------------------------------
    mm<kQ, kQ, P, false, true>(sT2, lMx, sG, lP, sX, lP, nullptr, nullptr, false);
    mm<kQ, N, P, false, false>(sT3, lMx, sG, lP, sSin, lN, nullptr, nullptr, false);
    __syncthreads();
    for (int s = tid; s < kQ; s += kThreads) {
      // column s of E, dgamma_s and dbeta_s (chunk-internal parts)
      float dg = 0.f, db = 0.f;
      for (int tau = s; tau < kQ; ++tau) {
        const float d = sDm[tau * (kQ + 1) + s + 1];
        dg = fmaf(d, sCB[tau * lQ + s] * sT2[tau * lMx + s], dg);
        const float m1 = s > 0 ? sCB[tau * lQ + s - 1] * sT2[tau * lMx + s - 1]
                               : sCbp[tau] * sGxp[tau];
        db = fmaf(d, m1, db);
      }
      sDgam[s] = dg;
      sDbet[s] = db;
    }
    for (int tau = tid; tau < kQ; tau += kThreads) {
      // a_tau = g_tau^T S_in Ct_tau
      float gs = 0.f;
      for (int n = 0; n < N; ++n) gs = fmaf(sT3[tau * lMx + n], sCt[tau * lN + n], gs);
      sRowE[tau] = gs;
    }
    {
      // the box sums sum_{tau>=s} sum_{j<=s-2} c(tau,j) M(tau,j) (c o M = W o G X^T),
      // four threads per s (rows tau = s + part, s + part + 4, ...), added in a
      // fixed butterfly
      static_assert(kThreads == 4 * kQ, "four threads per step");
      const int s = tid >> 2, part = tid & 3;
      float acc = 0.f;
      for (int tau = s + part; tau < kQ; tau += 4)
        for (int j = 0; j <= s - 2; ++j) acc = fmaf(sW[tau * lQ + j], sT2[tau * lMx + j], acc);
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      if (part == 0) sColE[s] = acc;
    }
    __syncthreads();
    // c o G X^T replaces Ct Bt^T
    for (int i = tid; i < kQ * kQ; i += kThreads) {
      const int t = i / kQ, s = i % kQ;
      float w = 0.f;
      if (s == t) w = sGa[t] * sT2[t * lMx + s];
      else if (s < t)
        w = sDm[t * (kQ + 1) + s + 2] * (sAl[s + 1] * sGa[s] + sBe[s + 1]) * sT2[t * lMx + s];
      sCB[t * lQ + s] = w;
    }
    __syncthreads();
    // ---- F. dx; X U; dBt; second scalar pass --------------------------------------
    mm<kQ, P, kQ, true, false>(sT1, lMx, sW, lQ, sG, lP, nullptr, nullptr, false);
    mm<kQ, P, N, false, true>(sT1, lMx, sBt, lN, sU, lN, sWu, nullptr, true);
    mm<kQ, N, P, false, false>(sT2, lMx, sX, lP, sU, lN, nullptr, nullptr, false);
    __syncthreads();
    for (int i = tid; i < kQ * P; i += kThreads) {
      const int t = i / P, pp = i % P;
      if (t < Qc) {
        const int64_t j = ((b * L + t0 + t) * H + h) * P + pp;
        float v = fmaf(Dh, sG[t * lP + pp], sT1[t * lMx + pp]);
        if (slab != kSlabWhole) {  // dx sums over the states: across the slabs
          if (slab != kSlabFirst) v = p.tok_dx[j] + v;
          if (!finish) {
            p.tok_dx[j] = v;
            continue;
          }
        }
        static_cast<T *>(p.dx)[j] = from_f32<T>(v);
      }
    }
    mm<kQ, N, kQ, true, false>(sW, lN, sCB, lQ, sCt, lN, nullptr, nullptr, false);
    // v_s = x_s^T U Bt_s (s >= 0), v_{-1} with the previous step; <U, S_in>
    for (int s = tid; s < kQ; s += kThreads) {
      float v = 0.f;
      for (int n = 0; n < N; ++n) v = fmaf(sT2[s * lMx + n], sBt[s * lN + n], v);
      sV[s] = v;
    }
    __syncthreads();
    // v_{-1} = x_prev^T U Bt_prev and <U, S_in>, as fixed-order block sums
    float us, vm1;
    {
      float part = 0.f;
      for (int i = tid; i < P * N; i += kThreads) {
        const int o = (i / N) * lN + i % N;
        part = fmaf(sU[o], sSin[o], part);
      }
      float xb = 0.f;
      if (tid < N) {
        float xu = 0.f;
        for (int q = 0; q < P; ++q) xu = fmaf(sXprev[q], sU[q * lN + tid], xu);
        xb = xu * sBprev[tid];
      }
      us = block_sum(part, sRed);
      vm1 = block_sum(xb, sRed);
    }
    for (int i = tid; i < kQ * N; i += kThreads) {
      const int t = i / N, n = i % N;
      sW[t * lN + n] = fmaf(sWu[t], sT2[t * lMx + n], sW[t * lN + n]);  // dBt
    }
    if (tid == 0) sV[-1] = vm1;
    __syncthreads();
    for (int s = tid; s < kQ; s += kThreads) {
      // parts that reach the next chunk through the last state
      const float dl = sDm[(kQ - 1) * (kQ + 1) + s + 1];
      const float fg = alQ * dl * sV[s], fb = alQ * dl * sV[s - 1];
      sDgam[s] += fg;
      sDbet[s] += fb;
    }
    __syncthreads();
    // dalpha of the chunk (above): the suffix sums over tau, the U row, the
    // box sums and gamma_{s-1} dbeta_s, each step by one thread in a fixed order
    for (int s = tid; s < kQ; s += kThreads) {
      float v;
      if (s == 0) {
        v = alQ * sDm[(kQ - 1) * (kQ + 1) + 1] * us;
        for (int tau = kQ - 1; tau >= 0; --tau) v = fmaf(sDm[tau * (kQ + 1) + 1], sRowE[tau], v);
      } else {
        float a1 = alQ * fmaf(sBe[0] * sDm[(kQ - 1) * (kQ + 1) + 1], sV[-1],
                              sDm[(kQ - 1) * (kQ + 1)] * us);
        for (int tau = kQ - 1; tau >= s; --tau)
          a1 += fmaf(sDm[tau * (kQ + 1)], sRowE[tau],
                     sBe[0] * sDm[tau * (kQ + 1) + 1] * (sCbp[tau] * sGxp[tau]));
        float bu = 0.f;  // the U row of the box sums: alpha_Q sum_{j<=s-2} c(Q-1,j) v_j
        for (int j = 0; j <= s - 2; ++j) bu = fmaf(sCrow[j], sV[j], bu);
        v = (a1 + sColE[s] + alQ * bu) / sAl[s] + sGa[s - 1] * sDbet[s];
      }
      sColE[s] = v;
    }
    __syncthreads();
    // ---- G. dCt ---------------------------------------------------------------------
    mm<kQ, N, kQ, false, false>(sT1, lMx, sCB, lQ, sBt, lN, nullptr, nullptr, false);
    __syncthreads();
    for (int i = tid; i < kQ * N; i += kThreads) {
      const int t = i / N, n = i % N;
      float v = sT1[t * lMx + n] + sD1[t] * sT3[t * lMx + n];
      v = fmaf(sBe[0] * sD0[t] * sGxp[t], sBprev[n], v);
      sT1[t * lMx + n] = v;
    }
    // dalpha (sColE), dbeta, dgamma of this chunk, warp 0 (lane l: steps 2l, 2l+1)
    if (tid < 32) {
      const int r0 = 2 * tid, r1 = 2 * tid + 1;
      const float a0 = sColE[r0], a1 = sColE[r1];
      // (slabs after the first add their sums over the states in place)
      const bool add = slab == kSlabMiddle || slab == kSlabLast;
      if (r0 < Qc) {
        const int64_t j = (b * L + t0 + r0) * H + h;
        p.dalpha[j] = (add ? p.dalpha[j] : 0.f) + a0;
        p.dbeta[j] = (add ? p.dbeta[j] : 0.f) + sDbet[r0];
        p.dgamma[j] = (add ? p.dgamma[j] : 0.f) + sDgam[r0];
      }
      if (r1 < Qc) {
        const int64_t j = (b * L + t0 + r1) * H + h;
        p.dalpha[j] = (add ? p.dalpha[j] : 0.f) + a1;
        p.dbeta[j] = (add ? p.dbeta[j] : 0.f) + sDbet[r1];
        p.dgamma[j] = (add ? p.dgamma[j] : 0.f) + sDgam[r1];
      }
    }
    __syncthreads();
    // ---- H. U_prev = G^T diag(d(.,0)) Ct + d(Q-1,0) alpha_Q U --------------------------
    mm<P, N, kQ, true, false>(sT3, lMx, sG, lP, sCt, lN, nullptr, sD0, false);
    // ---- J. RoPE backward: per-head dB, dC and dphi -----------------------------------
    for (int i = tid; i < kQ * (N / 2); i += kThreads) {
      const int t = i / (N / 2), k = i % (N / 2);
      const float db0 = sW[t * lN + 2 * k], db1 = sW[t * lN + 2 * k + 1];
      const float dc0 = sT1[t * lMx + 2 * k], dc1 = sT1[t * lMx + 2 * k + 1];
      float rb0 = db0, rb1 = db1, rc0 = dc0, rc1 = dc1;
      if (k < K) {
        float sn, cs;
        sincosf(sPhi[t * kK + k], &sn, &cs);
        rb0 = cs * db0 + sn * db1;
        rb1 = -sn * db0 + cs * db1;
        rc0 = cs * dc0 + sn * dc1;
        rc1 = -sn * dc0 + cs * dc1;
      }
      if (t < Qc) {
        const int64_t j = ((b * L + t0 + t) * H + h) * ldN + n0 + 2 * k;
        ws_dB[j] = rb0;
        ws_dB[j + 1] = rb1;
        ws_dC[j] = rc0;
        ws_dC[j + 1] = rc1;
      }
    }
    __syncthreads();
    for (int i = tid; i < kQ * K; i += kThreads) {
      const int t = i / (int)K, k = i % (int)K;
      const float b0 = sBt[t * lN + 2 * k], b1 = sBt[t * lN + 2 * k + 1];
      const float c0 = sCt[t * lN + 2 * k], c1 = sCt[t * lN + 2 * k + 1];
      const float db0 = sW[t * lN + 2 * k], db1 = sW[t * lN + 2 * k + 1];
      const float dc0 = sT1[t * lMx + 2 * k], dc1 = sT1[t * lMx + 2 * k + 1];
      sPhi[t * kK + k] = (db1 * b0 - db0 * b1) + (dc1 * c0 - dc0 * c1);  // dphi_t[k]
    }
    __syncthreads();
    if (tid < K) {
      float acc = sDth[tid];
      for (int t = Qc - 1; t >= 0; --t) {
        acc += sPhi[t * kK + tid];
        p.dtheta[((b * L + t0 + t) * H + h) * Kt + k0 + tid] = acc;
      }
      sDth[tid] = acc;
    }
    // ---- K. hand the adjoint to the previous chunk ----------------------------------
    {
      const float c = sD0[kQ - 1] * alQ;
      for (int i = tid; i < P * N; i += kThreads) {
        const int pp = i / N, n = i % N;
        sU[pp * lN + n] = fmaf(c, sU[pp * lN + n], sT3[pp * lMx + n]);
      }
    }
    alQ = sAl[0];
    beQ = sBe[0];
    __syncthreads();
  }

  if (p.dh0) {
    for (int i = tid; i < P * N; i += kThreads)
      p.dh0[((b * H + h) * P + i / N) * ldN + n0 + i % N] = alQ * sU[(i / N) * lN + i % N];  // alpha_0 Lambda_0
  }
  const float dD = block_sum(dD_l, sRed);
  if (tid == 0 && finish) ws_dD[b * H + h] = dD;
}

// dB, dC: the heads of each group added in ascending head order; dD: the
// batch rows added in ascending order.
__global__ void m3_bwd_reduce_kernel(const M3Params p, const float *ws_dB, const float *ws_dC,
                                     const float *ws_dD) {
  const int64_t Bsz = p.B, L = p.L, H = p.H, G = p.G, N = p.N;
  const int64_t hpg = H / G;
  const int64_t n_bc = Bsz * L * G * N;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_bc + H;
       i += (int64_t)gridDim.x * blockDim.x) {
    if (i < n_bc) {
      const int64_t n = i % N, g = (i / N) % G, bt = i / (N * G);  // bt = b * L + t
      float sb = 0.f, sc = 0.f;
      for (int64_t hh = g * hpg; hh < (g + 1) * hpg; ++hh) {
        sb += ws_dB[(bt * H + hh) * N + n];
        sc += ws_dC[(bt * H + hh) * N + n];
      }
      p.dB[i] = sb;
      p.dC[i] = sc;
    } else if (p.dD) {
      const int64_t h = i - n_bc;
      float s = 0.f;
      for (int64_t b = 0; b < Bsz; ++b) s += ws_dD[b * H + h];
      p.dD[h] = s;
    }
  }
}

template <typename T, int P, int N, bool kSlab>
cudaError_t launch_t(const M3Params &p, cudaStream_t s) {
  const size_t smem = sizeof(float) * (size_t)BwdSmem<P, N>::total;
  cudaError_t e = cudaFuncSetAttribute(m3_bwd_kernel<T, P, N, kSlab>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const M3BwdWs w = m3_bwd_ws_layout(p.B, p.L, p.H, p.P, p.ldN, p.K);
  char *ws = static_cast<char *>(p.ws);
  float *dB = reinterpret_cast<float *>(ws + w.dB);
  float *dC = reinterpret_cast<float *>(ws + w.dC);
  float *dD = reinterpret_cast<float *>(ws + w.dD);
  m3_bwd_kernel<T, P, N, kSlab><<<dim3((unsigned)p.H, (unsigned)p.B), kThreads, smem, s>>>(
      p, dB, dC, dD);
  return cudaGetLastError();
}

template <typename T, int P>
cudaError_t launch_n(const M3Params &p, cudaStream_t s) {
  if (p.slab != kSlabWhole) return launch_t<T, P, kM3Slab, true>(p, s);
  switch (p.N) {
    case 16: return launch_t<T, P, 16, false>(p, s);
    case 32: return launch_t<T, P, 32, false>(p, s);
    default: return launch_t<T, P, 64, false>(p, s);
  }
}

template <typename T>
cudaError_t launch_p(const M3Params &p, cudaStream_t s) {
  switch (p.P) {
    case 16: return launch_n<T, 16>(p, s);
    case 32: return launch_n<T, 32>(p, s);
    default: return launch_n<T, 64>(p, s);
  }
}

}  // namespace

// one layout serves both implementations (its regions are a superset of what
// this one uses), so the size does not depend on the io type
size_t m3_bwd_workspace_bytes(int64_t B, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G,
                              int64_t K) {
  (void)G;
  return m3_bwd_ws_layout(B, L, H, P, N, K).total;
}

// The whole d_state in one launch, or slabs of kM3Slab states in ascending
// order (sums over the states carried in the workspace and in dalpha, dbeta,
// dgamma), then the fixed-order sum of dB, dC over the heads of a group and
// of dD over the batch.
cudaError_t launch_m3_bwd(const M3Params &p0, cudaStream_t s) {
  if (p0.io == 1) return launch_m3_bwd_umma(p0, s);  // bf16 io: the tensor-core backward
  const int64_t n_tot = p0.N;
  const int64_t slabs = (n_tot + kM3Slab - 1) / kM3Slab;
  const M3BwdWs w = m3_bwd_ws_layout(p0.B, p0.L, p0.H, p0.P, n_tot, p0.K);
  char *ws = static_cast<char *>(p0.ws);
  for (int64_t k = 0; k < slabs; ++k) {
    M3Params p = p0;
    p.ldN = n_tot;
    p.n0 = k * kM3Slab;
    p.N = n_tot - p.n0 < kM3Slab ? n_tot - p.n0 : kM3Slab;
    p.slab = slabs == 1 ? kSlabWhole
                        : (k == 0 ? kSlabFirst : (k == slabs - 1 ? kSlabLast : kSlabMiddle));
    p.tok_y = slabs > 1 ? reinterpret_cast<float *>(ws + w.tok_y) : nullptr;
    p.tok_dx = slabs > 1 ? reinterpret_cast<float *>(ws + w.tok_dx) : nullptr;
    cudaError_t e;
    switch (p.io) {
      case 2: e = launch_p<f16>(p, s); break;
      default: e = launch_p<float>(p, s); break;
    }
    if (e != cudaSuccess) return e;
  }
  float *dB = reinterpret_cast<float *>(ws + w.dB);
  float *dC = reinterpret_cast<float *>(ws + w.dC);
  float *dD = reinterpret_cast<float *>(ws + w.dD);
  const int64_t total = p0.B * p0.L * p0.G * n_tot + p0.H;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  m3_bwd_reduce_kernel<<<(unsigned)blocks, 256, 0, s>>>(p0, dB, dC, dD);
  return cudaGetLastError();
}

}  // namespace msc
