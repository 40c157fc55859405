// m3_fwd.cu -- Mamba-3 SISO scan, forward (sm_100a).
//
// Per (batch b, head h) and t = 0..L-1 (mamba-rs 0.7.0 README, "Features";
// the three-term update and per-head cumulative angles are those whose
// gradients stages B3 and B4 of Mamba3Scratch in mamba-rs 0.4.2
// src/mamba3_siso/cpu/scratch.rs hold):
//   phi_t = sum_{s<=t} theta_s,  Bt_t = R(phi_t) B_t,  Ct_t = R(phi_t) C_t
//   S_t   = alpha_t S_{t-1} + beta_t K_{t-1} + gamma_t K_t,  K_t = x_t (outer) Bt_t
//   out_t = (S_t Ct_t + D x_t) silu(z_t)
//
// One CTA owns one (b, h) sequence and walks its 64-step chunks in order with
// the f32 state (transposed, [N][P]) resident in shared memory.  Per chunk it
// stages x, the rotated B and C, the decay products d(t, s) and the
// trapezoid weights, and evaluates the chunked form of m3_common.cuh with
// tile products; cumulative angles are summed sequentially per angle in f32
// (the order the backward pass repeats bit for bit).  The state entering every
// chunk goes to `saved` for the backward pass.
#include "m3_common.cuh"

namespace msc {
namespace {

using namespace m3;

template <int P, int N>
struct FwdSmem {
  static constexpr int kK = N / 2;                 // max angles
  static constexpr int X = 0;                      // [Q][P]
  static constexpr int Bt = X + kQ * P;            // [Q][N]   rotated B, row per step
  static constexpr int BtT = Bt + kQ * N;          // [N][Q]
  static constexpr int CtT = BtT + N * kQ;         // [N][Q]
  static constexpr int G = CtT + N * kQ;           // [Q][Q]   Ct Bt^T (raw C staged here first)
  static constexpr int WT = G + kQ * kQ;           // [Q][Q]   W transposed
  static constexpr int ST = WT + kQ * kQ;          // [N][P]   state, transposed
  static constexpr int Y = ST + N * P;             // [Q][P]
  static constexpr int Dm = Y + kQ * P;            // [Q][Q+1] d(t, s) at column s + 1
  static constexpr int Phi = Dm + kQ * (kQ + 1);   // [Q][kK]
  static constexpr int vec = Phi + kQ * kK;
  static constexpr int al = vec, be = al + kQ, ga = be + kQ, crow = ga + kQ, dlast = crow + kQ,
                       wc = dlast + kQ, xprev = wc + kQ, bprev = xprev + P, phiprev = bprev + N;
  static constexpr int total = phiprev + kK;
};

// kSlab: one slab of a wider d_state (runtime row length and offsets);
// otherwise the whole d_state with compile-time strides
template <typename T, int P, int N, bool kSlab>
__global__ void __launch_bounds__(kThreads, 1) m3_fwd_kernel(const M3Params p) {
  using S = FwdSmem<P, N>;
  extern __shared__ float4 smem4[];
  float *sm = reinterpret_cast<float *>(smem4);
  float *sX = sm + S::X, *sBt = sm + S::Bt, *sBtT = sm + S::BtT, *sCtT = sm + S::CtT;
  float *sG = sm + S::G, *sWT = sm + S::WT, *sST = sm + S::ST, *sY = sm + S::Y;
  float *sDm = sm + S::Dm, *sPhi = sm + S::Phi;
  float *sAl = sm + S::al, *sBe = sm + S::be, *sGa = sm + S::ga, *sCrow = sm + S::crow;
  float *sDlast = sm + S::dlast, *sWc = sm + S::wc, *sXprev = sm + S::xprev;
  float *sBprev = sm + S::bprev, *sPhiPrev = sm + S::phiprev;

  const int tid = threadIdx.x;
  const int64_t h = blockIdx.x, b = blockIdx.y;
  const int64_t L = p.L, H = p.H, G = p.G;
  // this slab's states n0 .. n0 + N - 1 of ldN; its angle pairs k0 .. k0 + K - 1 of Kt
  const int64_t ldN = kSlab ? p.ldN : N, n0 = kSlab ? p.n0 : 0, Kt = p.K, k0 = n0 / 2;
  const int64_t K = Kt - k0 < 0 ? 0 : (Kt - k0 > S::kK ? S::kK : Kt - k0);
  const int slab = kSlab ? p.slab : kSlabWhole;
  const bool finish = slab == kSlabWhole || slab == kSlabLast;
  const int64_t g = h / (H / G);
  const float Dh = (p.Dp && finish) ? p.Dp[h] : 0.f;  // the D x skip joins once
  const int64_t n_chunks = (L + kQ - 1) / kQ;

  for (int i = tid; i < N * P; i += kThreads) {
    const int n = i / P, pp = i % P;
    sST[i] = p.h0 ? p.h0[((b * H + h) * P + pp) * ldN + n0 + n] : 0.f;
  }
  for (int i = tid; i < P; i += kThreads) sXprev[i] = 0.f;
  for (int i = tid; i < N; i += kThreads) sBprev[i] = 0.f;
  for (int i = tid; i < S::kK; i += kThreads) sPhiPrev[i] = 0.f;

  for (int64_t ch = 0; ch < n_chunks; ++ch) {
    const int64_t t0 = ch * kQ;
    const int Qc = (int)((L - t0) < kQ ? (L - t0) : kQ);
    __syncthreads();
    // ---- 1. stage the chunk (steps past the end: identity, x = B = C = 0) ----
    for (int i = tid; i < kQ * P; i += kThreads) {
      const int t = i / P, pp = i % P;
      sX[i] = t < Qc ? ldv<T>(p.x, ((b * L + t0 + t) * H + h) * P + pp) : 0.f;
    }
    for (int i = tid; i < kQ * N; i += kThreads) {
      const int t = i / N, n = i % N;
      const bool in = t < Qc;
      const int64_t j = ((b * L + t0 + t) * G + g) * ldN + n0 + n;
      sBt[i] = in ? ldv<T>(p.Bm, j) : 0.f;
      sG[i] = in ? ldv<T>(p.Cm, j) : 0.f;  // raw C, [Q][N], until the rotation
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
      sPhi[t * S::kK + k] = t < Qc ? ldv<T>(p.theta, ((b * L + t0 + t) * H + h) * Kt + k0 + k) : 0.f;
    }
    __syncthreads();
    // ---- 2. cumulative angles; decay products d(t, s) ------------------------
    if (tid < K) {
      float acc = sPhiPrev[tid];
      for (int t = 0; t < kQ; ++t) {
        acc += sPhi[t * S::kK + tid];
        sPhi[t * S::kK + tid] = acc;
      }
    }
    for (int col = tid; col <= kQ; col += kThreads) {  // column col = s + 1, s in [-1, Q)
      const int s = col - 1;
      float v = 1.f;
      if (s >= 0) sDm[s * (kQ + 1) + col] = 1.f;
      for (int t = s + 1; t < kQ; ++t) {
        v *= sAl[t];
        sDm[t * (kQ + 1) + col] = v;
      }
    }
    __syncthreads();
    // ---- 3. rotate B and C by the cumulative angles ---------------------------
    for (int i = tid; i < kQ * (N / 2); i += kThreads) {
      const int t = i / (N / 2), k = i % (N / 2);
      const float b0 = sBt[t * N + 2 * k], b1 = sBt[t * N + 2 * k + 1];
      const float c0 = sG[t * N + 2 * k], c1 = sG[t * N + 2 * k + 1];
      float rb0 = b0, rb1 = b1, rc0 = c0, rc1 = c1;
      if (k < K) {
        float sn, cs;
        sincosf(sPhi[t * S::kK + k], &sn, &cs);
        rb0 = cs * b0 - sn * b1;
        rb1 = sn * b0 + cs * b1;
        rc0 = cs * c0 - sn * c1;
        rc1 = sn * c0 + cs * c1;
      }
      sBt[t * N + 2 * k] = rb0;
      sBt[t * N + 2 * k + 1] = rb1;
      sBtT[(2 * k) * kQ + t] = rb0;
      sBtT[(2 * k + 1) * kQ + t] = rb1;
      sCtT[(2 * k) * kQ + t] = rc0;
      sCtT[(2 * k + 1) * kQ + t] = rc1;
    }
    __syncthreads();
    // ---- 4. G = Ct Bt^T; per-step vectors --------------------------------------
    mm<kQ, kQ, N, true, false>(sG, kQ, sCtT, kQ, sBtT, kQ, nullptr, nullptr, false);
    for (int t = tid; t < kQ; t += kThreads) {
      sDlast[t] = sDm[t * (kQ + 1)];                       // d(t, -1)
      float dot = 0.f;
      for (int n = 0; n < N; ++n) dot = fmaf(sCtT[n * kQ + t], sBprev[n], dot);
      sWc[t] = sBe[0] * sDm[t * (kQ + 1) + 1] * dot;      // beta_0 d(t, 0) Ct_t . Bt_prev
      // c(Q-1, t): weight of K_t in the chunk's last state
      sCrow[t] = (t == kQ - 1) ? sGa[t]
                               : sDm[(kQ - 1) * (kQ + 1) + t + 2] * (sAl[t + 1] * sGa[t] + sBe[t + 1]);
    }
    __syncthreads();
    // ---- 5. W^T[s][t] = c(t, s) G[t][s] for s <= t -----------------------------
    for (int i = tid; i < kQ * kQ; i += kThreads) {
      const int s = i / kQ, t = i % kQ;
      float w = 0.f;
      if (s == t) w = sGa[t] * sG[t * kQ + s];
      else if (s < t)
        w = sDm[t * (kQ + 1) + s + 2] * (sAl[s + 1] * sGa[s] + sBe[s + 1]) * sG[t * kQ + s];
      sWT[i] = w;
    }
    __syncthreads();
    // ---- 6. Y = W X + diag(d(., -1)) Ct S_in^T ---------------------------------
    mm<kQ, P, kQ, true, false>(sY, P, sWT, kQ, sX, P, nullptr, nullptr, false);
    mm<kQ, P, N, true, false>(sY, P, sCtT, kQ, sST, P, sDlast, nullptr, true);
    __syncthreads();
    // ---- 7. outputs; the state entering this chunk goes to `saved` -------------
    for (int i = tid; i < kQ * P; i += kThreads) {
      const int t = i / P, pp = i % P;
      if (t < Qc) {
        float y = sY[i] + sWc[t] * sXprev[pp] + Dh * sX[i];
        const int64_t j = ((b * L + t0 + t) * H + h) * P + pp;
        if (slab != kSlabWhole) {  // the sums over the states cross the slabs
          if (slab != kSlabFirst) y = p.tok_y[j] + y;
          if (!finish) {
            p.tok_y[j] = y;
            continue;
          }
        }
        if (p.z) y *= silu(ldv<T>(p.z, j));
        static_cast<T *>(p.out)[j] = from_f32<T>(y);
      }
    }
    if (p.saved) {
      float *dst = p.saved + ((b * H + h) * n_chunks + ch) * P * ldN + n0;
      for (int i = tid; i < P * N; i += kThreads) {
        const int pp = i / N, n = i % N;
        dst[pp * ldN + n] = sST[n * P + pp];
      }
      // the cumulative angles at the chunk start, after all states
      float *ang = p.saved + p.B * H * n_chunks * P * ldN + ((b * H + h) * n_chunks + ch) * (ldN / 2) + k0;
      for (int i = tid; i < S::kK; i += kThreads) ang[i] = sPhiPrev[i];
    }
    __syncthreads();
    // ---- 8. S_out = d(Q-1,-1) S_in + beta_0 d(Q-1,0) K_prev + X^T diag(c) Bt ----
    {
      const float dl = sDlast[kQ - 1];
      const float w0 = sBe[0] * sDm[(kQ - 1) * (kQ + 1) + 1];
      for (int i = tid; i < N * P; i += kThreads) {
        const int n = i / P, pp = i % P;
        sST[i] = fmaf(dl, sST[i], w0 * sBprev[n] * sXprev[pp]);
      }
    }
    __syncthreads();
    mm<N, P, kQ, true, false>(sST, P, sBt, N, sX, P, nullptr, sCrow, true);
    __syncthreads();
    // ---- 9. carry the last step's key and angles into the next chunk ----------
    for (int i = tid; i < P; i += kThreads) sXprev[i] = sX[(Qc - 1) * P + i];
    for (int i = tid; i < N; i += kThreads) sBprev[i] = sBt[(Qc - 1) * N + i];
    for (int i = tid; i < K; i += kThreads) sPhiPrev[i] = sPhi[(Qc - 1) * S::kK + i];
  }
  __syncthreads();
  if (p.final_state) {
    float *dst = p.final_state + (b * H + h) * P * ldN + n0;
    for (int i = tid; i < P * N; i += kThreads) {
      const int pp = i / N, n = i % N;
      dst[pp * ldN + n] = sST[n * P + pp];
    }
  }
}

template <typename T, int P, int N, bool kSlab>
cudaError_t launch_t(const M3Params &p, cudaStream_t s) {
  const size_t smem = sizeof(float) * (size_t)FwdSmem<P, N>::total;
  cudaError_t e = cudaFuncSetAttribute(m3_fwd_kernel<T, P, N, kSlab>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  m3_fwd_kernel<T, P, N, kSlab><<<dim3((unsigned)p.H, (unsigned)p.B), kThreads, smem, s>>>(p);
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

// d_state 16, 32 or 64 in one launch; 128, 192 or 256 as slabs of 64 states
bool m3_supported(int64_t P, int64_t N) {
  return (P == 16 || P == 32 || P == 64) &&
         (N == 16 || N == 32 || N == 64 || (N > kM3Slab && N <= 4 * kM3Slab && N % kM3Slab == 0));
}

// bf16 io runs the tcgen05 kernel (m3_fwd_umma.cu); f32 and f16 io this one,
// whose contractions are f32 on the CUDA cores.
// The whole d_state in one launch, or slabs of kM3Slab states in ascending
// order, the output sums carried in tok_y.
cudaError_t launch_m3_fwd(const M3Params &p0, cudaStream_t s) {
  const int64_t n_tot = p0.N;
  const int64_t slabs = (n_tot + kM3Slab - 1) / kM3Slab;
  for (int64_t k = 0; k < slabs; ++k) {
    M3Params p = p0;
    p.ldN = n_tot;
    p.n0 = k * kM3Slab;
    p.N = n_tot - p.n0 < kM3Slab ? n_tot - p.n0 : kM3Slab;
    p.slab = slabs == 1 ? kSlabWhole
                        : (k == 0 ? kSlabFirst : (k == slabs - 1 ? kSlabLast : kSlabMiddle));
    cudaError_t e;
    switch (p.io) {
      case 1: e = launch_m3_fwd_umma(p, s); break;
      case 2: e = launch_p<f16>(p, s); break;
      default: e = launch_p<float>(p, s); break;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace msc
