// m3_fwd_tc.cu -- Mamba-3 SISO scan, forward, bf16 io (sm_100a tensor cores).
//
// Same recurrence, chunked form and outputs as m3_fwd.cu (mamba-rs 0.7.0
// README, "Features"; the three-term update and per-head cumulative angles
// whose gradients stages B3 and B4 of Mamba3Scratch, mamba-rs 0.4.2
// src/mamba3_siso/cpu/scratch.rs, hold), organised for throughput:
//
//   * one CTA of 8 warps per (b, h), two CTAs per SM; the f32 state lives in
//     registers in the MMA accumulator layout, with a tf32 copy in shared
//     memory as the operand of the next chunk's readout;
//   * the three contractions of a chunk -- G = Ct Bt^T, Y = W X + diag(d)
//     Ct S^T and the state update X^T diag(c) Bt -- are m16n8k8 tf32 MMAs
//     with split (hi + lo) operands and f32 accumulation (m3_tc.cuh);
//   * decay products come from a warp scan of log2(alpha) over the chunk,
//     d(t, s) = 2^(lc_t - lc_s); the cumulative angles from per-thread
//     8-step partial sums combined across the chunk, one thread per (angle,
//     8-step segment), which also rotates B and C of its steps;
//   * the next chunk's x, B, C and theta are copied into shared memory by
//     cp.async while the current chunk computes, and its alpha, beta, gamma
//     are prefetched into registers.
#include "m3_tc.cuh"

namespace msc {
namespace {

using namespace m3;

template <int P, int N>
struct TcFwdSmem {
  static constexpr int kKmax = N / 2;
  static constexpr int ldX = P + 8;  // X[s][p]
  static constexpr int ldB = N + 4;  // Bt[s][n], Ct[t][n]
  static constexpr int ldW = kQ + 4; // W[t][s], over Ct once Ct is consumed
  static constexpr int ldS = N + 4;  // S[p][n]
  // float offsets
  static constexpr int X = 0;
  static constexpr int Bt = X + kQ * ldX;
  static constexpr int CtW = Bt + kQ * ldB;
  static constexpr int S = CtW + kQ * (ldB > ldW ? ldB : ldW);
  static constexpr int lc = S + P * ldS;  // [Q] cumulative log2(alpha), inclusive
  static constexpr int al = lc + kQ, be = al + kQ, ga = be + kQ;
  static constexpr int ev = ga + kQ;     // [Q] alpha_{s+1} gamma_s + beta_{s+1}
  static constexpr int dl = ev + kQ;     // [Q] d(t, -1)
  static constexpr int wc = dl + kQ;     // [Q] beta_0 d(t, 0) Ct_t . Bt_prev
  static constexpr int crow = wc + kQ;   // [Q] c(Q-1, s)
  static constexpr int xprev = crow + kQ;
  static constexpr int bprev = xprev + P;
  static constexpr int phi0 = bprev + N;        // [kKmax] angle after the previous chunk
  static constexpr int segsum = phi0 + kKmax;   // [8][kKmax]
  static constexpr int f32_end = segsum + 8 * kKmax;
  // raw bf16 stage, byte offsets
  static constexpr int raw = (f32_end * 4 + 15) / 16 * 16;
  static constexpr int rx = 0;
  static constexpr int rB = rx + kQ * P * 2;
  static constexpr int rC = rB + kQ * N * 2;
  static constexpr int rth = rC + kQ * N * 2;
  static constexpr int total = raw + rth + kQ * kKmax * 2;
};

// cp.async the raw x, B, C, theta rows of the chunk starting at t0 (rows past
// L zero-filled); theta rows go by cp.async when they are whole 16-byte
// pieces (K % 8 == 0), else element by element.
template <int P, int N>
__device__ __forceinline__ void tc_issue_stage(const M3Params &p, unsigned char *raw, int64_t b,
                                               int64_t h, int64_t g, int64_t t0) {
  using S = TcFwdSmem<P, N>;
  const int tid = threadIdx.x;
  const int64_t L = p.L, H = p.H, G = p.G;
  const int K = (int)p.K;
  const bf16 *x = static_cast<const bf16 *>(p.x);
  const bf16 *Bm = static_cast<const bf16 *>(p.Bm);
  const bf16 *Cm = static_cast<const bf16 *>(p.Cm);
  const bf16 *th = static_cast<const bf16 *>(p.theta);
  for (int u = tid; u < kQ * (P / 8); u += kThreads) {
    const int t = u / (P / 8), pc = u % (P / 8);
    const bool in = t0 + t < L;
    const bf16 *src = in ? x + ((b * L + t0 + t) * H + h) * P + pc * 8 : x;
    cp_async16(raw + S::rx + (t * P + pc * 8) * 2, src, in ? 16 : 0);
  }
  for (int u = tid; u < 2 * kQ * (N / 8); u += kThreads) {
    const int k = u / (kQ * (N / 8)), v = u % (kQ * (N / 8));
    const int t = v / (N / 8), pc = v % (N / 8);
    const bool in = t0 + t < L;
    const bf16 *base = k == 0 ? Bm : Cm;
    const bf16 *src = in ? base + ((b * L + t0 + t) * G + g) * N + pc * 8 : base;
    cp_async16(raw + (k == 0 ? S::rB : S::rC) + (t * N + pc * 8) * 2, src, in ? 16 : 0);
  }
  if (K > 0 && K % 8 == 0) {
    for (int u = tid; u < kQ * (K / 8); u += kThreads) {
      const int t = u / (K / 8), pc = u % (K / 8);
      const bool in = t0 + t < L;
      const bf16 *src = in ? th + ((b * L + t0 + t) * H + h) * K + pc * 8 : th;
      cp_async16(raw + S::rth + (t * S::kKmax + pc * 8) * 2, src, in ? 16 : 0);
    }
  } else {
    bf16 *dst = reinterpret_cast<bf16 *>(raw + S::rth);
    for (int u = tid; u < kQ * K; u += kThreads) {
      const int t = u / K, k = u % K;
      dst[t * S::kKmax + k] =
          t0 + t < L ? th[((b * L + t0 + t) * H + h) * K + k] : __float2bfloat16_rn(0.f);
    }
  }
  cp_async_commit();
}

// 8 consecutive bf16 (16 bytes of shared memory) -> 8 floats
__device__ __forceinline__ void ld8_bf16(const unsigned char *src, float (&v)[8]) {
  const uint4 r = *reinterpret_cast<const uint4 *>(src);
  unpack_bf16x2(r.x, v[0], v[1]);
  unpack_bf16x2(r.y, v[2], v[3]);
  unpack_bf16x2(r.z, v[4], v[5]);
  unpack_bf16x2(r.w, v[6], v[7]);
}

template <int P, int N>
__global__ void __launch_bounds__(kThreads, 2) m3_fwd_tc_kernel(const M3Params p) {
  using S = TcFwdSmem<P, N>;
  using TQQ = TileSplit<kQ, kQ>;
  using TQP = TileSplit<kQ, P>;
  using TPN = TileSplit<P, N>;
  constexpr int kKmax = S::kKmax;
  extern __shared__ float4 smem4[];
  float *sm = reinterpret_cast<float *>(smem4);
  unsigned char *raw = reinterpret_cast<unsigned char *>(smem4) + S::raw;
  float *sX = sm + S::X, *sBt = sm + S::Bt, *sCt = sm + S::CtW, *sW = sm + S::CtW;
  float *sS = sm + S::S, *sLc = sm + S::lc, *sAl = sm + S::al, *sBe = sm + S::be;
  float *sGa = sm + S::ga, *sEv = sm + S::ev, *sDl = sm + S::dl, *sWc = sm + S::wc;
  float *sCrow = sm + S::crow, *sXprev = sm + S::xprev, *sBprev = sm + S::bprev;
  float *sPhi0 = sm + S::phi0, *sSeg = sm + S::segsum;

  const int tid = threadIdx.x;
  const int64_t h = blockIdx.x, b = blockIdx.y;
  const int64_t L = p.L, H = p.H, G = p.G;
  const int K = (int)p.K;
  const int64_t g = h / (H / G);
  const float Dh = p.Dp ? p.Dp[h] : 0.f;
  const int64_t nc = (L + kQ - 1) / kQ;
  const bf16 *al_g = static_cast<const bf16 *>(p.alpha);
  const bf16 *be_g = static_cast<const bf16 *>(p.beta);
  const bf16 *ga_g = static_cast<const bf16 *>(p.gamma);
  const bf16 *z_g = static_cast<const bf16 *>(p.z);
  bf16 *out_g = static_cast<bf16 *>(p.out);

  // the state, in registers (tiles of P x N) and as an operand in smem
  float s_acc[TPN::kPerWarp][4];
  for_acc<P, N>([&](int i, int j, int pp, int n) {
    const float v = p.h0 ? p.h0[((b * H + h) * P + pp) * N + n] : 0.f;
    s_acc[i][j] = v;
    sS[pp * S::ldS + n] = v;
  });
  for (int i = tid; i < P; i += kThreads) sXprev[i] = 0.f;
  for (int i = tid; i < N; i += kThreads) sBprev[i] = 0.f;
  for (int i = tid; i < kKmax; i += kThreads) sPhi0[i] = 0.f;

  // prologue: chunk 0's inputs
  tc_issue_stage<P, N>(p, raw, b, h, g, 0);
  float pa = 1.f, pb = 0.f, pg = 0.f;  // alpha, beta, gamma of step tid of the next chunk
  if (tid < kQ && tid < L) {
    const int64_t j = (b * L + tid) * H + h;
    pa = __bfloat162float(al_g[j]);
    pb = __bfloat162float(be_g[j]);
    pg = __bfloat162float(ga_g[j]);
  }

  // angle thread roles: angle pair ka = tid % 32, 8-step segment sg = tid / 32
  const int ka = tid & 31, sg = tid >> 5;

  for (int64_t ch = 0; ch < nc; ++ch) {
    const int64_t t0 = ch * kQ;
    const int Qc = (int)((L - t0) < kQ ? (L - t0) : kQ);
    cp_async_wait<0>();
    __syncthreads();  // (A) this chunk's raw inputs are in; the last chunk is done

    // ---- 1. convert x, B, C; alpha/beta/gamma; angle partial sums -------------
    for (int u = tid; u < kQ * (P / 8); u += kThreads) {
      const int t = u / (P / 8), pc = u % (P / 8);
      float v[8];
      ld8_bf16(raw + S::rx + (t * P + pc * 8) * 2, v);
      float4 *d = reinterpret_cast<float4 *>(sX + t * S::ldX + pc * 8);
      d[0] = make_float4(v[0], v[1], v[2], v[3]);
      d[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
    for (int u = tid; u < 2 * kQ * (N / 8); u += kThreads) {
      const int k = u / (kQ * (N / 8)), w = u % (kQ * (N / 8));
      const int t = w / (N / 8), pc = w % (N / 8);
      float v[8];
      ld8_bf16(raw + (k == 0 ? S::rB : S::rC) + (t * N + pc * 8) * 2, v);
      float4 *d = reinterpret_cast<float4 *>((k == 0 ? sBt : sCt) + t * S::ldB + pc * 8);
      d[0] = make_float4(v[0], v[1], v[2], v[3]);
      d[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
    if (tid < kQ) {
      const bool in = tid < Qc;
      sAl[tid] = in ? pa : 1.f;
      sBe[tid] = in ? pb : 0.f;
      sGa[tid] = in ? pg : 0.f;
    }
    float th[8];
    {
      const bf16 *rth = reinterpret_cast<const bf16 *>(raw + S::rth);
      float ssum = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        th[i] = ka < K ? __bfloat162float(rth[(sg * 8 + i) * kKmax + ka]) : 0.f;
        ssum += th[i];
      }
      if (ka < kKmax) sSeg[sg * kKmax + ka] = ssum;
    }
    __syncthreads();  // (B) raw stage consumed

    // ---- 2. next chunk's inputs; log-decay scan ---------------------------------
    if (ch + 1 < nc) {
      tc_issue_stage<P, N>(p, raw, b, h, g, t0 + kQ);
      if (tid < kQ && t0 + kQ + tid < L) {
        const int64_t j = (b * L + t0 + kQ + tid) * H + h;
        pa = __bfloat162float(al_g[j]);
        pb = __bfloat162float(be_g[j]);
        pg = __bfloat162float(ga_g[j]);
      } else {
        pa = 1.f; pb = 0.f; pg = 0.f;
      }
    }
    if (tid < 32) {
      // lane l: steps 2l, 2l+1; inclusive scan of log2(alpha)
      float la0, la1;
      asm("lg2.approx.f32 %0, %1;" : "=f"(la0) : "f"(sAl[2 * tid]));
      asm("lg2.approx.f32 %0, %1;" : "=f"(la1) : "f"(sAl[2 * tid + 1]));
      la0 = fmaxf(la0, -126.f);
      la1 = fmaxf(la1, -126.f);
      float incl = la0 + la1;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float v = __shfl_up_sync(0xffffffffu, incl, off);
        if (tid >= off) incl += v;
      }
      float excl = __shfl_up_sync(0xffffffffu, incl, 1);
      if (tid == 0) excl = 0.f;
      sLc[2 * tid] = excl + la0;
      sLc[2 * tid + 1] = incl;
    }
    // ---- 3. rotate B and C of this thread's 8 steps by the cumulative angles ----
    float phi_end = 0.f;
    if (ka < kKmax) {
      float phi = sPhi0[ka];
      for (int s2 = 0; s2 < sg; ++s2) phi += sSeg[s2 * kKmax + ka];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int t = sg * 8 + i;
        phi += th[i];
        if (ka < K) {
          float sn, cs;
          sincosf(phi, &sn, &cs);
          float *bt = sBt + t * S::ldB + 2 * ka;
          float *ct = sCt + t * S::ldB + 2 * ka;
          const float b0 = bt[0], b1 = bt[1], c0 = ct[0], c1 = ct[1];
          bt[0] = cs * b0 - sn * b1;
          bt[1] = sn * b0 + cs * b1;
          ct[0] = cs * c0 - sn * c1;
          ct[1] = sn * c0 + cs * c1;
        }
      }
      phi_end = phi;
    }
    __syncthreads();  // (C) rotated operands and the log-decays are in place

    // ---- 4. G = Ct Bt^T and Ct S^T (tensor cores); per-step vectors -------------
    if (tid < kQ) {
      const int t = tid;
      const float lct = sLc[t], lcl = sLc[kQ - 1];
      sDl[t] = ex2(lct);
      sEv[t] = t + 1 < kQ ? fmaf(sAl[t + 1], sGa[t], sBe[t + 1]) : 0.f;
      sCrow[t] = t + 1 < kQ ? ex2(lcl - sLc[t + 1]) * fmaf(sAl[t + 1], sGa[t], sBe[t + 1]) : sGa[t];
      float dot = 0.f;
      for (int n = 0; n < N; ++n) dot = fmaf(sCt[t * S::ldB + n], sBprev[n], dot);
      sWc[t] = sBe[0] * ex2(lct - sLc[0]) * dot;
    }
    float g_acc[TQQ::kPerWarp][4];
    zero_acc<kQ, kQ>(g_acc);
    mma_tiles<kQ, kQ, N, true, true>(g_acc, [&](int m, int k) { return sCt[m * S::ldB + k]; },
                         [&](int k, int n) { return sBt[n * S::ldB + k]; });
    float y_acc[TQP::kPerWarp][4];
    zero_acc<kQ, P>(y_acc);
    mma_tiles<kQ, P, N, true, true>(y_acc, [&](int m, int k) { return sCt[m * S::ldB + k]; },
                        [&](int k, int n) { return sS[n * S::ldS + k]; });
    // the state entering this chunk goes to `saved`
    if (p.saved) {
      float *dst = p.saved + ((b * H + h) * nc + ch) * P * N;
      for_acc<P, N>([&](int i, int j, int pp, int n) {
        if ((j & 1) == 0)
          *reinterpret_cast<float2 *>(dst + pp * N + n) = make_float2(s_acc[i][j], s_acc[i][j + 1]);
      });
      // the cumulative angles at the chunk start, after all states
      float *ang = p.saved + p.B * H * nc * P * N + ((b * H + h) * nc + ch) * kKmax;
      if (tid < kKmax) ang[tid] = sPhi0[tid];
    }
    __syncthreads();  // (D) Ct is consumed; the per-step vectors are visible

    // ---- 5. W = c o G over Ct's storage -------------------------------------------
    for_acc<kQ, kQ>([&](int i, int j, int t, int s) {
      float w = 0.f;
      if (s == t) w = sGa[t] * g_acc[i][j];
      else if (s < t) w = ex2(sLc[t] - sLc[s + 1]) * sEv[s] * g_acc[i][j];
      sW[t * S::ldW + s] = w;
    });
    for_acc<kQ, P>([&](int i, int j, int t, int pp) { y_acc[i][j] *= sDl[t]; });
    __syncthreads();  // (E) W is in place

    // ---- 6. Y += W X; outputs --------------------------------------------------------
    mma_tiles<kQ, P, kQ, true, false>(y_acc, [&](int m, int k) { return sW[m * S::ldW + k]; },
                         [&](int k, int n) { return sX[k * S::ldX + n]; });
    for_acc<kQ, P>([&](int i, int j, int t, int pp) {
      if ((j & 1) != 0 || t >= Qc) return;
      const int64_t o = ((b * L + t0 + t) * H + h) * P + pp;
      float y0 = y_acc[i][j] + sWc[t] * sXprev[pp] + Dh * sX[t * S::ldX + pp];
      float y1 = y_acc[i][j + 1] + sWc[t] * sXprev[pp + 1] + Dh * sX[t * S::ldX + pp + 1];
      if (z_g) {
        float z0, z1;
        unpack_bf16x2(*reinterpret_cast<const uint32_t *>(z_g + o), z0, z1);
        y0 *= silu(z0);
        y1 *= silu(z1);
      }
      *reinterpret_cast<uint32_t *>(out_g + o) = pack_bf16x2(y0, y1);
    });

    // ---- 7. state update: S = d(Q-1,-1) S + beta_0 d(Q-1,0) K_prev + X^T diag(c) Bt --
    {
      const float dlast = sDl[kQ - 1];
      const float w0 = sBe[0] * ex2(sLc[kQ - 1] - sLc[0]);
      for_acc<P, N>([&](int i, int j, int pp, int n) {
        s_acc[i][j] = fmaf(dlast, s_acc[i][j], w0 * sXprev[pp] * sBprev[n]);
      });
      mma_tiles<P, N, kQ, false, true>(s_acc, [&](int m, int k) { return sX[k * S::ldX + m]; },
                                       [&](int k, int n) { return sCrow[k] * sBt[k * S::ldB + n]; });
    }
    __syncthreads();  // (F) every read of X, Bt, S, the carries and the angles is done

    // ---- 8. carries into the next chunk ---------------------------------------------
    for_acc<P, N>([&](int i, int j, int pp, int n) { sS[pp * S::ldS + n] = s_acc[i][j]; });
    for (int i = tid; i < P; i += kThreads) sXprev[i] = sX[(Qc - 1) * S::ldX + i];
    for (int i = tid; i < N; i += kThreads) sBprev[i] = sBt[(Qc - 1) * S::ldB + i];
    if (sg == 7 && ka < kKmax) sPhi0[ka] = phi_end;
  }

  if (p.final_state) {
    float *dst = p.final_state + (b * H + h) * P * N;
    for_acc<P, N>([&](int i, int j, int pp, int n) {
      if ((j & 1) == 0)
        *reinterpret_cast<float2 *>(dst + pp * N + n) = make_float2(s_acc[i][j], s_acc[i][j + 1]);
    });
  }
}

template <int P, int N>
cudaError_t launch_tc(const M3Params &p, cudaStream_t s) {
  const size_t smem = (size_t)TcFwdSmem<P, N>::total;
  cudaError_t e = cudaFuncSetAttribute(m3_fwd_tc_kernel<P, N>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  m3_fwd_tc_kernel<P, N><<<dim3((unsigned)p.H, (unsigned)p.B), kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

template <int P>
cudaError_t launch_tc_n(const M3Params &p, cudaStream_t s) {
  switch (p.N) {
    case 16: return launch_tc<P, 16>(p, s);
    case 32: return launch_tc<P, 32>(p, s);
    default: return launch_tc<P, 64>(p, s);
  }
}

}  // namespace

cudaError_t launch_m3_fwd_tc(const M3Params &p, cudaStream_t s) {
  switch (p.P) {
    case 16: return launch_tc_n<16>(p, s);
    case 32: return launch_tc_n<32>(p, s);
    default: return launch_tc_n<64>(p, s);
  }
}

}  // namespace msc
