// m3_fwd_umma.cu -- Mamba-3 SISO scan, forward, bf16 io, on the sm_100a
// tensor cores through tcgen05 (umma.cuh).
//
// Same recurrence, chunked form (m3_common.cuh) and outputs as m3_fwd.cu
// (mamba-rs 0.7.0 README, "Features"; the three-term update and per-head
// cumulative angles whose gradients stages B3 and B4 of Mamba3Scratch,
// mamba-rs 0.4.2 src/mamba3_siso/cpu/scratch.rs, hold).  One CTA of 8 warps
// per (b, h) walks the 64-step chunks in order, two CTAs per SM.  A chunk is
// two rounds of tensor-core work:
//
//   round 1   G  = Ct Bt^T        (A: Ct [t][n], B: Bt [s][n])
//             Y1 = Ct S^T         (A: Ct,        B: S  [p][n])
//   epilogue  W  = c o G          (into Ct's planes)
//             Bc = diag(c(Q-1, .)) Bt   (into Bt's planes)
//   round 2   Y2 = W X            (A: W [t][s],  B: X^T [p][s])
//             dS = X^T Bc         (A: X^T,       B: Bc read MN-major)
//   epilogue  out = (d(t,-1) Y1 + Y2 + beta_0 d(t,0) (Ct.Bt_prev) x_prev + D x) silu(z)
//             S   = d(Q-1,-1) S + beta_0 d(Q-1,0) x_prev (outer) Bt_prev + dS
//
// f32 operands live in shared memory as three bf16 parts, the bf16 inputs as
// one, so every product carries f32 accuracy.  Thread 0 issues the MMAs; the
// CTA waits on an mbarrier (bounded) and reads the f32 accumulators from
// TMEM.  The state stays in registers, row r of the accumulator layout per
// thread, with its parts in shared memory for the next chunk's Y1.  x, B, C of
// the next chunk arrive by cp.async, and theta, alpha, beta, gamma into
// registers, while a chunk computes.
//
// Shared-memory access patterns follow the core-matrix layout: a warp stores
// a core matrix (8 rows x 16 bytes) per instruction, so that no two lanes
// share a bank.  The cumulative angles come from a scan over each warp's 8
// steps (lanes 4 i + q hold step i of angle pairs q, q + 4, ...) and the
// per-warp totals, which is also the layout the rotation writes in.
#include "m3_common.cuh"
#include "m3_disc_common.cuh"
#include "umma.cuh"

namespace msc {
namespace {

using namespace m3;
using umma::koff;

template <int P, int N>
struct UmFwdSmem {
  static constexpr int kK = N / 2;
  static constexpr int kG = kK / 4;         // groups of 4 angle pairs
  static constexpr int kRS = N * 2 + 16;    // raw B, C row stride in bytes (padded: no bank conflicts)
  // bytes; bf16 part planes, K-major core-matrix layout (umma.cuh)
  static constexpr int kCW = 64 * 64 * 2;  // one part of Ct (K = N) or W (K = Q)
  static constexpr int kBt = 64 * N * 2;   // one part of Bt / Bc [s][n]
  static constexpr int kSp = P * N * 2;    // one part of S [p][n]
  static constexpr int cw = 0;
  static constexpr int bt = cw + 3 * kCW;
  static constexpr int sp = bt + 3 * kBt;
  static constexpr int xp = sp + 3 * kSp;       // X^T [p][s], exact bf16, 64 rows (rows >= P zero)
  static constexpr int rx = xp + 64 * 64 * 2;   // raw x [t][p]
  static constexpr int rB = rx + 64 * P * 2;    // raw B [t][n]
  static constexpr int rC = rB + 64 * kRS;      // raw C [t][n]
  // f32 vectors
  static constexpr int vec = rC + 64 * kRS;
  static constexpr int al = vec, be = al + 256, ga = be + 256, lc = ga + 256, ev = lc + 256,
                       dl = ev + 256, crow = dl + 256,
                       wcd = crow + 256,           // [kG][Q] partial Ct_t . Bt_prev per angle group
                       xprev = wcd + kG * 256,     // [2][P], by chunk parity
                       bprev = xprev + 2 * P * 4,  // [2][N]
                       dtv = bprev + 2 * N * 4,    // [Q] dt of the next chunk's steps (raw input)
                       misc = dtv + 256;
  static constexpr int total = misc + 32;  // tmem slot, mbarrier, error flag
};

// cp.async the raw x, B, C rows of the chunk at t0 (rows past L zero-filled)
template <int P, int N, bool kSlab>
__device__ __forceinline__ void um_issue_raw(const M3Params &p, unsigned char *sm, int64_t b,
                                             int64_t h, int64_t g, int64_t t0) {
  using S = UmFwdSmem<P, N>;
  const int64_t L = p.L, H = p.H, G = p.G;
  const bf16 *x = static_cast<const bf16 *>(p.x);
  const bf16 *Bm = static_cast<const bf16 *>(p.Bm);
  const bf16 *Cm = static_cast<const bf16 *>(p.Cm);
  for (int u = threadIdx.x; u < kQ * (P / 8) + 2 * kQ * (N / 8); u += kThreads) {
    if (u < kQ * (P / 8)) {
      const int t = u / (P / 8), pc = u % (P / 8);
      const bool in = t0 + t < L;
      cp_async16(sm + S::rx + (t * P + pc * 8) * 2,
                 in ? x + ((b * L + t0 + t) * H + h) * P + pc * 8 : x, in ? 16 : 0);
    } else {
      const int v = u - kQ * (P / 8);
      const int k = v / (kQ * (N / 8)), w = v % (kQ * (N / 8));
      const int t = w / (N / 8), pc = w % (N / 8);
      const bool in = t0 + t < L;
      const bf16 *src = k == 0 ? Bm : Cm;
      cp_async16(sm + (k == 0 ? S::rB : S::rC) + t * S::kRS + pc * 16,
                 in ? src + ((b * L + t0 + t) * G + g) * (kSlab ? p.ldN : N) + (kSlab ? p.n0 : 0) + pc * 8
                    : src,
                 in ? 16 : 0);
    }
  }
  cp_async_commit();
}

__device__ __forceinline__ uint32_t bf16pair(bf16 lo, bf16 hi) {
  return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}

// the three parts of (v0, v1) at byte offset `off` of the planes at `base`
// (plane stride `stride`), one 4-byte store per plane
__device__ __forceinline__ void put3x2(unsigned char *base, int stride, int off, float v0,
                                       float v1) {
  uint32_t w[3];
  umma::split3x2(v0, v1, w);
#pragma unroll
  for (int q = 0; q < 3; ++q) *reinterpret_cast<uint32_t *>(base + q * stride + off) = w[q];
}

// Issue one product into TMEM column `col`: parts of A (nA of them, planes at
// aA, stride sA, K-major with Ka columns, 64 rows) times parts of B (nB,
// planes at aB, stride sB; K-major with Kb columns, or with kBMN the same
// bytes read MN-major, Kb then being the MN extent), over K / 16 steps.  Part
// pairs whose order is below f32 rounding are left out; the smallest go first.
template <int NMMA, bool kBMN>
__device__ __forceinline__ void issue_product(uint32_t tmem, int col, uint32_t aA, int sA, int nA,
                                              int Ka, uint32_t aB, int sB, int nB, int Kb, int K) {
  const uint32_t id = umma::idesc_bf16<NMMA, kBMN>();
  const int pa[6] = {2, 1, 0, 1, 0, 0}, pb[6] = {0, 1, 2, 0, 1, 0};
  bool first = true;
  for (int u = 0; u < 6; ++u) {
    if (pa[u] >= nA || pb[u] >= nB) continue;
    for (int ks = 0; ks < K / 16; ++ks) {
      const uint64_t da = umma::desc(aA + pa[u] * sA + ks * 256, 128, Ka * 16);
      const uint64_t db = kBMN ? umma::desc(aB + pb[u] * sB + ks * 2 * (Kb * 16), Kb * 16, 128)
                               : umma::desc(aB + pb[u] * sB + ks * 256, 128, Kb * 16);
      umma::mma(tmem + col, da, db, id, !first);
      first = false;
    }
  }
}

// kSlab: one slab of a wider d_state (runtime row length and offsets);
// otherwise the whole d_state with compile-time strides
template <int P, int N, bool kSlab, bool kRaw>
__global__ void __launch_bounds__(kThreads, 2) m3_fwd_umma_kernel(const M3Params p) {
  using S = UmFwdSmem<P, N>;
  constexpr int kK = N / 2;
  constexpr int kG = S::kG;    // angle groups
  constexpr int kWG = 8 / kG;  // warps per angle group
  constexpr int kM = 8 / kWG;  // 8-step segments a warp rotates
  constexpr int kSR = kK / 8;  // 8-column blocks of a state row half
  constexpr int kPR = P / 16;  // 8-column blocks of an output row half
  extern __shared__ __align__(1024) unsigned char sm[];
  float *sAl = reinterpret_cast<float *>(sm + S::al), *sBe = reinterpret_cast<float *>(sm + S::be);
  float *sGa = reinterpret_cast<float *>(sm + S::ga), *sLc = reinterpret_cast<float *>(sm + S::lc);
  float *sEv = reinterpret_cast<float *>(sm + S::ev), *sDl = reinterpret_cast<float *>(sm + S::dl);
  float *sCrow = reinterpret_cast<float *>(sm + S::crow);
  float *sWcd = reinterpret_cast<float *>(sm + S::wcd);
  float *sXprev = reinterpret_cast<float *>(sm + S::xprev);
  float *sBprev = reinterpret_cast<float *>(sm + S::bprev);
  uint32_t *sTmem = reinterpret_cast<uint32_t *>(sm + S::misc);
  uint64_t *sMbar = reinterpret_cast<uint64_t *>(sm + S::misc + 8);
  int *sErr = reinterpret_cast<int *>(sm + S::misc + 16);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t h = blockIdx.x, b = blockIdx.y;
  const int64_t L = p.L, H = p.H, G = p.G;
  // this slab's states n0 .. n0 + N - 1 of ldN, and its angle pairs k0 ..
  // k0 + K - 1 of the Kt
  const int64_t ldN = kSlab ? p.ldN : N, n0 = kSlab ? p.n0 : 0;
  const int Kt = (int)p.K, k0 = (int)(n0 / 2);
  const int K = Kt - k0 < 0 ? 0 : (Kt - k0 > kK ? kK : Kt - k0);
  const int slab = kSlab ? p.slab : kSlabWhole;
  const bool finish = slab == kSlabWhole || slab == kSlabLast;
  const int64_t g = h / (H / G);
  const float Dh = (p.Dp && finish) ? p.Dp[h] : 0.f;  // the D x skip joins once
  const int64_t nc = (L + kQ - 1) / kQ;
  const bf16 *x_g = static_cast<const bf16 *>(p.x);
  const bf16 *al_g = static_cast<const bf16 *>(p.alpha);
  const bf16 *be_g = static_cast<const bf16 *>(p.beta);
  const bf16 *ga_g = static_cast<const bf16 *>(p.gamma);
  const bf16 *th_g = static_cast<const bf16 *>(p.theta);
  const bf16 *z_g = static_cast<const bf16 *>(p.z);
  bf16 *out_g = static_cast<bf16 *>(p.out);
  const uint32_t base = umma::smem_addr(sm);
  const uint32_t mbar = umma::smem_addr(sMbar);

  // Roles.  Angles: lane (ri, rq) = (lane / 4, lane % 4) of warp w holds
  // angle pair ka = 4 (w % kG) + rq at steps 8 m + ri of the chunk, for all
  // eight segments m, and rotates segments sp kM .. sp kM + kM - 1 (sp = w /
  // kG).  Accumulators: warp w reads rows ra = 16 (w % 4) + ri and rb = ra + 8
  // (TMEM lane quarter w % 4), column half cb = w / 4, columns 2 rq, 2 rq + 1
  // of each 8-column block.
  const int ri = lane >> 2, rq = lane & 3;
  const int ag = warp % kG, sp = warp / kG;
  const int ka = 4 * ag + rq;
  const int q4 = warp & 3, cb = warp >> 2;
  const int ra = 16 * q4 + ri, rb = ra + 8, c2 = 2 * rq;
  const bool srow = 16 * q4 < P;
  const uint32_t tq = (uint32_t)(32 * q4) << 16;

  if (warp == 0) umma::tmem_alloc(sTmem, 256);
  if (tid == 0) {
    umma::mbar_init(mbar);
    *sErr = 0;
  }
  // the state: rows ra (sreg[4 i], [4 i + 1]) and rb (sreg[4 i + 2], [4 i + 3]),
  // columns cb * kK + 8 i + c2 + 0, 1
  float sreg[kK / 2];
  const float *h0 = p.h0 ? p.h0 + (b * H + h) * P * ldN + n0 : nullptr;  // rows of ldN
#pragma unroll
  for (int i = 0; i < kSR; ++i) {
    const int n = cb * kK + 8 * i + c2;
    const float2 va = (srow && h0) ? *reinterpret_cast<const float2 *>(h0 + ra * ldN + n) : make_float2(0.f, 0.f);
    const float2 vb = (srow && h0) ? *reinterpret_cast<const float2 *>(h0 + rb * ldN + n) : make_float2(0.f, 0.f);
    sreg[4 * i] = va.x; sreg[4 * i + 1] = va.y;
    sreg[4 * i + 2] = vb.x; sreg[4 * i + 3] = vb.y;
  }
  auto put_state = [&]() {
#pragma unroll
    for (int i = 0; i < kSR; ++i) {
      const int n = cb * kK + 8 * i + c2;
      put3x2(sm + S::sp, S::kSp, koff(ra, n, N), sreg[4 * i], sreg[4 * i + 1]);
      put3x2(sm + S::sp, S::kSp, koff(rb, n, N), sreg[4 * i + 2], sreg[4 * i + 3]);
    }
  };
  auto store_state = [&](float *dst) {  // dst: this (b, h, slab)'s P x N block, rows of ldN
#pragma unroll
    for (int i = 0; i < kSR; ++i) {
      const int n = cb * kK + 8 * i + c2;
      *reinterpret_cast<float2 *>(dst + ra * ldN + n) = make_float2(sreg[4 * i], sreg[4 * i + 1]);
      *reinterpret_cast<float2 *>(dst + rb * ldN + n) = make_float2(sreg[4 * i + 2], sreg[4 * i + 3]);
    }
  };
  if (srow) put_state();
  for (int i = tid; i < 2 * P; i += kThreads) sXprev[i] = 0.f;
  for (int i = tid; i < 2 * N; i += kThreads) sBprev[i] = 0.f;
  // rows P..63 of X^T take part in dS (rows of the result that are dropped)
  for (int i = tid; i < (64 - P) * 64 / 8; i += kThreads)
    *reinterpret_cast<uint4 *>(sm + S::xp + P * 128 + i * 16) = make_uint4(0, 0, 0, 0);

  // the next chunk's theta (angle roles) and alpha, beta, gamma (warp 0: steps
  // 2 lane, 2 lane + 1)
  float thv[8];
  float pa0, pa1, pb0, pb1, pg0, pg1;
  // from raw projections: the discretisation of step s (the expressions of
  // the discretisation kernel, each value rounded to bf16 as it stores them)
  const float dtb = (kRaw && p.dt_bias) ? p.dt_bias[h] : 0.f;
  float *sDt = reinterpret_cast<float *>(sm + S::dtv);
  auto raw_coef = [&](int64_t j, float &a, float &bt, float &gm) {
    const DiscCoef cf = disc_coef(__bfloat162float(static_cast<const bf16 *>(p.dd_dt)[j]), dtb,
                                  __bfloat162float(static_cast<const bf16 *>(p.dd_a)[j]),
                                  __bfloat162float(static_cast<const bf16 *>(p.trap)[j]), p.A_floor);
    a = to_f32(from_f32<bf16>(cf.alpha));
    bt = to_f32(from_f32<bf16>(disc_beta(cf)));
    gm = to_f32(from_f32<bf16>(disc_gamma(cf)));
    return cf.dt;
  };
  // the next chunk's per-step values into registers (and, from raw
  // projections, warp 0's dt of each step into sDt: the chunk's readers of
  // sDt are past barrier (C), where this is called, so one buffer serves)
  auto load_small = [&](int64_t t0) {
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int64_t t = t0 + 8 * m + ri;
      float v = 0.f;
      if (ka < K && t < L) {
        if constexpr (kRaw)  // the raw angle (shared by the heads); theta = dt x angle once dt is in
          v = __bfloat162float(static_cast<const bf16 *>(p.angles)[(b * L + t) * Kt + k0 + ka]);
        else
          v = __bfloat162float(th_g[((b * L + t) * H + h) * Kt + k0 + ka]);
      }
      thv[m] = v;
    }
    pa0 = pa1 = 1.f;
    pb0 = pb1 = pg0 = pg1 = 0.f;
    if (warp == 0) {
      const int64_t s = t0 + 2 * lane;
      float dt0 = 0.f, dt1 = 0.f;
      if (s < L) {
        const int64_t j = (b * L + s) * H + h;
        if constexpr (kRaw) {
          dt0 = raw_coef(j, pa0, pb0, pg0);
        } else {
          pa0 = __bfloat162float(al_g[j]);
          pb0 = __bfloat162float(be_g[j]);
          pg0 = __bfloat162float(ga_g[j]);
        }
      }
      if (s + 1 < L) {
        const int64_t j = (b * L + s + 1) * H + h;
        if constexpr (kRaw) {
          dt1 = raw_coef(j, pa1, pb1, pg1);
        } else {
          pa1 = __bfloat162float(al_g[j]);
          pb1 = __bfloat162float(be_g[j]);
          pg1 = __bfloat162float(ga_g[j]);
        }
      }
      if constexpr (kRaw) {
        sDt[2 * lane] = dt0;
        sDt[2 * lane + 1] = dt1;
      }
    }
  };
  um_issue_raw<P, N, kSlab>(p, sm, b, h, g, 0);
  load_small(0);
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = *sTmem;
  float phi_c = 0.f;  // cumulative angle of pair ka before the chunk
  float2 brot[8];     // rotated B of pair ka at steps 8 m + ri (this warp's segments)

  for (int64_t ch = 0; ch < nc; ++ch) {
    const int64_t t0 = ch * kQ;
    const int Qc = (int)((L - t0) < kQ ? (L - t0) : kQ);
    const int cur = (int)(ch & 1);
    const float *xp_c = sXprev + cur * P, *bp_c = sBprev + cur * N;
    float *xp_n = sXprev + (cur ^ 1) * P, *bp_n = sBprev + (cur ^ 1) * N;
    cp_async_wait<0>();
    __syncthreads();  // (A) this chunk's raw inputs are in; the last chunk is done
    if (*sErr) break;
    if constexpr (kRaw) {
      // theta = dt x angle, rounded to bf16 as the discretisation stores it
      // (sDt was written by warp 0 ahead of barrier (A))
#pragma unroll
      for (int m = 0; m < 8; ++m) thv[m] = to_f32(from_f32<bf16>(sDt[8 * m + ri] * thv[m]));
    }

    // ---- 1. state and angles entering the chunk; X^T; per-step vectors ----------
    if (p.saved) {
      if (srow) store_state(p.saved + ((b * H + h) * nc + ch) * P * ldN + n0);
      if (sp == 0 && ri == 0)
        p.saved[p.B * H * nc * P * ldN + ((b * H + h) * nc + ch) * (ldN / 2) + k0 + ka] = phi_c;
    }
    for (int u = tid; u < P * 8; u += kThreads) {
      const int pp = u % P, t8 = u / P;
      const bf16 *src = reinterpret_cast<const bf16 *>(sm + S::rx) + t8 * 8 * P + pp;
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) w[e] = bf16pair(src[2 * e * P], src[(2 * e + 1) * P]);
      *reinterpret_cast<uint4 *>(sm + S::xp + koff(pp, t8 * 8, 64)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    for (int i = tid; i < P; i += kThreads)
      xp_n[i] = __bfloat162float(reinterpret_cast<const bf16 *>(sm + S::rx)[(Qc - 1) * P + i]);
    if (warp == 0) {
      const int s0 = 2 * lane;
      sAl[s0] = pa0; sAl[s0 + 1] = pa1;
      sBe[s0] = pb0; sBe[s0 + 1] = pb1;
      sGa[s0] = pg0; sGa[s0 + 1] = pg1;
      // inclusive scan of log2(alpha)
      float la0, la1;
      asm("lg2.approx.f32 %0, %1;" : "=f"(la0) : "f"(pa0));
      asm("lg2.approx.f32 %0, %1;" : "=f"(la1) : "f"(pa1));
      la0 = fmaxf(la0, -126.f);
      la1 = fmaxf(la1, -126.f);
      float incl = la0 + la1;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      float excl = __shfl_up_sync(0xffffffffu, incl, 1);
      if (lane == 0) excl = 0.f;
      sLc[s0] = excl + la0;
      sLc[s0 + 1] = incl;
      __syncwarp();
      const float lcl = sLc[kQ - 1];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = s0 + e;
        const float ev = t + 1 < kQ ? fmaf(sAl[t + 1], sGa[t], sBe[t + 1]) : 0.f;
        sDl[t] = ex2(sLc[t]);
        sEv[t] = ev;
        sCrow[t] = t + 1 < kQ ? ex2(lcl - sLc[t + 1]) * ev : sGa[t];
      }
    }

    // ---- 2. cumulative angles; rotate B and C into the Bt and Ct planes ------------
    {
      float T[8];  // segment totals
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        float v = thv[m];
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          const float u = __shfl_up_sync(0xffffffffu, v, off);
          if (lane >= off) v += u;
        }
        thv[m] = v;  // inclusive within segment m
        T[m] = __shfl_sync(0xffffffffu, v, 28 + rq);
      }
      float phi = phi_c;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        if (m >= sp * kM && m < sp * kM + kM) {
          const int t = 8 * m + ri;
          float b0, b1, c0, c1;
          unpack_bf16x2(*reinterpret_cast<const uint32_t *>(sm + S::rB + t * S::kRS + 4 * ka), b0, b1);
          unpack_bf16x2(*reinterpret_cast<const uint32_t *>(sm + S::rC + t * S::kRS + 4 * ka), c0, c1);
          if (ka < K) {
            float sn, cs;
            sincos_reduced(phi + thv[m], sn, cs);
            const float rb0 = cs * b0 - sn * b1, rb1 = sn * b0 + cs * b1;
            const float rc0 = cs * c0 - sn * c1, rc1 = sn * c0 + cs * c1;
            b0 = rb0; b1 = rb1; c0 = rc0; c1 = rc1;
          }
          brot[m] = make_float2(b0, b1);
          put3x2(sm + S::bt, S::kBt, koff(t, 2 * ka, N), b0, b1);
          put3x2(sm + S::cw, S::kCW, koff(t, 2 * ka, N), c0, c1);
          float d = fmaf(c0, bp_c[2 * ka], c1 * bp_c[2 * ka + 1]);
          d += __shfl_xor_sync(0xffffffffu, d, 1);
          d += __shfl_xor_sync(0xffffffffu, d, 2);
          if (rq == 0) sWcd[ag * kQ + t] = d;
          if (t == Qc - 1) {
            bp_n[2 * ka] = b0;
            bp_n[2 * ka + 1] = b1;
          }
        }
        phi += T[m];
      }
      phi_c = phi;
    }
    umma::fence_async_smem();
    __syncthreads();  // (C) operands of round 1 in place; raw stage consumed

    if (tid == 0) {
      umma::fence_after();
      issue_product<64, false>(tmem, 0, base + S::cw, S::kCW, 3, N, base + S::bt, S::kBt, 3, N, N);
      issue_product<P, false>(tmem, 64, base + S::cw, S::kCW, 3, N, base + S::sp, S::kSp, 3, N, N);
      umma::commit(mbar);
    }
    if (ch + 1 < nc) {
      um_issue_raw<P, N, kSlab>(p, sm, b, h, g, t0 + kQ);
      load_small(t0 + kQ);
    }
    // x and z of this thread's outputs (rows ra, rb)
    uint32_t xo[2 * kPR], zo[2 * kPR];
#pragma unroll
    for (int i = 0; i < kPR; ++i)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = e ? rb : ra;
        const int64_t o = ((b * L + t0 + t) * H + h) * P + cb * (P / 2) + 8 * i + c2;
        const bool in = t < Qc;
        xo[2 * i + e] = in ? *reinterpret_cast<const uint32_t *>(x_g + o) : 0u;
        zo[2 * i + e] = (in && z_g) ? *reinterpret_cast<const uint32_t *>(z_g + o) : 0u;
      }

    // ---- 3. W = c o G over Ct's planes; Bc = diag(c(Q-1, .)) Bt over Bt's planes
    if (!umma::mbar_wait(mbar, 0)) *sErr = 1;
    umma::fence_after();
    {
      float gv[16];
      umma::tmem_ld16<4>(tmem + tq + cb * 32, gv);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = e ? rb : ra;
        const float lct = sLc[t], gt = sGa[t];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int s0 = cb * 32 + 8 * i + c2;
          float w[2];
#pragma unroll
          for (int f = 0; f < 2; ++f) {
            const int s = s0 + f;
            const float gval = gv[4 * i + 2 * e + f];
            w[f] = s == t ? gt * gval : (s < t ? ex2(lct - sLc[s + 1]) * sEv[s] * gval : 0.f);
          }
          put3x2(sm + S::cw, S::kCW, koff(t, s0, 64), w[0], w[1]);
        }
      }
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      if (m >= sp * kM && m < sp * kM + kM) {
        const int t = 8 * m + ri;
        const float cr = sCrow[t];
        put3x2(sm + S::bt, S::kBt, koff(t, 2 * ka, N), cr * brot[m].x, cr * brot[m].y);
      }
    }
    umma::fence_async_smem();
    umma::fence_before();
    __syncthreads();  // (D) operands of round 2 in place
    if (*sErr) break;
    if (tid == 0) {
      umma::fence_after();
      issue_product<P, false>(tmem, 128, base + S::cw, S::kCW, 3, 64, base + S::xp, 0, 1, 64, 64);
      issue_product<N, true>(tmem, 192, base + S::xp, 0, 1, 64, base + S::bt, S::kBt, 3, N, 64);
      umma::commit(mbar);
    }

    // ---- 4. outputs; the state update ------------------------------------------------
    if (!umma::mbar_wait(mbar, 1)) *sErr = 1;
    umma::fence_after();
    {
      float y1[4 * kPR], y2[4 * kPR];
      umma::tmem_ld16_pair<kPR>(tmem + tq + 64 + cb * (P / 2), tmem + tq + 128 + cb * (P / 2), y1, y2);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = e ? rb : ra;
        if (t < Qc) {
          float wcd = 0.f;
#pragma unroll
          for (int a = 0; a < kG; ++a) wcd += sWcd[a * kQ + t];
          const float dlt = sDl[t], wct = sBe[0] * ex2(sLc[t] - sLc[0]) * wcd;
#pragma unroll
          for (int i = 0; i < kPR; ++i) {
            const int p0 = cb * (P / 2) + 8 * i + c2;
            float xf0, xf1;
            unpack_bf16x2(xo[2 * i + e], xf0, xf1);
            float o0 = fmaf(dlt, y1[4 * i + 2 * e], y2[4 * i + 2 * e]) + wct * xp_c[p0] + Dh * xf0;
            float o1 = fmaf(dlt, y1[4 * i + 2 * e + 1], y2[4 * i + 2 * e + 1]) + wct * xp_c[p0 + 1] + Dh * xf1;
            const int64_t oi = ((b * L + t0 + t) * H + h) * P + p0;
            if (slab != kSlabWhole) {  // the sums over the states cross the slabs
              float2 *ty = reinterpret_cast<float2 *>(p.tok_y + oi);
              if (slab != kSlabFirst) {
                const float2 prev = *ty;
                o0 = prev.x + o0;
                o1 = prev.y + o1;
              }
              if (!finish) {
                *ty = make_float2(o0, o1);
                continue;
              }
            }
            if (z_g) {
              float zf0, zf1;
              unpack_bf16x2(zo[2 * i + e], zf0, zf1);
              o0 *= silu(zf0);
              o1 *= silu(zf1);
            }
            *reinterpret_cast<uint32_t *>(out_g + oi) = pack_bf16x2(o0, o1);
          }
        }
      }
    }
    {
      float dv[kK / 2];
      umma::tmem_ld16<kSR>(tmem + tq + 192 + cb * kK, dv);
      if (srow) {
        const float dlast = sDl[kQ - 1], w0 = sBe[0] * ex2(sLc[kQ - 1] - sLc[0]);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float wx = w0 * xp_c[e ? rb : ra];
#pragma unroll
          for (int i = 0; i < kSR; ++i) {
            const int n = cb * kK + 8 * i + c2;
#pragma unroll
            for (int f = 0; f < 2; ++f) {
              float &sv = sreg[4 * i + 2 * e + f];
              sv = fmaf(dlast, sv, wx * bp_c[n + f]) + dv[4 * i + 2 * e + f];
            }
          }
        }
        put_state();
      }
    }
    umma::fence_async_smem();
    umma::fence_before();
  }

  cp_async_wait<0>();
  __syncthreads();
  const bool failed = *sErr != 0;
  if (p.final_state && srow) {
    if (failed) {
#pragma unroll
      for (int j = 0; j < kK / 2; ++j) sreg[j] = __int_as_float(0x7fc00000);
    }
    store_state(p.final_state + (b * H + h) * P * ldN + n0);
  }
  if (failed) {  // a tensor-core round never completed: the outputs of this (b, h) are NaN
    const bf16 qnan = __ushort_as_bfloat16((unsigned short)0x7fc0);
    for (int64_t i = tid; i < L * P; i += kThreads)
      out_g[((b * L + i / P) * H + h) * P + i % P] = qnan;
  }
  umma::fence_before();
  __syncthreads();
  if (warp == 0) {
    umma::fence_after();
    umma::tmem_dealloc(tmem, 256);
  }
}

template <int P, int N, bool kSlab, bool kRaw = false>
cudaError_t launch_um(const M3Params &p, cudaStream_t s) {
  // at least 80 KB of shared memory per CTA, so that no more than two CTAs
  // (2 x 256 TMEM columns) share an SM
  const size_t smem = UmFwdSmem<P, N>::total > 80 * 1024 ? (size_t)UmFwdSmem<P, N>::total : 80 * 1024;
  cudaError_t e = cudaFuncSetAttribute(m3_fwd_umma_kernel<P, N, kSlab, kRaw>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  m3_fwd_umma_kernel<P, N, kSlab, kRaw><<<dim3((unsigned)p.H, (unsigned)p.B), kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

template <int P>
cudaError_t launch_um_n(const M3Params &p, cudaStream_t s) {
  if (p.slab != kSlabWhole) return launch_um<P, kM3Slab, true>(p, s);
  // from raw projections: d_state 16, 32 or 64 (the API refuses others)
  if (p.raw) {
    switch (p.N) {
      case 16: return launch_um<P, 16, false, true>(p, s);
      case 32: return launch_um<P, 32, false, true>(p, s);
      default: return launch_um<P, 64, false, true>(p, s);
    }
  }
  switch (p.N) {
    case 16: return launch_um<P, 16, false>(p, s);
    case 32: return launch_um<P, 32, false>(p, s);
    default: return launch_um<P, 64, false>(p, s);
  }
}

}  // namespace

cudaError_t launch_m3_fwd_umma(const M3Params &p, cudaStream_t s) {
  switch (p.P) {
    case 16: return launch_um_n<16>(p, s);
    case 32: return launch_um_n<32>(p, s);
    default: return launch_um_n<64>(p, s);
  }
}

}  // namespace msc
