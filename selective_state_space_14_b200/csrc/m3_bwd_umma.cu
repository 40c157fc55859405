// m3_bwd_umma.cu -- Mamba-3 SISO scan, backward, bf16 io, chunk-parallel on
// the sm_100a tensor cores (tcgen05, accumulators in TMEM; umma.cuh).
//
// Backward stages B2 (output gating), B3 (BPTT through the trapezoidal state,
// with its per-head d_alpha, d_beta, d_gamma and the beta carry d_k_carry)
// and B4 (RoPE) of Mamba3Scratch, mamba-rs 0.4.2
// src/mamba3_siso/cpu/scratch.rs.  Chunk notation as in m3_common.cuh and
// m3_bwd.cu: chunks of Q steps, d(t,s) the decay products, c(t,s) the
// trapezoid weights, g_t = dout_t silu(z_t), U the state adjoint entering the
// chunk from the next one (its first step's alpha, beta written alpha_Q,
// beta_Q).  Every quantity of a chunk is a function of the chunk's own inputs,
// its starting state S_in (saved by the forward) and U, and U obeys a short
// linear recurrence over the chunks,
//   U_{ch-1} = V_ch + rho_ch U_ch,   V_ch = sum_tau d(tau,0) g_tau (outer) Ct_tau,
//   rho_ch = d(Q-1,0) alpha_Q,       U_{last} = 0,
// so the backward runs as four launches, the two heavy ones over all chunks
// of all (b, h) at once rather than one sequential walk per (b, h):
//   1. m3b_prep_kernel (one CTA per chunk): Ct Bt^T, Ct S_in^T and
//      (diag d(.,0) G)^T Ct on the tensor cores, then W X; y and dz; V_ch and
//      rho_ch to the workspace.
//   2. m3b_carry_kernel: the recurrence above, element by element of P x N,
//      chunks last to first, U_ch written over V_ch; dh0 = alpha_0 U_{-1}.
//   3. m3b_grad_kernel (one CTA per chunk): Ct Bt^T, G X^T, G S_in, X U in a
//      first round, then
//        dX  = W^T G + diag(wU) Bt U^T     (wU_t = alpha_Q c(Q-1,t) + [t = Q-1] beta_Q)
//        dBt = Z^T Ct + diag(wU) X U       (Z = c o G X^T)
//        dCt = Z Bt + diag(d(.,-1)) G S_in + beta_0 diag(d(.,0)) (G x_prev) Bt_prev^T
//      in a second; dalpha, dbeta, dgamma from the first round's products
//      (sums in which every term carries its factor, see m3_bwd.cu); the
//      RoPE backward, per-head dB and dC to the workspace, dphi summed in
//      reverse within the chunk, the chunk's dphi total to the workspace.
//   4. m3b_theta_carry_kernel and m3b_finish_kernel: the dtheta carries from
//      later chunks, the heads of a group added into dB and dC in ascending
//      head order, dD in ascending (b, chunk) order.
// f32 operands enter the tensor cores as three bf16 parts v = v0 + v1 + v2
// (each part the bf16 rounding of what the previous ones leave, about 24
// significant bits); a product adds the six part products whose order is above
// 2^-24 (a0 b0, a0 b1, a1 b0, a0 b2, a1 b1, a2 b0), smallest first, so it
// carries f32 accuracy, as the forward's do.  Two parts (16 bits) are not
// enough: dtheta is a sum over the whole sequence of a cancelling cross
// product of dBt with Bt, and at 2048 steps two-part products left its small
// entries 2 % off.  The bf16 inputs x go as one exact part.  Every sum has a fixed order: the
// results are the same bits on every run.
#include "m3_common.cuh"
#include "umma.cuh"

namespace msc {

// Workspace of the Mamba-3 backward (both implementations); byte offsets.
M3BwdWs m3_bwd_ws_layout(int64_t B, int64_t L, int64_t H, int64_t P, int64_t N, int64_t K) {
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  const int64_t nc = (L + MSC_M3_CHUNK_STEPS - 1) / MSC_M3_CHUNK_STEPS;
  M3BwdWs w;
  w.dB = 0;
  w.dC = w.dB + up(sizeof(float) * (size_t)(B * L * H * N));
  w.dD = w.dC + up(sizeof(float) * (size_t)(B * L * H * N));
  w.vu = w.dD + up(sizeof(float) * (size_t)(B * H * nc));
  w.rho = w.vu + up(sizeof(float) * (size_t)(B * H * nc * P * N));
  w.th = w.rho + up(sizeof(float) * (size_t)(B * H * nc));
  w.tok_y = w.th + up(sizeof(float) * (size_t)(B * H * nc * (K > 0 ? K : 1)));
  const size_t tok = N > kM3Slab ? up(sizeof(float) * (size_t)(B * L * H * P)) : 0;
  w.tok_dx = w.tok_y + tok;
  w.total = w.tok_dx + tok;
  return w;
}

namespace {

using namespace m3;
using umma::koff;

constexpr int kPl = 64 * 64 * 2;  // bytes of one bf16 part of a 64 x 64 tile
constexpr int kParts = 3;         // bf16 parts of an f32 operand
constexpr int kMat = kParts * kPl;  // bytes of the planes of one f32 operand

// ---------------------------------------------------------------------------
// kParts-part operand stores (core-matrix layout of umma.cuh)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t bits2(__nv_bfloat162 v) {
  return *reinterpret_cast<const uint32_t *>(&v);
}
// the kParts parts of (v0, v1) at byte offset off of the planes at base
// (plane stride kPl): one 4-byte store per part
__device__ __forceinline__ void put2x2(unsigned char *base, int off, float v0, float v1) {
#pragma unroll
  for (int q = 0; q < kParts; ++q) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
    const float2 hf = __bfloat1622float2(h);
    *reinterpret_cast<uint32_t *>(base + q * kPl + off) = bits2(h);
    v0 -= hf.x;
    v1 -= hf.y;
  }
}
// eight consecutive K elements of one row (16 bytes per part)
__device__ __forceinline__ void put8x2(unsigned char *base, int off, const float (&v8)[8]) {
  float v[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = v8[e];
#pragma unroll
  for (int q = 0; q < kParts; ++q) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
      const float2 hf = __bfloat1622float2(h);
      w[j] = bits2(h);
      v[2 * j] -= hf.x;
      v[2 * j + 1] -= hf.y;
    }
    *reinterpret_cast<uint4 *>(base + q * kPl + off) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}
// the value the parts at off represent (pairs: off 4-byte aligned), the
// smallest part first
__device__ __forceinline__ float2 get2x2(const unsigned char *base, int off) {
  float2 r = make_float2(0.f, 0.f);
#pragma unroll
  for (int q = kParts - 1; q >= 0; --q) {
    float a0, a1;
    unpack_bf16x2(*reinterpret_cast<const uint32_t *>(base + q * kPl + off), a0, a1);
    r.x += a0;
    r.y += a1;
  }
  return r;
}

// One product into the TMEM accumulator at column `col`: A (nA parts, 64
// rows; K-major with row length Ka, or kAMN: a tile stored [K][M] K-major read
// MN-major, Ka its row length) times B (nB parts; K-major with rows the N
// dimension and row length Kb, or kBMN: a tile stored [K][N] read MN-major, Kb
// its row length), K / 16 steps.  An MN-major operand whose stored rows are
// shorter than the MMA's extent (A with P < 64 rows) reads bytes of the same
// tile for the rows beyond, which land in accumulator rows nobody reads.  The
// part pairs whose order is above 2^-24 (pa + pb < kParts), smallest first;
// the first MMA overwrites unless acc.
template <int NMMA, bool kBMN, bool kAMN = false>
__device__ __forceinline__ void product(uint32_t tmem, int col, uint32_t aA, int nA, int Ka,
                                        uint32_t aB, int nB, int Kb, int K, bool acc) {
  const uint32_t id = umma::idesc_bf16<NMMA, kBMN, kAMN>();
  const int pa[6] = {2, 1, 0, 1, 0, 0}, pb[6] = {0, 1, 2, 0, 1, 0};
  bool first = !acc;
  for (int u = 0; u < 6; ++u) {
    if (pa[u] >= nA || pb[u] >= nB || pa[u] + pb[u] >= kParts) continue;
    for (int ks = 0; ks < K / 16; ++ks) {
      const uint64_t da = kAMN ? umma::desc(aA + pa[u] * kPl + ks * 2 * (Ka * 16), Ka * 16, 128)
                               : umma::desc(aA + pa[u] * kPl + ks * 256, 128, Ka * 16);
      const uint64_t db = kBMN ? umma::desc(aB + pb[u] * kPl + ks * 2 * (Kb * 16), Kb * 16, 128)
                               : umma::desc(aB + pb[u] * kPl + ks * 256, 128, Kb * 16);
      umma::mma(tmem + col, da, db, id, !first);
      first = false;
    }
  }
}

// The staging unit u of a 64-row tile with kR runs of 8 elements per row:
// the eight rows of a core matrix go to eight consecutive lanes (their 16-byte
// pieces fill all 32 banks), and a warp's 32 lanes take four runs of those
// rows (contiguous bytes of each row in global memory).
template <int kR>
__device__ __forceinline__ void row_run(int u, int &row, int &run) {
  const int rest = u >> 3;
  run = rest % kR;
  row = (rest / kR) * 8 + (u & 7);
}

// TMEM load of an accumulator W columns wide: this thread's rows ra, rb of
// its lane quarter, columns cb * W/2 + 8 i + 2 rq + {0, 1}, i < W / 16
template <int W>
__device__ __forceinline__ void tld(uint32_t taddr, float *v) {
  umma::tmem_ld16<W / 16>(taddr, v);
}

// ---------------------------------------------------------------------------
// shared memory
// ---------------------------------------------------------------------------
// f32 vectors of one chunk (floats)
struct Vec {
  static constexpr int al = 0, be = 65, ga = 130, eps = 195, d1 = 260, d0 = 325, crow = 390,
                       wu = 455, cbp = 520, gxp = 585, a = 650, v = 715, dg = 780, db = 845,
                       bx = 910, da = 975, xprev = 1040, bprev = 1104, phist = 1168,
                       part = 1200 /* [2][64] partial row sums */, red = 1328 /* [3][8] */,
                       rowb = 1352 /* [8][64] per-run parts of Ct.Bt_prev */,
                       rowx = 1864 /* [8][64] per-run parts of g.x_prev */, total = 2376;
};

// Row stride (floats) of the angle table tPhi [t][k]: padded so that the
// threads of a warp that hold steps 2 lane, 2 lane + 1 (the angle scans) or
// eight consecutive steps (the rotations) fall on different banks.
constexpr int kPhS = 33;

struct PrepSmem {
  static constexpr int pC = 0, pB = pC + kMat, pS = pB + kMat, pGd = pS + kMat,
                       pW = pGd + kMat, pX = pW + kMat;
  static constexpr int tD = pX + kPl;                // f32 [64][65]: d(t,-1), d(t,0..63)
  static constexpr int tPhi = tD + 64 * 65 * 4;      // f32 [64][kPhS] cumulative angles
  static constexpr int vec = tPhi + 64 * kPhS * 4;   // Vec
  static constexpr int misc = vec + Vec::total * 4;  // tmem slot, mbarrier, error flag
  static constexpr int total = misc + 32;
};

struct GradSmem {
  static constexpr int pC = 0, pB = pC + kMat, pG = pB + kMat, pX = pG + kMat,
                       pS = pX + kPl /* S_in, then W */, pU = pS + kMat, pZ = pU + kMat;
  static constexpr int tD = pZ + kMat;                // f32 [64][65]
  static constexpr int tM = tD + 64 * 65 * 4;         // f32 [64][65]: (Ct.Bt)(g.x)
  static constexpr int tPhi = tM + 64 * 65 * 4;       // f32 [64][kPhS] angles, then dphi
  static constexpr int vec = tPhi + 64 * kPhS * 4;
  static constexpr int misc = vec + Vec::total * 4;
  static constexpr int total = misc + 32;
  static_assert(total <= 232448, "one CTA's shared memory");
};

// ---------------------------------------------------------------------------
// staging shared by both chunk kernels
// ---------------------------------------------------------------------------
struct Chunk {
  int64_t b, h, g, ch, t0, nc;
  int Qc;          // valid steps of the chunk
  int64_t ldN, n0;  // full d_state and this slab's first state
  int Kt, k0, K;   // angle pairs: total, this slab's first, this slab's count
};

// unit u of the persistent loop: chunk u % nc of head (u / nc) % H of batch
// row u / (nc H)
__device__ __forceinline__ Chunk chunk_of(const M3Params &p, int P, int64_t u) {
  Chunk c;
  const int64_t nc = (p.L + kQ - 1) / kQ;
  c.ch = u % nc;
  c.h = (u / nc) % p.H;
  c.b = u / (nc * p.H);
  c.g = c.h / (p.H / p.G);
  c.t0 = c.ch * kQ;
  c.nc = (p.L + kQ - 1) / kQ;
  c.Qc = (int)((p.L - c.t0) < kQ ? (p.L - c.t0) : kQ);
  c.ldN = p.ldN;
  c.n0 = p.n0;
  c.Kt = (int)p.K;
  c.k0 = (int)(p.n0 / 2);
  const int kmax = (int)(p.N / 2);
  c.K = c.Kt - c.k0 < 0 ? 0 : (c.Kt - c.k0 > kmax ? kmax : c.Kt - c.k0);
  (void)P;
  return c;
}

// Every global load of a chunk, issued by each thread before any of them is
// used, so that a thread keeps all of its loads in flight at once (with one
// CTA per SM, loads issued phase by phase would leave the SM waiting on each
// phase's latency in turn).  Units of 8 elements follow row_run: B and C rows
// (Q x N), x, dout and z rows (Q x P), the state rows S_in and U (P x N; the
// rows are counted to 64 and those past P skipped).
template <int P, int N, bool kU>
struct Loads {
  static constexpr int kBC = (kQ * (N / 8) + kThreads - 1) / kThreads;
  static constexpr int kXG = (kQ * (P / 8) + kThreads - 1) / kThreads;
  static constexpr int kST = (64 * (N / 8) + kThreads - 1) / kThreads;
  static constexpr int kTH = kQ * 32 / kThreads;  // theta elements per thread
  uint4 bb[kBC], cc[kBC], xx[kXG], dd[kXG], zz[kXG];
  float4 s0[kST], s1[kST], u0[kST], u1[kST];
  bf16 th[kTH];
  bf16 al, be, ga, prev;
  float phist;

  __device__ __forceinline__ void issue(const M3Params &p, const Chunk &c, const float *sin,
                                        const float *usrc) {
    const int tid = threadIdx.x;
    const uint4 zero4 = make_uint4(0, 0, 0, 0);
    const bf16 *Bm = static_cast<const bf16 *>(p.Bm), *Cm = static_cast<const bf16 *>(p.Cm);
    const bf16 *x = static_cast<const bf16 *>(p.x), *dout = static_cast<const bf16 *>(p.dout),
               *z = static_cast<const bf16 *>(p.z);
#pragma unroll
    for (int k = 0; k < kBC; ++k) {
      const int u = tid + k * kThreads;
      int t, r;
      row_run<N / 8>(u, t, r);
      bb[k] = cc[k] = zero4;
      if (u < kQ * (N / 8) && t < c.Qc) {
        const int64_t j = ((c.b * p.L + c.t0 + t) * p.G + c.g) * c.ldN + c.n0 + r * 8;
        bb[k] = __ldg(reinterpret_cast<const uint4 *>(Bm + j));
        cc[k] = __ldg(reinterpret_cast<const uint4 *>(Cm + j));
      }
    }
#pragma unroll
    for (int k = 0; k < kXG; ++k) {
      const int u = tid + k * kThreads;
      int t, r;
      row_run<P / 8>(u, t, r);
      xx[k] = dd[k] = zz[k] = zero4;
      if (u < kQ * (P / 8) && t < c.Qc) {
        const int64_t j = ((c.b * p.L + c.t0 + t) * p.H + c.h) * P + r * 8;
        xx[k] = __ldg(reinterpret_cast<const uint4 *>(x + j));
        dd[k] = __ldg(reinterpret_cast<const uint4 *>(dout + j));
        if (z) zz[k] = __ldg(reinterpret_cast<const uint4 *>(z + j));
      }
    }
#pragma unroll
    for (int k = 0; k < kST; ++k) {
      const int u = tid + k * kThreads;
      int pp, r;
      row_run<N / 8>(u, pp, r);
      if (u < 64 * (N / 8) && pp < P) {
        s0[k] = __ldg(reinterpret_cast<const float4 *>(sin + pp * c.ldN + r * 8));
        s1[k] = __ldg(reinterpret_cast<const float4 *>(sin + pp * c.ldN + r * 8 + 4));
        if (kU) {
          u0[k] = __ldg(reinterpret_cast<const float4 *>(usrc + pp * c.ldN + r * 8));
          u1[k] = __ldg(reinterpret_cast<const float4 *>(usrc + pp * c.ldN + r * 8 + 4));
        }
      }
    }
    const bf16 *thp = static_cast<const bf16 *>(p.theta);
#pragma unroll
    for (int q = 0; q < kTH; ++q) {
      const int i = tid + q * kThreads, t = i >> 5, k = i & 31;
      th[q] = (k < c.K && t < c.Qc)
                  ? thp[((c.b * p.L + c.t0 + t) * p.H + c.h) * c.Kt + c.k0 + k]
                  : __float2bfloat16_rn(0.f);
    }
    const bf16 one = __float2bfloat16_rn(1.f), nil = __float2bfloat16_rn(0.f);
    al = one;
    be = ga = nil;
    if (tid <= kQ) {
      const int64_t tg = c.t0 + tid;
      const bool in = tid < kQ ? tid < c.Qc : tg < p.L;  // row Q: the next chunk's first step
      const int64_t j = (c.b * p.L + tg) * p.H + c.h;
      if (in) {
        al = static_cast<const bf16 *>(p.alpha)[j];
        be = static_cast<const bf16 *>(p.beta)[j];
        if (tid < kQ) ga = static_cast<const bf16 *>(p.gamma)[j];
      }
    }
    phist = 0.f;
    if (tid < c.K) {
      const float *ps = p.saved_in + p.B * p.H * c.nc * P * c.ldN +
                        (c.b * p.H + c.h) * c.nc * (c.ldN / 2);
      phist = ps[c.ch * (c.ldN / 2) + c.k0 + tid];
    }
    prev = nil;
    if (c.t0 > 0 && tid < P + N) {
      prev = tid < P ? x[((c.b * p.L + c.t0 - 1) * p.H + c.h) * P + tid]
                     : Bm[((c.b * p.L + c.t0 - 1) * p.G + c.g) * c.ldN + c.n0 + tid - P];
    }
  }
};

// Phase 1 (from the loads): alpha, beta, gamma (and the next chunk's alpha,
// beta), theta into the angle table, the chunk-start angles, x_prev and B_prev
// (raw).
template <class LD>
__device__ __forceinline__ void stage_small(const LD &ld, float *sv, float *tPhi, int P, int N) {
  const int tid = threadIdx.x;
  if (tid <= kQ) {
    sv[Vec::al + tid] = __bfloat162float(ld.al);
    sv[Vec::be + tid] = __bfloat162float(ld.be);
    if (tid < kQ) sv[Vec::ga + tid] = __bfloat162float(ld.ga);
  }
#pragma unroll
  for (int q = 0; q < LD::kTH; ++q) {
    const int i = tid + q * kThreads;
    tPhi[(i >> 5) * kPhS + (i & 31)] = __bfloat162float(ld.th[q]);
  }
  if (tid < 32) sv[Vec::phist + tid] = ld.phist;
  if (tid < P) sv[Vec::xprev + tid] = __bfloat162float(ld.prev);
  else if (tid < P + N) sv[Vec::bprev + tid - P] = __bfloat162float(ld.prev);
}

// Phase 2: cumulative angles (per angle pair a warp scan over the chunk,
// lane l holding steps 2l and 2l + 1), B_prev rotated by the chunk-start
// angles, the decay table d(t, s) = prod_{r=s+1..t} alpha_r (column s + 1;
// column 0: d(t, -1); zero above the diagonal; per column a product scan in
// the same layout), and the per-step coefficients.
__device__ __forceinline__ void stage_decays(const Chunk &c, float *sv, float *tPhi, float *tD) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = 2 * lane, t1 = t0 + 1;
  for (int k = warp; k < c.K; k += kThreads / 32) {
    const float a0 = tPhi[t0 * kPhS + k], a1 = tPhi[t1 * kPhS + k];
    float incl = a0 + a1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    float excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = 0.f;
    const float st = sv[Vec::phist + k];
    tPhi[t0 * kPhS + k] = st + (excl + a0);
    tPhi[t1 * kPhS + k] = st + incl;
  }
  if (tid < c.K) {
    float sn, cs;
    sincos_reduced(sv[Vec::phist + tid], sn, cs);
    const float b0 = sv[Vec::bprev + 2 * tid], b1 = sv[Vec::bprev + 2 * tid + 1];
    sv[Vec::bprev + 2 * tid] = cs * b0 - sn * b1;
    sv[Vec::bprev + 2 * tid + 1] = sn * b0 + cs * b1;
  }
  for (int col = warp; col <= kQ; col += kThreads / 32) {
    const int s = col - 1;  // column col holds d(., s)
    const float f0 = t0 > s ? sv[Vec::al + t0] : 1.f, f1 = t1 > s ? sv[Vec::al + t1] : 1.f;
    float incl = f0 * f1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl *= u;
    }
    float excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = 1.f;
    tD[t0 * 65 + col] = t0 >= s ? excl * f0 : 0.f;
    tD[t1 * 65 + col] = t1 >= s ? excl * f0 * f1 : 0.f;
  }
  __syncthreads();
  if (tid < kQ) {
    const int t = tid;
    sv[Vec::d1 + t] = tD[t * 65];
    sv[Vec::d0 + t] = tD[t * 65 + 1];
    // eps_t = alpha_{t+1} gamma_t + beta_{t+1} (alpha_Q, beta_Q: the next chunk's)
    sv[Vec::eps + t] = fmaf(sv[Vec::al + t + 1], sv[Vec::ga + t], sv[Vec::be + t + 1]);
  }
  __syncthreads();
  if (tid < kQ) {
    const int t = tid;
    // c(Q-1, t) and wU_t = alpha_Q c(Q-1, t) + [t = Q-1] beta_Q
    const float cr = t == kQ - 1 ? sv[Vec::ga + t] : tD[(kQ - 1) * 65 + t + 2] * sv[Vec::eps + t];
    sv[Vec::crow + t] = cr;
    sv[Vec::wu + t] = fmaf(sv[Vec::al + kQ], cr, t == kQ - 1 ? sv[Vec::be + kQ] : 0.f);
  }
}

// c(t, s) from the decay table and the per-step coefficients
__device__ __forceinline__ float cw(const float *tD, const float *sv, int t, int s) {
  return s == t ? sv[Vec::ga + t] : (s < t ? tD[t * 65 + s + 2] * sv[Vec::eps + s] : 0.f);
}

// Phase 3 (after phase 2): the rotated B and C rows of the chunk into the
// operand planes; the per-run parts of Ct_t . Bt_prev into rowb (added in run
// order by row_sums).  A unit is 8 consecutive states of one step.
template <int N, class LD>
__device__ __forceinline__ void stage_bc(const LD &ld, const Chunk &c, float *sv,
                                         const float *tPhi, unsigned char *pB, unsigned char *pC) {
  constexpr int kR = N / 8;  // runs per row
#pragma unroll
  for (int k = 0; k < LD::kBC; ++k) {
    const int u = threadIdx.x + k * kThreads;
    if (u >= kQ * kR) break;
    int t, r;
    row_run<kR>(u, t, r);
    float bv[8], cv[8];
    unpack_bf16x2(ld.bb[k].x, bv[0], bv[1]); unpack_bf16x2(ld.bb[k].y, bv[2], bv[3]);
    unpack_bf16x2(ld.bb[k].z, bv[4], bv[5]); unpack_bf16x2(ld.bb[k].w, bv[6], bv[7]);
    unpack_bf16x2(ld.cc[k].x, cv[0], cv[1]); unpack_bf16x2(ld.cc[k].y, cv[2], cv[3]);
    unpack_bf16x2(ld.cc[k].z, cv[4], cv[5]); unpack_bf16x2(ld.cc[k].w, cv[6], cv[7]);
    float dot = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int kk = r * 4 + q;
      if (kk < c.K) {
        float sn, cs;
        sincos_reduced(tPhi[t * kPhS + kk], sn, cs);
        const float b0 = bv[2 * q], b1 = bv[2 * q + 1], c0 = cv[2 * q], c1 = cv[2 * q + 1];
        bv[2 * q] = cs * b0 - sn * b1;
        bv[2 * q + 1] = sn * b0 + cs * b1;
        cv[2 * q] = cs * c0 - sn * c1;
        cv[2 * q + 1] = sn * c0 + cs * c1;
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) dot = fmaf(cv[e], sv[Vec::bprev + r * 8 + e], dot);
    const int off = koff(t, r * 8, N);
    put8x2(pB, off, bv);
    put8x2(pC, off, cv);
    sv[Vec::rowb + r * 64 + t] = dot;
  }
}

// Phase 3: x, dout, z of the chunk: g = dout silu(z) into planes pG ([t][p],
// when given) and d(t, 0) g into pGd ([t][p], when given); x into pX (one
// exact part); the per-run parts of g . x_prev into rowx; the thread's sum of
// g x.
template <int P, class LD>
__device__ __forceinline__ float stage_xg(const LD &ld, bool has_z, float *sv, unsigned char *pX,
                                          unsigned char *pG, unsigned char *pGd) {
  constexpr int kR = P / 8;
  float gx_sum = 0.f;
#pragma unroll
  for (int k = 0; k < LD::kXG; ++k) {
    const int u = threadIdx.x + k * kThreads;
    if (u >= kQ * kR) break;
    int t, r;
    row_run<kR>(u, t, r);
    float xv[8], gv[8], dv[8];
    unpack_bf16x2(ld.dd[k].x, dv[0], dv[1]); unpack_bf16x2(ld.dd[k].y, dv[2], dv[3]);
    unpack_bf16x2(ld.dd[k].z, dv[4], dv[5]); unpack_bf16x2(ld.dd[k].w, dv[6], dv[7]);
    if (has_z) {
      float zv[8];
      unpack_bf16x2(ld.zz[k].x, zv[0], zv[1]); unpack_bf16x2(ld.zz[k].y, zv[2], zv[3]);
      unpack_bf16x2(ld.zz[k].z, zv[4], zv[5]); unpack_bf16x2(ld.zz[k].w, zv[6], zv[7]);
#pragma unroll
      for (int e = 0; e < 8; ++e) gv[e] = dv[e] * silu(zv[e]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) gv[e] = dv[e];
    }
    unpack_bf16x2(ld.xx[k].x, xv[0], xv[1]); unpack_bf16x2(ld.xx[k].y, xv[2], xv[3]);
    unpack_bf16x2(ld.xx[k].z, xv[4], xv[5]); unpack_bf16x2(ld.xx[k].w, xv[6], xv[7]);
    const int off = koff(t, r * 8, P);
    *reinterpret_cast<uint4 *>(pX + off) = ld.xx[k];
    if (pG) put8x2(pG, off, gv);
    if (pGd) {
      const float d0 = sv[Vec::d0 + t];
      float gd[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) gd[e] = d0 * gv[e];
      put8x2(pGd, off, gd);
    }
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      dot = fmaf(gv[e], sv[Vec::xprev + r * 8 + e], dot);
      gx_sum = fmaf(gv[e], xv[e], gx_sum);
    }
    sv[Vec::rowx + r * 64 + t] = dot;
  }
  return gx_sum;
}

// After phase 3 (and a barrier): cbp_t and gxp_t, the runs added in order.
template <int P, int N>
__device__ __forceinline__ void row_sums(float *sv) {
  const int t = threadIdx.x;
  if (t < kQ) {
    float a = 0.f, b = 0.f;
#pragma unroll
    for (int r = 0; r < N / 8; ++r) a += sv[Vec::rowb + r * 64 + t];
#pragma unroll
    for (int r = 0; r < P / 8; ++r) b += sv[Vec::rowx + r * 64 + t];
    sv[Vec::cbp + t] = a;
    sv[Vec::gxp + t] = b;
  }
}

// Phase 3: the state tile S_in (and U, with kU) into planes [p][n]; with U,
// the sums <U, S_in> and x_prev^T U Bt_prev of the thread's elements are
// added to us and vm1.
template <int P, int N, bool kU, class LD>
__device__ __forceinline__ void stage_state(const LD &ld, unsigned char *pl, unsigned char *pu,
                                            const float *sv, float &us, float &vm1) {
  constexpr int kR = N / 8;
#pragma unroll
  for (int k = 0; k < LD::kST; ++k) {
    const int u = threadIdx.x + k * kThreads;
    int pp, r;
    row_run<kR>(u, pp, r);
    if (u >= 64 * kR || pp >= P) continue;
    const float v[8] = {ld.s0[k].x, ld.s0[k].y, ld.s0[k].z, ld.s0[k].w,
                        ld.s1[k].x, ld.s1[k].y, ld.s1[k].z, ld.s1[k].w};
    put8x2(pl, koff(pp, r * 8, N), v);
    if (kU) {
      const float w[8] = {ld.u0[k].x, ld.u0[k].y, ld.u0[k].z, ld.u0[k].w,
                          ld.u1[k].x, ld.u1[k].y, ld.u1[k].z, ld.u1[k].w};
      put8x2(pu, koff(pp, r * 8, N), w);
      float ub = 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        us = fmaf(w[q], v[q], us);
        ub = fmaf(w[q], sv[Vec::bprev + r * 8 + q], ub);
      }
      vm1 = fmaf(sv[Vec::xprev + pp], ub, vm1);
    }
  }
}

// fixed-order sums over the CTA of three values (warp butterflies, then the
// warps in order); every thread gets the three sums
__device__ __forceinline__ float3 block_sum3(float3 v, float *red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    v.x += __shfl_xor_sync(0xffffffffu, v.x, o);
    v.y += __shfl_xor_sync(0xffffffffu, v.y, o);
    v.z += __shfl_xor_sync(0xffffffffu, v.z, o);
  }
  if ((threadIdx.x & 31) == 0) {
    red[threadIdx.x >> 5] = v.x;
    red[8 + (threadIdx.x >> 5)] = v.y;
    red[16 + (threadIdx.x >> 5)] = v.z;
  }
  __syncthreads();
  float3 s = make_float3(0.f, 0.f, 0.f);
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) {
    s.x += red[w];
    s.y += red[8 + w];
    s.z += red[16 + w];
  }
  return s;
}

// ---------------------------------------------------------------------------
// 1. preparation: y (for dz), V_ch, rho_ch
// ---------------------------------------------------------------------------
template <int P, int N>
__global__ void __launch_bounds__(kThreads, 1) m3b_prep_kernel(const M3Params p, float *vu,
                                                               float *rho) {
  using S = PrepSmem;
  extern __shared__ __align__(1024) unsigned char sm[];
  float *sv = reinterpret_cast<float *>(sm + S::vec);
  float *tD = reinterpret_cast<float *>(sm + S::tD);
  float *tPhi = reinterpret_cast<float *>(sm + S::tPhi);
  uint32_t *sTmem = reinterpret_cast<uint32_t *>(sm + S::misc);
  uint64_t *sMbar = reinterpret_cast<uint64_t *>(sm + S::misc + 8);
  int *sErr = reinterpret_cast<int *>(sm + S::misc + 16);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slab = p.slab;
  const bool finish = slab == kSlabWhole || slab == kSlabLast;
  const uint32_t base = umma::smem_addr(sm);
  const uint32_t mbar = umma::smem_addr(sMbar);
  const int64_t n_units = ((p.L + kQ - 1) / kQ) * p.H * p.B;

  if (warp == 0) umma::tmem_alloc(sTmem, 256);
  if (tid == 0) {
    umma::mbar_init(mbar);
    *sErr = 0;
  }
  auto sin_of = [&](const Chunk &c) {
    return p.saved_in + ((c.b * p.H + c.h) * c.nc + c.ch) * P * c.ldN + c.n0;
  };
  Loads<P, N, false> ld;
  if ((int64_t)blockIdx.x < n_units) {
    const Chunk c0 = chunk_of(p, P, blockIdx.x);
    ld.issue(p, c0, sin_of(c0), nullptr);
  }
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = *sTmem;
  for (int64_t unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
  const Chunk c = chunk_of(p, P, unit);
  const float Dh = (p.Dp && finish) ? p.Dp[c.h] : 0.f;
  stage_small(ld, sv, tPhi, P, N);
  __syncthreads();
  stage_decays(c, sv, tPhi, tD);
  __syncthreads();
  stage_bc<N>(ld, c, sv, tPhi, sm + S::pB, sm + S::pC);
  stage_xg<P>(ld, p.z != nullptr, sv, sm + S::pX, nullptr, sm + S::pGd);
  {
    float us = 0.f, vm1 = 0.f;
    stage_state<P, N, false>(ld, sm + S::pS, nullptr, sv, us, vm1);
  }
  if (unit + gridDim.x < n_units) {  // the next unit's loads fly while this one computes
    const Chunk cn = chunk_of(p, P, unit + gridDim.x);
    ld.issue(p, cn, sin_of(cn), nullptr);
  }
  umma::fence_async_smem();
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  if (tid == 0) {
    product<64, false>(tmem, 0, base + S::pC, kParts, N, base + S::pB, kParts, N, N, false);  // Ct Bt^T
    product<P, false>(tmem, 64, base + S::pC, kParts, N, base + S::pS, kParts, N, N, false);  // Ct S_in^T
    // V = (diag d(., 0) G)^T Ct: A read MN-major from [t][p]
    product<N, true, true>(tmem, 128, base + S::pGd, kParts, P, base + S::pC, kParts, N, 64, false);
    umma::commit(mbar);
  }
  row_sums<P, N>(sv);
  const int ri = lane >> 2, rq = lane & 3, q4 = warp & 3, cb = warp >> 2;
  const int ra = 16 * q4 + ri, rb = ra + 8, c2 = 2 * rq;
  const uint32_t tq = (uint32_t)(32 * q4) << 16;
  if (!umma::mbar_wait(mbar, 0)) *sErr = 1;
  umma::fence_after();
  // ---- W = c o Ct Bt^T; V to the workspace ------------------------------------
  {
    float v[16];
    tld<64>(tmem + tq + cb * 32, v);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int t = e ? rb : ra;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int s = cb * 32 + 8 * i + c2;
        put2x2(sm + S::pW, koff(t, s, 64), cw(tD, sv, t, s) * v[4 * i + 2 * e],
               cw(tD, sv, t, s + 1) * v[4 * i + 2 * e + 1]);
      }
    }
    float vv[N / 4];
    tld<N>(tmem + tq + 128 + cb * (N / 2), vv);
    float *dst = vu + ((c.b * p.H + c.h) * c.nc + c.ch) * P * c.ldN + c.n0;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int pp = e ? rb : ra;
      if (pp < P) {
#pragma unroll
        for (int i = 0; i < N / 16; ++i)
          *reinterpret_cast<float2 *>(dst + pp * c.ldN + cb * (N / 2) + 8 * i + c2) =
              make_float2(vv[4 * i + 2 * e], vv[4 * i + 2 * e + 1]);
      }
    }
    if (tid == 0) rho[(c.b * p.H + c.h) * c.nc + c.ch] = tD[(kQ - 1) * 65 + 1] * sv[Vec::al + kQ];
  }
  umma::fence_async_smem();
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  if (tid == 0) {
    product<P, true>(tmem, 192, base + S::pW, kParts, 64, base + S::pX, 1, P, 64, false);  // W X
    umma::commit(mbar);
  }
  if (!umma::mbar_wait(mbar, 1)) *sErr = 1;
  umma::fence_after();
  // ---- y and dz ----------------------------------------------------------------------
  {
    float y1[P / 4], y2[P / 4];
    umma::tmem_ld16_pair<P / 16>(tmem + tq + 192 + cb * (P / 2), tmem + tq + 64 + cb * (P / 2), y1, y2);
    const bf16 *dout = static_cast<const bf16 *>(p.dout), *z = static_cast<const bf16 *>(p.z);
    const bool failed = *sErr != 0;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int t = e ? rb : ra;
      if (t >= c.Qc) continue;
      const float dl = sv[Vec::d1 + t];
      const float wc = sv[Vec::be] * sv[Vec::d0 + t] * sv[Vec::cbp + t];
#pragma unroll
      for (int i = 0; i < P / 16; ++i) {
        const int p0 = cb * (P / 2) + 8 * i + c2;
        float xf0, xf1;
        unpack_bf16x2(*reinterpret_cast<const uint32_t *>(sm + S::pX + koff(t, p0, P)), xf0, xf1);
        float o0 = fmaf(dl, y2[4 * i + 2 * e], y1[4 * i + 2 * e]) + wc * sv[Vec::xprev + p0] + Dh * xf0;
        float o1 = fmaf(dl, y2[4 * i + 2 * e + 1], y1[4 * i + 2 * e + 1]) + wc * sv[Vec::xprev + p0 + 1] + Dh * xf1;
        const int64_t j = ((c.b * p.L + c.t0 + t) * p.H + c.h) * P + p0;
        if (slab != kSlabWhole) {  // y sums over the states: across the slabs
          float2 *ty = reinterpret_cast<float2 *>(p.tok_y + j);
          if (slab != kSlabFirst) {
            const float2 pr = *ty;
            o0 = pr.x + o0;
            o1 = pr.y + o1;
          }
          if (!finish) {
            *ty = make_float2(o0, o1);
            continue;
          }
        }
        if (p.dz) {
          float d0, d1, z0, z1;
          unpack_bf16x2(*reinterpret_cast<const uint32_t *>(dout + j), d0, d1);
          unpack_bf16x2(*reinterpret_cast<const uint32_t *>(z + j), z0, z1);
          float r0 = o0 * d0 * dsilu(z0), r1 = o1 * d1 * dsilu(z1);
          if (failed) r0 = r1 = __int_as_float(0x7fc00000);
          *reinterpret_cast<uint32_t *>(static_cast<bf16 *>(p.dz) + j) = pack_bf16x2(r0, r1);
        }
      }
    }
  }
  umma::fence_before();
  __syncthreads();  // this unit's TMEM reads and shared-memory uses are done
  umma::fence_after();
  if (*sErr) break;  // a tensor-core round never completed: stop (outputs are NaN)
  }
  umma::fence_before();
  __syncthreads();
  if (warp == 0) {
    umma::fence_after();
    umma::tmem_dealloc(tmem, 256);
  }
}

// ---------------------------------------------------------------------------
// 2. the adjoint carried across the chunks
// ---------------------------------------------------------------------------
// Element e of P x N of (b, h): U = 0, then for ch from last to first
// U_ch = U and U <- V_ch + rho_ch U.  The loads of a batch of kB chunks are
// issued before any of its stores, so that each thread keeps kB loads in
// flight instead of one.
__global__ void __launch_bounds__(256) m3b_carry_kernel(const M3Params p, float *__restrict__ vu,
                                                        const float *__restrict__ rho) {
  constexpr int kB = 8;
  const int64_t PN = p.P * p.ldN;
  const int64_t nc = (p.L + kQ - 1) / kQ;
  const int64_t n = (int64_t)p.B * p.H * PN;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t bh = i / PN, e = i % PN;
    float *col = vu + bh * nc * PN + e;
    const float *r = rho + bh * nc;
    float U = 0.f;
    for (int64_t top = nc - 1; top >= 0; top -= kB) {
      float v[kB], rr[kB];
#pragma unroll
      for (int k = 0; k < kB; ++k) {
        const int64_t ch = top - k;
        v[k] = ch >= 0 ? __ldcs(col + ch * PN) : 0.f;
        rr[k] = ch >= 0 ? r[ch] : 0.f;
      }
#pragma unroll
      for (int k = 0; k < kB; ++k) {
        const int64_t ch = top - k;
        if (ch >= 0) {
          __stcs(col + ch * PN, U);  // the adjoint chunk ch receives from chunk ch + 1
          U = fmaf(rr[k], U, v[k]);
        }
      }
    }
    if (p.dh0) {
      const int64_t b = bh / p.H, h = bh % p.H;
      const float a0 = __bfloat162float(static_cast<const bf16 *>(p.alpha)[(b * p.L) * p.H + h]);
      p.dh0[bh * PN + e] = a0 * U;  // alpha_0 Lambda_0
    }
  }
}

// ---------------------------------------------------------------------------
// 3. the gradients of a chunk
// ---------------------------------------------------------------------------
template <int P, int N>
__global__ void __launch_bounds__(kThreads, 1) m3b_grad_kernel(const M3Params p, const float *vu,
                                                               float *ws_dB, float *ws_dC,
                                                               float *ws_dD, float *ws_th) {
  using S = GradSmem;
  extern __shared__ __align__(1024) unsigned char sm[];
  float *sv = reinterpret_cast<float *>(sm + S::vec);
  float *tD = reinterpret_cast<float *>(sm + S::tD);
  float *tM = reinterpret_cast<float *>(sm + S::tM);
  float *tPhi = reinterpret_cast<float *>(sm + S::tPhi);
  uint32_t *sTmem = reinterpret_cast<uint32_t *>(sm + S::misc);
  uint64_t *sMbar = reinterpret_cast<uint64_t *>(sm + S::misc + 8);
  int *sErr = reinterpret_cast<int *>(sm + S::misc + 16);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slab = p.slab;
  const bool finish = slab == kSlabWhole || slab == kSlabLast;
  const uint32_t base = umma::smem_addr(sm);
  const uint32_t mbar = umma::smem_addr(sMbar);
  const int64_t n_units = ((p.L + kQ - 1) / kQ) * p.H * p.B;

  if (warp == 0) umma::tmem_alloc(sTmem, 512);
  if (tid == 0) {
    umma::mbar_init(mbar);
    *sErr = 0;
  }
  auto off_of = [&](const Chunk &c) { return ((c.b * p.H + c.h) * c.nc + c.ch) * P * c.ldN + c.n0; };
  Loads<P, N, true> ld;
  if ((int64_t)blockIdx.x < n_units) {
    const Chunk c0 = chunk_of(p, P, blockIdx.x);
    ld.issue(p, c0, p.saved_in + off_of(c0), vu + off_of(c0));
  }
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = *sTmem;
  for (int64_t unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
  const Chunk c = chunk_of(p, P, unit);
  const float Dh = (p.Dp && finish) ? p.Dp[c.h] : 0.f;
  stage_small(ld, sv, tPhi, P, N);
  __syncthreads();
  stage_decays(c, sv, tPhi, tD);
  __syncthreads();
  stage_bc<N>(ld, c, sv, tPhi, sm + S::pB, sm + S::pC);
  const float gx_l = stage_xg<P>(ld, p.z != nullptr, sv, sm + S::pX, sm + S::pG, nullptr);
  float us_l = 0.f, vm1_l = 0.f;
  stage_state<P, N, true>(ld, sm + S::pS, sm + S::pU, sv, us_l, vm1_l);
  if (unit + gridDim.x < n_units) {  // the next unit's loads fly while this one computes
    const Chunk cn = chunk_of(p, P, unit + gridDim.x);
    ld.issue(p, cn, p.saved_in + off_of(cn), vu + off_of(cn));
  }
  umma::fence_async_smem();
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  if (tid == 0) {
    product<64, false>(tmem, 0, base + S::pC, kParts, N, base + S::pB, kParts, N, N, false);   // Ct Bt^T
    product<64, false>(tmem, 64, base + S::pG, kParts, P, base + S::pX, 1, P, P, false);       // G X^T
    product<N, true>(tmem, 128, base + S::pG, kParts, P, base + S::pS, kParts, N, P, false);   // G S_in
    product<N, true>(tmem, 192, base + S::pX, 1, P, base + S::pU, kParts, N, P, false);        // X U
    umma::commit(mbar);
  }
  row_sums<P, N>(sv);
  // block sums while the tensor cores work (every thread takes part)
  const float3 sums = block_sum3(make_float3(us_l, vm1_l, gx_l), sv + Vec::red);
  const float us = sums.x, vm1 = sums.y, dD = sums.z;
  const int ri = lane >> 2, rq = lane & 3, q4 = warp & 3, cb = warp >> 2;
  const int ra = 16 * q4 + ri, rb = ra + 8, c2 = 2 * rq;
  const uint32_t tq = (uint32_t)(32 * q4) << 16;
  if (!umma::mbar_wait(mbar, 0)) *sErr = 1;
  umma::fence_after();
  // ---- W and Z = c o (Ct Bt^T, G X^T) into planes [t][s] (W over S_in's);
  // M = (Ct.Bt)(g.x) into the table; the row dots a_t = (G S_in)_t . Ct_t and
  // v_s = (X U)_s . Bt_s -------------------------------------------------------------
  {
    float cbv[16], gxv[16];
    umma::tmem_ld16_pair<4>(tmem + tq + cb * 32, tmem + tq + 64 + cb * 32, cbv, gxv);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int t = e ? rb : ra;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int s = cb * 32 + 8 * i + c2;
        const float c0 = cw(tD, sv, t, s), c1 = cw(tD, sv, t, s + 1);
        const float g0 = cbv[4 * i + 2 * e], g1 = cbv[4 * i + 2 * e + 1];
        const float x0 = gxv[4 * i + 2 * e], x1 = gxv[4 * i + 2 * e + 1];
        put2x2(sm + S::pS, koff(t, s, 64), c0 * g0, c1 * g1);
        put2x2(sm + S::pZ, koff(t, s, 64), c0 * x0, c1 * x1);
        tM[t * 65 + s] = s <= t ? g0 * x0 : 0.f;  // rows of 65 floats: 4-byte stores
        tM[t * 65 + s + 1] = s + 1 <= t ? g1 * x1 : 0.f;
      }
    }
    float gs[N / 4], xu[N / 4];
    umma::tmem_ld16_pair<N / 16>(tmem + tq + 128 + cb * (N / 2), tmem + tq + 192 + cb * (N / 2), gs, xu);
    float pa[2] = {0.f, 0.f}, pv[2] = {0.f, 0.f};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int t = e ? rb : ra;
#pragma unroll
      for (int i = 0; i < N / 16; ++i) {
        const int n = cb * (N / 2) + 8 * i + c2;
        const float2 cc = get2x2(sm + S::pC, koff(t, n, N)), bb = get2x2(sm + S::pB, koff(t, n, N));
        pa[e] = fmaf(gs[4 * i + 2 * e], cc.x, pa[e]);
        pa[e] = fmaf(gs[4 * i + 2 * e + 1], cc.y, pa[e]);
        pv[e] = fmaf(xu[4 * i + 2 * e], bb.x, pv[e]);
        pv[e] = fmaf(xu[4 * i + 2 * e + 1], bb.y, pv[e]);
      }
#pragma unroll
      for (int o = 1; o < 4; o <<= 1) {
        pa[e] += __shfl_xor_sync(0xffffffffu, pa[e], o);
        pv[e] += __shfl_xor_sync(0xffffffffu, pv[e], o);
      }
    }
    if (rq == 0) {  // [2][64] for a, then [2][64] for v in the row-part area
      sv[Vec::part + cb * 64 + ra] = pa[0];
      sv[Vec::part + cb * 64 + rb] = pa[1];
      sv[Vec::rowb + cb * 64 + ra] = pv[0];
      sv[Vec::rowb + cb * 64 + rb] = pv[1];
    }
  }
  umma::fence_async_smem();
  umma::fence_before();
  __syncthreads();  // operands of round 2 in place; the partial row dots written
  umma::fence_after();
  if (tid == 0) {
    // W^T G and Z^T Ct read W and Z MN-major
    product<P, true, true>(tmem, 256, base + S::pS, kParts, 64, base + S::pG, kParts, P, 64, false);
    product<P, false>(tmem, 448, base + S::pB, kParts, N, base + S::pU, kParts, N, N, false);   // Bt U^T
    product<N, true, true>(tmem, 320, base + S::pZ, kParts, 64, base + S::pC, kParts, N, 64, false);
    product<N, true>(tmem, 384, base + S::pZ, kParts, 64, base + S::pB, kParts, N, 64, false);  // Z Bt
    umma::commit(mbar);
  }
  if (tid < kQ) {
    sv[Vec::a + tid] = sv[Vec::part + tid] + sv[Vec::part + 64 + tid];
    sv[Vec::v + tid] = sv[Vec::rowb + tid] + sv[Vec::rowb + 64 + tid];
  }
  __syncthreads();
  // ---- dgamma, dbeta, the box sums, four threads per step (the tensor cores run
  // round 2 meanwhile); the parts are added in a fixed butterfly --------------------
  const float alQ = sv[Vec::al + kQ];
  {
    const int s = tid >> 2, part = tid & 3;
    float dg = 0.f, db = 0.f;
    for (int tau = s + part; tau < kQ; tau += 4) {
      const float dts = tD[tau * 65 + s + 1];
      dg = fmaf(dts, tM[tau * 65 + s], dg);
      if (s > 0) db = fmaf(dts, tM[tau * 65 + s - 1], db);
    }
    if (s == 0) {
      for (int tau = part; tau < kQ; tau += 4)
        db = fmaf(tD[tau * 65 + 1], sv[Vec::gxp + tau] * sv[Vec::cbp + tau], db);
    }
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
      dg += __shfl_xor_sync(0xffffffffu, dg, o);
      db += __shfl_xor_sync(0xffffffffu, db, o);
    }
    if (part == 0) {
      const float dq = alQ * tD[(kQ - 1) * 65 + s + 1];  // the U row
      sv[Vec::dg + s] = fmaf(dq, sv[Vec::v + s], dg);
      sv[Vec::db + s] = fmaf(dq, s == 0 ? vm1 : sv[Vec::v + s - 1], db);
    }
  }
  __syncthreads();
  // the box sums BX_s = sum_{tau>=s} sum_{j<=s-2} c(tau,j) M(tau,j): each row's
  // prefix over j, written over M (a row keeps the two M values it still needs
  // in registers), then the column sums over tau >= s
  if (tid < kQ) {
    const int tau = tid;
    float run = 0.f, m2 = 0.f, m1 = 0.f;  // M(tau, s-2), M(tau, s-1)
    for (int s2 = 0; s2 <= tau; ++s2) {
      const float m0 = tM[tau * 65 + s2];
      if (s2 >= 2) run = fmaf(tD[tau * 65 + s2] * sv[Vec::eps + s2 - 2], m2, run);  // c(tau, s2-2)
      tM[tau * 65 + s2] = run;
      m2 = m1;
      m1 = m0;
    }
  }
  __syncthreads();
  {
    const int s = tid >> 2, part = tid & 3;
    float bx = 0.f;
    for (int tau = s + part; tau < kQ; tau += 4) bx += tM[tau * 65 + s];
    bx += __shfl_xor_sync(0xffffffffu, bx, 1);
    bx += __shfl_xor_sync(0xffffffffu, bx, 2);
    if (part == 0) sv[Vec::bx + s] = bx;
  }
  __syncthreads();
  {
    // dalpha_s: the suffix sums over tau and the U row's sums over j, four
    // threads per step
    const int s = tid >> 2, part = tid & 3;
    const float be0 = sv[Vec::be];
    float a1 = 0.f, bu = 0.f;
    if (s == 0) {
      for (int tau = part; tau < kQ; tau += 4) a1 = fmaf(tD[tau * 65 + 1], sv[Vec::a + tau], a1);
    } else {
      for (int tau = s + part; tau < kQ; tau += 4)
        a1 += fmaf(tD[tau * 65], sv[Vec::a + tau],
                   be0 * tD[tau * 65 + 1] * (sv[Vec::gxp + tau] * sv[Vec::cbp + tau]));
      for (int j = part; j <= s - 2; j += 4) bu = fmaf(sv[Vec::crow + j], sv[Vec::v + j], bu);
    }
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
      a1 += __shfl_xor_sync(0xffffffffu, a1, o);
      bu += __shfl_xor_sync(0xffffffffu, bu, o);
    }
    if (part == 0) {
      float v;
      if (s == 0) {
        v = fmaf(alQ * tD[(kQ - 1) * 65 + 1], us, a1);
      } else {
        a1 += alQ * fmaf(be0 * tD[(kQ - 1) * 65 + 1], vm1, tD[(kQ - 1) * 65] * us);
        v = (a1 + sv[Vec::bx + s] + alQ * bu) / sv[Vec::al + s] + sv[Vec::ga + s - 1] * sv[Vec::db + s];
      }
      sv[Vec::da + s] = v;
    }
  }
  if (!umma::mbar_wait(mbar, 1)) *sErr = 1;
  umma::fence_after();
  __syncthreads();
  const bool failed = *sErr != 0;
  const float qnan = __int_as_float(0x7fc00000);
  // ---- dx ----------------------------------------------------------------------------
  {
    float dxv[P / 4], buv[P / 4];
    umma::tmem_ld16_pair<P / 16>(tmem + tq + 256 + cb * (P / 2), tmem + tq + 448 + cb * (P / 2), dxv, buv);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int s = e ? rb : ra;
      if (s >= c.Qc) continue;
      const float wu = sv[Vec::wu + s];
#pragma unroll
      for (int i = 0; i < P / 16; ++i) {
        const int p0 = cb * (P / 2) + 8 * i + c2;
        const float2 gv = get2x2(sm + S::pG, koff(s, p0, P));
        float o0 = fmaf(Dh, gv.x, fmaf(wu, buv[4 * i + 2 * e], dxv[4 * i + 2 * e]));
        float o1 = fmaf(Dh, gv.y, fmaf(wu, buv[4 * i + 2 * e + 1], dxv[4 * i + 2 * e + 1]));
        const int64_t j = ((c.b * p.L + c.t0 + s) * p.H + c.h) * P + p0;
        if (slab != kSlabWhole) {  // dx sums over the states: across the slabs
          float2 *td = reinterpret_cast<float2 *>(p.tok_dx + j);
          if (slab != kSlabFirst) {
            const float2 pr = *td;
            o0 = pr.x + o0;
            o1 = pr.y + o1;
          }
          if (!finish) {
            *td = make_float2(o0, o1);
            continue;
          }
        }
        if (failed) o0 = o1 = qnan;
        *reinterpret_cast<uint32_t *>(static_cast<bf16 *>(p.dx) + j) = pack_bf16x2(o0, o1);
      }
    }
  }
  // ---- dBt, dCt; RoPE backward: per-head dB, dC; dphi ----------------------------------
  {
    float dbv[N / 4], dcv[N / 4], xu[N / 4], gs[N / 4];
    umma::tmem_ld16_pair<N / 16>(tmem + tq + 320 + cb * (N / 2), tmem + tq + 384 + cb * (N / 2), dbv, dcv);
    umma::tmem_ld16_pair<N / 16>(tmem + tq + 192 + cb * (N / 2), tmem + tq + 128 + cb * (N / 2), xu, gs);
    const float be0 = sv[Vec::be];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int t = e ? rb : ra;
      const float wu = sv[Vec::wu + t], d1 = sv[Vec::d1 + t];
      const float wprev = be0 * sv[Vec::d0 + t] * sv[Vec::gxp + t];
#pragma unroll
      for (int i = 0; i < N / 16; ++i) {
        const int n = cb * (N / 2) + 8 * i + c2, kk = n >> 1;
        const float db0 = fmaf(wu, xu[4 * i + 2 * e], dbv[4 * i + 2 * e]);
        const float db1 = fmaf(wu, xu[4 * i + 2 * e + 1], dbv[4 * i + 2 * e + 1]);
        const float dc0 = fmaf(wprev, sv[Vec::bprev + n], fmaf(d1, gs[4 * i + 2 * e], dcv[4 * i + 2 * e]));
        const float dc1 = fmaf(wprev, sv[Vec::bprev + n + 1], fmaf(d1, gs[4 * i + 2 * e + 1], dcv[4 * i + 2 * e + 1]));
        float rb0 = db0, rb1 = db1, rc0 = dc0, rc1 = dc1, dphi = 0.f;
        if (kk < c.K) {
          float sn, cs;
          sincos_reduced(tPhi[t * kPhS + kk], sn, cs);
          rb0 = cs * db0 + sn * db1;
          rb1 = -sn * db0 + cs * db1;
          rc0 = cs * dc0 + sn * dc1;
          rc1 = -sn * dc0 + cs * dc1;
          const float2 bb = get2x2(sm + S::pB, koff(t, n, N)), cc = get2x2(sm + S::pC, koff(t, n, N));
          dphi = (db1 * bb.x - db0 * bb.y) + (dc1 * cc.x - dc0 * cc.y);
        }
        if (t < c.Qc) {
          const int64_t j = ((c.b * p.L + c.t0 + t) * p.H + c.h) * c.ldN + c.n0 + n;
          if (failed) rb0 = rb1 = rc0 = rc1 = qnan;
          *reinterpret_cast<float2 *>(ws_dB + j) = make_float2(rb0, rb1);
          *reinterpret_cast<float2 *>(ws_dC + j) = make_float2(rc0, rc1);
        }
        if (kk < c.K) tPhi[t * kPhS + kk] = dphi;  // this thread alone reads and writes it
      }
    }
  }
  __syncthreads();
  // ---- dtheta within the chunk (reverse sum), the chunk's total; dalpha, dbeta,
  // dgamma; dD -----------------------------------------------------------------------
  if (warp < 2) {
    // reverse sums over the chunk per angle pair: warp w takes pairs w, w + 2,
    // ...; lane l holds steps 2l, 2l + 1 (steps past Qc carry zero)
    const int t0 = 2 * lane, t1 = t0 + 1;
    for (int k = warp; k < c.K; k += 2) {
      const float a0 = tPhi[t0 * kPhS + k], a1 = tPhi[t1 * kPhS + k];
      float incl = a0 + a1;  // suffix sums: lanes >= l
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_down_sync(0xffffffffu, incl, o);
        if (lane + o < 32) incl += u;
      }
      float excl = __shfl_down_sync(0xffffffffu, incl, 1);
      if (lane == 31) excl = 0.f;
      const float v1 = excl + a1, v0 = v1 + a0;
      const int64_t j = ((c.b * p.L + c.t0 + t0) * p.H + c.h) * c.Kt + c.k0 + k;
      if (t0 < c.Qc) p.dtheta[j] = failed ? qnan : v0;
      if (t1 < c.Qc) p.dtheta[j + p.H * c.Kt] = failed ? qnan : v1;
      if (lane == 0) ws_th[((c.b * p.H + c.h) * c.nc + c.ch) * c.Kt + c.k0 + k] = v0;
    }
  } else if (tid >= 64 && tid < 64 + kQ) {
    const int s = tid - 64;
    if (s < c.Qc) {
      const bool add = slab == kSlabMiddle || slab == kSlabLast;
      const int64_t j = (c.b * p.L + c.t0 + s) * p.H + c.h;
      float va = sv[Vec::da + s], vb = sv[Vec::db + s], vg = sv[Vec::dg + s];
      if (failed) va = vb = vg = qnan;
      p.dalpha[j] = (add ? p.dalpha[j] : 0.f) + va;
      p.dbeta[j] = (add ? p.dbeta[j] : 0.f) + vb;
      p.dgamma[j] = (add ? p.dgamma[j] : 0.f) + vg;
    }
  } else if (tid == 128 && finish) {
    ws_dD[(c.b * p.H + c.h) * c.nc + c.ch] = dD;
  }
  umma::fence_before();
  __syncthreads();  // this unit's TMEM reads and shared-memory uses are done
  umma::fence_after();
  if (*sErr) break;  // a tensor-core round never completed: stop (outputs are NaN)
  }
  umma::fence_before();
  __syncthreads();
  if (warp == 0) {
    umma::fence_after();
    umma::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// 4. dtheta carries; sums over heads (dB, dC) and over batch and chunks (dD)
// ---------------------------------------------------------------------------
// in place: the chunk totals become the sums over all later chunks
__global__ void m3b_theta_carry_kernel(const M3Params p, float *ws_th) {
  const int64_t nc = (p.L + kQ - 1) / kQ, K = p.K;
  const int64_t n = p.B * p.H * K;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t bh = i / K, k = i % K;
    float acc = 0.f;
    for (int64_t ch = nc - 1; ch >= 0; --ch) {
      float *slot = ws_th + (bh * nc + ch) * K + k;
      const float v = *slot;
      *slot = acc;
      acc += v;
    }
  }
}

__global__ void m3b_finish_kernel(const M3Params p, const float *ws_dB, const float *ws_dC,
                                  const float *ws_dD, const float *ws_th) {
  const int64_t Bsz = p.B, L = p.L, H = p.H, G = p.G, N = p.N, K = p.K;
  const int64_t nc = (L + kQ - 1) / kQ;
  const int64_t hpg = H / G;
  const int64_t n_bc = Bsz * L * G * N;
  const int64_t n_th = Bsz * L * H * K;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_bc + n_th + H;
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
    } else if (i < n_bc + n_th) {
      const int64_t j = i - n_bc;  // (b, t, h, k)
      const int64_t k = j % K, h = (j / K) % H, t = (j / (K * H)) % L, b = j / (K * H * L);
      p.dtheta[j] += ws_th[((b * H + h) * nc + t / kQ) * K + k];
    } else if (p.dD) {
      const int64_t h = i - n_bc - n_th;
      float s = 0.f;
      for (int64_t b = 0; b < Bsz; ++b)
        for (int64_t ch = 0; ch < nc; ++ch) s += ws_dD[(b * H + h) * nc + ch];
      p.dD[h] = s;
    }
  }
}

// ---------------------------------------------------------------------------
template <int P, int N>
cudaError_t launch_chunks(const M3Params &p, char *ws, const M3BwdWs &w, bool prep,
                          cudaStream_t s) {
  const int64_t units = ((p.L + kQ - 1) / kQ) * p.H * p.B;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // persistent: one CTA per SM (shared memory admits no second) walking the units
  const dim3 grid((unsigned)(units < sms ? units : sms));
  float *vu = reinterpret_cast<float *>(ws + w.vu);
  if (prep) {
    const size_t smem = (size_t)PrepSmem::total;
    cudaError_t e = cudaFuncSetAttribute(m3b_prep_kernel<P, N>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    m3b_prep_kernel<P, N><<<grid, kThreads, smem, s>>>(p, vu, reinterpret_cast<float *>(ws + w.rho));
  } else {
    const size_t smem = (size_t)GradSmem::total;
    cudaError_t e = cudaFuncSetAttribute(m3b_grad_kernel<P, N>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    m3b_grad_kernel<P, N><<<grid, kThreads, smem, s>>>(
        p, vu, reinterpret_cast<float *>(ws + w.dB), reinterpret_cast<float *>(ws + w.dC),
        reinterpret_cast<float *>(ws + w.dD), reinterpret_cast<float *>(ws + w.th));
  }
  return cudaGetLastError();
}

template <int P>
cudaError_t launch_chunks_n(const M3Params &p, char *ws, const M3BwdWs &w, bool prep,
                            cudaStream_t s) {
  switch (p.N) {
    case 16: return launch_chunks<P, 16>(p, ws, w, prep, s);
    case 32: return launch_chunks<P, 32>(p, ws, w, prep, s);
    default: return launch_chunks<P, 64>(p, ws, w, prep, s);
  }
}

cudaError_t launch_chunks_p(const M3Params &p, char *ws, const M3BwdWs &w, bool prep,
                            cudaStream_t s) {
  switch (p.P) {
    case 16: return launch_chunks_n<16>(p, ws, w, prep, s);
    case 32: return launch_chunks_n<32>(p, ws, w, prep, s);
    default: return launch_chunks_n<64>(p, ws, w, prep, s);
  }
}

unsigned grid_for(int64_t n) {
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  return (unsigned)(blocks < 1 ? 1 : blocks);
}

}  // namespace

// bf16 io: the whole d_state, or slabs of kM3Slab states in ascending order,
// first the preparation of every slab (y carried across them in tok_y), then
// the carry over all of d_state, then the gradients of every slab (dx carried
// in tok_dx, dalpha, dbeta, dgamma added in place), then the sums.
cudaError_t launch_m3_bwd_umma(const M3Params &p0, cudaStream_t s) {
  const int64_t n_tot = p0.N;
  const int64_t slabs = (n_tot + kM3Slab - 1) / kM3Slab;
  const M3BwdWs w = m3_bwd_ws_layout(p0.B, p0.L, p0.H, p0.P, n_tot, p0.K);
  char *ws = static_cast<char *>(p0.ws);
  M3Params pp = p0;
  pp.ldN = n_tot;
  pp.n0 = 0;
  pp.tok_y = slabs > 1 ? reinterpret_cast<float *>(ws + w.tok_y) : nullptr;
  pp.tok_dx = slabs > 1 ? reinterpret_cast<float *>(ws + w.tok_dx) : nullptr;
  for (int pass = 0; pass < 2; ++pass) {
    for (int64_t k = 0; k < slabs; ++k) {
      M3Params p = pp;
      p.n0 = k * kM3Slab;
      p.N = n_tot - p.n0 < kM3Slab ? n_tot - p.n0 : kM3Slab;
      p.slab = slabs == 1 ? kSlabWhole
                          : (k == 0 ? kSlabFirst : (k == slabs - 1 ? kSlabLast : kSlabMiddle));
      cudaError_t e = launch_chunks_p(p, ws, w, pass == 0, s);
      if (e != cudaSuccess) return e;
    }
    if (pass == 0) {
      m3b_carry_kernel<<<grid_for(pp.B * pp.H * pp.P * n_tot), 256, 0, s>>>(
          pp, reinterpret_cast<float *>(ws + w.vu), reinterpret_cast<const float *>(ws + w.rho));
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
  }
  if (pp.K > 0) {
    m3b_theta_carry_kernel<<<grid_for(pp.B * pp.H * pp.K), 256, 0, s>>>(
        pp, reinterpret_cast<float *>(ws + w.th));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int64_t total = pp.B * pp.L * pp.G * n_tot + pp.B * pp.L * pp.H * pp.K + pp.H;
  m3b_finish_kernel<<<grid_for(total), 256, 0, s>>>(
      pp, reinterpret_cast<const float *>(ws + w.dB), reinterpret_cast<const float *>(ws + w.dC),
      reinterpret_cast<const float *>(ws + w.dD), reinterpret_cast<const float *>(ws + w.th));
  return cudaGetLastError();
}

}  // namespace msc
