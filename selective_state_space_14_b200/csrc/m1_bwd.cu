// m1_bwd.cu -- Mamba-1 selective scan, backward through the recurrent state
// (sm_100a).  "Full backward pass through the recurrent SSM state", mamba-rs
// 0.7.0 README, "Features".
//
// With g_t = dout_t silu(z_t) and a_t[n] = exp(delta_t A[c,n]), the state
// adjoint runs backwards in time,
//   lambda_t[n] = g_t C_t[n] + a_{t+1}[n] lambda_{t+1}[n],
// and every gradient is a product of lambda with forward quantities:
//   dB_t[n] += lambda_t delta_t x_t      dC_t[n] += g_t h_t[n]   (over channels)
//   dA[n]   += lambda_t delta_t a_t h_{t-1}          (over batch and time)
//   ddelta_t = sum_n lambda_t (A[n] a_t h_{t-1} + B_t[n] x_t)
//   dx_t     = g_t D + delta_t sum_n lambda_t B_t[n]
//
// Work decomposition (m1_common.cuh): a thread owns a (b, c) sequence and one
// pair of state indices and walks the sequence backwards in 8-step chunks
// (the forward's saved-state interval).  Per chunk it re-runs the 8 forward
// steps from the saved state, keeping a_t and h_{t-1} in registers, then walks
// them backwards carrying mu = a lambda (the adjoint handed to the earlier
// step) in registers; dA accumulates per thread in registers.  The sums over
// state pairs (y for dz, ddelta, sum_n lambda B) go through shared memory per
// token, the sums over channels (dB, dC) through shared memory in channel
// order within the CTA, then in rank order across the 8 CTAs of a
// thread-block cluster through distributed shared memory, and one partial
// per cluster and chunk goes to the workspace.  A second kernel adds a
// group's partials in ascending order and the per-(b, c) partials of dA, dD
// and dbias over the batch in ascending order.  No atomics: the bits are the
// same on every run.
#include <cooperative_groups.h>

#include "m1_common.cuh"

namespace cg = cooperative_groups;

namespace msc {
namespace {

using namespace m1;

constexpr int kWarps = 4;
constexpr int kS = kM1SaveInterval;  // steps per backward chunk
constexpr int kCS = kM1BwdCluster;   // CTAs per cluster
constexpr int kAccT = 64;            // steps of dB/dC exchanged across the cluster at once
constexpr int kAccChunks = kAccT / kS;

template <int kN>
struct BwdSmem {
  using Lay = Layout<kN, kWarps>;
  static constexpr int kP = Lay::kP;
  static constexpr int kCh = Lay::kCh;
  // warp-local tile of per-token partials (y, ddelta, lambda.B, -):
  // [channel in warp][step][pair] float4 with the pair stride padded to kP + 1
  // so that the transposed read (one step, all pairs) is conflict-free
  static constexpr int kTileRow = kP + 1;                          // float4 per step row
  static constexpr int kTile = Lay::kChPerWarp * kS * kTileRow * 4;  // floats per warp
  // float offsets
  static constexpr int kTk = kS + 1;  // token tile channel stride (float4, bank spread)
  static constexpr int tok = 0;                           // [kCh][kTk] float4 (dt, dtx, g, x)
  static constexpr int tok2 = tok + kCh * kTk * 4;        // [kCh][kTk] float4 (Dx, sig, dzf, gD)
  static constexpr int bc = tok2 + kCh * kTk * 4;         // [kS][kP] float4
  static constexpr int tile = bc + kS * kP * 4;           // [kWarps][kTile]
  static constexpr int rbc = tile + kWarps * kTile;       // [kCh][kS][kP] float4: (dB pair, dC pair)
  static constexpr int acc = rbc + kCh * kS * kP * 4;     // [2 tensor][kN][kAccT]
  static constexpr int total = acc + 2 * kN * kAccT;
};

template <typename T>
__device__ __forceinline__ float ld1(const void *base, int64_t i) {
  return to_f32(static_cast<const T *>(base)[i]);
}

template <typename T, int kN>
__global__ void __launch_bounds__(kWarps * 32, 4) m1_bwd_kernel(const M1Params p) {
  using S = BwdSmem<kN>;
  using Lay = Layout<kN, kWarps>;
  constexpr int kP = Lay::kP;
  constexpr int kCh = Lay::kCh;
  constexpr int kThreads = Lay::kThreads;
  extern __shared__ float4 smem4[];
  float *smem = reinterpret_cast<float *>(smem4);
  float4 *sTok = reinterpret_cast<float4 *>(smem + S::tok);
  float4 *sTok2 = reinterpret_cast<float4 *>(smem + S::tok2);
  float4 *sBC = reinterpret_cast<float4 *>(smem + S::bc);
  float4 *sRbc = reinterpret_cast<float4 *>(smem + S::rbc);
  cg::cluster_group cluster = cg::this_cluster();
  const unsigned rank = cluster.block_rank();

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int pr = lane % kP;
  const int chl = warp * Lay::kChPerWarp + lane / kP;
  float4 *sTile = reinterpret_cast<float4 *>(smem + S::tile) + (size_t)warp * (S::kTile / 4) +
                  (lane / kP) * kS * S::kTileRow;
  const int64_t D = p.D, L = p.L, N = p.N, Bsz = p.B;
  const int64_t b = blockIdx.y;
  const int64_t per_group = D / p.G;
  const int64_t ctas_per_group = (per_group + kCh - 1) / kCh;
  // CTAs past the last group only pad the grid to whole clusters
  const int64_t gq = blockIdx.x / ctas_per_group;
  const int64_t g = gq < p.G ? gq : p.G - 1;
  const int64_t c_first = g * per_group + (blockIdx.x % ctas_per_group) * kCh;
  const int64_t c_end = gq < p.G ? (g + 1) * per_group : 0;
  const int64_t c = c_first + chl;
  const bool active = c < c_end;
  const int64_t part = blockIdx.x / kCS;  // dB/dC partial (kCh * kCS channels)
  const T *Bg = static_cast<const T *>(p.Bm) + (b * p.G + g) * N * L;
  const T *Cg = static_cast<const T *>(p.Cm) + (b * p.G + g) * N * L;
  const int64_t n_chunks = (L + kS - 1) / kS;

  const int n0 = 2 * pr, n1 = 2 * pr + 1;
  float2 Ap = make_float2(0.f, 0.f);
  if (active) {
    if (n0 < N) Ap.x = p.A[c * N + n0];
    if (n1 < N) Ap.y = p.A[c * N + n1];
  }
  const float2 A2 = mul2(Ap, splat2(kLog2e));
  float2 mu = make_float2(0.f, 0.f);   // a_{t+1} lambda_{t+1}, handed backwards
  float2 dA = make_float2(0.f, 0.f);   // this (b, c)'s dA for the pair
  float dD_l = 0.f, dbias_l = 0.f;     // per lane (tokens it finishes), summed per channel

  for (int64_t ch = n_chunks - 1; ch >= 0; --ch) {
    const int64_t tc = ch * kS;
    // 64-step accumulator of the CTA's dB/dC sums
    const int64_t blk = ch / kAccChunks;
    const int tacc = (int)(ch % kAccChunks) * kS;  // this chunk's offset in the block
    float *acc = smem + S::acc;

    // ---- stage the chunk's per-token values and B, C -----------------------
    for (int u = tid; u < kCh * kS; u += kThreads) {
      const int cl = u / kS, tt = u % kS;
      const int64_t cc = c_first + cl;
      const int64_t t = tc + tt;
      float4 tk = make_float4(0.f, 0.f, 0.f, 0.f), tk2 = make_float4(0.f, 0.f, 0.f, 0.f);
      if (cc < c_end && t < L) {
        const int64_t i = (b * D + cc) * L + t;
        const float x = ld1<T>(p.u, i);
        const float v = ld1<T>(p.delta, i) + (p.bias ? p.bias[cc] : 0.f);
        const float dy = ld1<T>(p.dout, i);
        const float d = p.softplus ? softplus(v) : v;
        const float Dc = p.Dp ? p.Dp[cc] : 0.f;
        float gz = dy, dzf = 0.f;
        if (p.z) {
          const float zv = ld1<T>(p.z, i);
          gz = dy * silu(zv);
          dzf = dy * dsilu(zv);
        }
        tk = make_float4(d, d * x, gz, x);
        tk2 = make_float4(Dc * x, p.softplus ? sigmoid(v) : 1.f, dzf, gz * Dc);
      }
      sTok[cl * S::kTk + tt] = tk;
      sTok2[cl * S::kTk + tt] = tk2;
    }
    stage_bc<T, kN, kS>(sBC, Bg, Cg, N, L, tc, p.vec, tid, kThreads);
    float2 h = make_float2(0.f, 0.f);
    if (active) {
      const float *sv = p.saved_in + ((b * D + c) * n_chunks + ch) * N;
      if (n0 < N) h.x = sv[n0];
      if (n1 < N) h.y = sv[n1];
    }
    __syncthreads();

    // ---- forward over the chunk, keeping a_t, h_{t-1} and the token values ----
    float2 a[kS], hp[kS];
    float tdt[kS], tdtx[kS], tg[kS], yv[kS];
#pragma unroll
    for (int t = 0; t < kS; ++t) {
      const float4 tk = sTok[chl * S::kTk + t];
      const float4 bcv = sBC[t * kP + pr];
      tdt[t] = tk.x; tdtx[t] = tk.y; tg[t] = tk.z;
      a[t] = ex2_2(mul2(splat2(tk.x), A2));
      hp[t] = h;
      h = fma2(a[t], h, mul2(splat2(tk.y), make_float2(bcv.x, bcv.y)));
      yv[t] = fmaf(bcv.w, h.y, bcv.z * h.x);
    }
    // ---- backwards over the chunk --------------------------------------------
#pragma unroll
    for (int t = kS - 1; t >= 0; --t) {
      const float4 bcv = sBC[t * kP + pr];
      const float2 Bv = make_float2(bcv.x, bcv.y), Cv = make_float2(bcv.z, bcv.w);
      const float2 lam = fma2(splat2(tg[t]), Cv, mu);
      const float2 bb = mul2(splat2(tdtx[t]), Bv);
      const float2 hcur = fma2(a[t], hp[t], bb);
      const float2 q = mul2(a[t], hp[t]);
      const float2 dC = mul2(splat2(tg[t]), hcur);
      const float2 dB = mul2(lam, splat2(tdtx[t]));
      const float2 lq = mul2(lam, q);
      dA = fma2(splat2(tdt[t]), lq, dA);
      sTile[t * S::kTileRow + pr] =
          make_float4(yv[t], fmaf(Ap.y, lq.y, Ap.x * lq.x), fmaf(lam.y, Bv.y, lam.x * Bv.x), 0.f);
      sRbc[(chl * kS + t) * kP + pr] = make_float4(dB.x, dB.y, dC.x, dC.y);
      mu = mul2(a[t], lam);
    }
    // ---- per token (warp-local): lane pr < kS of a channel sums step pr ------
    __syncwarp();
    if (pr < kS) {
      const int tt = pr;
      const int64_t t = tc + tt;
      const float4 tk = sTok[chl * S::kTk + tt];
      const float4 tk2 = sTok2[chl * S::kTk + tt];
      float y = tk2.x, dd = 0.f, sb = 0.f;
#pragma unroll
      for (int q = 0; q < kP; ++q) {
        const float4 r = sTile[tt * S::kTileRow + q];
        y += r.x; dd += r.y; sb += r.z;
      }
      if (active && t < L) {
        const int64_t i = (b * D + c) * L + t;
        const float draw = fmaf(tk.w, sb, dd) * tk2.y;
        static_cast<T *>(p.du)[i] = from_f32<T>(fmaf(tk.x, sb, tk2.w));
        static_cast<T *>(p.ddelta)[i] = from_f32<T>(draw);
        if (p.dz) static_cast<T *>(p.dz)[i] = from_f32<T>(y * tk2.z);
        dbias_l += draw;
        dD_l = fmaf(tk.z, tk.w, dD_l);
      }
    }
    __syncthreads();
    // ---- dB, dC: the CTA's channels, added in channel order -------------------
    for (int u = tid; u < kS * kP; u += kThreads) {
      const int tt = u / kP, q = u % kP;
      float4 s = sRbc[tt * kP + q];
#pragma unroll
      for (int cl = 1; cl < kCh; ++cl) {
        const float4 o = sRbc[(cl * kS + tt) * kP + q];
        s.x += o.x; s.y += o.y; s.z += o.z; s.w += o.w;
      }
      acc[(0 * kN + 2 * q) * kAccT + tacc + tt] = s.x;
      acc[(0 * kN + 2 * q + 1) * kAccT + tacc + tt] = s.y;
      acc[(1 * kN + 2 * q) * kAccT + tacc + tt] = s.z;
      acc[(1 * kN + 2 * q + 1) * kAccT + tacc + tt] = s.w;
    }

    if (tacc == 0) {
      // block complete: the cluster's CTA sums, added in rank order, go to the
      // workspace
      cluster.sync();
      constexpr int E = 2 * kN * kAccT;
      constexpr int per = E / kCS;
      const int64_t t_blk = blk * kAccT;
      for (int e = rank * per + tid; e < (int)(rank + 1) * per; e += kThreads) {
        float s = *(cluster.map_shared_rank(acc, 0) + e);
#pragma unroll
        for (int qq = 1; qq < kCS; ++qq) s += *(cluster.map_shared_rank(acc, qq) + e);
        const int te = e / (kN * kAccT);
        const int n = (e / kAccT) % kN;
        const int64_t t = t_blk + e % kAccT;
        if (n < N && t < L) p.ws_bc[(((part * Bsz + b) * 2 + te) * N + n) * L + t] = s;
      }
      cluster.sync();  // the accumulator is free again
    } else {
      __syncthreads();  // this chunk's shared buffers are free for the next one
    }
  }
  cluster.sync();  // no CTA leaves while a peer may still read its shared memory

  // per-(b, c) partials: dA (per thread), dD and dbias (the lanes of a channel
  // added by a fixed butterfly), dh0 = the carry left after step 0
#pragma unroll
  for (int off = kP / 2; off > 0; off >>= 1) {
    dD_l += __shfl_xor_sync(0xffffffffu, dD_l, off, kP);
    dbias_l += __shfl_xor_sync(0xffffffffu, dbias_l, off, kP);
  }
  if (active) {
    float *m = p.ws_misc + (b * D + c) * (N + 2);
    if (n0 < N) m[n0] = dA.x;
    if (n1 < N) m[n1] = dA.y;
    if (p.dh0) {
      if (n0 < N) p.dh0[(b * D + c) * N + n0] = mu.x;
      if (n1 < N) p.dh0[(b * D + c) * N + n1] = mu.y;
    }
  }
  if (active && pr == 0) {
    float *m = p.ws_misc + (b * D + c) * (N + 2);
    m[N] = dD_l;
    m[N + 1] = dbias_l;
  }
}

// dB/dC: sum of a group's partials in ascending order; dA, dD, dbias: sum of
// the per-(b, c) partials over the batch in ascending order.
__global__ void m1_bwd_reduce_kernel(const M1Params p) {
  const int64_t Bsz = p.B, D = p.D, N = p.N, L = p.L, G = p.G;
  const int64_t per_group = p.n_part / G;  // partials per group
  const int64_t n_bc = Bsz * G * 2 * N * L;
  const int64_t n_total = n_bc + D * (N + 2);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_total;
       i += (int64_t)gridDim.x * blockDim.x) {
    if (i < n_bc) {
      // i enumerates (b, g, tensor, n, t)
      const int64_t t = i % L;
      const int64_t n = (i / L) % N;
      const int64_t tensor = (i / (L * N)) % 2;
      const int64_t g = (i / (L * N * 2)) % G;
      const int64_t b = i / (L * N * 2 * G);
      float s = 0.f;
      for (int64_t q = g * per_group; q < (g + 1) * per_group; ++q)
        s += p.ws_bc[(((q * Bsz + b) * 2 + tensor) * N + n) * L + t];
      float *dst = tensor == 0 ? p.dB : p.dC;
      dst[((b * G + g) * N + n) * L + t] = s;
    } else {
      const int64_t j = i - n_bc;  // (c, k), k < N + 2
      const int64_t c = j / (N + 2), k = j % (N + 2);
      float s = 0.f;
      for (int64_t b = 0; b < Bsz; ++b) s += p.ws_misc[(b * D + c) * (N + 2) + k];
      if (k < N) p.dA[c * N + k] = s;
      else if (k == N) { if (p.dD) p.dD[c] = s; }
      else if (p.dbias) p.dbias[c] = s;
    }
  }
}

template <typename T, int kN>
cudaError_t launch_t(const M1Params &p, cudaStream_t s) {
  using Lay = Layout<kN, kWarps>;
  const size_t smem = sizeof(float) * (size_t)BwdSmem<kN>::total;
  cudaError_t err = cudaFuncSetAttribute(m1_bwd_kernel<T, kN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int64_t per_group = p.D / p.G;
  const int64_t ctas_per_group = (per_group + Lay::kCh - 1) / Lay::kCh;
  const int64_t grid_x = (p.G * ctas_per_group + kCS - 1) / kCS * kCS;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid_x, (unsigned)p.B);
  cfg.blockDim = dim3(Lay::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kCS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, m1_bwd_kernel<T, kN>, p);
  if (err != cudaSuccess) return err;
  const int64_t total = p.B * p.G * 2 * p.N * p.L + p.D * (p.N + 2);
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  m1_bwd_reduce_kernel<<<(unsigned)blocks, threads, 0, s>>>(p);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_n(const M1Params &p, cudaStream_t s) {
  switch (pad_n(p.N)) {
    case 16: return launch_t<T, 16>(p, s);
    case 32: return launch_t<T, 32>(p, s);
    default: return launch_t<T, 64>(p, s);
  }
}

}  // namespace

// Partials: one per cluster of CTAs; with ngroups > 1 the channels of a group
// are a whole number of clusters (checked by the caller).
int64_t m1_bwd_partials(int64_t D, int64_t N, int64_t G) {
  const int64_t kch = m1_bwd_block(N) / kM1BwdCluster;
  const int64_t per_group = D / G;
  const int64_t ctas = G * ((per_group + kch - 1) / kch);
  return (ctas + kM1BwdCluster - 1) / kM1BwdCluster;
}

size_t m1_bwd_workspace_bytes(int64_t B, int64_t D, int64_t N, int64_t L, int64_t G) {
  const int64_t n_part = m1_bwd_partials(D, N, G);
  size_t bc = sizeof(float) * (size_t)(n_part * B * 2 * N * L);
  bc = (bc + 255) / 256 * 256;
  return bc + sizeof(float) * (size_t)(B * D * (N + 2));
}

cudaError_t launch_m1_bwd(const M1Params &p, cudaStream_t s) {
  return p.io_bf16 ? launch_n<bf16>(p, s) : launch_n<float>(p, s);
}

}  // namespace msc
