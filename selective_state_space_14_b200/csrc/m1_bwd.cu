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
// Work decomposition.  As in the forward, one warp owns one (b, c) sequence,
// 32 lanes x kItems steps form a chunk of 256 steps (= the forward's state
// save interval), and the warp walks the chunks from last to first.  Per chunk
// and state index n:
//   * the forward states are re-materialised from the state the forward
//     saved at the chunk start (warp scan of (prod a, h) pairs, as forward);
//   * the adjoint is scanned from the right with the carry mu = a lambda
//     handed over from the later chunk (warp suffix scan of the same monoid);
//   * each lane then walks its steps backwards and forms the contributions.
// dB and dC sum over the channels of a group.  Each warp's per-(n, t)
// contributions go to shared memory, where the CTA adds its 8 warps in warp
// order; the 8 CTAs of a thread-block cluster then add their CTA sums in rank
// order through distributed shared memory, and one 64-channel partial per
// chunk goes to the workspace.  A second kernel adds the partials of a group
// in ascending order, and the per-(b, c) partials of dA, dD and dbias over the
// batch in ascending order.  No atomics anywhere, so the bits are the same on
// every run.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace msc {
namespace {

constexpr int kItems = 8;               // steps per lane per chunk
constexpr int kT = 32 * kItems;         // chunk length
constexpr int kW = kM1BwdWarps;         // warps (channels) per CTA
constexpr int kCS = kM1BwdCluster;      // CTAs per cluster
constexpr int kNG = 2;                  // state indices per shared-memory round
static_assert(kT == kM1SaveInterval, "backward chunk must equal the save interval");

struct Smem {
  // float offsets into dynamic shared memory
  static constexpr int stage = 0;                        // [kW][2][kNG][kT]
  static constexpr int mu = stage + kW * 2 * kNG * kT;   // [kW][MSC_MAX_N]
  static constexpr int A = mu + kW * MSC_MAX_N;          // [kW][MSC_MAX_N]
  static constexpr int dA = A + kW * MSC_MAX_N;          // [kW][MSC_MAX_N]
  static constexpr int acc = dA + kW * MSC_MAX_N;        // [2][N][kT]
  static size_t bytes(int64_t N) { return sizeof(float) * (size_t)(acc + 2 * N * kT); }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

template <typename T>
__global__ void __launch_bounds__(kW * 32, 2) m1_bwd_kernel(const M1Params p) {
  extern __shared__ float4 smem4[];
  float *smem = reinterpret_cast<float *>(smem4);
  float *stage = smem + Smem::stage;
  float *acc = smem + Smem::acc;
  cg::cluster_group cluster = cg::this_cluster();
  const unsigned rank = cluster.block_rank();

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int64_t D = p.D, L = p.L, N = p.N, Bsz = p.B;
  const int64_t b = blockIdx.y;
  const int64_t c = (int64_t)blockIdx.x * kW + warp;
  const bool active = c < D;
  const int64_t part = blockIdx.x / kCS;  // 64-channel partial index
  const int64_t g = active ? c / (D / p.G) : 0;
  const int64_t row = (b * D + (active ? c : 0)) * L;
  const T *u = static_cast<const T *>(p.u) + row;
  const T *dl = static_cast<const T *>(p.delta) + row;
  const T *zr = p.z ? static_cast<const T *>(p.z) + row : nullptr;
  const T *dout = static_cast<const T *>(p.dout) + row;
  T *du = static_cast<T *>(p.du) + row;
  T *ddl = static_cast<T *>(p.ddelta) + row;
  T *dz = p.dz ? static_cast<T *>(p.dz) + row : nullptr;
  const T *Bg = static_cast<const T *>(p.Bm) + (b * p.G + g) * N * L;
  const T *Cg = static_cast<const T *>(p.Cm) + (b * p.G + g) * N * L;
  const float Dc = (active && p.Dp) ? p.Dp[c] : 0.f;
  const float bias = (active && p.bias) ? p.bias[c] : 0.f;
  const int64_t n_chunks = (L + kT - 1) / kT;
  const float *saved = p.saved_in + (b * D + (active ? c : 0)) * n_chunks * N;

  float *s_mu = smem + Smem::mu + warp * MSC_MAX_N;
  float *s_A = smem + Smem::A + warp * MSC_MAX_N;
  float *s_dA = smem + Smem::dA + warp * MSC_MAX_N;
  for (int n = lane; n < N; n += 32) {
    s_mu[n] = 0.f;
    s_A[n] = active ? p.A[c * N + n] : 0.f;
    s_dA[n] = 0.f;
  }
  __syncwarp();
  float dD_l = 0.f, dbias_l = 0.f;

  for (int64_t ch = n_chunks - 1; ch >= 0; --ch) {
    const int64_t t0 = ch * kT + (int64_t)lane * kItems;
    float dt[kItems], dtx[kItems], gg[kItems], y[kItems], ddt[kItems], SB[kItems];
    {
      float x[kItems], v[kItems], dy[kItems], zv[kItems];
      if (active) {
        load_run<kItems, Cache::kKeep>(u, t0, L, p.vec, x, 0.f);
        load_run<kItems, Cache::kKeep>(dl, t0, L, p.vec, v, 0.f);
        load_run<kItems, Cache::kKeep>(dout, t0, L, p.vec, dy, 0.f);
        if (zr) load_run<kItems, Cache::kKeep>(zr, t0, L, p.vec, zv, 0.f);
      } else {
#pragma unroll
        for (int i = 0; i < kItems; ++i) x[i] = v[i] = dy[i] = zv[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < kItems; ++i) {
        const float vv = v[i] + bias;
        float d = p.softplus ? softplus(vv) : vv;
        if (!active || t0 + i >= L) d = 0.f;
        dt[i] = d;
        dtx[i] = d * x[i];
        gg[i] = zr ? dy[i] * silu(zv[i]) : dy[i];
        y[i] = Dc * x[i];
        ddt[i] = 0.f;
        SB[i] = 0.f;
      }
    }

    for (int64_t n0 = 0; n0 < N; n0 += kNG) {
#pragma unroll
      for (int j = 0; j < kNG; ++j) {
        const int64_t n = n0 + j;
        float dBc[kItems], dCc[kItems];
        if (n < N) {
          float Bv[kItems], Cv[kItems], a[kItems], hp[kItems];
          load_run<kItems, Cache::kKeep>(Bg + n * L, t0, L, p.vec, Bv, 0.f);
          load_run<kItems, Cache::kKeep>(Cg + n * L, t0, L, p.vec, Cv, 0.f);
          const float An = s_A[n];
          const float A2 = An * kLog2e;
          // forward: local fold, then scan from the saved chunk-start state
          float pl = 1.f, hl = 0.f;
#pragma unroll
          for (int i = 0; i < kItems; ++i) {
            a[i] = ex2(dt[i] * A2);
            hl = fmaf(a[i], hl, dtx[i] * Bv[i]);
            pl = pl * a[i];
          }
          float pe, he;
          warp_scan_fwd(pl, hl, pe, he);
          float h = fmaf(pe, saved[ch * N + n], he);
#pragma unroll
          for (int i = 0; i < kItems; ++i) {
            hp[i] = h;
            h = fmaf(a[i], h, dtx[i] * Bv[i]);
            y[i] = fmaf(Cv[i], h, y[i]);
          }
          // adjoint: local fold from the right, then suffix scan with the
          // carry handed over from the later chunk
          float ml = 0.f;
#pragma unroll
          for (int i = kItems - 1; i >= 0; --i) ml = a[i] * fmaf(gg[i], Cv[i], ml);
          float ps, ms;
          warp_scan_rev(pl, ml, ps, ms);
          float mu = fmaf(ps, s_mu[n], ms);
          float dA_l = 0.f;
#pragma unroll
          for (int i = kItems - 1; i >= 0; --i) {
            const float lam = fmaf(gg[i], Cv[i], mu);
            const float bb = dtx[i] * Bv[i];
            const float q = a[i] * hp[i];
            const float hcur = fmaf(a[i], hp[i], bb);
            dCc[i] = gg[i] * hcur;
            dBc[i] = lam * dtx[i];
            const float lq = lam * q;
            dA_l = fmaf(dt[i], lq, dA_l);
            ddt[i] = fmaf(An, lq, ddt[i]);
            SB[i] = fmaf(lam, Bv[i], SB[i]);
            mu = a[i] * lam;
          }
          mu = __shfl_sync(0xffffffffu, mu, 0);
          dA_l = warp_sum(dA_l);
          __syncwarp();
          if (lane == 0) {
            s_mu[n] = mu;
            s_dA[n] += dA_l;
          }
        } else {
#pragma unroll
          for (int i = 0; i < kItems; ++i) dBc[i] = dCc[i] = 0.f;
        }
        float *sB = stage + ((warp * 2 + 0) * kNG + j) * kT + lane * kItems;
        float *sC = stage + ((warp * 2 + 1) * kNG + j) * kT + lane * kItems;
#pragma unroll
        for (int i = 0; i < kItems; i += 4) {
          *reinterpret_cast<float4 *>(sB + i) = make_float4(dBc[i], dBc[i + 1], dBc[i + 2], dBc[i + 3]);
          *reinterpret_cast<float4 *>(sC + i) = make_float4(dCc[i], dCc[i + 1], dCc[i + 2], dCc[i + 3]);
        }
      }
      __syncthreads();
      // add the warps' contributions in warp order: acc[tensor][n0 + j][t]
      for (int e = tid * 4; e < 2 * kNG * kT; e += kW * 32 * 4) {
        const int tensor = e / (kNG * kT);
        const int j = (e / kT) % kNG;
        const int t = e % kT;
        if (n0 + j < N) {
          float4 s = *reinterpret_cast<const float4 *>(stage + e);
#pragma unroll
          for (int w = 1; w < kW; ++w) {
            const float4 o = *reinterpret_cast<const float4 *>(stage + w * 2 * kNG * kT + e);
            s.x += o.x; s.y += o.y; s.z += o.z; s.w += o.w;
          }
          *reinterpret_cast<float4 *>(acc + (tensor * N + n0 + j) * kT + t) = s;
        }
      }
      __syncthreads();
    }

    // per-(b, c, t) gradients of this chunk
    if (active) {
      float x[kItems], v[kItems];
      load_run<kItems, Cache::kKeep>(u, t0, L, p.vec, x, 0.f);
      load_run<kItems, Cache::kKeep>(dl, t0, L, p.vec, v, 0.f);
      float dxo[kItems], ddo[kItems];
#pragma unroll
      for (int i = 0; i < kItems; ++i) {
        dxo[i] = fmaf(gg[i], Dc, dt[i] * SB[i]);
        const float dd = fmaf(x[i], SB[i], ddt[i]);
        float draw = p.softplus ? dd * sigmoid(v[i] + bias) : dd;
        if (t0 + i >= L) draw = 0.f;
        ddo[i] = draw;
        dbias_l += draw;
        dD_l = fmaf(gg[i], x[i], dD_l);
      }
      store_run<kItems>(du, t0, L, p.vec, dxo);
      store_run<kItems>(ddl, t0, L, p.vec, ddo);
      if (dz && zr) {
        float dy[kItems], zv[kItems];
        load_run<kItems, Cache::kKeep>(dout, t0, L, p.vec, dy, 0.f);
        load_run<kItems, Cache::kKeep>(zr, t0, L, p.vec, zv, 0.f);
#pragma unroll
        for (int i = 0; i < kItems; ++i) y[i] = dy[i] * y[i] * dsilu(zv[i]);
        store_run<kItems>(dz, t0, L, p.vec, y);
      }
    }

    // the cluster's 8 CTA sums, added in rank order, go to the workspace
    cluster.sync();
    {
      const int64_t E = 2 * N * kT;
      const int64_t per = E / kCS;  // N * kT * 2 is a multiple of kCS * 4
      const float *peer[kCS];
#pragma unroll
      for (int q = 0; q < kCS; ++q) peer[q] = cluster.map_shared_rank(acc, q);
      for (int64_t e = rank * per + tid * 4; e < (rank + 1) * per; e += kW * 32 * 4) {
        float4 s = *reinterpret_cast<const float4 *>(peer[0] + e);
#pragma unroll
        for (int q = 1; q < kCS; ++q) {
          const float4 o = *reinterpret_cast<const float4 *>(peer[q] + e);
          s.x += o.x; s.y += o.y; s.z += o.z; s.w += o.w;
        }
        const int64_t tensor = e / (N * kT);
        const int64_t n = (e / kT) % N;
        const int64_t t = ch * kT + e % kT;
        float *dst = p.ws_bc + (((part * Bsz + b) * 2 + tensor) * N + n) * L + t;
        if ((L % 4 == 0) && t + 4 <= L) {
          *reinterpret_cast<float4 *>(dst) = s;
        } else {
          const float sv[4] = {s.x, s.y, s.z, s.w};
          for (int k = 0; k < 4; ++k)
            if (t + k < L) dst[k] = sv[k];
        }
      }
    }
    cluster.sync();
  }

  // per-(b, c) partials: dA row (already summed over lanes and chunks in a
  // fixed order), dD and dbias (summed over lanes by a fixed butterfly)
  dD_l = warp_sum(dD_l);
  dbias_l = warp_sum(dbias_l);
  if (active) {
    float *m = p.ws_misc + (b * D + c) * (N + 2);
    for (int n = lane; n < N; n += 32) {
      m[n] = s_dA[n];
      if (p.dh0) p.dh0[(b * D + c) * N + n] = s_mu[n];
    }
    if (lane == 0) {
      m[N] = dD_l;
      m[N + 1] = dbias_l;
    }
  }
}

// dB/dC: sum of a group's partials in ascending order; dA, dD, dbias: sum of
// the per-(b, c) partials over the batch in ascending order.
__global__ void m1_bwd_reduce_kernel(const M1Params p) {
  const int64_t Bsz = p.B, D = p.D, N = p.N, L = p.L, G = p.G;
  const int64_t per_group = (p.n_part + G - 1) / G;  // partials per group
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
      for (int64_t q = g * per_group; q < (g + 1) * per_group && q < p.n_part; ++q)
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

template <typename T>
cudaError_t launch_t(const M1Params &p, cudaStream_t s) {
  const size_t smem = Smem::bytes(p.N);
  cudaError_t err = cudaFuncSetAttribute(m1_bwd_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.n_part * kCS), (unsigned)p.B);
  cfg.blockDim = dim3(kW * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kCS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, m1_bwd_kernel<T>, p);
  if (err != cudaSuccess) return err;
  const int64_t total = p.B * p.G * 2 * p.N * p.L + p.D * (p.N + 2);
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  m1_bwd_reduce_kernel<<<(unsigned)blocks, threads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

size_t m1_bwd_workspace_bytes(int64_t B, int64_t D, int64_t N, int64_t L, int64_t G) {
  (void)G;
  const int64_t n_part = (D + kM1BwdBlock - 1) / kM1BwdBlock;
  size_t bc = sizeof(float) * (size_t)(n_part * B * 2 * N * L);
  bc = (bc + 255) / 256 * 256;
  return bc + sizeof(float) * (size_t)(B * D * (N + 2));
}

cudaError_t launch_m1_bwd(const M1Params &p, cudaStream_t s) {
  return p.io_bf16 ? launch_t<bf16>(p, s) : launch_t<float>(p, s);
}

}  // namespace msc
