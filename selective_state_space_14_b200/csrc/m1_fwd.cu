// m1_fwd.cu -- Mamba-1 selective scan, forward (sm_100a).
//
// Computes, per (batch b, channel c) and t = 0..L-1 (the selective SSM layer,
// state-spaces/mamba README "Usage / Selective SSM"; mamba-rs 0.7.0 README
// "Features"):
//   delta_t = softplus(delta_raw + bias[c])
//   h_t[n]  = exp(delta_t A[c,n]) h_{t-1}[n] + delta_t B_t[n] x_t
//   out_t   = (sum_n C_t[n] h_t[n] + D[c] x_t) * silu(z_t)
//
// Work decomposition (m1_common.cuh): a thread owns a (b, c) sequence and one
// pair of state indices, and steps through time with the pair of states in
// registers; exp(delta A) is taken as 2^(delta * A log2 e) on the SFU.  Per
// 64-step chunk the CTA stages the per-token values of its channels (softplus
// and the silu gate computed once per token) and the batch row's B, C in
// shared memory.  y_t sums over the state pairs of a channel: every kP steps
// each lane writes its kP pair partials to a padded shared-memory tile and
// then sums one step's partials in pair order (a transpose through shared
// memory, no shuffles).  Gated outputs collect in shared memory and leave in
// 16-byte stores.  The state entering every 8-step block goes to `saved` for
// the backward pass.  Two block barriers per chunk; no atomics.
#include "m1_common.cuh"

namespace msc {
namespace {

using namespace m1;

constexpr int kWarps = 4;

template <int kN>
struct FwdSmem {
  using Lay = Layout<kN, kWarps>;
  static constexpr int kP = Lay::kP;
  static constexpr int kCh = Lay::kCh;
  // per-warp transpose tile: [channel in warp][pair][kP + 4], channel blocks
  // padded so that channels of a warp fall on different banks
  static constexpr int kRow = kP + 4;
  static constexpr int kChBlock = kP * kRow + (kP == 8 ? 8 : (kP == 16 ? 16 : 0));
  // float offsets
  static constexpr int kOut = kT + 8;  // output tile channel stride (bank spread)
  static constexpr int tok = 0;                               // [kT][kCh] float4
  static constexpr int bc = tok + kCh * kT * 4;               // [kT][kP] float4
  static constexpr int ytile = bc + kT * kP * 4;              // [kWarps][32/kP][kChBlock]
  static constexpr int out = ytile + kWarps * (32 / kP) * kChBlock;  // [kCh][kOut]
  static constexpr int total = out + kCh * kOut;
};

// Store the gated outputs of the chunk starting at tc from shared memory.
template <typename T, int kCh, int kOut>
__device__ __forceinline__ void store_chunk(T *out_base, const float *sout, int64_t c_first,
                                            int64_t c_end, int64_t b, int64_t D, int64_t L,
                                            int64_t tc, bool vec, int tid, int nthreads) {
  for (int u = tid; u < kCh * (kT / 8); u += nthreads) {
    const int chl = u / (kT / 8);
    const int seg = u % (kT / 8);
    const int64_t c = c_first + chl;
    if (c >= c_end) continue;
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = sout[chl * kOut + seg * 8 + i];
    store_run<8>(out_base + (b * D + c) * L, tc + seg * 8, L, vec, v);
  }
}

template <typename T, int kN>
__global__ void __launch_bounds__(kWarps * 32, 6) m1_fwd_kernel(const M1Params p) {
  using S = FwdSmem<kN>;
  using Lay = Layout<kN, kWarps>;
  constexpr int kP = Lay::kP;
  constexpr int kCh = Lay::kCh;
  constexpr int kThreads = Lay::kThreads;
  extern __shared__ float4 smem4[];
  float *smem = reinterpret_cast<float *>(smem4);
  float4 *sTok = reinterpret_cast<float4 *>(smem + S::tok);
  float4 *sBC = reinterpret_cast<float4 *>(smem + S::bc);
  float *sOut = smem + S::out;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int chw = lane / kP;                 // channel within the warp
  const int pr = lane % kP;                  // state pair
  const int chl = warp * Lay::kChPerWarp + chw;
  float *ytile = smem + S::ytile + (warp * Lay::kChPerWarp + chw) * S::kChBlock;

  const int64_t D = p.D, L = p.L, N = p.N;
  const int64_t b = blockIdx.y;
  // CTAs tile each B/C group separately, so a CTA never straddles two groups
  const int64_t per_group = D / p.G;
  const int64_t ctas_per_group = (per_group + kCh - 1) / kCh;
  const int64_t g = blockIdx.x / ctas_per_group;
  const int64_t c_first = g * per_group + (blockIdx.x % ctas_per_group) * kCh;
  const int64_t c_end = (g + 1) * per_group;
  const int64_t c = c_first + chl;
  const bool active = c < c_end;
  const T *Bg = static_cast<const T *>(p.Bm) + (b * p.G + g) * N * L;
  const T *Cg = static_cast<const T *>(p.Cm) + (b * p.G + g) * N * L;
  const int64_t n_chunks = (L + kT - 1) / kT;
  const int64_t n_save = (L + kM1SaveInterval - 1) / kM1SaveInterval;

  // this thread's state pair and its A * log2(e)
  const int n0 = 2 * pr, n1 = 2 * pr + 1;
  float2 h = make_float2(0.f, 0.f), A2 = make_float2(0.f, 0.f);
  if (active) {
    if (n0 < N) A2.x = p.A[c * N + n0] * kLog2e;
    if (n1 < N) A2.y = p.A[c * N + n1] * kLog2e;
    if (p.h0) {
      if (n0 < N) h.x = p.h0[(b * D + c) * N + n0];
      if (n1 < N) h.y = p.h0[(b * D + c) * N + n1];
    }
  }

  for (int64_t ch = 0; ch <= n_chunks; ++ch) {
    const int64_t tc = ch * kT;
    // ---- outputs of the previous chunk, and staging of this chunk ----------
    if (ch > 0)
      store_chunk<T, kCh, S::kOut>(static_cast<T *>(p.out), sOut, c_first, c_end, b, D, L,
                                   tc - kT, p.vec, tid, kThreads);
    if (ch == n_chunks) break;
    // (channel fastest: stores to the [step][channel] tile are contiguous, and
    // lanes cl and cl + kCh read the two halves of one 32-byte sector)
    for (int u = tid; u < kCh * (kT / 8); u += kThreads) {
      const int cl = u % kCh, seg = u / kCh;
      const int64_t cc = c_first + cl;
      const int64_t t = tc + seg * 8;
      float x[8], v[8], zv[8];
      const bool act = cc < c_end;
      if (act) {
        const int64_t row = (b * D + cc) * L;
        load_run<8>(static_cast<const T *>(p.u) + row, t, L, p.vec, x, 0.f);
        load_run<8>(static_cast<const T *>(p.delta) + row, t, L, p.vec, v, 0.f);
        if (p.z) load_run<8>(static_cast<const T *>(p.z) + row, t, L, p.vec, zv, 0.f);
      }
      const float Dc = (act && p.Dp) ? p.Dp[cc] : 0.f;
      const float bias = (act && p.bias) ? p.bias[cc] : 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float4 tk = make_float4(0.f, 0.f, 0.f, 0.f);
        if (act && t + i < L) {
          const float vv = v[i] + bias;
          const float d = p.softplus ? softplus(vv) : vv;
          tk = make_float4(d, d * x[i], Dc * x[i], p.z ? silu(zv[i]) : 1.f);
        }
        sTok[(seg * 8 + i) * kCh + cl] = tk;
      }
    }
    stage_bc<T, kN, kT>(sBC, Bg, Cg, N, L, tc, p.vec, tid, kThreads);
    __syncthreads();

    // ---- the recurrence over the chunk -------------------------------------
#pragma unroll 1
    for (int grp = 0; grp < kT / kP; ++grp) {
      float yp[kP];
#pragma unroll
      for (int k = 0; k < kP; ++k) {
        const int t = grp * kP + k;
        if (t % kM1SaveInterval == 0 && active && p.saved && tc + t < L) {
          float *dst = p.saved + ((b * D + c) * n_save + (tc + t) / kM1SaveInterval) * N;
          if (n0 < N) dst[n0] = h.x;
          if (n1 < N) dst[n1] = h.y;
        }
        const float4 tk = sTok[t * kCh + chl];
        const float4 bcv = sBC[t * kP + pr];
        const float2 a = ex2_2(mul2(splat2(tk.x), A2));
        h = fma2(a, h, mul2(splat2(tk.y), make_float2(bcv.x, bcv.y)));
        yp[k] = fmaf(bcv.w, h.y, bcv.z * h.x);
      }
      // transpose through shared memory: lane pr sums step grp*kP + pr
#pragma unroll
      for (int k = 0; k < kP; k += 4)
        *reinterpret_cast<float4 *>(ytile + pr * S::kRow + k) =
            make_float4(yp[k], yp[k + 1], yp[k + 2], yp[k + 3]);
      __syncwarp();
      const int t = grp * kP + pr;
      const float4 tk = sTok[t * kCh + chl];
      float y = tk.z;
#pragma unroll
      for (int q = 0; q < kP; ++q) y += ytile[q * S::kRow + pr];
      sOut[chl * S::kOut + t] = y * tk.w;
      __syncwarp();
    }
    __syncthreads();
  }

  if (active && p.final_state) {
    float *dst = p.final_state + (b * D + c) * N;
    if (n0 < N) dst[n0] = h.x;
    if (n1 < N) dst[n1] = h.y;
  }
}

template <typename T, int kN>
cudaError_t launch_t(const M1Params &p, cudaStream_t s) {
  using Lay = Layout<kN, kWarps>;
  const size_t smem = sizeof(float) * (size_t)FwdSmem<kN>::total;
  cudaError_t e = cudaFuncSetAttribute(m1_fwd_kernel<T, kN>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t per_group = p.D / p.G;
  dim3 grid((unsigned)(p.G * ((per_group + Lay::kCh - 1) / Lay::kCh)), (unsigned)p.B);
  m1_fwd_kernel<T, kN><<<grid, Lay::kThreads, smem, s>>>(p);
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

cudaError_t launch_m1_fwd(const M1Params &p, cudaStream_t s) {
  return p.io_bf16 ? launch_n<bf16>(p, s) : launch_n<float>(p, s);
}

}  // namespace msc
