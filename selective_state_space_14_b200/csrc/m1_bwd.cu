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
// pair of state indices; a CTA of kWarps warps owns kCh channels of one batch
// row and walks the sequence backwards.
//
//   * Blocks of kBlk = 32 steps.  The raw inputs of a block (u, delta, z,
//     dout of the CTA's channels, the B and C rows, and the forward's saved
//     states) are brought into shared memory by cp.async one block ahead,
//     into the other half of a double buffer, so no warp waits on a global
//     load; B and C are converted once per block into an f32 table of
//     (B[2p], B[2p+1], C[2p], C[2p+1]) per (step, pair).
//   * Windows of kS = 8 steps (the forward's saved-state interval), walked
//     in reverse.  Per window the lanes p < kS of a channel first derive the
//     per-token values of step p (softplus, gates) and share them through a
//     warp-private slot; every lane then re-runs the 8 forward steps from
//     the saved state, keeping a_t and h_{t-1} in registers, and walks them
//     backwards carrying mu = a lambda in registers.  dA accumulates per
//     thread in registers.
//   * Sums over the state pairs of a token (y for dz, ddelta, sum_n lambda B)
//     go through a warp-private tile: lane p of the channel adds step p's
//     pair partials in pair order and writes du, ddelta and dz.
//   * Sums over channels (dB, dC) go through a CTA tile: after one block
//     barrier each thread adds one (step, pair, tensor) entry over the CTA's
//     channels in channel order into the block accumulator.  At the end of a
//     block the kCS CTAs of a thread-block cluster add their accumulators in
//     rank order through distributed shared memory, one slice per rank, and
//     one partial per cluster goes to the workspace.
//   * A second kernel adds a group's partials in ascending order and the
//     per-(b, c) partials of dA, dD and dbias over the batch in ascending
//     order.  No atomics: the bits are the same on every run.
#include <cooperative_groups.h>

#include "m1_common.cuh"

namespace cg = cooperative_groups;

namespace msc {
namespace {

using namespace m1;

constexpr int kWarps = kM1BwdWarps;
constexpr int kS = kM1SaveInterval;  // steps per window (saved-state interval)
constexpr int kCS = kM1BwdCluster;   // CTAs per cluster
constexpr int kBlk = 32;             // steps per staged block and per dB/dC exchange
constexpr int kWin = kBlk / kS;      // windows per block
static_assert(kBlk % kS == 0, "a block holds whole windows");

template <typename T, int kN>
struct BwdSmem {
  using Lay = Layout<kN, kWarps>;
  static constexpr int kP = Lay::kP;
  static constexpr int kCh = Lay::kCh;
  static constexpr int kChW = Lay::kChPerWarp;
  // raw stage (one buffer; two are kept): tokens [4][kCh][kBlk] T in the
  // order u, delta, z, dout; bc [2][kN][kBlk] T; saved [kCh][kWin][kN] f32
  static constexpr int kTokBytes = 4 * kCh * kBlk * (int)sizeof(T);
  static constexpr int kBCBytes = 2 * kN * kBlk * (int)sizeof(T);
  static constexpr int kSavBytes = kCh * kWin * kN * 4;
  static constexpr int kStageBytes = kTokBytes + kBCBytes + kSavBytes;
  // byte offsets
  static constexpr int stage = 0;                                   // [2][kStageBytes]
  static constexpr int bcf = stage + 2 * kStageBytes;               // [2][kBlk][kP] float4
  // per (warp channel, step): (d, d, d x, d x) and (g, g), pairs ready for
  // the packed arithmetic of the state pairs
  static constexpr int tok = bcf + 2 * kBlk * kP * 16;              // [kWarps][kChW][kS] float4
  static constexpr int tokg = tok + kWarps * kChW * kS * 16;        // [kWarps][kChW][kS] float2
  static constexpr int kTileRow = kP + 1;                           // float4 per (chw, step) row
  static constexpr int tile = tokg + kWarps * kChW * kS * 8;        // [kWarps][kChW][kS][kP+1] float4
  static constexpr int rbc = tile + kWarps * kChW * kS * kTileRow * 16;  // [kCh][kS][kP] float4
  static constexpr int kAccRow = kBlk + 1;                          // floats per (tensor, n) row
  static constexpr int acc = rbc + kCh * kS * kP * 16;              // [2][kN][kBlk+1] f32
  static constexpr int total = acc + 2 * kN * kAccRow * 4;
  static_assert(kStageBytes % 16 == 0 && kTokBytes % 16 == 0 && kBCBytes % 16 == 0,
                "stage regions must stay 16-byte aligned");
};

template <typename T>
__device__ __forceinline__ float ldsm(const unsigned char *base, int i) {
  return to_f32(reinterpret_cast<const T *>(base)[i]);
}

// Issue the copies of block kb's raw inputs into one stage buffer: token runs
// of the CTA's channels, the B and C rows and the saved states of the block's
// windows.  With vec (16-byte aligned rows) every 16-byte piece is one
// cp.async that zero-fills what lies past the end of its row; otherwise the
// elements are copied one by one (synchronously).  Entries past L, past the
// last channel, past d_state or past the last saved state are never read as
// data: the consumers test those bounds themselves.
template <typename T, int kN>
__device__ __forceinline__ void issue_stage(const M1Params &p, unsigned char *st, int64_t b,
                                            int64_t c_first, int64_t c_end, const T *Bg,
                                            const T *Cg, int64_t kb, int64_t n_chunks,
                                            bool vec_sav, int tid) {
  using S = BwdSmem<T, kN>;
  constexpr int kCh = S::kCh;
  constexpr int kThreads = kWarps * 32;
  constexpr int E = 16 / (int)sizeof(T);  // elements per 16-byte piece
  constexpr int kPieces = kBlk / E;       // pieces per token / B / C run
  const int64_t L = p.L, N = p.N;
  const int64_t t0 = kb * kBlk;
  // token runs: (tensor k, channel cl, piece j)
#pragma unroll 1
  for (int u = tid; u < 4 * kCh * kPieces; u += kThreads) {
    const int j = u % kPieces, r = u / kPieces;
    const int cl = r % kCh, k = r / kCh;
    const int64_t c = c_first + cl;
    const void *src = k == 0 ? p.u : (k == 1 ? p.delta : (k == 2 ? p.z : p.dout));
    const bool ok = src != nullptr && c < c_end;
    const T *row = ok ? static_cast<const T *>(src) + (b * p.D + c) * L : static_cast<const T *>(p.u);
    const int64_t t = t0 + j * E;
    const int64_t left = L - t;
    const int valid = !ok || left <= 0 ? 0 : (left >= E ? E : (int)left);
    T *dst = reinterpret_cast<T *>(st) + r * kBlk + j * E;
    if (p.vec) {
      cp_async16(dst, valid > 0 ? row + t : row, valid * (int)sizeof(T));
    } else {
#pragma unroll
      for (int i = 0; i < E; ++i) dst[i] = i < valid ? row[t + i] : from_f32<T>(0.f);
    }
  }
  // B and C rows: (tensor k, state n, piece j)
#pragma unroll 1
  for (int u = tid; u < 2 * kN * kPieces; u += kThreads) {
    const int j = u % kPieces, r = u / kPieces;
    const int n = r % kN, k = r / kN;
    const bool ok = n < N;
    const T *row = ok ? (k == 0 ? Bg : Cg) + n * L : Bg;
    const int64_t t = t0 + j * E;
    const int64_t left = L - t;
    const int valid = !ok || left <= 0 ? 0 : (left >= E ? E : (int)left);
    T *dst = reinterpret_cast<T *>(st + S::kTokBytes) + r * kBlk + j * E;
    if (p.vec) {
      cp_async16(dst, valid > 0 ? row + t : row, valid * (int)sizeof(T));
    } else {
#pragma unroll
      for (int i = 0; i < E; ++i) dst[i] = i < valid ? row[t + i] : from_f32<T>(0.f);
    }
  }
  // saved states: (channel cl, window w, 4 states); a channel's windows are
  // consecutive in memory, kWin * N floats from chunk kb * kWin on
#pragma unroll 1
  for (int u = tid; u < kCh * kWin * (kN / 4); u += kThreads) {
    const int j = u % (kWin * (kN / 4)), cl = u / (kWin * (kN / 4));
    const int w = j / (kN / 4);
    const int64_t n = 4 * (j % (kN / 4));
    const int64_t c = c_first + cl;
    const int64_t chunk = kb * kWin + w;
    float *dst = reinterpret_cast<float *>(st + S::kTokBytes + S::kBCBytes) + (cl * kWin + w) * kN + n;
    const bool ok = c < c_end && chunk < n_chunks && n < N;
    const float *src = ok ? p.saved_in + ((b * p.D + c) * n_chunks + chunk) * N + n : p.saved_in;
    const int valid = ok ? (int)(N - n < 4 ? N - n : 4) : 0;
    if (vec_sav) {
      cp_async16(dst, src, valid * 4);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) dst[i] = i < valid ? src[i] : 0.f;
    }
  }
  cp_async_commit();
}

// Block kb's B and C rows (raw stage) -> bcf[tt][p] = (B[2p], B[2p+1], C[2p],
// C[2p+1]) in f32, zero past d_state and past L.
template <typename T, int kN>
__device__ __forceinline__ void convert_bc(const unsigned char *st, float4 *bcf, int64_t N,
                                           int64_t L, int64_t kb, int tid) {
  using S = BwdSmem<T, kN>;
  constexpr int kP = S::kP;
  const unsigned char *raw = st + S::kTokBytes;
  for (int i = tid; i < kBlk * kP; i += kWarps * 32) {
    const int tt = i % kBlk, pr = i / kBlk;
    const bool tin = kb * kBlk + tt < L;
    float v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int n = 2 * pr + (k & 1);
      v[k] = (tin && n < N) ? ldsm<T>(raw, ((k >> 1) * kN + n) * kBlk + tt) : 0.f;
    }
    bcf[tt * kP + pr] = make_float4(v[0], v[1], v[2], v[3]);
  }
}

template <typename T, int kN>
__global__ void __launch_bounds__(kWarps * 32, 4) m1_bwd_kernel(const M1Params p) {
  using S = BwdSmem<T, kN>;
  using Lay = Layout<kN, kWarps>;
  constexpr int kP = Lay::kP;
  constexpr int kCh = Lay::kCh;
  constexpr int kChW = Lay::kChPerWarp;
  constexpr int kThreads = Lay::kThreads;
  extern __shared__ float4 smem4[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(smem4);
  float4 *const sRbc = reinterpret_cast<float4 *>(smem + S::rbc);
  float *const acc = reinterpret_cast<float *>(smem + S::acc);
  cg::cluster_group cluster = cg::this_cluster();
  const unsigned rank = cluster.block_rank();

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int pr = lane % kP;
  const int chw = lane / kP;
  const int chl = warp * kChW + chw;
  float4 *const sTok = reinterpret_cast<float4 *>(smem + S::tok) + (warp * kChW + chw) * kS;
  float2 *const sTokG = reinterpret_cast<float2 *>(smem + S::tokg) + (warp * kChW + chw) * kS;
  float4 *const sTile =
      reinterpret_cast<float4 *>(smem + S::tile) + (warp * kChW + chw) * kS * S::kTileRow;
  const int64_t D = p.D, L = p.L, N = p.N, Bsz = p.B;
  const int64_t b = blockIdx.y;
  // a group's channels fill whole clusters; the CTAs past them own no channel
  const int64_t per_group = D / p.G;
  const int64_t ctas_per_group = (per_group + kCh - 1) / kCh;
  const int64_t ctas_padded = (ctas_per_group + kCS - 1) / kCS * kCS;
  const int64_t g = blockIdx.x / ctas_padded;
  const int64_t cig = blockIdx.x % ctas_padded;
  const int64_t c_first = g * per_group + cig * kCh;
  const int64_t c_end = cig < ctas_per_group ? (g + 1) * per_group : 0;
  const int64_t c = c_first + chl;
  const bool active = c < c_end;
  const int64_t part = blockIdx.x / kCS;  // dB/dC partial of this cluster
  const T *Bg = static_cast<const T *>(p.Bm) + (b * p.G + g) * N * L;
  const T *Cg = static_cast<const T *>(p.Cm) + (b * p.G + g) * N * L;
  const int64_t n_chunks = (L + kS - 1) / kS;
  const int64_t nb = (L + kBlk - 1) / kBlk;
  const bool vec_sav = (N % 4 == 0) && ((reinterpret_cast<uintptr_t>(p.saved_in) & 15) == 0);

  const int n0 = 2 * pr, n1 = 2 * pr + 1;
  float2 Ap = make_float2(0.f, 0.f);
  if (active) {
    if (n0 < N) Ap.x = p.A[c * N + n0];
    if (n1 < N) Ap.y = p.A[c * N + n1];
  }
  const float2 A2 = mul2(Ap, splat2(kLog2e));
  const float bias_c = (active && p.bias) ? p.bias[c] : 0.f;
  const float D_c = (active && p.Dp) ? p.Dp[c] : 0.f;
  float2 mu = make_float2(0.f, 0.f);  // a_{t+1} lambda_{t+1}, handed backwards
  float2 dA = make_float2(0.f, 0.f);  // this (b, c)'s dA for the pair
  float dD_l = 0.f, dbias_l = 0.f;    // per lane (the tokens it finishes)

  unsigned char *const stage0 = smem + S::stage;
  float4 *const bcf0 = reinterpret_cast<float4 *>(smem + S::bcf);

  // ---- prologue: the last block's inputs (and the one before, in flight) ----
  issue_stage<T, kN>(p, stage0 + ((nb - 1) & 1) * S::kStageBytes, b, c_first, c_end, Bg, Cg,
                     nb - 1, n_chunks, vec_sav, tid);
  if (nb >= 2) {
    issue_stage<T, kN>(p, stage0 + ((nb - 2) & 1) * S::kStageBytes, b, c_first, c_end, Bg, Cg,
                       nb - 2, n_chunks, vec_sav, tid);
    cp_async_wait<1>();
  } else {
    cp_async_wait<0>();
  }
  __syncthreads();
  convert_bc<T, kN>(stage0 + ((nb - 1) & 1) * S::kStageBytes, bcf0 + ((nb - 1) & 1) * kBlk * kP,
                    N, L, nb - 1, tid);
  __syncthreads();

  for (int64_t kb = nb - 1; kb >= 0; --kb) {
    const unsigned char *const st = stage0 + (kb & 1) * S::kStageBytes;
    const float4 *const bcf = bcf0 + (kb & 1) * kBlk * kP;
    const float *const sav = reinterpret_cast<const float *>(st + S::kTokBytes + S::kBCBytes);

    for (int w = kWin - 1; w >= 0; --w) {
      const int tw = w * kS;  // the window's first step within the block
      const int64_t t_win = kb * kBlk + tw;

      // ---- lanes p < kS: the per-token values of step p --------------------
      float tx = 0.f, tD = 0.f, tdx = 0.f, tsig = 0.f, tdzf = 0.f, tg = 0.f;
      if (pr < kS) {
        float4 tk = make_float4(0.f, 0.f, 0.f, 0.f);
        float2 tk2 = make_float2(0.f, 0.f);
        const int tb = tw + pr;
        if (active && t_win + pr < L) {
          const float x = ldsm<T>(st, (0 * kCh + chl) * kBlk + tb);
          const float v = ldsm<T>(st, (1 * kCh + chl) * kBlk + tb) + bias_c;
          const float dy = ldsm<T>(st, (3 * kCh + chl) * kBlk + tb);
          const float d = p.softplus ? softplus(v) : v;
          float gz = dy, dzf = 0.f;
          if (p.z) {
            const float zv = ldsm<T>(st, (2 * kCh + chl) * kBlk + tb);
            const float sz = sigmoid(zv);
            gz = dy * (zv * sz);
            dzf = dy * (sz * fmaf(zv, 1.f - sz, 1.f));
          }
          tk = make_float4(d, d, d * x, d * x);
          tk2 = make_float2(gz, gz);
          tx = x; tD = d; tdx = D_c * x; tg = gz; tdzf = dzf;
          tsig = p.softplus ? sigmoid(v) : 1.f;
        }
        sTok[pr] = tk;
        sTokG[pr] = tk2;
      }
      __syncwarp();

      // ---- forward over the window from the saved state ---------------------
      float2 h = make_float2(0.f, 0.f);
      if (active && kb * kWin + w < n_chunks) {
        const float2 sv = *reinterpret_cast<const float2 *>(sav + (chl * kWin + w) * kN + n0);
        h = make_float2(n0 < N ? sv.x : 0.f, n1 < N ? sv.y : 0.f);
      }
      float2 a[kS], hp[kS];
      float yv[kS];
#pragma unroll
      for (int t = 0; t < kS; ++t) {
        const float4 tk = sTok[t];
        const float4 bcv = bcf[(tw + t) * kP + pr];
        a[t] = ex2_2(mul2(make_float2(tk.x, tk.y), A2));
        hp[t] = h;
        h = fma2(a[t], h, mul2(make_float2(tk.z, tk.w), make_float2(bcv.x, bcv.y)));
        yv[t] = fmaf(bcv.w, h.y, bcv.z * h.x);
      }
      // ---- backwards over the window ----------------------------------------
#pragma unroll
      for (int t = kS - 1; t >= 0; --t) {
        const float4 bcv = bcf[(tw + t) * kP + pr];
        const float4 tk = sTok[t];
        const float2 g2 = sTokG[t];
        const float2 dt2 = make_float2(tk.x, tk.y), dtx2 = make_float2(tk.z, tk.w);
        const float2 Bv = make_float2(bcv.x, bcv.y), Cv = make_float2(bcv.z, bcv.w);
        const float2 lam = fma2(g2, Cv, mu);
        const float2 q = mul2(a[t], hp[t]);
        const float2 hcur = fma2(dtx2, Bv, q);
        const float2 dC = mul2(g2, hcur);
        const float2 dB = mul2(lam, dtx2);
        const float2 lq = mul2(lam, q);
        dA = fma2(dt2, lq, dA);
        sTile[t * S::kTileRow + pr] =
            make_float4(yv[t], fmaf(Ap.y, lq.y, Ap.x * lq.x), fmaf(lam.y, Bv.y, lam.x * Bv.x), 0.f);
        sRbc[(chl * kS + t) * kP + pr] = make_float4(dB.x, dB.y, dC.x, dC.y);
        mu = mul2(a[t], lam);
      }
      __syncwarp();

      // ---- lanes p < kS: step p's sums over the pairs, in pair order --------
      if (pr < kS) {
        float y = tdx, dd = 0.f, sb = 0.f;
#pragma unroll
        for (int qq = 0; qq < kP; ++qq) {
          const float4 r = sTile[pr * S::kTileRow + qq];
          y += r.x; dd += r.y; sb += r.z;
        }
        const int64_t t = t_win + pr;
        if (active && t < L) {
          const int64_t i = (b * D + c) * L + t;
          const float draw = fmaf(tx, sb, dd) * tsig;
          static_cast<T *>(p.du)[i] = from_f32<T>(fmaf(tD, sb, tg * D_c));
          static_cast<T *>(p.ddelta)[i] = from_f32<T>(draw);
          if (p.dz) static_cast<T *>(p.dz)[i] = from_f32<T>(y * tdzf);
          dbias_l += draw;
          dD_l = fmaf(tg, tx, dD_l);
        }
      }
      __syncthreads();  // every channel's dB/dC entries of the window are in place

      // ---- dB, dC of the window's steps: the CTA's channels in channel order --
      const float2 *const r2 = reinterpret_cast<const float2 *>(sRbc);
      for (int it = tid; it < kS * kP * 2; it += kThreads) {
        const int half = it & 1, qq = (it >> 1) % kP, t = (it >> 1) / kP;
        float2 s = r2[(t * kP + qq) * 2 + half];
#pragma unroll
        for (int cl = 1; cl < kCh; ++cl) s = add2(s, r2[((cl * kS + t) * kP + qq) * 2 + half]);
        float *row = acc + (half * kN + 2 * qq) * S::kAccRow + tw + t;
        row[0] = s.x;
        row[S::kAccRow] = s.y;
      }
      __syncthreads();  // the entries are free for the next window
    }

    // ---- end of block: the cluster's sums in rank order, next block's inputs --
    cp_async_wait<0>();  // block kb - 1's inputs (issued one block ago) have landed
    cluster.sync();      // accumulators complete; block kb's buffers free
    {
      constexpr int E = 2 * kN * kBlk;
      constexpr int per = E / kCS;
      for (int e = (int)rank * per + tid; e < ((int)rank + 1) * per; e += kThreads) {
        const int te = e / (kN * kBlk), n = (e / kBlk) % kN, tt = e % kBlk;
        const int off = (te * kN + n) * S::kAccRow + tt;
        float s = *(cluster.map_shared_rank(acc, 0) + off);
#pragma unroll
        for (int qq = 1; qq < kCS; ++qq) s += *(cluster.map_shared_rank(acc, qq) + off);
        const int64_t t = kb * kBlk + tt;
        if (n < N && t < L) p.ws_bc[(((part * Bsz + b) * 2 + te) * N + n) * L + t] = s;
      }
    }
    if (kb >= 1)
      convert_bc<T, kN>(stage0 + ((kb - 1) & 1) * S::kStageBytes, bcf0 + ((kb - 1) & 1) * kBlk * kP,
                        N, L, kb - 1, tid);
    if (kb >= 2)
      issue_stage<T, kN>(p, stage0 + (kb & 1) * S::kStageBytes, b, c_first, c_end, Bg, Cg, kb - 2,
                         n_chunks, vec_sav, tid);
    // peers are done reading (the values read are consumed before the arrive);
    // the new B/C table is visible CTA-wide
    __syncthreads();
    asm volatile("barrier.cluster.arrive.relaxed.aligned;\n" ::: "memory");
    asm volatile("barrier.cluster.wait.aligned;\n" ::: "memory");
  }

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
    if (pr == 0) {
      m[N] = dD_l;
      m[N + 1] = dbias_l;
    }
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

int64_t ctas_padded_per_group(int64_t D, int64_t N, int64_t G) {
  const int64_t kch = m1_bwd_cta_channels(N);
  const int64_t ctas = ((D / G) + kch - 1) / kch;
  return (ctas + kCS - 1) / kCS * kCS;
}

template <typename T, int kN>
cudaError_t launch_t(const M1Params &p, cudaStream_t s) {
  using Lay = Layout<kN, kWarps>;
  const size_t smem = (size_t)BwdSmem<T, kN>::total;
  cudaError_t err = cudaFuncSetAttribute(m1_bwd_kernel<T, kN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int64_t grid_x = p.G * ctas_padded_per_group(p.D, p.N, p.G);
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

// Partials: one per cluster of CTAs; a group's channels fill whole clusters.
int64_t m1_bwd_partials(int64_t D, int64_t N, int64_t G) {
  return G * ctas_padded_per_group(D, N, G) / kM1BwdCluster;
}

size_t m1_bwd_workspace_bytes(int64_t B, int64_t D, int64_t N, int64_t L, int64_t G) {
  const int64_t n_part = m1_bwd_partials(D, N, G);
  size_t bc = sizeof(float) * (size_t)(n_part * B * 2 * N * L);
  bc = (bc + 255) / 256 * 256;
  return bc + sizeof(float) * (size_t)(B * D * (N + 2));
}

cudaError_t launch_m1_bwd(const M1Params &p, cudaStream_t s) {
  switch (p.io) {
    case 1: return launch_n<bf16>(p, s);
    case 2: return launch_n<f16>(p, s);
    default: return launch_n<float>(p, s);
  }
}

}  // namespace msc
