// m1_bwd.cu -- Mamba-1 selective scan, backward through the recurrent state
// (sm_100a): backpropagation through time over the SSM state, mamba-rs 0.7.0
// README, "Features".
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
//     dout of the CTA's channels, the B and C rows) are brought into shared
//     memory by cp.async one block ahead, into the other half of a double
//     buffer, from a table of row addresses built once per CTA, so no warp
//     waits on a global load; B and C are converted once per block, eight
//     steps of a pair at a time, into an f32 table of (B[2p], B[2p+1], C[2p],
//     C[2p+1]) per (step, pair).  Each thread loads its pair of the
//     forward's saved state straight into registers, one window ahead.
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
  // order u, delta, z, dout; bc [2][kN][kBCRow] T
  static constexpr int kTokBytes = 4 * kCh * kBlk * (int)sizeof(T);
  // B and C rows padded by 16 bytes: the eight rows a conversion reads at
  // once fall on different banks
  static constexpr int kBCRow = kBlk + 16 / (int)sizeof(T);
  static constexpr int kBCBytes = 2 * kN * kBCRow * (int)sizeof(T);
  static constexpr int kStageBytes = kTokBytes + kBCBytes;
  static constexpr int kRows = 4 * kCh + 2 * kN;  // staged rows: tokens, then B and C
  // byte offsets
  static constexpr int stage = 0;                                   // [2][kStageBytes]
  static constexpr int bcf = stage + 2 * kStageBytes;               // [2][kBlk][kP] float4
  // per (warp channel, step): (d, d, d x, d x) and (g, g), pairs ready for
  // the packed arithmetic of the state pairs
  // (per channel kS + 1 slots: the channels of a warp, read at the same step,
  // fall on different banks)
  static constexpr int kTokRow = kS + 1;
  static constexpr int tok = bcf + 2 * kBlk * kP * 16;              // [kWarps][kChW][kTokRow] float4
  static constexpr int tokg = tok + kWarps * kChW * kTokRow * 16;   // [kWarps][kChW][kTokRow] float2
  static constexpr int kTileRow = kP + 1;                           // float4 per (chw, step) row
  static constexpr int tile = (tokg + kWarps * kChW * kTokRow * 8 + 15) / 16 * 16;  // [kWarps][kChW][kS][kP+1] float4
  static constexpr int rbc = tile + kWarps * kChW * kS * kTileRow * 16;  // [kCh][kS][kP] float4
  static constexpr int kAccRow = kBlk + 1;                          // floats per (tensor, n) row
  // the block's dB/dC sums over the CTA's channels, [2][kN][kBlk+1] f32, one
  // buffer per block parity (the cluster reads one while the next fills)
  static constexpr int kAccFloats = 2 * kN * kAccRow;
  static constexpr int acc = rbc + kCh * kS * kP * 16;              // [2 parities]
  // global address of every staged row at t = 0 (0: absent row, zero-filled)
  static constexpr int rows = (acc + 2 * kAccFloats * 4 + 7) / 8 * 8;  // [kRows] pointers
  static constexpr int total = rows + kRows * 8;
  static_assert(kStageBytes % 16 == 0 && kTokBytes % 16 == 0 && kBCBytes % 16 == 0,
                "stage regions must stay 16-byte aligned");
};

template <typename T>
__device__ __forceinline__ float ldsm(const unsigned char *base, int i) {
  return to_f32(reinterpret_cast<const T *>(base)[i]);
}

// The global address of every row the stage copies, at t = 0, once per CTA:
// token rows (tensor k of u, delta, z, dout; channel cl) at k * kCh + cl, then
// the B and C rows (state n) at 4 kCh + k * kN + n.  Rows that do not exist
// (absent z, a channel past the group, a state past d_state) hold 0.
template <typename T, int kN>
__device__ __forceinline__ void fill_rows(const M1Params &p, const T **rows, int64_t b,
                                          int64_t c_first, int64_t c_end, const T *Bg,
                                          const T *Cg, int tid) {
  using S = BwdSmem<T, kN>;
  constexpr int kCh = S::kCh;
  for (int r = tid; r < S::kRows; r += kWarps * 32) {
    const T *row = nullptr;
    if (r < 4 * kCh) {
      const int k = r / kCh, cl = r % kCh;
      const void *src = k == 0 ? p.u : (k == 1 ? p.delta : (k == 2 ? p.z : p.dout));
      const int64_t c = c_first + cl;
      if (src != nullptr && c < c_end) row = static_cast<const T *>(src) + (b * p.D + c) * p.L;
    } else {
      const int k = (r - 4 * kCh) / kN, n = (r - 4 * kCh) % kN;
      if (n < p.N) row = (k == 0 ? Bg : Cg) + n * p.L;
    }
    rows[r] = row;
  }
}

// Issue the copies of block kb's raw inputs into one stage buffer: the token
// runs of the CTA's channels and the B and C rows, 16-byte pieces taken from
// the row table.  With vec (16-byte aligned rows) every piece is one cp.async
// that zero-fills what lies past the end of its row or past L; otherwise the
// elements are copied one by one (synchronously).  Absent rows are zeros.
template <typename T, int kN>
__device__ __forceinline__ void issue_stage(const M1Params &p, unsigned char *st,
                                            const T *const *rows, int64_t kb, int tid) {
  using S = BwdSmem<T, kN>;
  constexpr int E = 16 / (int)sizeof(T);  // elements per 16-byte piece
  constexpr int kPieces = kBlk / E;       // pieces per row
  static_assert((kPieces & (kPieces - 1)) == 0, "pieces per row: a power of two");
  const int64_t L = p.L;
  const int64_t t0 = kb * kBlk;
  const T *const fallback = static_cast<const T *>(p.Bm);  // a valid address for empty copies
#pragma unroll 1
  for (int u = tid; u < S::kRows * kPieces; u += kWarps * 32) {
    const int j = u & (kPieces - 1), r = u / kPieces;
    const T *row = rows[r];
    const int64_t t = t0 + j * E;
    const int64_t left = L - t;
    const int valid = row == nullptr || left <= 0 ? 0 : (left >= E ? E : (int)left);
    T *dst = r < 4 * S::kCh
                 ? reinterpret_cast<T *>(st) + r * kBlk + j * E
                 : reinterpret_cast<T *>(st + S::kTokBytes) + (r - 4 * S::kCh) * S::kBCRow + j * E;
    if (p.vec) {
      cp_async16(dst, valid > 0 ? row + t : fallback, valid * (int)sizeof(T));
    } else {
#pragma unroll
      for (int i = 0; i < E; ++i) dst[i] = i < valid ? row[t + i] : from_f32<T>(0.f);
    }
  }
  cp_async_commit();
}

// Block kb's B and C rows (raw stage) -> bcf[tt][p] = (B[2p], B[2p+1], C[2p],
// C[2p+1]) in f32.  The stage already holds zeros past d_state and past L.
// One unit is a pair p and 8 consecutive steps: four 8-element row pieces in,
// eight float4 out.
template <typename T, int kN>
__device__ __forceinline__ void convert_bc(const unsigned char *st, float4 *bcf, int tid) {
  using S = BwdSmem<T, kN>;
  constexpr int kP = S::kP;
  const T *raw = reinterpret_cast<const T *>(st + S::kTokBytes);
  for (int u = tid; u < kP * (kBlk / 8); u += kWarps * 32) {
    const int pr = u % kP, seg = u / kP;
    float v[4][8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const T *src = raw + ((k >> 1) * kN + 2 * pr + (k & 1)) * S::kBCRow + seg * 8;
      if constexpr (sizeof(T) == 2) {
        const uint4 w = *reinterpret_cast<const uint4 *>(src);
        unpack2<T>(w.x, v[k][0], v[k][1]);
        unpack2<T>(w.y, v[k][2], v[k][3]);
        unpack2<T>(w.z, v[k][4], v[k][5]);
        unpack2<T>(w.w, v[k][6], v[k][7]);
      } else {
        const float4 a = reinterpret_cast<const float4 *>(src)[0];
        const float4 c = reinterpret_cast<const float4 *>(src)[1];
        v[k][0] = a.x; v[k][1] = a.y; v[k][2] = a.z; v[k][3] = a.w;
        v[k][4] = c.x; v[k][5] = c.y; v[k][6] = c.z; v[k][7] = c.w;
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
      bcf[(seg * 8 + i) * kP + pr] = make_float4(v[0][i], v[1][i], v[2][i], v[3][i]);
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
  float *const acc0 = reinterpret_cast<float *>(smem + S::acc);
  cg::cluster_group cluster = cg::this_cluster();
  const unsigned rank = cluster.block_rank();

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int pr = lane % kP;
  const int chw = lane / kP;
  const int chl = warp * kChW + chw;
  float4 *const sTok = reinterpret_cast<float4 *>(smem + S::tok) + (warp * kChW + chw) * S::kTokRow;
  float2 *const sTokG = reinterpret_cast<float2 *>(smem + S::tokg) + (warp * kChW + chw) * S::kTokRow;
  float4 *const sTile =
      reinterpret_cast<float4 *>(smem + S::tile) + (warp * kChW + chw) * kS * S::kTileRow;
  const int64_t D = p.D, L = p.L, N = p.N, Bsz = p.B;
  const int64_t ldN = p.ldN, ns = p.n0;  // row length of A and the states; this slab's first state
  const bool finish = p.slab == kSlabWhole || p.slab == kSlabLast;  // this launch finishes the tokens
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
  const T *Bg = static_cast<const T *>(p.Bm) + ((b * p.G + g) * ldN + ns) * L;
  const T *Cg = static_cast<const T *>(p.Cm) + ((b * p.G + g) * ldN + ns) * L;
  const int64_t n_chunks = (L + kS - 1) / kS;
  // this CTA's blocks: the whole sequence, or time segment blockIdx.z
  const int64_t seg = blockIdx.z, n_seg = gridDim.z;
  const int64_t tb = p.seg_len > 0 ? seg * p.seg_len : 0;
  const int64_t te = p.seg_len > 0 && tb + p.seg_len < L ? tb + p.seg_len : L;
  const int64_t kb_lo = tb / kBlk, kb_hi = (te + kBlk - 1) / kBlk;
  const int n0 = 2 * pr, n1 = 2 * pr + 1;
  // this thread's pair of the saved states, one window ahead (windows run
  // backwards: chunk kb * kWin + w)
  const float *const sav_row = p.saved_in + (b * D + c) * n_chunks * ldN + ns;
  auto load_saved = [&](int64_t chunk) {
    float2 v = make_float2(0.f, 0.f);
    if (active && chunk >= 0 && chunk < n_chunks) {
      if (n0 < N) v.x = sav_row[chunk * ldN + n0];
      if (n1 < N) v.y = sav_row[chunk * ldN + n1];
    }
    return v;
  };

  float2 Ap = make_float2(0.f, 0.f);
  if (active) {
    if (n0 < N) Ap.x = p.A[c * ldN + ns + n0];
    if (n1 < N) Ap.y = p.A[c * ldN + ns + n1];
  }
  const float2 A2 = mul2(Ap, splat2(kLog2e));
  const float bias_c = (active && p.bias) ? p.bias[c] : 0.f;
  const float D_c = (active && p.Dp && finish) ? p.Dp[c] : 0.f;  // the D terms join once
  float2 mu = make_float2(0.f, 0.f);  // a_{t+1} lambda_{t+1}, handed backwards
  if (seg < n_seg - 1 && active) {     // the carry entering this segment from the right
    const float *cs = p.seg_ws + p.B * D * N * (n_seg + seg + 1) + (b * D + c) * N;
    if (n0 < N) mu.x = cs[n0];
    if (n1 < N) mu.y = cs[n1];
  }
  float2 dA = make_float2(0.f, 0.f);  // this (b, c)'s dA for the pair
  float dD_l = 0.f, dbias_l = 0.f;    // per lane (the tokens it finishes)

  unsigned char *const stage0 = smem + S::stage;
  float4 *const bcf0 = reinterpret_cast<float4 *>(smem + S::bcf);
  const T **const rows = reinterpret_cast<const T **>(smem + S::rows);

  // ---- prologue: the row table; the last block's inputs (and the one
  // before, in flight); the first window's saved state ------------------------
  fill_rows<T, kN>(p, rows, b, c_first, c_end, Bg, Cg, tid);
  __syncthreads();
  issue_stage<T, kN>(p, stage0 + ((kb_hi - 1) & 1) * S::kStageBytes, rows, kb_hi - 1, tid);
  if (kb_hi - kb_lo >= 2) {
    issue_stage<T, kN>(p, stage0 + ((kb_hi - 2) & 1) * S::kStageBytes, rows, kb_hi - 2, tid);
    cp_async_wait<1>();
  } else {
    cp_async_wait<0>();
  }
  float2 sv_next = load_saved((kb_hi - 1) * kWin + kWin - 1);
  __syncthreads();
  convert_bc<T, kN>(stage0 + ((kb_hi - 1) & 1) * S::kStageBytes,
                    bcf0 + ((kb_hi - 1) & 1) * kBlk * kP, tid);
  __syncthreads();

  for (int64_t kb = kb_hi - 1; kb >= kb_lo; --kb) {
    const unsigned char *const st = stage0 + (kb & 1) * S::kStageBytes;
    const float4 *const bcf = bcf0 + (kb & 1) * kBlk * kP;
    float *const acc = acc0 + (kb & 1) * S::kAccFloats;

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
      float2 h = sv_next;
      sv_next = load_saved(kb * kWin + w - 1);  // the next window walked
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
          if (p.slab != kSlabWhole) {  // the sums over the states cross the slabs
            float *tp = p.tok_part + i;
            const int64_t plane = Bsz * D * L;
            if (p.slab != kSlabFirst) {
              y = tp[0] + y;
              dd = tp[plane] + dd;
              sb = tp[2 * plane] + sb;
            }
            if (!finish) {
              tp[0] = y;
              tp[plane] = dd;
              tp[2 * plane] = sb;
            }
          }
        }
        if (finish && active && t < L) {
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
      for (int it = tid; it < kS * kP; it += kThreads) {
        const int qq = it % kP, t = it / kP;
        const float4 v0 = sRbc[t * kP + qq];
        float2 sb = make_float2(v0.x, v0.y), sc = make_float2(v0.z, v0.w);
#pragma unroll
        for (int cl = 1; cl < kCh; ++cl) {
          const float4 v = sRbc[(cl * kS + t) * kP + qq];
          sb = add2(sb, make_float2(v.x, v.y));
          sc = add2(sc, make_float2(v.z, v.w));
        }
        float *rb = acc + 2 * qq * S::kAccRow + tw + t;
        float *rc = acc + (kN + 2 * qq) * S::kAccRow + tw + t;
        rb[0] = sb.x;
        rb[S::kAccRow] = sb.y;
        rc[0] = sc.x;
        rc[S::kAccRow] = sc.y;
      }
      __syncthreads();  // the entries are free for the next window
    }

    // ---- end of block: next block's inputs, the cluster's sums in rank order --
    cp_async_wait<0>();  // block kb - 1's inputs (issued one block ago) have landed
    cluster.sync();      // every CTA's accumulators of block kb are complete; block kb's buffers free
    if (kb - 1 >= kb_lo)
      convert_bc<T, kN>(stage0 + ((kb - 1) & 1) * S::kStageBytes, bcf0 + ((kb - 1) & 1) * kBlk * kP,
                        tid);
    if (kb - 2 >= kb_lo) issue_stage<T, kN>(p, stage0 + (kb & 1) * S::kStageBytes, rows, kb - 2, tid);
    __syncthreads();  // the new B/C table is visible CTA-wide
    // The peers' accumulators of block kb stay intact until their block kb - 2,
    // which starts after the next cluster barrier: this CTA reaches that
    // barrier only after these reads.
    {
      constexpr int E = 2 * kN * kBlk;
      constexpr int per = E / kCS;
      const float *racc[kCS];
#pragma unroll
      for (int qq = 0; qq < kCS; ++qq) racc[qq] = cluster.map_shared_rank(acc, qq);
      for (int e = (int)rank * per + tid; e < ((int)rank + 1) * per; e += kThreads) {
        const int te = e / (kN * kBlk), n = (e / kBlk) % kN, tt = e % kBlk;
        const int off = (te * kN + n) * S::kAccRow + tt;
        float s = racc[0][off];
#pragma unroll
        for (int qq = 1; qq < kCS; ++qq) s += racc[qq][off];
        const int64_t t = kb * kBlk + tt;
        if (n < N && t < L) p.ws_bc[(((part * Bsz + b) * 2 + te) * ldN + ns + n) * L + t] = s;
      }
    }
  }
  // no CTA leaves while a peer may still read its accumulators
  cluster.sync();

  // per-(b, c) partials: dA (per thread), dD and dbias (the lanes of a channel
  // added by a fixed butterfly), dh0 = the carry left after step 0
#pragma unroll
  for (int off = kP / 2; off > 0; off >>= 1) {
    dD_l += __shfl_xor_sync(0xffffffffu, dD_l, off, kP);
    dbias_l += __shfl_xor_sync(0xffffffffu, dbias_l, off, kP);
  }
  if (active) {
    float *m = p.ws_misc + ((seg * Bsz + b) * D + c) * (ldN + 2);
    if (n0 < N) m[ns + n0] = dA.x;
    if (n1 < N) m[ns + n1] = dA.y;
    if (p.dh0 && seg == 0) {
      if (n0 < N) p.dh0[(b * D + c) * ldN + ns + n0] = mu.x;
      if (n1 < N) p.dh0[(b * D + c) * ldN + ns + n1] = mu.y;
    }
    if (pr == 0 && finish) {
      m[ldN] = dD_l;
      m[ldN + 1] = dbias_l;
    }
  }
}

// dB/dC: sum of a group's partials in ascending order; dA, dD, dbias: sum of
// the per-(segment, b, c) partials over the segments and the batch in
// ascending order.
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
      const int64_t n_seg = p.seg_len > 0 ? (L + p.seg_len - 1) / p.seg_len : 1;
      float s = 0.f;
      for (int64_t q = 0; q < n_seg * Bsz; ++q) s += p.ws_misc[(q * D + c) * (N + 2) + k];
      if (k < N) p.dA[c * N + k] = s;
      else if (k == N) { if (p.dD) p.dD[c] = s; }
      else if (p.dbias) p.dbias[c] = s;
    }
  }
}

// Time segments, first pass: per state element, segment blockIdx.y walked
// backwards from a zero adjoint carry, as the backward walks it (mu <- a_t
// (g_t C_t + mu)), without the states: the product of its decays and the
// carry it reaches at its left end, to seg_ws.  A thread takes one pair of
// states of one (b, c); the kPw lanes of a channel (kPw the power of two at
// or above its pairs) take the token values of kPw steps at a time, one step
// each, and hand them round by shuffles.
template <typename T, int kPw>
__global__ void __launch_bounds__(256) m1_bwd_seg_sum_kernel(const M1Params p) {
  const int64_t N = p.N, D = p.D, L = p.L;
  const int64_t kPr = (N + 1) / 2;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int q = (int)(threadIdx.x % kPw);
  const int64_t bc = i / kPw;
  const bool live = bc < p.B * D;  // every lane of a warp stays for the shuffles
  const bool act = live && q < kPr;
  const int64_t c = live ? bc % D : 0, b = live ? bc / D : 0;
  const int64_t seg = blockIdx.y, n_seg = gridDim.y;
  const int64_t tb = seg * p.seg_len, te = tb + p.seg_len < L ? tb + p.seg_len : L;
  const int64_t g = c / (D / p.G);
  const int64_t n0 = 2 * (int64_t)q, n1 = n0 + 1;
  const bool has0 = act && n0 < N, has1 = act && n1 < N;
  const float2 A2 = mul2(make_float2(has0 ? p.A[c * N + n0] : 0.f, has1 ? p.A[c * N + n1] : 0.f),
                         splat2(kLog2e));
  const float bias = (live && p.bias) ? p.bias[c] : 0.f;
  const int64_t row = (live ? bc : 0) * L;
  const T *drow = static_cast<const T *>(p.delta) + row;
  const T *yrow = static_cast<const T *>(p.dout) + row;
  const T *zrow = p.z ? static_cast<const T *>(p.z) + row : nullptr;
  const T *c0 = static_cast<const T *>(p.Cm) + ((b * p.G + g) * N + (has0 ? n0 : 0)) * L;
  const T *c1 = has1 ? c0 + L : c0;
  float2 mu = make_float2(0.f, 0.f), dec = make_float2(1.f, 1.f);
  for (int64_t th = te - 1; th >= tb; th -= kPw) {
    // this lane's step of the group: th - q
    const int64_t tq = th - q;
    float d_own = 0.f, g_own = 0.f;
    if (live && tq >= tb) {
      const float v = to_f32(drow[tq]) + bias;
      d_own = p.softplus ? softplus(v) : v;
      g_own = to_f32(yrow[tq]);
      if (zrow) {
        const float zv = to_f32(zrow[tq]);
        g_own = g_own * (zv * sigmoid(zv));
      }
    }
#pragma unroll
    for (int s = 0; s < kPw; ++s) {
      const int64_t t = th - s;
      if (t < tb) break;  // the same for every thread of the block
      const float d = __shfl_sync(0xffffffffu, d_own, s, kPw);
      const float gz = __shfl_sync(0xffffffffu, g_own, s, kPw);
      if (act) {
        const float2 a = ex2_2(mul2(splat2(d), A2));
        const float2 Cv = make_float2(has0 ? to_f32(c0[t]) : 0.f, has1 ? to_f32(c1[t]) : 0.f);
        mu = mul2(a, fma2(splat2(gz), Cv, mu));
        dec = mul2(dec, a);
      }
    }
  }
  if (!act) return;
  const int64_t elems = p.B * D * N;
  float *dd = p.seg_ws + elems * seg + bc * N;
  float *mm = p.seg_ws + elems * (n_seg + seg) + bc * N;
  if (has0) {
    dd[n0] = dec.x;
    mm[n0] = mu.x;
  }
  if (has1) {
    dd[n1] = dec.y;
    mm[n1] = mu.y;
  }
}

// the summary pass: kPw lanes per channel, the power of two at or above its
// state pairs (d_state <= 64: at most 32)
template <typename T, int kPw>
cudaError_t launch_seg_sum_w(const M1Params &p, int64_t n_seg, cudaStream_t s) {
  const int64_t items = p.B * p.D * kPw;
  const dim3 grid((unsigned)((items + 255) / 256), (unsigned)n_seg);
  m1_bwd_seg_sum_kernel<T, kPw><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}
template <typename T>
cudaError_t launch_seg_sum(const M1Params &p, int64_t n_seg, cudaStream_t s) {
  const int64_t pr = (p.N + 1) / 2;
  if (pr <= 1) return launch_seg_sum_w<T, 1>(p, n_seg, s);
  if (pr <= 2) return launch_seg_sum_w<T, 2>(p, n_seg, s);
  if (pr <= 4) return launch_seg_sum_w<T, 4>(p, n_seg, s);
  if (pr <= 8) return launch_seg_sum_w<T, 8>(p, n_seg, s);
  if (pr <= 16) return launch_seg_sum_w<T, 16>(p, n_seg, s);
  return launch_seg_sum_w<T, 32>(p, n_seg, s);
}

// The segments' summaries combined from the sequence's end: segment s takes
// the carry entering it from the right, x, to decay_s x + carry_s at its left
// end, so the carry entering segment s is the composition of segments
// n_seg - 1 .. s + 1 applied to 0.  A warp takes one state element, lane l
// segment n_seg - 1 - l (lane order = the order of the walk), composed with
// the warp-shuffle scan of the linear-recurrence monoid; the carry leaving
// segment s goes over carry_s, which only this warp reads.
__global__ void m1_bwd_seg_combine_kernel(const M1Params p, int n_seg) {
  const int64_t elems = p.B * p.D * p.N;
  const int lane = threadIdx.x & 31;
  const int s = n_seg - 1 - lane;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t e = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); e < elems;
       e += warps) {
    float dc = 1.f, st = 0.f;  // lanes past the segments compose as the identity
    if (s >= 0) {
      dc = p.seg_ws[elems * s + e];
      st = p.seg_ws[elems * (n_seg + s) + e];
    }
    float pe, he;
    warp_scan_fwd(dc, st, pe, he);
    if (s >= 1) p.seg_ws[elems * (n_seg + s) + e] = fmaf(dc, he, st);  // inclusive, applied to 0
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
  const int64_t grid_x = p.G * ctas_padded_per_group(p.D, kN, p.G);  // the layout's channels per CTA
  cudaLaunchConfig_t cfg = {};
  const int64_t n_seg = p.seg_len > 0 ? (p.L + p.seg_len - 1) / p.seg_len : 1;
  cfg.gridDim = dim3((unsigned)grid_x, (unsigned)p.B, (unsigned)n_seg);
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
  return cudaLaunchKernelEx(&cfg, m1_bwd_kernel<T, kN>, p);
}

// one slab (or the whole d_state); slabs all run at the widest layout, so
// that every slab has the same CTAs and dB/dC partials
template <typename T>
cudaError_t launch_n(const M1Params &p, cudaStream_t s) {
  switch (p.slab == kSlabWhole ? pad_n(p.N) : kM1Slab) {
    case 16: return launch_t<T, 16>(p, s);
    case 32: return launch_t<T, 32>(p, s);
    default: return launch_t<T, 64>(p, s);
  }
}

}  // namespace

// Partials: one per cluster of CTAs; a group's channels fill whole clusters.
int64_t m1_bwd_partials(int64_t D, int64_t N, int64_t G) {
  return G * ctas_padded_per_group(D, N > kM1Slab ? kM1Slab : N, G) / kM1BwdCluster;
}

// Time segments of the backward: as the forward's (m1_fwd_segments), only
// when the CTAs of the (batch, channel-block) grid number fewer than the SMs,
// aiming at about two CTAs per SM, each segment at least two staged blocks
// long, at most 32 segments; d_state up to one slab.
int64_t m1_bwd_segments(int64_t B, int64_t D, int64_t N, int64_t L, int64_t G) {
  if (N > kM1Slab || B <= 0 || D <= 0 || L <= 0 || G <= 0 || D % G != 0) return 1;
  const int64_t ctas = B * G * ctas_padded_per_group(D, N, G);
  constexpr int64_t kSMs = 148;
  if (ctas >= kSMs) return 1;
  int64_t n = (2 * kSMs + ctas - 1) / ctas;
  const int64_t by_len = L / (2 * kBlk);
  if (n > by_len) n = by_len;
  if (n > 32) n = 32;
  if (n < 2) return 1;
  return (L + m1_fwd_seg_len(L, n) - 1) / m1_fwd_seg_len(L, n);  // segments of whole blocks
}

// Workspace: dB/dC partials [n_part][B][2][N][L], per-(segment, b, c)
// partials [S][B][D][N + 2], above one slab the token sums [3][B][D][L], and
// with time segments their summaries [2][S][B][D][N].
M1BwdWorkspace m1_bwd_workspace(int64_t B, int64_t D, int64_t N, int64_t L, int64_t G) {
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  M1BwdWorkspace w;
  w.n_part = m1_bwd_partials(D, N, G);
  w.n_seg = m1_bwd_segments(B, D, N, L, G);
  w.bc = 0;
  w.misc = up(sizeof(float) * (size_t)(w.n_part * B * 2 * N * L));
  w.tok = w.misc + up(sizeof(float) * (size_t)(w.n_seg * B * D * (N + 2)));
  w.seg = w.tok + up(N > kM1Slab ? sizeof(float) * (size_t)(3 * B * D * L) : 0);
  w.bytes = w.seg + (w.n_seg > 1 ? sizeof(float) * (size_t)(2 * w.n_seg * B * D * N) : 0);
  return w;
}

size_t m1_bwd_workspace_bytes(int64_t B, int64_t D, int64_t N, int64_t L, int64_t G) {
  return m1_bwd_workspace(B, D, N, L, G).bytes;
}

// The whole d_state in one launch, or slabs of kM1Slab states in ascending
// order (the token sums carried in tok_part), then the fixed-order reduction
// of the partials over the full d_state.
cudaError_t launch_m1_bwd(const M1Params &p0, cudaStream_t s) {
  const int64_t n_tot = p0.N;
  const int64_t slabs = (n_tot + kM1Slab - 1) / kM1Slab;
  if (p0.seg_len > 0) {
    // time segments: each one's summary from a zero carry, then the carries
    // entering them, composed from the sequence's end
    const int64_t n_seg = (p0.L + p0.seg_len - 1) / p0.seg_len;
    cudaError_t e;
    switch (p0.io) {
      case 1: e = launch_seg_sum<bf16>(p0, n_seg, s); break;
      case 2: e = launch_seg_sum<f16>(p0, n_seg, s); break;
      default: e = launch_seg_sum<float>(p0, n_seg, s); break;
    }
    if (e != cudaSuccess) return e;
    const int64_t elems = p0.B * p0.D * p0.N;
    int64_t blocks = (elems + 7) / 8;  // 8 warps of 32 per block, a warp per element
    if (blocks > 148 * 16) blocks = 148 * 16;
    m1_bwd_seg_combine_kernel<<<(unsigned)blocks, 256, 0, s>>>(p0, (int)n_seg);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  for (int64_t k = 0; k < slabs; ++k) {
    M1Params p = p0;
    p.ldN = n_tot;
    p.n0 = k * kM1Slab;
    p.N = n_tot - p.n0 < kM1Slab ? n_tot - p.n0 : kM1Slab;
    p.slab = slabs == 1 ? kSlabWhole
                        : (k == 0 ? kSlabFirst : (k == slabs - 1 ? kSlabLast : kSlabMiddle));
    cudaError_t e;
    switch (p.io) {
      case 1: e = launch_n<bf16>(p, s); break;
      case 2: e = launch_n<f16>(p, s); break;
      default: e = launch_n<float>(p, s); break;
    }
    if (e != cudaSuccess) return e;
  }
  const int64_t total = p0.B * p0.G * 2 * n_tot * p0.L + p0.D * (n_tot + 2);
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  m1_bwd_reduce_kernel<<<(unsigned)blocks, threads, 0, s>>>(p0);
  return cudaGetLastError();
}

}  // namespace msc
