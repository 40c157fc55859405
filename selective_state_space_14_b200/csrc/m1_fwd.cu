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
// registers; exp(delta A) is taken as 2^(delta * A log2 e) on the SFU.  The
// raw inputs of a 32-step chunk (u, delta, z of the CTA's channels and the
// batch row's B, C) arrive by cp.async one chunk ahead; per chunk the CTA
// turns them into per-token values (softplus and the silu gate computed once
// per token) and an f32 table of B, C pairs in shared memory.  y_t sums over the state pairs of a channel: every kP steps
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
constexpr int kTF = 32;  // steps per forward chunk
static_assert(kTF % kM1SaveInterval == 0, "chunk must hold whole saved-state intervals");

template <int kN, bool kConv>
struct FwdSmem {
  using Lay = Layout<kN, kWarps>;
  static constexpr int kP = Lay::kP;
  static constexpr int kCh = Lay::kCh;
  // per-warp transpose tile: [channel in warp][pair][kP + 4], channel blocks
  // padded so that channels of a warp fall on different banks
  static constexpr int kRow = kP + 4;
  static constexpr int kChBlock = kP * kRow + (kP == 8 ? 8 : (kP == 16 ? 16 : 0));
  // float offsets
  static constexpr int kOut = kTF + 8;  // output tile channel stride (bank spread)
  static constexpr int tok = 0;                               // [kTF][kCh] float4
  static constexpr int bc = tok + kCh * kTF * 4;              // [kTF][kP] float4
  static constexpr int ytile = bc + kTF * kP * 4;             // [kWarps][32/kP][kChBlock]
  static constexpr int out = ytile + kWarps * (32 / kP) * kChBlock;  // [kCh][kOut]
  static constexpr int gate = out + kCh * kOut;               // [kCh][kOut] silu(z), last slab
  // with the conv fused ahead: [2][kCh][4] conv inputs before a chunk,
  // [kCh][8] the conv's taps (4, right-aligned: a width-W conv uses taps
  // 4-W..3) and bias, and [2][kCh][kUOut] the conv's output u (a chunk's tile
  // is stored out with the chunk's outputs, while the next chunk fills the
  // other one; the stride of 36 floats makes a warp's 16-byte stores and
  // loads conflict-free)
  static constexpr int kUOut = kTF + 4;
  static constexpr int halo = gate + kCh * kOut;
  static constexpr int cw = halo + (kConv ? 2 * kCh * 4 : 0);
  static constexpr int su = cw + (kConv ? kCh * 8 : 0);
  static constexpr int raw = (su + (kConv ? 2 * kCh * kUOut : 0) + 3) / 4 * 4;  // 16-byte aligned
  static constexpr int total_floats = raw;
};

// raw inputs of one chunk, bytes: u, delta, z [3][kCh][kTokRow] T; B, C [2][kN][kTokRow] T;
// then the row table
template <typename T, int kN>
struct FwdRaw {
  static constexpr int kCh = Layout<kN, kWarps>::kCh;
  static constexpr int kRows = 3 * kCh + 2 * kN;  // staged rows: u, delta, z, then B and C
  // rows padded by 16 bytes: the threads that convert one step of
  // consecutive channels (or state pairs) read from different banks
  static constexpr int kTokRow = kTF + 16 / (int)sizeof(T);
  static constexpr int tok = 0;
  static constexpr int bc = 3 * kCh * kTokRow * (int)sizeof(T);
  // global address of every staged row at t = 0 (0: absent row, zero-filled)
  static constexpr int rows = (bc + 2 * kN * kTokRow * (int)sizeof(T) + 7) / 8 * 8;
  static constexpr int bytes = rows + kRows * 8;
};

// The row table, once per CTA: token rows (tensor k of u, delta, z; channel
// cl) at k * kCh + cl, then the B and C rows (state n) at 3 kCh + k * kN + n.
template <typename T, int kN>
__device__ __forceinline__ void fwd_fill_rows(const M1Params &p, const T **rows, int64_t b,
                                              int64_t c_first, int64_t c_end, const T *Bg,
                                              const T *Cg, int tid) {
  using R = FwdRaw<T, kN>;
  constexpr int kCh = R::kCh;
  for (int r = tid; r < R::kRows; r += kWarps * 32) {
    const T *row = nullptr;
    if (r < 3 * kCh) {
      const int k = r / kCh, cl = r % kCh;
      const void *src = k == 0 ? p.u : (k == 1 ? p.delta : p.z);
      const int64_t c = c_first + cl;
      if (src != nullptr && c < c_end) row = static_cast<const T *>(src) + (b * p.D + c) * p.L;
    } else {
      const int k = (r - 3 * kCh) / kN, n = (r - 3 * kCh) % kN;
      if (n < p.N) row = (k == 0 ? Bg : Cg) + n * p.L;
    }
    rows[r] = row;
  }
}

// Issue the copies of the chunk starting at tc into the raw buffer: 16-byte
// pieces of the rows in the row table, by cp.async (zero-filled past the end
// of a row) when rows are 16-byte aligned, element copies otherwise.  Absent
// rows are zeros.
template <typename T, int kN>
__device__ __forceinline__ void fwd_issue_raw(const M1Params &p, unsigned char *raw,
                                              const T *const *rows, int64_t tc, int tid) {
  using R = FwdRaw<T, kN>;
  constexpr int E = 16 / (int)sizeof(T);
  constexpr int kPieces = kTF / E;
  static_assert((kPieces & (kPieces - 1)) == 0, "pieces per row: a power of two");
  const int64_t L = p.L;
  const T *const fallback = static_cast<const T *>(p.Bm);  // a valid address for empty copies
  for (int u = tid; u < R::kRows * kPieces; u += kWarps * 32) {
    const int j = u & (kPieces - 1), r = u / kPieces;
    const T *row = rows[r];
    const int64_t t = tc + j * E;
    const int64_t left = L - t;
    const int valid = row == nullptr || left <= 0 ? 0 : (left >= E ? E : (int)left);
    T *dst = r < 3 * R::kCh ? reinterpret_cast<T *>(raw) + r * R::kTokRow + j * E
                            : reinterpret_cast<T *>(raw + R::bc) + (r - 3 * R::kCh) * R::kTokRow + j * E;
    if (p.vec) {
      cp_async16(dst, valid > 0 ? row + t : fallback, valid * (int)sizeof(T));
    } else {
#pragma unroll
      for (int i = 0; i < E; ++i) dst[i] = i < valid ? row[t + i] : from_f32<T>(0.f);
    }
  }
  cp_async_commit();
}

// Store the outputs of the chunk starting at tc from shared memory.  Whole
// d_state: the gated outputs.  Slabs: the first writes its sums over its
// states to tok_part (f32), a middle one adds to them, the last adds them to
// its own and stores the gated outputs.
template <typename T, int kCh, int kOut, int kUOut>
__device__ __forceinline__ void store_chunk(const M1Params &p, const float *sout,
                                            const float *sgate, const float *su,
                                            int64_t c_first, int64_t c_end, int64_t b,
                                            int64_t tc, int64_t t_end, int tid, int nthreads) {
  const int64_t D = p.D, L = t_end;  // rows are L long; this pass ends at t_end
  for (int u = tid; u < kCh * (kTF / 8); u += nthreads) {
    const int chl = u / (kTF / 8);
    const int seg = u % (kTF / 8);
    const int64_t c = c_first + chl;
    if (c >= c_end) continue;
    const float4 a = *reinterpret_cast<const float4 *>(sout + chl * kOut + seg * 8);
    const float4 e = *reinterpret_cast<const float4 *>(sout + chl * kOut + seg * 8 + 4);
    float v[8] = {a.x, a.y, a.z, a.w, e.x, e.y, e.z, e.w};
    const int64_t row = (b * D + c) * p.L, t0 = tc + seg * 8;
    if (su) {  // the conv's output u (exact: values already rounded to T)
      const float4 ua = *reinterpret_cast<const float4 *>(su + chl * kUOut + seg * 8);
      const float4 ue = *reinterpret_cast<const float4 *>(su + chl * kUOut + seg * 8 + 4);
      const float uv[8] = {ua.x, ua.y, ua.z, ua.w, ue.x, ue.y, ue.z, ue.w};
      store_run<8>(static_cast<T *>(p.u_out) + row, t0, L, p.vec, uv);
    }
    if (p.slab == kSlabWhole) {
      store_run<8>(static_cast<T *>(p.out) + row, t0, L, p.vec, v);
      continue;
    }
    if (p.slab != kSlabFirst) {
      float prev[8];
      load_run<8>(p.tok_part + row, t0, L, p.vec, prev, 0.f);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = prev[i] + v[i];
    }
    if (p.slab == kSlabLast) {
      const float4 ga = *reinterpret_cast<const float4 *>(sgate + chl * kOut + seg * 8);
      const float4 ge = *reinterpret_cast<const float4 *>(sgate + chl * kOut + seg * 8 + 4);
      const float g[8] = {ga.x, ga.y, ga.z, ga.w, ge.x, ge.y, ge.z, ge.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] *= g[i];
      store_run<8>(static_cast<T *>(p.out) + row, t0, L, p.vec, v);
    } else {
      store_run<8>(p.tok_part + row, t0, L, p.vec, v);
    }
  }
}

// kConv: the causal conv1d + SiLU fused ahead: the token runs read the conv's
// input x (from the stage, the W-1 inputs before a chunk from the halo) and
// turn it into u.
// Time segments (p.seg_len > 0): the CTA covers segment blockIdx.z.  kSum:
// the segment's summary alone, from a zero state -- the product of its decays
// and the state it reaches, per state element, to seg_ws -- with no outputs;
// otherwise the segment runs from its carried state (seg_ws, written by the
// combine kernel; h0 for the first segment) and writes its outputs.
template <typename T, int kN, bool kConv, bool kSum>
__global__ void __launch_bounds__(kWarps * 32, 6) m1_fwd_kernel(const M1Params p) {
  using S = FwdSmem<kN, kConv>;
  using Lay = Layout<kN, kWarps>;
  constexpr int kP = Lay::kP;
  constexpr int kCh = Lay::kCh;
  constexpr int kThreads = Lay::kThreads;
  extern __shared__ float4 smem4[];
  float *smem = reinterpret_cast<float *>(smem4);
  float4 *sTok = reinterpret_cast<float4 *>(smem + S::tok);
  float4 *sBC = reinterpret_cast<float4 *>(smem + S::bc);
  float *sOut = smem + S::out;
  float *sGate = smem + S::gate;
  float *sHalo = smem + S::halo;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int chw = lane / kP;                 // channel within the warp
  const int pr = lane % kP;                  // state pair
  const int chl = warp * Lay::kChPerWarp + chw;
  float *ytile = smem + S::ytile + (warp * Lay::kChPerWarp + chw) * S::kChBlock;

  const int64_t D = p.D, L = p.L, N = p.N;
  const int64_t ldN = p.ldN, ns = p.n0;  // row length of A and the states; this slab's first state
  const int64_t b = blockIdx.y;
  // CTAs tile each B/C group separately, so a CTA never straddles two groups
  const int64_t per_group = D / p.G;
  const int64_t ctas_per_group = (per_group + kCh - 1) / kCh;
  const int64_t g = blockIdx.x / ctas_per_group;
  const int64_t c_first = g * per_group + (blockIdx.x % ctas_per_group) * kCh;
  const int64_t c_end = (g + 1) * per_group;
  const int64_t c = c_first + chl;
  const bool active = c < c_end;
  const T *Bg = static_cast<const T *>(p.Bm) + ((b * p.G + g) * ldN + ns) * L;
  const T *Cg = static_cast<const T *>(p.Cm) + ((b * p.G + g) * ldN + ns) * L;
  // this pass's steps [tb, te): the whole sequence, or time segment blockIdx.z
  const int64_t seg = blockIdx.z, n_seg = gridDim.z;
  const int64_t tb = p.seg_len > 0 ? seg * p.seg_len : 0;
  const int64_t te = p.seg_len > 0 && tb + p.seg_len < L ? tb + p.seg_len : L;
  const int64_t n_chunks = (te - tb + kTF - 1) / kTF;
  const int64_t n_save = (L + kM1SaveInterval - 1) / kM1SaveInterval;
  const int64_t seg_elems = p.B * D * N;  // state elements (whole d_state: N == ldN)
  using R = FwdRaw<T, kN>;
  unsigned char *raw = reinterpret_cast<unsigned char *>(smem + S::raw);

  // this thread's state pair and its A * log2(e)
  const int n0 = 2 * pr, n1 = 2 * pr + 1;
  float2 h = make_float2(0.f, 0.f), A2 = make_float2(0.f, 0.f);
  float2 decay = make_float2(1.f, 1.f);  // kSum: the product of the segment's decays
  if (active) {
    if (n0 < N) A2.x = p.A[c * ldN + ns + n0] * kLog2e;
    if (n1 < N) A2.y = p.A[c * ldN + ns + n1] * kLog2e;
    if (!kSum && seg > 0) {  // the state carried into this segment
      const float *cs = p.seg_ws + seg_elems * (n_seg + seg - 1) + (b * D + c) * N;
      if (n0 < N) h.x = cs[n0];
      if (n1 < N) h.y = cs[n1];
    } else if (!kSum && p.h0) {
      if (n0 < N) h.x = p.h0[(b * D + c) * ldN + ns + n0];
      if (n1 < N) h.y = p.h0[(b * D + c) * ldN + ns + n1];
    }
  }
  // token conversion role: channel tcl, a run of kRun steps tseg (one run per thread)
  constexpr int kRun = kCh * kTF / kThreads;  // 4, 2, 1 for d_state 16, 32, 64
  static_assert(kRun >= 1 && kCh * kTF == kRun * kThreads, "one token run per thread");
  const int tcl = tid % kCh, tseg = tid / kCh;
  const int64_t tcc = c_first + tcl;
  const bool tact = tcc < c_end;
  // the D x skip joins the sums once: in the whole or the last slab
  const bool with_skip = p.slab == kSlabWhole || p.slab == kSlabLast;
  const float tDc = (tact && p.Dp && with_skip) ? p.Dp[tcc] : 0.f;
  const float tbias = (tact && p.bias) ? p.bias[tcc] : 0.f;

  const T **const rows = reinterpret_cast<const T **>(raw + R::rows);
  fwd_fill_rows<T, kN>(p, rows, b, c_first, c_end, Bg, Cg, tid);
  if constexpr (kConv) {
    // the inputs before the sequence: the conv state (entry j holds x at time
    // j - (W-1)) or zeros
    // (a time segment after the first takes them from x itself)
    const int Wd = (int)p.conv_W;
    for (int i = tid; i < kCh * 3; i += kThreads) {
      const int cl = i / 3, k = i % 3, pos = k - 3;
      const int64_t cc = c_first + cl;
      float v = 0.f;
      if (cc < c_end && pos >= -(Wd - 1)) {
        if (tb > 0) v = to_f32(static_cast<const T *>(p.u)[(b * D + cc) * L + tb + pos]);
        else if (p.conv_xs_in) v = p.conv_xs_in[(b * D + cc) * (Wd - 1) + (Wd - 1) + pos];
      }
      sHalo[cl * 4 + k] = v;
    }
    for (int i = tid; i < kCh * 5; i += kThreads) {  // taps right-aligned, then the bias
      const int cl = i / 5, k = i % 5, k0 = 4 - Wd;
      const int64_t cc = c_first + cl;
      float v = 0.f;
      if (cc < c_end) {
        if (k == 4) v = p.conv_b ? p.conv_b[cc] : 0.f;
        else if (k >= k0) v = p.conv_w[cc * Wd + k - k0];
      }
      smem[S::cw + cl * 8 + k] = v;
    }
  }
  __syncthreads();
  fwd_issue_raw<T, kN>(p, raw, rows, tb, tid);
  for (int64_t ch = 0; ch <= n_chunks; ++ch) {
    const int64_t tc = tb + ch * kTF;
    cp_async_wait<0>();
    __syncthreads();  // this chunk's raw inputs are in; the last chunk is done
    if (ch > 0 && !kSum)
      store_chunk<T, kCh, S::kOut, S::kUOut>(
          p, sOut, sGate,
          kConv && p.u_out ? smem + S::su + ((ch - 1) & 1) * kCh * S::kUOut : nullptr,
                                   c_first, c_end, b, tc - kTF, te, tid, kThreads);
    if (ch == n_chunks) break;
    // ---- per-token values: kRun steps of one channel per thread ---------------
    {
      const T *ru = reinterpret_cast<const T *>(raw + R::tok);
      float x[kRun], v[kRun], zv[kRun];
#pragma unroll
      for (int i = 0; i < kRun; ++i) {
        const int o = tcl * R::kTokRow + tseg * kRun + i;
        x[i] = to_f32(ru[o]);
        v[i] = to_f32(ru[kCh * R::kTokRow + o]);
        zv[i] = p.z ? to_f32(ru[2 * kCh * R::kTokRow + o]) : 0.f;
      }
      if constexpr (kConv) {
        // u = silu(b + sum_k w[k] x[t-(W-1)+k]) over this run; x before the
        // chunk from the halo, and this chunk's last three inputs become the
        // next chunk's halo (other parity: this chunk's halo is still read)
        const float *hl = sHalo + ((ch & 1) * kCh + tcl) * 4;  // x at tc-3 .. tc-1
        float xs[kRun + 3];  // x at tseg*kRun - 3 .. tseg*kRun + kRun - 1
        if constexpr (kRun == 4 && sizeof(T) == 2) {
          // this run and the run before it, 8 bytes each (rows and runs are
          // 8-byte aligned); the first run takes the chunk's halo
          const T *row = ru + tcl * R::kTokRow + tseg * 4;
          float prev[4];
          const uint2 w1 = *reinterpret_cast<const uint2 *>(row);
          if (tseg > 0) {
            const uint2 w0 = *reinterpret_cast<const uint2 *>(row - 4);
            unpack2<T>(w0.x, prev[0], prev[1]);
            unpack2<T>(w0.y, prev[2], prev[3]);
          } else {
            prev[1] = hl[0]; prev[2] = hl[1]; prev[3] = hl[2];
          }
          xs[0] = prev[1]; xs[1] = prev[2]; xs[2] = prev[3];
          unpack2<T>(w1.x, xs[3], xs[4]);
          unpack2<T>(w1.y, xs[5], xs[6]);
        } else {
#pragma unroll
          for (int j = 0; j < kRun + 3; ++j) {
            const int pos = tseg * kRun - 3 + j;
            xs[j] = pos >= 0 ? to_f32(ru[tcl * R::kTokRow + pos]) : hl[pos + 3];
          }
        }
        // tap k of 4 meets x at t-3+k; a width-W conv uses taps 4-W .. 3 (the
        // taps stay compile-time indexes: xs lives in registers)
        const int k0 = 4 - (int)p.conv_W;
        const float4 wq = *reinterpret_cast<const float4 *>(smem + S::cw + tcl * 8);
        const float wv[4] = {wq.x, wq.y, wq.z, wq.w};
        const float cb = smem[S::cw + tcl * 8 + 4];
#pragma unroll
        for (int i = 0; i < kRun; ++i) {
          float a = cb;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (k >= k0) a = fmaf(wv[k], xs[i + k], a);
          // u rounded to the io type, as the unfused conv would store it
          x[i] = to_f32(from_f32<T>(silu(a)));
        }
        float *ud = smem + S::su + ((ch & 1) * kCh + tcl) * S::kUOut + tseg * kRun;
        if constexpr (kRun == 4) {
          *reinterpret_cast<float4 *>(ud) = make_float4(x[0], x[1], x[2], x[3]);
        } else {
#pragma unroll
          for (int i = 0; i < kRun; ++i) ud[i] = x[i];
        }
        if (tseg == kTF / kRun - 1) {
          float *hn = sHalo + (((ch + 1) & 1) * kCh + tcl) * 4;
#pragma unroll
          for (int k = 0; k < 3; ++k) hn[k] = xs[kRun + k];
        }
      }
#pragma unroll
      for (int i = 0; i < kRun; ++i) {
        float4 tk = make_float4(0.f, 0.f, 0.f, 0.f);
        if (tact && tc + tseg * kRun + i < te) {
          const float vv = v[i] + tbias;
          const float d = p.softplus ? softplus(vv) : vv;
          tk = make_float4(d, d * x[i], tDc * x[i], p.z ? silu(zv[i]) : 1.f);
        }
        sTok[(tseg * kRun + i) * kCh + tcl] = tk;
      }
    }
    // ---- B, C pairs in f32 (the raw rows hold zeros past d_state and past L):
    // a unit is a pair and 8 consecutive steps, four row pieces in, eight
    // float4 out
    {
      const T *rb = reinterpret_cast<const T *>(raw + R::bc);
      for (int u = tid; u < kP * (kTF / 8); u += kThreads) {
        const int q = u % kP, seg = u / kP;
        float e[4][8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const T *src = rb + ((k >> 1) * kN + 2 * q + (k & 1)) * R::kTokRow + seg * 8;
          if constexpr (sizeof(T) == 2) {
            const uint4 w = *reinterpret_cast<const uint4 *>(src);
            unpack2<T>(w.x, e[k][0], e[k][1]);
            unpack2<T>(w.y, e[k][2], e[k][3]);
            unpack2<T>(w.z, e[k][4], e[k][5]);
            unpack2<T>(w.w, e[k][6], e[k][7]);
          } else {
            const float4 a = reinterpret_cast<const float4 *>(src)[0];
            const float4 c = reinterpret_cast<const float4 *>(src)[1];
            e[k][0] = a.x; e[k][1] = a.y; e[k][2] = a.z; e[k][3] = a.w;
            e[k][4] = c.x; e[k][5] = c.y; e[k][6] = c.z; e[k][7] = c.w;
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
          sBC[(seg * 8 + i) * kP + q] = make_float4(e[0][i], e[1][i], e[2][i], e[3][i]);
      }
    }
    __syncthreads();  // tables ready; the raw buffer and the output tile are free
    if (ch + 1 < n_chunks) fwd_issue_raw<T, kN>(p, raw, rows, tc + kTF, tid);
    if constexpr (kSum) {
      // no outputs: the state walk alone
#pragma unroll 1
      for (int t = 0; t < kTF; ++t) {
        const float4 tk = sTok[t * kCh + chl];
        const float4 bcv = sBC[t * kP + pr];
        const float2 a = ex2_2(mul2(splat2(tk.x), A2));
        h = fma2(a, h, mul2(splat2(tk.y), make_float2(bcv.x, bcv.y)));
        decay = mul2(decay, a);
      }
      continue;
    }

    // ---- the recurrence over the chunk -------------------------------------
    if constexpr (!kSum) {
#pragma unroll 1
    for (int grp = 0; grp < kTF / kP; ++grp) {
      float yp[kP];
#pragma unroll
      for (int k = 0; k < kP; ++k) {
        const int t = grp * kP + k;
        if (!kSum && t % kM1SaveInterval == 0 && active && p.saved && tc + t < te) {
          float *dst = p.saved + ((b * D + c) * n_save + (tc + t) / kM1SaveInterval) * ldN + ns;
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
      if (p.slab == kSlabWhole) {
        sOut[chl * S::kOut + t] = y * tk.w;
      } else {
        sOut[chl * S::kOut + t] = y;
        sGate[chl * S::kOut + t] = tk.w;
      }
      __syncwarp();
    }
    }
  }

  if constexpr (kConv) {
    // the conv state for the next call: the last W-1 inputs (the last
    // segment's outputs pass writes it)
    const int Wd = (int)p.conv_W;
    if (p.conv_xs_out && !kSum && seg == n_seg - 1) {
      for (int i = tid; i < kCh * (Wd - 1); i += kThreads) {
        const int cl = i / (Wd - 1), j = i % (Wd - 1);
        const int64_t cc = c_first + cl;
        if (cc >= c_end) continue;
        const int64_t t = L - (Wd - 1) + j;
        p.conv_xs_out[(b * D + cc) * (Wd - 1) + j] =
            t >= 0 ? to_f32(static_cast<const T *>(p.u)[(b * D + cc) * L + t])
                   : (p.conv_xs_in ? p.conv_xs_in[(b * D + cc) * (Wd - 1) + (Wd - 1) + t] : 0.f);
      }
    }
  }
  if (kSum) {
    if (active) {  // the segment's summary: decays [seg], state [n_seg + seg]
      float *dd = p.seg_ws + seg_elems * seg + (b * D + c) * N;
      float *hh = p.seg_ws + seg_elems * (n_seg + seg) + (b * D + c) * N;
      if (n0 < N) { dd[n0] = decay.x; hh[n0] = h.x; }
      if (n1 < N) { dd[n1] = decay.y; hh[n1] = h.y; }
    }
    return;
  }
  if (active && p.final_state && seg == n_seg - 1) {
    float *dst = p.final_state + (b * D + c) * ldN + ns;
    if (n0 < N) dst[n0] = h.x;
    if (n1 < N) dst[n1] = h.y;
  }
}

// The segments' summaries combined in time order: for state element e, with
// segment s taking a state x to decay_s x + state_s, the state entering
// segment s + 1 is the composition of segments 0..s applied to h0.  A warp
// takes one element, its lanes the segments (at most 32), and composes them
// with the warp-shuffle scan of the linear-recurrence monoid
// (p, h) o (p', h') = (p p', p' h + h'); the result for segment s goes over
// state_s, which only this warp reads.
__global__ void m1_seg_combine_kernel(const M1Params p, int n_seg) {
  const int64_t elems = p.B * p.D * p.N;
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t e = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); e < elems;
       e += warps) {
    float dc = 1.f, st = 0.f;  // segments past the last compose as the identity
    if (lane < n_seg) {
      dc = p.seg_ws[elems * lane + e];
      st = p.seg_ws[elems * (n_seg + lane) + e];
    }
    float pe, he;
    warp_scan_fwd(dc, st, pe, he);
    // inclusive: segments 0..lane, applied to the initial state
    const float pi = pe * dc, hi = fmaf(dc, he, st);
    const float x0 = p.h0 ? p.h0[e] : 0.f;
    if (lane < n_seg - 1) p.seg_ws[elems * (n_seg + lane) + e] = fmaf(pi, x0, hi);
  }
}

template <typename T, int kN, bool kConv, bool kSum>
cudaError_t launch_c(const M1Params &p, int64_t n_seg, cudaStream_t s) {
  using Lay = Layout<kN, kWarps>;
  const size_t smem =
      sizeof(float) * (size_t)FwdSmem<kN, kConv>::total_floats + FwdRaw<T, kN>::bytes;
  cudaError_t e = cudaFuncSetAttribute(m1_fwd_kernel<T, kN, kConv, kSum>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t per_group = p.D / p.G;
  dim3 grid((unsigned)(p.G * ((per_group + Lay::kCh - 1) / Lay::kCh)), (unsigned)p.B,
            (unsigned)n_seg);
  m1_fwd_kernel<T, kN, kConv, kSum><<<grid, Lay::kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename T, int kN, bool kConv>
cudaError_t launch_seg(const M1Params &p, cudaStream_t s) {
  if (p.seg_len <= 0) return launch_c<T, kN, kConv, false>(p, 1, s);
  // time segments: summaries, their combination, then every segment from its
  // carried state
  const int64_t n_seg = (p.L + p.seg_len - 1) / p.seg_len;
  cudaError_t e = launch_c<T, kN, kConv, true>(p, n_seg, s);
  if (e != cudaSuccess) return e;
  const int64_t elems = p.B * p.D * p.N;
  int64_t blocks = (elems + 7) / 8;  // 8 warps of 32 per block, a warp per element
  if (blocks > 148 * 16) blocks = 148 * 16;
  m1_seg_combine_kernel<<<(unsigned)blocks, 256, 0, s>>>(p, (int)n_seg);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return launch_c<T, kN, kConv, false>(p, n_seg, s);
}

template <typename T, int kN>
cudaError_t launch_t(const M1Params &p, cudaStream_t s) {
  return p.conv_w ? launch_seg<T, kN, true>(p, s) : launch_seg<T, kN, false>(p, s);
}

template <typename T>
cudaError_t launch_n(const M1Params &p, cudaStream_t s) {
  switch (p.slab == kSlabWhole ? pad_n(p.N) : kM1Slab) {
    case 16: return launch_t<T, 16>(p, s);
    case 32: return launch_t<T, 32>(p, s);
    default: return launch_t<T, 64>(p, s);
  }
}

}  // namespace

// Time segments of the forward: only when the (batch, channel-block) grid
// gives fewer CTAs than SMs (small batch, few channels), aiming at about two
// CTAs per SM, each segment at least two chunks long and at most 32 segments
// (one warp's lanes compose them).  d_state up to one slab; the forward with
// the conv fused ahead takes the same segments, so that it stays bit-equal to
// the conv followed by the plain forward.
int64_t m1_fwd_segments(int64_t B, int64_t D, int64_t N, int64_t L) {
  if (N > kM1Slab || B <= 0 || D <= 0 || L <= 0) return 1;
  const int64_t kch = pad_n(N) == 16 ? 16 : (pad_n(N) == 32 ? 8 : 4);  // channels per CTA
  const int64_t ctas = B * ((D + kch - 1) / kch);
  constexpr int64_t kSMs = 148;
  if (ctas >= kSMs) return 1;
  int64_t n = (2 * kSMs + ctas - 1) / ctas;
  const int64_t by_len = L / (2 * kM1SegSteps);
  if (n > by_len) n = by_len;
  if (n > 32) n = 32;
  if (n < 2) return 1;
  return (L + m1_fwd_seg_len(L, n) - 1) / m1_fwd_seg_len(L, n);  // segments of whole chunks
}

int64_t m1_fwd_seg_len(int64_t L, int64_t n_seg) {
  const int64_t per = (L + n_seg - 1) / n_seg;
  return (per + kM1SegSteps - 1) / kM1SegSteps * kM1SegSteps;
}

// The whole d_state in one launch, or slabs of kM1Slab states in ascending
// order, the sums over the states carried in tok_part.
cudaError_t launch_m1_fwd(const M1Params &p0, cudaStream_t s) {
  const int64_t n_tot = p0.N;
  const int64_t slabs = (n_tot + kM1Slab - 1) / kM1Slab;
  for (int64_t k = 0; k < slabs; ++k) {
    M1Params p = p0;
    p.seg_len = 0;
    if (slabs == 1) {
      const int64_t n_seg = m1_fwd_segments(p0.B, p0.D, n_tot, p0.L);
      if (n_seg > 1) p.seg_len = m1_fwd_seg_len(p0.L, n_seg);
    }
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
  return cudaSuccess;
}

}  // namespace msc
