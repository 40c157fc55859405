// kernels.h -- internal launch interface between the C ABI layer (api.cu) and
// the kernel translation units.  Not installed; msc.h is the public surface.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace msc {

// ---------------------------------------------------------------- Mamba-1 --
struct M1Params {
  int io;  // msc_dtype: 0 f32, 1 bf16, 2 f16
  int64_t B, D, N, L, G;
  int softplus;
  bool vec;  // rows of length L are 16-byte aligned for vector access
  const void *u, *delta, *Bm, *Cm, *z;
  const float *A, *Dp, *bias, *h0;
  // forward with the causal conv1d + SiLU fused ahead (conv_w non-null): u
  // holds the conv's input x; u_out (optional) receives the scan input u
  const float *conv_w, *conv_b, *conv_xs_in;
  float *conv_xs_out;
  void *u_out;
  int64_t conv_W;
  // forward outputs
  void *out;
  float *final_state, *saved;
  // backward
  const float *saved_in;
  const void *dout;
  void *du, *ddelta, *dz;
  float *dA, *dB, *dC, *dD, *dbias, *dh0;
  float *ws_bc;    // [n_part][B][2][ldN][L] partial sums of dB, dC
  float *ws_misc;  // [B][D][ldN + 2]: per-(b, c) dA row, dD, dbias
  int64_t n_part;  // dB/dC partials per batch row (one per cluster of CTAs)
  // d_state above kM1Slab runs as slabs of at most kM1Slab states, one launch
  // each: N is the slab's width, n0 its first state, ldN the full d_state
  // (the row length of A, h0, the states and dA).  The per-token sums over
  // the states (y, and in the backward also the dΔ and du sums) collect in
  // tok_part across the slabs in slab order; the last slab finishes them.
  int64_t n0, ldN;
  int slab;         // kSlabWhole, kSlabFirst, kSlabMiddle or kSlabLast
  float *tok_part;  // fwd: [B][D][L] (y); bwd: [3][B][D][L] (y, dΔ sum, Σ λ B)
  // time segments (when the (batch, channel) grid alone cannot fill the
  // GPU): segment blockIdx.z covers steps [z seg_len, (z+1) seg_len).  seg_ws
  // holds per segment and state element ([2][S][B][D][N], f32) the decay
  // product and, forward, the state reached from zero, then the carried
  // state; backward, the adjoint carry reached from zero at the segment's
  // left end, then the carry entering it from the right
  int64_t seg_len;  // 0: the whole sequence in one segment
  float *seg_ws;
};
constexpr int kM1Slab = 64;  // widest d_state one launch handles
// time segments of the Mamba-1 forward for these sizes (1: none)
int64_t m1_fwd_segments(int64_t B, int64_t D, int64_t N, int64_t L);
int64_t m1_fwd_seg_len(int64_t L, int64_t n_seg);
constexpr int kM1SegSteps = 32;  // segments are whole multiples of the forward's chunk
constexpr int kSlabWhole = 0, kSlabFirst = 1, kSlabMiddle = 2, kSlabLast = 3;

constexpr int MSC_MAX_N = 256;            // largest Mamba-1 d_state (slabs of 64 above 64)
constexpr int kM1SaveInterval = 8;        // saved-state spacing (time steps)
constexpr int kM1BwdCluster = 8;          // CTAs per cluster in the backward
constexpr int kM1BwdWarps = 3;            // warps per backward CTA
// channels of one backward CTA: kM1BwdWarps x (32 lanes / (padded d_state / 2))
inline int64_t m1_bwd_cta_channels(int64_t N) {
  const int64_t kn = N <= 16 ? 16 : (N <= 32 ? 32 : 64);
  return kM1BwdWarps * (32 / (kn / 2));
}

int64_t m1_bwd_partials(int64_t D, int64_t N, int64_t G);
// time segments of the Mamba-1 backward for these sizes (1: none)
int64_t m1_bwd_segments(int64_t B, int64_t D, int64_t N, int64_t L, int64_t G);
cudaError_t launch_m1_fwd(const M1Params &p, cudaStream_t s);
cudaError_t launch_m1_bwd(const M1Params &p, cudaStream_t s);
size_t m1_bwd_workspace_bytes(int64_t B, int64_t D, int64_t N, int64_t L, int64_t G);
struct M1BwdWorkspace {
  int64_t n_part, n_seg;
  size_t bc, misc, tok, seg, bytes;  // byte offsets of the regions, total size
};
M1BwdWorkspace m1_bwd_workspace(int64_t B, int64_t D, int64_t N, int64_t L, int64_t G);

// ------------------------------------------------------------ decode step --
struct SUParams {
  int io;  // msc_dtype: 0 f32, 1 bf16, 2 f16
  int64_t B, D, N, G;
  int softplus;
  float *state;
  const void *x, *delta, *Bm, *Cm, *z;
  const float *A, *Dp, *bias;
  void *out;
};
cudaError_t launch_state_update(const SUParams &p, cudaStream_t s);

// ---------------------------------------------------------- Mamba-3 SISO --
#define MSC_M3_CHUNK_STEPS 64  // steps per chunk (= the saved-state interval)
struct M3Params {
  int io;  // msc_dtype: 0 f32, 1 bf16, 2 f16
  int64_t B, L, H, P, N, G, K;
  const void *x, *z, *Bm, *Cm, *alpha, *beta, *gamma, *theta;
  const float *Dp, *h0;
  void *out;
  float *final_state, *saved;
  // backward
  const float *saved_in;
  const void *dout;
  void *dx, *dz;
  float *dB, *dC, *dalpha, *dbeta, *dgamma, *dtheta, *dD, *dh0;
  void *ws;
  size_t ws_bytes;
  // d_state above kM3Slab runs as slabs (N the slab's width, n0 its first
  // state, ldN the full d_state; angle pairs n0/2 .. n0/2 + N/2 - 1 of the
  // K); the sums over the states of each output carry from slab to slab:
  // fwd y in tok_y, bwd y (for dz) in tok_y and dx in tok_dx, dalpha, dbeta,
  // dgamma in place.  The last slab finishes them.
  int64_t n0, ldN;
  int slab;  // kSlabWhole, kSlabFirst, kSlabMiddle or kSlabLast
  float *tok_y, *tok_dx;  // [B, L, H, P] f32
  // forward from raw projections (bf16 io, d_state <= kM3Slab): alpha, beta,
  // gamma and theta are derived in the kernel from these, each rounded to
  // bf16 as the discretisation kernel stores it (alpha .. theta are unused;
  // Bm, Cm are BCNorm's rows, normalised once per row ahead of the scan)
  bool raw;
  const void *dd_dt, *dd_a, *trap, *angles;  // [B, L, H] x3, [B, L, K]
  const float *dt_bias;                      // [H] or null
  float A_floor, eps;
};
constexpr int kM3Slab = 64;  // widest d_state one launch handles
cudaError_t launch_m3_fwd(const M3Params &p, cudaStream_t s);
cudaError_t launch_m3_fwd_umma(const M3Params &p, cudaStream_t s);  // bf16 io, tcgen05
cudaError_t launch_m3_bwd(const M3Params &p, cudaStream_t s);
cudaError_t launch_m3_bwd_umma(const M3Params &p, cudaStream_t s);  // bf16 io, tcgen05
// Workspace of the Mamba-3 backward, byte offsets of its regions: per-head dB,
// dC [B, L, H, N]; per-(b, h, chunk) dD [B, H, nc]; the chunk adjoints V / U
// [B, H, nc, P, N] and their decays rho [B, H, nc]; the dtheta chunk totals
// [B, H, nc, K]; above one slab the token sums of y and dx [B, L, H, P].
struct M3BwdWs {
  size_t dB, dC, dD, vu, rho, th, tok_y, tok_dx, total;
};
M3BwdWs m3_bwd_ws_layout(int64_t B, int64_t L, int64_t H, int64_t P, int64_t N, int64_t K);
size_t m3_bwd_workspace_bytes(int64_t B, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G,
                              int64_t K);
bool m3_supported(int64_t P, int64_t N);

// Mamba-3 SISO discretisation (dd_dt, dd_a, trap, angles -> alpha, beta,
// gamma, theta) and BCNorm (B_raw, C_raw -> Bm, Cm), and their backward
struct M3DiscParams {
  int io;  // msc_dtype
  int64_t B, L, H, N, G, K;
  bool bc_only;  // forward: BCNorm alone (Bm, Cm), no alpha .. theta
  float A_floor, eps;
  const void *dd_dt, *dd_a, *trap, *angles;  // io [B, L, H] x3, [B, L, K]
  const float *dt_bias;                      // [H] or null
  const void *B_raw, *C_raw;                 // io [B, L, G, N]
  // forward outputs (io)
  void *alpha, *beta, *gamma, *theta, *Bm, *Cm;
  // backward: upstream f32 gradients and f32 results
  const float *dalpha, *dbeta, *dgamma, *dtheta, *dB, *dC;
  float *ddd_dt, *ddd_a, *dtrap, *dangles, *ddt_bias, *dB_raw, *dC_raw;
};
cudaError_t launch_m3_disc_fwd(const M3DiscParams &p, cudaStream_t s);
cudaError_t launch_m3_disc_bwd(const M3DiscParams &p, cudaStream_t s);

// causal depthwise conv1d + SiLU ahead of the Mamba-1 scan
struct ConvParams {
  int io;  // msc_dtype
  int64_t B, D, L, W;
  bool vec;  // rows of length L are 16-byte aligned for vector access
  const void *x;
  const float *w, *bias, *xs_in;
  void *u;
  float *xs_out;
  // backward
  const void *du;
  void *dx;
  float *dw, *dbias, *dxs_in;
  float *ws;  // per-run partials of dw, dbias
};
cudaError_t launch_conv1d_fwd(const ConvParams &p, cudaStream_t s);
cudaError_t launch_conv1d_bwd(const ConvParams &p, cudaStream_t s);
size_t conv1d_bwd_workspace_bytes(int64_t B, int64_t D, int64_t L, int64_t W);

// Mamba-3 SISO single-token state update (decode)
struct M3SUParams {
  int io;  // msc_dtype: 0 f32, 1 bf16, 2 f16
  int64_t B, H, P, N, G, K;
  float *state, *x_prev, *bt_prev, *phi;
  const void *x, *z, *Bm, *Cm, *alpha, *beta, *gamma, *theta;
  const float *Dp;
  void *out;
  // with the discretisation and BCNorm fused ahead (raw): alpha .. theta, Bm,
  // Cm are derived in the kernel from these step inputs instead
  bool raw;
  const void *dd_dt, *dd_a, *trap, *angles;  // io [B, H] x3, [B, K]
  const float *dt_bias;                      // [H] or null
  const void *B_raw, *C_raw;                 // io [B, G, N]
  float A_floor, eps;
};
cudaError_t launch_m3_state_update(const M3SUParams &p, cudaStream_t s);

}  // namespace msc
