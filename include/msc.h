/*
 * msc.h -- C ABI of the B200 selective state-space scan library (libmsc.so).
 *
 * The library computes the hot path of the Mamba family's selective SSM:
 *
 *   - the Mamba-1 selective scan, forward and backward (the selective SSM
 *     layer of "Mamba: Linear-Time Sequence Modeling with Selective State
 *     Spaces", Section 3 / Algorithm 2, as the state-spaces/mamba README's
 *     "Usage / Selective SSM" section names it; the mamba-rs 0.7.0 README,
 *     "Features", lists the Gu and Dao 2023 SSM with backpropagation
 *     through its recurrent state);
 *   - the Mamba-3 SISO scan, forward and backward (mamba-rs 0.7.0 README,
 *     "Features"; backward stages B2 output gating, B3 BPTT and B4 RoPE of
 *     Mamba3Scratch in mamba-rs 0.4.2 src/mamba3_siso/cpu/scratch.rs);
 *   - the single-token recurrent state update used in decoding (mamba_step /
 *     GpuMambaBackbone::step, mamba-rs 0.7.0 README, "Quick start"), for
 *     Mamba-1 and for Mamba-3 SISO (mamba3_step, the same README);
 *   - the steps either side of the scans: the causal conv1d + SiLU ahead of
 *     the Mamba-1 scan, standalone and fused into its forward, and the
 *     Mamba-3 discretisation and BCNorm stages (B6, B5 of Mamba3Scratch),
 *     each with its backward.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *   * Every function returns an msc_status.  On failure nothing is launched
 *     and msc_last_error() returns a message (thread-local, valid until the
 *     next call on the same thread) that names the offending argument.  The
 *     one exception is MSC_ERR_CUDA, returned when a launch itself fails.
 *   * Every tensor pointer is a caller-owned DEVICE pointer to a dense,
 *     contiguous, row-major array with the layout stated below.  The library
 *     allocates no memory, never synchronises, and launches all of its work
 *     on the caller's stream; results are ready when the stream reaches them.
 *   * Optional pointers may be NULL, meaning "absent": no h0 (zero initial
 *     state), no z (no gate), no D (no skip), no delta_bias, no final state.
 *   * io tensors (MSC_F32, MSC_BF16 or MSC_F16, chosen per call; "f32, bf16
 *     and f16 storage", mamba-rs README, "Features") are read and written in
 *     that dtype; every accumulation is f32 (the same README: "every kernel
 *     accumulates in f32"), and recurrent states and reduced gradients are
 *     always f32.  f16 values are IEEE binary16: results past its range
 *     (65504) become infinite in the stored outputs.
 *   * Results are bit-identical from run to run for the same inputs on the
 *     same GPU and build: there are no atomics and every cross-thread
 *     reduction has a fixed order (the "same bits run to run" guarantee of
 *     mamba-rs docs/gemm-modes.md, "What is guaranteed").
 *   * Argument structs begin with struct_size; callers set it to
 *     sizeof(the struct) so that later fields can be added compatibly.
 *   * Scratch memory, where an operation needs it, is passed in by the caller
 *     (the "zero-allocation rule" of Mamba3Scratch: hot-path buffers are
 *     preallocated once and reused); its size comes from the matching
 *     *_bytes() query.
 *   * Pointers must be 16-byte aligned.  Sequences of any length are
 *     accepted; when a row's byte length is not a multiple of 16 the kernels
 *     fall back to element loads for it.
 */
#ifndef MSC_H_
#define MSC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *msc_stream_t;

typedef enum {
  MSC_OK = 0,
  MSC_ERR_INVALID_ARG = 1, /* a NULL required pointer, a bad size or flag       */
  MSC_ERR_UNSUPPORTED = 2, /* a valid request this build does not implement     */
  MSC_ERR_ALIGNMENT = 3,   /* a pointer not 16-byte aligned                     */
  MSC_ERR_CUDA = 4,        /* a CUDA launch error (message carries the reason)  */
  MSC_ERR_WORKSPACE = 5    /* workspace pointer NULL or smaller than required   */
} msc_status;

typedef enum { MSC_F32 = 0, MSC_BF16 = 1, MSC_F16 = 2 } msc_dtype;

/* Message for the last failure on this thread ("" after a success). */
const char *msc_last_error(void);

/* Library version, e.g. "msc 0.1.0 sm_100a". */
const char *msc_version(void);

/* ======================================================================
 * Mamba-1 selective scan
 * ======================================================================
 * Shapes: B = batch, D = dim (d_inner channels), N = dstate, L = seqlen,
 * G = ngroups (B/C are shared by the D/G channels of a group; G divides D).
 *
 *   u, delta, z, out          io  [B, D, L]
 *   Bm, Cm                    io  [B, G, N, L]
 *   A                         f32 [D, N]
 *   D, delta_bias             f32 [D]
 *   h0, final_state           f32 [B, D, N]
 *   saved_states              f32 [B, D, ceil(L / MSC_M1_SAVE_INTERVAL), N]
 *
 * Forward, per (b, c) and t = 0..L-1, with g the group of channel c:
 *   delta_t = softplus(delta[b,c,t] + delta_bias[c])  if delta_softplus,
 *             delta[b,c,t] + delta_bias[c]            otherwise
 *   h[n]    = exp(delta_t * A[c,n]) * h[n] + delta_t * Bm[b,g,n,t] * u[b,c,t]
 *   y       = sum_n Cm[b,g,n,t] * h[n] + D[c] * u[b,c,t]
 *   out     = y * silu(z[b,c,t])                        (y if z is NULL)
 * starting from h = h0[b,c,:] (or 0).  final_state receives h after the last
 * step.  saved_states receives h at the start of every block of
 * MSC_M1_SAVE_INTERVAL steps (the first is h0); the backward pass needs it.
 * N may be 1..256 (the largest state the mamba-rs README lists under
 * "Features"); L >= 1.  Above 64 states the scan runs in slabs of 64 states;
 * with few (batch, channel) rows for the GPU's SMs it splits time into
 * segments whose summaries a warp-shuffle scan composes (the associative
 * combine of the recurrence).  In both cases the forward needs a workspace
 * of msc_selective_scan_fwd_workspace_bytes() bytes (0 otherwise): the sums
 * over the earlier slabs, or the segments' summaries.  The segments change
 * only the rounding order, not the result's accuracy; every configuration
 * gives the same bits from run to run.
 */
#define MSC_M1_SAVE_INTERVAL 8
#define MSC_M1_MAX_DSTATE 256

typedef struct {
  uint32_t struct_size;
  int32_t io_dtype;       /* msc_dtype of u, delta, z, Bm, Cm, out              */
  int64_t batch, dim, dstate, seqlen, ngroups;
  int32_t delta_softplus; /* 0 or 1                                            */
  const void *u, *delta;
  const float *A;
  const void *Bm, *Cm;
  const float *D;          /* optional */
  const float *delta_bias; /* optional */
  const void *z;           /* optional */
  const float *h0;         /* optional */
  void *out;
  float *final_state;      /* optional */
  float *saved_states;     /* optional; required if the backward pass follows */
  void *workspace;         /* required when the workspace query is > 0, else ignored */
  size_t workspace_bytes;
} msc_ss_fwd_args;

/* Bytes of the forward's workspace for these sizes (0 when the forward needs
 * none: up to 64 states, with enough rows to fill the GPU). */
size_t msc_selective_scan_fwd_workspace_bytes(int64_t batch, int64_t dim, int64_t dstate,
                                              int64_t seqlen);

/* Bytes of the saved_states array for these sizes. */
size_t msc_selective_scan_saved_states_bytes(int64_t batch, int64_t dim, int64_t dstate,
                                             int64_t seqlen);

msc_status msc_selective_scan_fwd(const msc_ss_fwd_args *args, msc_stream_t stream);

/*
 * Backward (BPTT through the recurrent state).  Inputs are the forward's
 * inputs, the saved_states it wrote, and dout [B, D, L] (io).  With
 * g_t = dout_t * silu(z_t) and the state adjoint
 *   lambda_t[n] = g_t Cm_t[n] + exp(delta_{t+1} A[c,n]) lambda_{t+1}[n]
 * (lambda after the last step = 0: the final state is not differentiated):
 *   du[b,c,t]        = g_t D[c] + delta_t sum_n lambda_t[n] Bm_t[n]       io
 *   ddelta[b,c,t]    = d loss / d delta (raw, before bias and softplus)  io
 *   dz[b,c,t]        = dout_t y_t silu'(z_t)                              io
 *   dA[c,n]          = sum_{b,t} lambda_t delta_t exp(delta_t A) h_{t-1}  f32
 *   dB[b,g,n,t]      = sum_{c in g} lambda_t[n] delta_t u_t               f32
 *   dC[b,g,n,t]      = sum_{c in g} g_t h_t[n]                            f32
 *   dD[c]            = sum_{b,t} g_t u_t                                  f32
 *   ddelta_bias[c]   = sum_{b,t} ddelta[b,c,t]                            f32
 *   dh0[b,c,n]       = exp(delta_0 A) lambda_0[n]                         f32
 * dD, ddelta_bias, dz and dh0 are optional outputs (NULL: not computed).
 * Every output is overwritten (not accumulated into).
 * Workspace: msc_selective_scan_bwd_workspace_bytes() bytes of device memory,
 * contents on entry irrelevant (the dB/dC partials of each cluster of
 * channel blocks, and with few (batch, channel) rows the summaries of the
 * time segments the backward then splits into).
 */
typedef struct {
  uint32_t struct_size;
  int32_t io_dtype;
  int64_t batch, dim, dstate, seqlen, ngroups;
  int32_t delta_softplus;
  const void *u, *delta;
  const float *A;
  const void *Bm, *Cm;
  const float *D;          /* optional */
  const float *delta_bias; /* optional */
  const void *z;           /* optional */
  const float *h0;         /* optional */
  const float *saved_states; /* required: written by the forward            */
  const void *dout;
  void *du, *ddelta;
  void *dz;                /* optional (only meaningful with z)              */
  float *dA, *dB, *dC;
  float *dD;               /* optional */
  float *ddelta_bias;      /* optional */
  float *dh0;              /* optional */
} msc_ss_bwd_args;

size_t msc_selective_scan_bwd_workspace_bytes(int64_t batch, int64_t dim, int64_t dstate,
                                              int64_t seqlen, int64_t ngroups);

msc_status msc_selective_scan_bwd(const msc_ss_bwd_args *args, void *workspace,
                                  size_t workspace_bytes, msc_stream_t stream);

/*
 * The same backward pass without a workspace argument, for callers that may
 * not allocate device memory when they run it (a fixed memory budget
 * reserved up front, a pooled allocator that must not be bypassed, a path
 * that must not synchronise the device).  This entry point has no
 * counterpart in the pages; it is an addition of this library.
 *
 * The scratch lives in a static device array of MSC_STATIC_SCRATCH_BYTES
 * inside the library, held on every GPU that loads the library until the
 * process exits.  Sizes whose msc_selective_scan_bwd_workspace_bytes()
 * exceeds it are rejected with MSC_ERR_WORKSPACE (nothing launched).  The
 * first call on a device looks up the array's device address on that device
 * (cudaGetSymbolAddress); make that first call before any stream capture.
 * The address is kept for the life of the process, so the entry point must
 * not be used across a cudaDeviceReset of that device (the reset may move the
 * array).  Arguments are checked as msc_selective_scan_bwd checks them, before
 * the scratch size is computed.  All calls share the array: calls that may overlap on the GPU race on it
 * and must be serialised by the caller.  Results equal those of
 * msc_selective_scan_bwd.  Allocates nothing, never synchronises.
 */
#define MSC_STATIC_SCRATCH_BYTES (64u << 20)
msc_status msc_selective_scan_bwd_static(const msc_ss_bwd_args *args, msc_stream_t stream);

/* ======================================================================
 * Single-token state update (decode)
 * ======================================================================
 *   state                     f32 [B, D, N]   read and written in place
 *   x, delta, z, out          io  [B, D]
 *   Bm, Cm                    io  [B, G, N]
 *   A f32 [D, N]; D, delta_bias f32 [D]
 * One step of the Mamba-1 recurrence above, for every (b, c):
 *   state[b,c,n] <- exp(delta A[c,n]) state[b,c,n] + delta Bm[b,g,n] x[b,c]
 *   out[b,c]      = (sum_n Cm[b,g,n] state[b,c,n] + D[c] x[b,c]) silu(z[b,c])
 * It equals the scan's step exactly in arithmetic order per element.
 */
typedef struct {
  uint32_t struct_size;
  int32_t io_dtype;
  int64_t batch, dim, dstate, ngroups;
  int32_t delta_softplus;
  float *state;
  const void *x, *delta;
  const float *A;
  const void *Bm, *Cm;
  const float *D;          /* optional */
  const float *delta_bias; /* optional */
  const void *z;           /* optional */
  void *out;
} msc_su_args;

msc_status msc_ssm_state_update(const msc_su_args *args, msc_stream_t stream);

/* ======================================================================
 * Causal depthwise conv1d + SiLU ahead of the Mamba-1 scan
 * ======================================================================
 * The Mamba block's local convolution (the Mamba README, "Usage / Mamba
 * Block": d_conv, the "local convolution width"; its causal-conv1d extra;
 * MambaState carries d_conv per layer, mamba-rs 0.7.0 README, "Quick start
 * (CPU)"), producing the scan's input u from x:
 *   v[b,c,t] = bias[c] + sum_{k<W} w[c,k] x[b,c,t-(W-1)+k]
 *   u[b,c,t] = silu(v[b,c,t])
 * x before the sequence comes from conv_state_in[b,c,0..W-2] (the W-1 inputs
 * before t = 0, oldest first) or is 0; conv_state_out receives the last W-1
 * inputs (the state for the next call).
 *
 *   x, u                      io  [B, D, L]
 *   w                         f32 [D, W]        1 <= W <= 4
 *   bias                      f32 [D]           optional
 *   conv_state_in/out         f32 [B, D, W-1]   optional
 * Backward, for an upstream gradient du (io, [B, D, L]):
 *   dv = du silu'(v);  dx[t] = sum_k w[c,k] dv[t+(W-1)-k]  (terms with t+(W-1)-k < L)
 *   dw[c,k] = sum_{b,t} dv[t] x[t-(W-1)+k];  dbias[c] = sum_{b,t} dv[t]
 *   dconv_state_in[b,c,j] = the gradient of conv_state_in[b,c,j]
 * dw and dbias are summed over the batch in a fixed order (a workspace of
 * msc_causal_conv1d_bwd_workspace_bytes() bytes holds the per-row partials).
 */
#define MSC_CONV_MAX_WIDTH 4
typedef struct {
  uint32_t struct_size;
  int32_t io_dtype;
  int64_t batch, dim, seqlen, width;
  const void *x;
  const float *w;
  const float *bias;            /* optional */
  const float *conv_state_in;   /* optional */
  void *u;
  float *conv_state_out;        /* optional */
} msc_conv_fwd_args;

msc_status msc_causal_conv1d_fwd(const msc_conv_fwd_args *args, msc_stream_t stream);

typedef struct {
  uint32_t struct_size;
  int32_t io_dtype;
  int64_t batch, dim, seqlen, width;
  const void *x;
  const float *w;
  const float *bias;            /* optional */
  const float *conv_state_in;   /* optional */
  const void *du;
  void *dx;
  float *dw;
  float *dbias;                 /* optional */
  float *dconv_state_in;        /* optional */
} msc_conv_bwd_args;

size_t msc_causal_conv1d_bwd_workspace_bytes(int64_t batch, int64_t dim, int64_t seqlen,
                                             int64_t width);
msc_status msc_causal_conv1d_bwd(const msc_conv_bwd_args *args, void *workspace,
                                 size_t workspace_bytes, msc_stream_t stream);

/*
 * The conv fused ahead of the Mamba-1 scan forward: one launch computes
 * u = silu(conv(x)) per token as the scan consumes it, so u is never read
 * back from memory (and written only when u_out asks for it).  scan->u holds x (the conv's input, io
 * [B, D, L]); every other field of scan keeps its meaning in
 * msc_selective_scan_fwd, and conv gives the conv's parameters with the
 * layouts of msc_conv_fwd_args.  u_out (optional, io [B, D, L]) receives
 * u = silu(conv(x)), which the backward pass of the scan takes as its u;
 * the backward stays two calls: msc_selective_scan_bwd (on u_out) and then
 * msc_causal_conv1d_bwd (with its du).  The fused form is an addition of
 * this library; its results are those of msc_causal_conv1d_fwd followed by
 * msc_selective_scan_fwd, bit for bit (the scan takes u rounded to the io
 * type, as the unfused conv stores it).
 */
typedef struct {
  uint32_t struct_size;
  int64_t width;                /* 1 <= width <= MSC_CONV_MAX_WIDTH          */
  const float *w;               /* f32 [D, W]                                */
  const float *bias;            /* optional, f32 [D]                         */
  const float *conv_state_in;   /* optional, f32 [B, D, W-1]                 */
  float *conv_state_out;        /* optional, f32 [B, D, W-1]                 */
  void *u_out;                  /* optional, io [B, D, L]                    */
} msc_ss_conv_args;

msc_status msc_selective_scan_conv_fwd(const msc_ss_fwd_args *scan,
                                       const msc_ss_conv_args *conv, msc_stream_t stream);

/* ======================================================================
 * Mamba-3 SISO scan
 * ======================================================================
 * Shapes: B = batch, L = seqlen, H = nheads, P = headdim, N = dstate,
 * G = ngroups (G divides H), K = nangles (2K <= N).
 *
 *   x, z, out                 io  [B, L, H, P]
 *   Bm, Cm                    io  [B, L, G, N]
 *   alpha, beta, gamma        io  [B, L, H]
 *   theta                     io  [B, L, H, K]   per-step angle increments
 *   D                         f32 [H]
 *   h0, final_state           f32 [B, H, P, N]
 *
 * Per (b, h), with g the group of head h and t = 0..L-1:
 *   phi_t[k] = sum_{s<=t} theta[b,s,h,k]
 *   Bt_t = R(phi_t) Bm[b,t,g,:],  Ct_t = R(phi_t) Cm[b,t,g,:]
 *      (R rotates each pair (2k, 2k+1), k < K, counter-clockwise by phi_t[k];
 *       components 2K..N-1 are not rotated)
 *   K_t  = x[b,t,h,:] (outer) Bt_t                                  [P, N]
 *   S_t  = alpha_t S_{t-1} + beta_t K_{t-1} + gamma_t K_t,   K_{-1} = 0,
 *          S_{-1} = h0 (or 0)
 *   y_t  = S_t Ct_t + D[h] x[b,t,h,:];  out = y_t * silu(z[b,t,h,:])
 * final_state receives S_{L-1}.
 * Supported: P in {16, 32, 64}; N in {16, 32, 64} and, as slabs of 64
 * states, {128, 192, 256} ("state dimensions up to 256", mamba-rs README,
 * "Features"; the Mamba README's Mamba-3 example uses 128); L >= 0 (L = 0
 * copies h0 to final_state).  Above 64 states the forward needs a workspace
 * of msc_mamba3_siso_scan_fwd_workspace_bytes() bytes (0 up to 64 states).
 */
typedef struct {
  uint32_t struct_size;
  int32_t io_dtype;
  int64_t batch, seqlen, nheads, headdim, dstate, ngroups, nangles;
  const void *x;
  const void *z;           /* optional */
  const void *Bm, *Cm;
  const void *alpha, *beta, *gamma, *theta;
  const float *D;          /* optional */
  const float *h0;         /* optional */
  void *out;
  float *final_state;      /* optional */
  float *saved_states;     /* optional; required if the backward pass follows */
  void *workspace;         /* required when dstate > 64, else ignored (may be NULL) */
  size_t workspace_bytes;
} msc_m3_fwd_args;

/* Bytes of the forward's workspace for these sizes (0 when dstate <= 64). */
size_t msc_mamba3_siso_scan_fwd_workspace_bytes(int64_t batch, int64_t seqlen, int64_t nheads,
                                                int64_t headdim, int64_t dstate);

/* saved_states holds S at the start of every block of MSC_M3_CHUNK steps,
 * f32 [B, H, ceil(L / MSC_M3_CHUNK), P, N], followed by the cumulative angles
 * phi at the start of every block, f32 [B, H, ceil(L / MSC_M3_CHUNK), N / 2]
 * (entries k >= K are zero); the backward pass reads both.  This returns its
 * size in bytes. */
#define MSC_M3_CHUNK 64
size_t msc_mamba3_siso_saved_states_bytes(int64_t batch, int64_t seqlen, int64_t nheads,
                                          int64_t headdim, int64_t dstate);

msc_status msc_mamba3_siso_scan_fwd(const msc_m3_fwd_args *args, msc_stream_t stream);

/*
 * Backward.  Inputs are the forward's inputs, the saved_states it wrote and
 * dout [B, L, H, P] (io).  With g_t = dout_t * silu(z_t) and the state adjoint
 *   Lambda_t = g_t (outer) Ct_t + alpha_{t+1} Lambda_{t+1}:
 *   dK_t        = gamma_t Lambda_t + beta_{t+1} Lambda_{t+1}
 *   dx          = dK_t Bt_t + D g_t                                     io
 *   dz          = dout_t y_t silu'(z_t)                                 io
 *   dalpha_t    = <Lambda_t, S_{t-1}>, dbeta_t = <Lambda_t, K_{t-1}>,
 *   dgamma_t    = <Lambda_t, K_t>                                       f32 [B,L,H]
 *   dB, dC      = R(phi_t)^T (dK_t^T x_t), R(phi_t)^T (S_t^T g_t),
 *                 summed over the heads of the group                    f32 [B,L,G,N]
 *   dtheta_t[k] = sum_{s>=t} dphi_s[k]                                  f32 [B,L,H,K]
 *   dD[h]       = sum g_t . x_t                                         f32 [H]
 *   dh0         = alpha_0 Lambda_0                                      f32 [B,H,P,N]
 * dz, dD and dh0 are optional outputs.  Every output is overwritten.
 */
typedef struct {
  uint32_t struct_size;
  int32_t io_dtype;
  int64_t batch, seqlen, nheads, headdim, dstate, ngroups, nangles;
  const void *x;
  const void *z;           /* optional */
  const void *Bm, *Cm;
  const void *alpha, *beta, *gamma, *theta;
  const float *D;          /* optional */
  const float *h0;         /* optional */
  const float *saved_states; /* required: written by the forward            */
  const void *dout;
  void *dx;
  void *dz;                /* optional */
  float *dB, *dC;
  float *dalpha, *dbeta, *dgamma, *dtheta;
  float *dD;               /* optional */
  float *dh0;              /* optional */
} msc_m3_bwd_args;

size_t msc_mamba3_siso_scan_bwd_workspace_bytes(int64_t batch, int64_t seqlen, int64_t nheads,
                                                int64_t headdim, int64_t dstate,
                                                int64_t ngroups, int64_t nangles);

msc_status msc_mamba3_siso_scan_bwd(const msc_m3_bwd_args *args, void *workspace,
                                    size_t workspace_bytes, msc_stream_t stream);

/* ======================================================================
 * Mamba-3 SISO single-token state update (decode)
 * ======================================================================
 * The step that mamba3_step applies to a Mamba3State (mamba-rs 0.7.0 README,
 * "Quick start (CPU)", Mamba-3), reduced to the scan: one step t of the
 * Mamba-3 SISO recurrence above for every (b, h).  The recurrent state is
 * everything that step needs from the past:
 *
 *   state     f32 [B, H, P, N]   S_{t-1} in, S_t out
 *   x_prev    f32 [B, H, P]      x_{t-1} in, x_t out      (K_{t-1} = x_prev (outer) bt_prev)
 *   bt_prev   f32 [B, H, N]      Bt_{t-1} in, Bt_t out    (the rotated B of the last step)
 *   phi       f32 [B, H, K]      phi_{t-1} in, phi_t out  (cumulative angles)
 * all read and written in place; a fresh sequence starts from zeros (then
 * L steps equal msc_mamba3_siso_scan_fwd over those L tokens with h0 = 0).
 * Inputs of the step:
 *   x, z, out                 io  [B, H, P]
 *   Bm, Cm                    io  [B, G, N]
 *   alpha, beta, gamma        io  [B, H]
 *   theta                     io  [B, H, K]
 *   D                         f32 [H]
 * Per (b, h), with g the group of head h:
 *   phi   <- phi + theta;  Bt = R(phi) Bm[b,g,:],  Ct = R(phi) Cm[b,g,:]
 *   S     <- alpha S + beta x_prev (outer) bt_prev + gamma x (outer) Bt
 *   out    = (S Ct + D[h] x) * silu(z)
 *   x_prev <- x,  bt_prev <- Bt
 * Supported: P in {16, 32, 64}, N in {16, 32, 64, 128, 192, 256}, 2K <= N.  Every pointer is
 * 16-byte aligned; z and D are optional, theta and phi may be NULL when K = 0.
 */
typedef struct {
  uint32_t struct_size;
  int32_t io_dtype;
  int64_t batch, nheads, headdim, dstate, ngroups, nangles;
  float *state, *x_prev, *bt_prev, *phi;
  const void *x;
  const void *z;           /* optional */
  const void *Bm, *Cm;
  const void *alpha, *beta, *gamma, *theta;
  const float *D;          /* optional */
  void *out;
} msc_m3_su_args;

msc_status msc_mamba3_siso_state_update(const msc_m3_su_args *args, msc_stream_t stream);

/*
 * The same step with the discretisation and BCNorm (msc_mamba3_siso_discretize
 * below) fused ahead: the step's alpha, beta, gamma, theta, Bm and Cm are
 * derived in the kernel from this token's raw values instead of being read
 * (the corresponding fields of `step` are ignored and may be NULL):
 *   dd_dt, dd_a, trap         io  [B, H]
 *   angles                    io  [B, K]   (may be NULL when K = 0)
 *   dt_bias                   f32 [H]      optional
 *   B_raw, C_raw              io  [B, G, N]
 * Every derived value is rounded to the io type, so the result equals, bit
 * for bit, msc_mamba3_siso_discretize over the token followed by
 * msc_mamba3_siso_state_update.  An addition of this library (one launch per
 * generated token instead of two).
 */
typedef struct {
  uint32_t struct_size;
  float A_floor, eps;
  const void *dd_dt, *dd_a, *trap, *angles;
  const float *dt_bias;    /* optional */
  const void *B_raw, *C_raw;
} msc_m3_disc_step_args;

msc_status msc_mamba3_siso_disc_state_update(const msc_m3_su_args *step,
                                             const msc_m3_disc_step_args *raw,
                                             msc_stream_t stream);

/* ======================================================================
 * Mamba-3 SISO discretisation and BCNorm (the stages ahead of the scan)
 * ======================================================================
 * Stage B6 "discretization" and stage B5 "BCNorm" of Mamba3Scratch (mamba-rs
 * 0.4.2 src/mamba3_siso/cpu/scratch.rs: per-token, per-head dd_dt, dd_a,
 * trap [T * nheads], per-token raw angles [T * n_angles], raw B and C
 * [T * ngroups * d_state]).  The pages name the buffers but print no
 * formulas; this library reads them as the exponential-trapezoid
 * discretisation of the Mamba-3 paper (the README's citation), per (b, t, h):
 *   dt    = softplus(dd_dt + dt_bias[h])
 *   A     = min(-softplus(dd_a), -A_floor)
 *   alpha = exp(dt A),   lam = sigmoid(trap)
 *   beta  = (1 - lam) dt alpha,   gamma = lam dt
 *   theta[k] = dt angles[b,t,k]            (k < K; per head through dt)
 * and per (b, t, g):
 *   Bm = B_raw / sqrt(mean_n B_raw^2 + eps),   Cm likewise (no weight)
 * The outputs are the scan's inputs of the same names (io, layouts of
 * msc_m3_fwd_args).
 *
 *   dd_dt, dd_a, trap         io  [B, L, H]
 *   angles                    io  [B, L, K]      (may be NULL when K = 0)
 *   dt_bias                   f32 [H]            optional
 *   B_raw, C_raw              io  [B, L, G, N]
 *   alpha, beta, gamma        io  [B, L, H]      out
 *   theta                     io  [B, L, H, K]   out (may be NULL when K = 0)
 *   Bm, Cm                    io  [B, L, G, N]   out
 * Any N >= 1 and K with 2K <= N, and H (K + 2) + K <= 6144 (a token's
 * per-head values and angle gradients are staged in shared memory); A_floor
 * >= 0, eps >= 0 (eps > 0 unless no raw row is all zeros).
 */
typedef struct {
  uint32_t struct_size;
  int32_t io_dtype;
  int64_t batch, seqlen, nheads, dstate, ngroups, nangles;
  float A_floor, eps;
  const void *dd_dt, *dd_a, *trap, *angles;
  const float *dt_bias;    /* optional */
  const void *B_raw, *C_raw;
  void *alpha, *beta, *gamma, *theta, *Bm, *Cm;
} msc_m3_disc_args;

msc_status msc_mamba3_siso_discretize(const msc_m3_disc_args *args, msc_stream_t stream);

/*
 * Backward of msc_mamba3_siso_discretize for upstream f32 gradients of its
 * outputs (as msc_mamba3_siso_scan_bwd writes them: dalpha, dbeta, dgamma
 * [B, L, H], dtheta [B, L, H, K], dB, dC [B, L, G, N]).  Writes, all f32:
 *   ddd_dt, ddd_a, dtrap      [B, L, H]
 *   dangles                   [B, L, K]   sum over heads, ascending
 *   ddt_bias                  [H]         optional; sum over (b, t) of ddd_dt
 *   dB_raw, dC_raw            [B, L, G, N]
 * ddd_a is 0 where A is held at -A_floor.  Every output is overwritten.
 */
typedef struct {
  uint32_t struct_size;
  int32_t io_dtype;
  int64_t batch, seqlen, nheads, dstate, ngroups, nangles;
  float A_floor, eps;
  const void *dd_dt, *dd_a, *trap, *angles;
  const float *dt_bias;    /* optional */
  const void *B_raw, *C_raw;
  const float *dalpha, *dbeta, *dgamma, *dtheta, *dB, *dC;
  float *ddd_dt, *ddd_a, *dtrap, *dangles;
  float *ddt_bias;         /* optional */
  float *dB_raw, *dC_raw;
} msc_m3_disc_bwd_args;

msc_status msc_mamba3_siso_discretize_bwd(const msc_m3_disc_bwd_args *args, msc_stream_t stream);

/* ======================================================================
 * Mamba-3 SISO scan from raw projections (discretisation fused in)
 * ======================================================================
 * The scan forward and backward taking the raw projections of the
 * discretisation and BCNorm above (the pages list the stages B6
 * "discretization" and B5 "BCNorm" of Mamba3Scratch either side of the BPTT
 * and RoPE stages, mamba-rs 0.4.2 src/mamba3_siso/cpu/scratch.rs), so that
 * nothing derived from them is kept between the forward and the backward.
 *   forward   the per-head discretisation is fused into the scan's kernel:
 *             it derives alpha, beta, gamma and theta from dd_dt, dd_a,
 *             trap and angles as it stages each chunk, so theta
 *             [B, L, H, K] and alpha .. gamma are never written or read in
 *             global memory.  BCNorm acts per (b, t, g), on rows the group's
 *             heads share, so it runs once per row, by the discretisation
 *             kernel, into the call's workspace, ahead of the scan.
 *   backward  the discretisation and BCNorm are re-derived once, by the
 *             discretisation kernel, into the workspace; the scan's backward
 *             kernels read them there (deriving them inside both of its
 *             chunk kernels measured slower), and the discretisation's
 *             backward turns the scan's gradients into the raw ones.
 * Every derived value is rounded to bf16 exactly as
 * msc_mamba3_siso_discretize stores it, so:
 *   msc_mamba3_siso_scan_fwd_raw  equals, bit for bit,
 *     msc_mamba3_siso_discretize followed by msc_mamba3_siso_scan_fwd;
 *   msc_mamba3_siso_scan_bwd_raw  equals, bit for bit,
 *     msc_mamba3_siso_scan_bwd (on the discretised inputs) followed by
 *     msc_mamba3_siso_discretize_bwd.
 * bf16 io and dstate 16, 32 or 64 (the tensor-core kernels; other sizes:
 * MSC_ERR_UNSUPPORTED -- take the two calls).
 *
 * In the scan arguments (msc_m3_fwd_args / msc_m3_bwd_args) alpha, beta,
 * gamma, theta, Bm and Cm are ignored (may be NULL), and so, in the backward,
 * are dB, dC, dalpha, dbeta, dgamma and dtheta: the scan's gradients of the
 * derived inputs live in the workspace, and the raw gradients go to `grads`.
 * dx, dz, dD and dh0 are the scan's, as in msc_mamba3_siso_scan_bwd.
 * Workspaces (device memory, 16-byte aligned, caller-owned, contents
 * undefined on return; MSC_ERR_WORKSPACE when missing or short):
 *   forward   the `workspace` fields of msc_m3_fwd_args, at least
 *             msc_mamba3_siso_scan_fwd_raw_workspace_bytes (BCNorm's rows);
 *   backward  the `workspace` argument, at least
 *             msc_mamba3_siso_scan_bwd_raw_workspace_bytes.
 * Layouts as in msc_mamba3_siso_discretize:
 *   dd_dt, dd_a, trap         bf16 [B, L, H]
 *   angles                    bf16 [B, L, K]      (may be NULL when K = 0)
 *   dt_bias                   f32  [H]            optional
 *   B_raw, C_raw              bf16 [B, L, G, N]
 *   ddd_dt, ddd_a, dtrap      f32  [B, L, H]      out
 *   dangles                   f32  [B, L, K]      out (may be NULL when K = 0)
 *   ddt_bias                  f32  [H]            out, optional
 *   dB_raw, dC_raw            f32  [B, L, G, N]   out
 */
typedef struct {
  uint32_t struct_size;
  float A_floor, eps;
  const void *dd_dt, *dd_a, *trap, *angles;
  const float *dt_bias;    /* optional */
  const void *B_raw, *C_raw;
} msc_m3_raw_args;

typedef struct {
  uint32_t struct_size;
  float *ddd_dt, *ddd_a, *dtrap, *dangles;
  float *ddt_bias;         /* optional */
  float *dB_raw, *dC_raw;
} msc_m3_raw_grads;

msc_status msc_mamba3_siso_scan_fwd_raw(const msc_m3_fwd_args *scan, const msc_m3_raw_args *raw,
                                        msc_stream_t stream);
size_t msc_mamba3_siso_scan_fwd_raw_workspace_bytes(int64_t batch, int64_t seqlen,
                                                    int64_t nheads, int64_t headdim,
                                                    int64_t dstate, int64_t ngroups,
                                                    int64_t nangles);
size_t msc_mamba3_siso_scan_bwd_raw_workspace_bytes(int64_t batch, int64_t seqlen,
                                                    int64_t nheads, int64_t headdim,
                                                    int64_t dstate, int64_t ngroups,
                                                    int64_t nangles);
msc_status msc_mamba3_siso_scan_bwd_raw(const msc_m3_bwd_args *scan, const msc_m3_raw_args *raw,
                                        const msc_m3_raw_grads *grads, void *workspace,
                                        size_t workspace_bytes, msc_stream_t stream);

/* ======================================================================
 * Measurement probes: the compute ceiling of the Mamba-1 scans
 * ======================================================================
 * Every state element of every step of the Mamba-1 recurrence takes one
 * 2^x for its decay exp(delta A) (the discretisation of the selective SSM,
 * Mamba paper, Section 3 / Algorithm 2), so the GPU's rate of 2^x bounds the
 * scans from below independently of their memory traffic (mamba-rs 0.7.0
 * README, "Performance", names the scan and the other kernels outside the
 * GEMMs as the bulk of a training step).  These probes measure that rate and
 * the FMA pipe's, for the roofline's compute side.  They are not part of
 * the scan path.
 *
 * Each launches `blocks` CTAs of msc_probe_threads_per_block() threads; a
 * thread runs 8 independent chains for `iters` rounds and writes one float
 * to out[thread] (caller-owned device memory of blocks * threads floats, its
 * values meaningless).  *ops (host memory) receives the number of
 * operations the launch performs: 2^x evaluations (ex2.approx.ftz.f32), or
 * element fused multiply-adds (packed = 1: fma.rn.f32x2, two per
 * instruction; packed = 0: scalar fma.rn.f32).  Time the launch with events
 * on `stream`; rate = ops / time.  blocks must be in 1..2^20, iters in
 * 1..2^24; otherwise MSC_ERR_INVALID_ARG and nothing is launched.
 */
int64_t msc_probe_threads_per_block(void);
msc_status msc_probe_sfu_ex2(float *out, int64_t blocks, int64_t iters, int64_t *ops,
                             msc_stream_t stream);
msc_status msc_probe_ffma(float *out, int64_t blocks, int64_t iters, int32_t packed, int64_t *ops,
                          msc_stream_t stream);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* MSC_H_ */
