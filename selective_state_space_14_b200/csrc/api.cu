// api.cu -- the extern "C" entry points of libmsc.so (declared in msc.h).
//
// Each entry point checks its arguments on the host, translates them into the
// internal launch parameters and enqueues the kernels on the caller's stream.
// Nothing here allocates device memory or synchronises.  Errors are reported
// as msc_status codes plus a thread-local message that names the argument
// (the mamba-rs docs/gemm-modes.md "Errors" section: messages name the call or
// value that failed).
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstddef>
#include <cstdio>
#include <cstring>

#include "../../include/msc.h"
#include "kernels.h"

namespace {

thread_local char g_err[512] = "";

msc_status fail(msc_status st, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

msc_status ok() {
  g_err[0] = '\0';
  return MSC_OK;
}

msc_status cuda_status(cudaError_t e, const char *what) {
  if (e == cudaSuccess) return ok();
  return fail(MSC_ERR_CUDA, "%s: CUDA error %s (%s)", what, cudaGetErrorName(e),
              cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define REQUIRE_PTR(fn, name, ptr)                                                   \
  do {                                                                              \
    if ((ptr) == nullptr) return fail(MSC_ERR_INVALID_ARG, "%s: %s is NULL", fn, name); \
    if (!aligned16(ptr))                                                            \
      return fail(MSC_ERR_ALIGNMENT, "%s: %s is not 16-byte aligned", fn, name);    \
  } while (0)

#define OPTIONAL_PTR(fn, name, ptr)                                                 \
  do {                                                                              \
    if ((ptr) != nullptr && !aligned16(ptr))                                        \
      return fail(MSC_ERR_ALIGNMENT, "%s: %s is not 16-byte aligned", fn, name);    \
  } while (0)

size_t io_size(int32_t dt) { return dt == MSC_F32 ? 4 : 2; }

msc_status check_dtype(const char *fn, int32_t dt) {
  if (dt != MSC_F32 && dt != MSC_BF16 && dt != MSC_F16)
    return fail(MSC_ERR_INVALID_ARG,
                "%s: io_dtype %d is not MSC_F32 (0), MSC_BF16 (1) or MSC_F16 (2)", fn,
                (int)dt);
  return MSC_OK;
}

msc_status check_flag(const char *fn, const char *name, int32_t v) {
  if (v != 0 && v != 1) return fail(MSC_ERR_INVALID_ARG, "%s: %s must be 0 or 1, got %d", fn, name, (int)v);
  return MSC_OK;
}

// Shared size checks of the Mamba-1 scans.
msc_status check_m1_sizes(const char *fn, int64_t B, int64_t D, int64_t N, int64_t L, int64_t G) {
  if (B < 0 || D < 0 || L < 0)
    return fail(MSC_ERR_INVALID_ARG, "%s: batch, dim and seqlen must be >= 0 (got %lld, %lld, %lld)",
                fn, (long long)B, (long long)D, (long long)L);
  if (N < 1 || N > MSC_M1_MAX_DSTATE)
    return fail(MSC_ERR_UNSUPPORTED, "%s: dstate %lld outside the supported range 1..%d", fn,
                (long long)N, MSC_M1_MAX_DSTATE);
  if (G < 1 || (D > 0 && D % G != 0))
    return fail(MSC_ERR_INVALID_ARG, "%s: ngroups %lld must be >= 1 and divide dim %lld", fn,
                (long long)G, (long long)D);
  if (B > 65535)
    return fail(MSC_ERR_UNSUPPORTED, "%s: batch %lld exceeds 65535", fn, (long long)B);
  return MSC_OK;
}

}  // namespace

namespace msc {
// shared with the Mamba-3 entry points (api_m3.cu): one thread-local message
msc_status api_fail(msc_status st, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}
msc_status api_ok() { return ok(); }
// the backward's checks of dtype, flags and sizes (before any size is computed)
msc_status m1_bwd_check_sizes(const char *fn, const msc_ss_bwd_args *a) {
  msc_status st;
  if ((st = check_dtype(fn, a->io_dtype)) != MSC_OK) return st;
  if ((st = check_flag(fn, "delta_softplus", a->delta_softplus)) != MSC_OK) return st;
  return check_m1_sizes(fn, a->batch, a->dim, a->dstate, a->seqlen, a->ngroups);
}
msc_status api_cuda(cudaError_t e, const char *what) { return cuda_status(e, what); }
}  // namespace msc

extern "C" {

const char *msc_last_error(void) { return g_err; }

const char *msc_version(void) { return "msc 0.1.0 sm_100a"; }

// ============================================================== Mamba-1 ====
size_t msc_selective_scan_saved_states_bytes(int64_t batch, int64_t dim, int64_t dstate,
                                             int64_t seqlen) {
  if (batch <= 0 || dim <= 0 || dstate <= 0 || seqlen <= 0) return 0;
  const int64_t n_save = (seqlen + MSC_M1_SAVE_INTERVAL - 1) / MSC_M1_SAVE_INTERVAL;
  return sizeof(float) * (size_t)(batch * dim * n_save * dstate);
}

size_t msc_selective_scan_fwd_workspace_bytes(int64_t batch, int64_t dim, int64_t dstate,
                                              int64_t seqlen) {
  if (batch <= 0 || dim <= 0 || dstate <= 0 || seqlen <= 0) return 0;
  if (dstate > msc::kM1Slab)
    return sizeof(float) * (size_t)(batch * dim * seqlen);  // the sums over the earlier slabs
  // time segments: per segment and state element a decay product and a state
  const int64_t n_seg = msc::m1_fwd_segments(batch, dim, dstate, seqlen);
  return n_seg > 1 ? sizeof(float) * (size_t)(2 * n_seg * batch * dim * dstate) : 0;
}

}  // extern "C"

namespace {
// the Mamba-1 forward, with the causal conv1d fused ahead when conv is non-null
msc_status m1_fwd(const char *fn, const msc_ss_fwd_args *a, const msc_ss_conv_args *conv,
                  msc_stream_t stream) {
  if (!a) return fail(MSC_ERR_INVALID_ARG, "%s: args is NULL", fn);
  // callers built before the workspace fields pass a shorter struct: no workspace
  constexpr size_t kNoWorkspaceSize = offsetof(msc_ss_fwd_args, workspace);
  if (a->struct_size < kNoWorkspaceSize)
    return fail(MSC_ERR_INVALID_ARG, "%s: struct_size %u < %zu", fn, a->struct_size,
                kNoWorkspaceSize);
  const bool has_ws_fields = a->struct_size >= sizeof(msc_ss_fwd_args);
  void *const workspace = has_ws_fields ? a->workspace : nullptr;
  const size_t workspace_bytes = has_ws_fields ? a->workspace_bytes : 0;
  msc_status st;
  if ((st = check_dtype(fn, a->io_dtype)) != MSC_OK) return st;
  if ((st = check_flag(fn, "delta_softplus", a->delta_softplus)) != MSC_OK) return st;
  if ((st = check_m1_sizes(fn, a->batch, a->dim, a->dstate, a->seqlen, a->ngroups)) != MSC_OK)
    return st;
  const int64_t B = a->batch, D = a->dim, N = a->dstate, L = a->seqlen;
  int64_t W = 0;
  if (conv) {
    if (conv->struct_size < sizeof(msc_ss_conv_args))
      return fail(MSC_ERR_INVALID_ARG, "%s: conv struct_size %u < sizeof(msc_ss_conv_args) %zu",
                  fn, conv->struct_size, sizeof(msc_ss_conv_args));
    W = conv->width;
    if (W < 1 || W > MSC_CONV_MAX_WIDTH)
      return fail(MSC_ERR_UNSUPPORTED, "%s: width %lld outside 1..%d", fn, (long long)W,
                  MSC_CONV_MAX_WIDTH);
    REQUIRE_PTR(fn, "w", conv->w);
    OPTIONAL_PTR(fn, "bias", conv->bias);
    OPTIONAL_PTR(fn, "conv_state_in", conv->conv_state_in);
    OPTIONAL_PTR(fn, "conv_state_out", conv->conv_state_out);
    OPTIONAL_PTR(fn, "u_out", conv->u_out);
  }
  if (B == 0 || D == 0) return ok();
  REQUIRE_PTR(fn, "A", a->A);
  OPTIONAL_PTR(fn, "D", a->D);
  OPTIONAL_PTR(fn, "delta_bias", a->delta_bias);
  OPTIONAL_PTR(fn, "h0", a->h0);
  OPTIONAL_PTR(fn, "final_state", a->final_state);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (L == 0) {  // no steps: the final states are the initial states
    cudaError_t e = cudaSuccess;
    if (a->final_state) {
      const size_t bytes = sizeof(float) * (size_t)(B * D * N);
      e = a->h0 ? cudaMemcpyAsync(a->final_state, a->h0, bytes, cudaMemcpyDeviceToDevice, s)
                : cudaMemsetAsync(a->final_state, 0, bytes, s);
    }
    if (e == cudaSuccess && conv && conv->conv_state_out && W > 1) {
      const size_t bytes = sizeof(float) * (size_t)(B * D * (W - 1));
      e = conv->conv_state_in ? cudaMemcpyAsync(conv->conv_state_out, conv->conv_state_in, bytes,
                                                cudaMemcpyDeviceToDevice, s)
                              : cudaMemsetAsync(conv->conv_state_out, 0, bytes, s);
    }
    return cuda_status(e, fn);
  }
  REQUIRE_PTR(fn, "u", a->u);
  REQUIRE_PTR(fn, "delta", a->delta);
  REQUIRE_PTR(fn, "Bm", a->Bm);
  REQUIRE_PTR(fn, "Cm", a->Cm);
  REQUIRE_PTR(fn, "out", a->out);
  OPTIONAL_PTR(fn, "z", a->z);
  OPTIONAL_PTR(fn, "saved_states", a->saved_states);
  const size_t need = msc_selective_scan_fwd_workspace_bytes(B, D, N, L);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need))
    return fail(MSC_ERR_WORKSPACE, "%s: these sizes need a workspace of %zu bytes, %zu given",
                fn, need, workspace ? workspace_bytes : (size_t)0);
  OPTIONAL_PTR(fn, "workspace", workspace);

  msc::M1Params p = {};
  p.io = a->io_dtype;
  p.B = B; p.D = D; p.N = N; p.L = L; p.G = a->ngroups;
  p.softplus = a->delta_softplus;
  p.vec = (L * (int64_t)io_size(a->io_dtype)) % 16 == 0;
  p.u = a->u; p.delta = a->delta; p.Bm = a->Bm; p.Cm = a->Cm; p.z = a->z;
  p.A = a->A; p.Dp = a->D; p.bias = a->delta_bias; p.h0 = a->h0;
  p.out = a->out; p.final_state = a->final_state; p.saved = a->saved_states;
  p.tok_part = need > 0 && N > msc::kM1Slab ? static_cast<float *>(workspace) : nullptr;
  p.seg_ws = need > 0 && N <= msc::kM1Slab ? static_cast<float *>(workspace) : nullptr;
  if (conv) {
    p.conv_W = W;
    p.conv_w = conv->w; p.conv_b = conv->bias;
    p.conv_xs_in = W > 1 ? conv->conv_state_in : nullptr;
    p.conv_xs_out = W > 1 ? conv->conv_state_out : nullptr;
    p.u_out = conv->u_out;
  }
  return cuda_status(msc::launch_m1_fwd(p, s), fn);
}
}  // namespace

extern "C" {

msc_status msc_selective_scan_fwd(const msc_ss_fwd_args *a, msc_stream_t stream) {
  return m1_fwd("msc_selective_scan_fwd", a, nullptr, stream);
}

msc_status msc_selective_scan_conv_fwd(const msc_ss_fwd_args *scan,
                                       const msc_ss_conv_args *conv, msc_stream_t stream) {
  const char *fn = "msc_selective_scan_conv_fwd";
  if (!conv) return fail(MSC_ERR_INVALID_ARG, "%s: conv is NULL", fn);
  return m1_fwd(fn, scan, conv, stream);
}

size_t msc_selective_scan_bwd_workspace_bytes(int64_t batch, int64_t dim, int64_t dstate,
                                              int64_t seqlen, int64_t ngroups) {
  if (batch <= 0 || dim <= 0 || dstate <= 0 || seqlen <= 0) return 0;
  // sizes the backward refuses need no workspace (and ngroups is a divisor)
  if (dstate > MSC_M1_MAX_DSTATE || ngroups < 1 || dim % ngroups != 0) return 0;
  return msc::m1_bwd_workspace_bytes(batch, dim, dstate, seqlen, ngroups);
}

msc_status msc_selective_scan_bwd(const msc_ss_bwd_args *a, void *workspace,
                                  size_t workspace_bytes, msc_stream_t stream) {
  const char *fn = "msc_selective_scan_bwd";
  if (!a) return fail(MSC_ERR_INVALID_ARG, "%s: args is NULL", fn);
  if (a->struct_size < sizeof(msc_ss_bwd_args))
    return fail(MSC_ERR_INVALID_ARG, "%s: struct_size %u < sizeof(msc_ss_bwd_args) %zu", fn,
                a->struct_size, sizeof(msc_ss_bwd_args));
  msc_status st;
  if ((st = check_dtype(fn, a->io_dtype)) != MSC_OK) return st;
  if ((st = check_flag(fn, "delta_softplus", a->delta_softplus)) != MSC_OK) return st;
  if ((st = check_m1_sizes(fn, a->batch, a->dim, a->dstate, a->seqlen, a->ngroups)) != MSC_OK)
    return st;
  const int64_t B = a->batch, D = a->dim, N = a->dstate, L = a->seqlen, G = a->ngroups;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (D == 0) return ok();
  REQUIRE_PTR(fn, "A", a->A);
  REQUIRE_PTR(fn, "dA", a->dA);
  OPTIONAL_PTR(fn, "dD", a->dD);
  OPTIONAL_PTR(fn, "ddelta_bias", a->ddelta_bias);
  OPTIONAL_PTR(fn, "dh0", a->dh0);
  if (B == 0 || L == 0) {  // nothing depends on any parameter: zero gradients
    cudaError_t e = cudaMemsetAsync(a->dA, 0, sizeof(float) * (size_t)(D * N), s);
    if (e == cudaSuccess && a->dD) e = cudaMemsetAsync(a->dD, 0, sizeof(float) * (size_t)D, s);
    if (e == cudaSuccess && a->ddelta_bias)
      e = cudaMemsetAsync(a->ddelta_bias, 0, sizeof(float) * (size_t)D, s);
    if (e == cudaSuccess && a->dh0 && B > 0)
      e = cudaMemsetAsync(a->dh0, 0, sizeof(float) * (size_t)(B * D * N), s);
    return cuda_status(e, fn);
  }
  REQUIRE_PTR(fn, "u", a->u);
  REQUIRE_PTR(fn, "delta", a->delta);
  REQUIRE_PTR(fn, "Bm", a->Bm);
  REQUIRE_PTR(fn, "Cm", a->Cm);
  REQUIRE_PTR(fn, "saved_states", a->saved_states);
  REQUIRE_PTR(fn, "dout", a->dout);
  REQUIRE_PTR(fn, "du", a->du);
  REQUIRE_PTR(fn, "ddelta", a->ddelta);
  REQUIRE_PTR(fn, "dB", a->dB);
  REQUIRE_PTR(fn, "dC", a->dC);
  OPTIONAL_PTR(fn, "D", a->D);
  OPTIONAL_PTR(fn, "delta_bias", a->delta_bias);
  OPTIONAL_PTR(fn, "z", a->z);
  OPTIONAL_PTR(fn, "h0", a->h0);
  OPTIONAL_PTR(fn, "dz", a->dz);
  const size_t need = msc::m1_bwd_workspace_bytes(B, D, N, L, G);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(MSC_ERR_WORKSPACE, "%s: workspace of %zu bytes given, %zu required", fn,
                workspace ? workspace_bytes : (size_t)0, need);
  if (!aligned16(workspace))
    return fail(MSC_ERR_ALIGNMENT, "%s: workspace is not 16-byte aligned", fn);

  msc::M1Params p = {};
  p.io = a->io_dtype;
  p.B = B; p.D = D; p.N = N; p.L = L; p.G = G;
  p.softplus = a->delta_softplus;
  p.vec = (L * (int64_t)io_size(a->io_dtype)) % 16 == 0;
  p.u = a->u; p.delta = a->delta; p.Bm = a->Bm; p.Cm = a->Cm; p.z = a->z;
  p.A = a->A; p.Dp = a->D; p.bias = a->delta_bias; p.h0 = a->h0;
  p.saved_in = a->saved_states; p.dout = a->dout;
  p.du = a->du; p.ddelta = a->ddelta; p.dz = a->z ? a->dz : nullptr;
  p.dA = a->dA; p.dB = a->dB; p.dC = a->dC; p.dD = a->dD; p.dbias = a->ddelta_bias;
  p.dh0 = a->dh0;
  const msc::M1BwdWorkspace w = msc::m1_bwd_workspace(B, D, N, L, G);
  char *const ws = static_cast<char *>(workspace);
  p.n_part = w.n_part;
  p.ws_bc = reinterpret_cast<float *>(ws + w.bc);
  p.ws_misc = reinterpret_cast<float *>(ws + w.misc);
  p.tok_part = N > msc::kM1Slab ? reinterpret_cast<float *>(ws + w.tok) : nullptr;
  if (w.n_seg > 1) {
    p.seg_len = msc::m1_fwd_seg_len(L, w.n_seg);
    p.seg_ws = reinterpret_cast<float *>(ws + w.seg);
  }
  return cuda_status(msc::launch_m1_bwd(p, s), fn);
}

// ======================================================== decode step ====
msc_status msc_ssm_state_update(const msc_su_args *a, msc_stream_t stream) {
  const char *fn = "msc_ssm_state_update";
  if (!a) return fail(MSC_ERR_INVALID_ARG, "%s: args is NULL", fn);
  if (a->struct_size < sizeof(msc_su_args))
    return fail(MSC_ERR_INVALID_ARG, "%s: struct_size %u < sizeof(msc_su_args) %zu", fn,
                a->struct_size, sizeof(msc_su_args));
  msc_status st;
  if ((st = check_dtype(fn, a->io_dtype)) != MSC_OK) return st;
  if ((st = check_flag(fn, "delta_softplus", a->delta_softplus)) != MSC_OK) return st;
  if ((st = check_m1_sizes(fn, 0, a->dim, a->dstate, 0, a->ngroups)) != MSC_OK) return st;
  if (a->batch < 0) return fail(MSC_ERR_INVALID_ARG, "%s: batch must be >= 0", fn);
  if (a->batch == 0 || a->dim == 0) return ok();
  REQUIRE_PTR(fn, "state", a->state);
  REQUIRE_PTR(fn, "x", a->x);
  REQUIRE_PTR(fn, "delta", a->delta);
  REQUIRE_PTR(fn, "A", a->A);
  REQUIRE_PTR(fn, "Bm", a->Bm);
  REQUIRE_PTR(fn, "Cm", a->Cm);
  REQUIRE_PTR(fn, "out", a->out);
  OPTIONAL_PTR(fn, "D", a->D);
  OPTIONAL_PTR(fn, "delta_bias", a->delta_bias);
  OPTIONAL_PTR(fn, "z", a->z);
  msc::SUParams p = {};
  p.io = a->io_dtype;
  p.B = a->batch; p.D = a->dim; p.N = a->dstate; p.G = a->ngroups;
  p.softplus = a->delta_softplus;
  p.state = a->state; p.x = a->x; p.delta = a->delta; p.Bm = a->Bm; p.Cm = a->Cm; p.z = a->z;
  p.A = a->A; p.Dp = a->D; p.bias = a->delta_bias; p.out = a->out;
  return cuda_status(msc::launch_state_update(p, reinterpret_cast<cudaStream_t>(stream)), fn);
}

// ============================================ causal conv1d ahead of the scan ====
size_t msc_causal_conv1d_bwd_workspace_bytes(int64_t batch, int64_t dim, int64_t seqlen,
                                             int64_t width) {
  if (batch <= 0 || dim <= 0 || seqlen <= 0 || width < 1 || width > MSC_CONV_MAX_WIDTH) return 0;
  return msc::conv1d_bwd_workspace_bytes(batch, dim, seqlen, width);
}

}  // extern "C"

namespace {
template <typename Args>
msc_status check_conv(const char *fn, const Args *a) {
  if (!a) return fail(MSC_ERR_INVALID_ARG, "%s: args is NULL", fn);
  if (a->struct_size < sizeof(Args))
    return fail(MSC_ERR_INVALID_ARG, "%s: struct_size %u < sizeof(args) %zu", fn, a->struct_size,
                sizeof(Args));
  msc_status st;
  if ((st = check_dtype(fn, a->io_dtype)) != MSC_OK) return st;
  if (a->batch < 0 || a->dim < 0 || a->seqlen < 0)
    return fail(MSC_ERR_INVALID_ARG, "%s: batch, dim and seqlen must be >= 0", fn);
  if (a->width < 1 || a->width > MSC_CONV_MAX_WIDTH)
    return fail(MSC_ERR_UNSUPPORTED, "%s: width %lld outside 1..%d", fn, (long long)a->width,
                MSC_CONV_MAX_WIDTH);
  REQUIRE_PTR(fn, "w", a->w);
  OPTIONAL_PTR(fn, "bias", a->bias);
  OPTIONAL_PTR(fn, "conv_state_in", a->conv_state_in);
  return MSC_OK;
}
}  // namespace

extern "C" {

msc_status msc_causal_conv1d_fwd(const msc_conv_fwd_args *a, msc_stream_t stream) {
  const char *fn = "msc_causal_conv1d_fwd";
  msc_status st = check_conv(fn, a);
  if (st != MSC_OK) return st;
  OPTIONAL_PTR(fn, "conv_state_out", a->conv_state_out);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t B = a->batch, D = a->dim, L = a->seqlen, W = a->width;
  if (B == 0 || D == 0) return ok();
  if (L == 0) {  // no steps: the state passes through
    if (a->conv_state_out && W > 1) {
      const size_t bytes = sizeof(float) * (size_t)(B * D * (W - 1));
      return cuda_status(a->conv_state_in ? cudaMemcpyAsync(a->conv_state_out, a->conv_state_in,
                                                            bytes, cudaMemcpyDeviceToDevice, s)
                                          : cudaMemsetAsync(a->conv_state_out, 0, bytes, s),
                         fn);
    }
    return ok();
  }
  REQUIRE_PTR(fn, "x", a->x);
  REQUIRE_PTR(fn, "u", a->u);
  msc::ConvParams p = {};
  p.io = a->io_dtype;
  p.B = B; p.D = D; p.L = L; p.W = W;
  p.vec = (L * (int64_t)io_size(a->io_dtype)) % 16 == 0;
  p.x = a->x; p.w = a->w; p.bias = a->bias; p.xs_in = W > 1 ? a->conv_state_in : nullptr;
  p.u = a->u; p.xs_out = W > 1 ? a->conv_state_out : nullptr;
  return cuda_status(msc::launch_conv1d_fwd(p, s), fn);
}

msc_status msc_causal_conv1d_bwd(const msc_conv_bwd_args *a, void *workspace,
                                 size_t workspace_bytes, msc_stream_t stream) {
  const char *fn = "msc_causal_conv1d_bwd";
  msc_status st = check_conv(fn, a);
  if (st != MSC_OK) return st;
  REQUIRE_PTR(fn, "dw", a->dw);
  OPTIONAL_PTR(fn, "dbias", a->dbias);
  OPTIONAL_PTR(fn, "dconv_state_in", a->dconv_state_in);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t B = a->batch, D = a->dim, L = a->seqlen, W = a->width;
  if (B == 0 || D == 0 || L == 0) {  // no steps: zero gradients
    cudaError_t e = D > 0 ? cudaMemsetAsync(a->dw, 0, sizeof(float) * (size_t)(D * W), s)
                          : cudaSuccess;
    if (e == cudaSuccess && a->dbias && D > 0)
      e = cudaMemsetAsync(a->dbias, 0, sizeof(float) * (size_t)D, s);
    if (e == cudaSuccess && a->dconv_state_in && W > 1 && B * D > 0)
      e = cudaMemsetAsync(a->dconv_state_in, 0, sizeof(float) * (size_t)(B * D * (W - 1)), s);
    return cuda_status(e, fn);
  }
  REQUIRE_PTR(fn, "x", a->x);
  REQUIRE_PTR(fn, "du", a->du);
  REQUIRE_PTR(fn, "dx", a->dx);
  const size_t need = msc::conv1d_bwd_workspace_bytes(B, D, L, W);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(MSC_ERR_WORKSPACE, "%s: workspace of %zu bytes given, %zu required", fn,
                workspace ? workspace_bytes : (size_t)0, need);
  if (!aligned16(workspace))
    return fail(MSC_ERR_ALIGNMENT, "%s: workspace is not 16-byte aligned", fn);
  msc::ConvParams p = {};
  p.io = a->io_dtype;
  p.B = B; p.D = D; p.L = L; p.W = W;
  p.vec = (L * (int64_t)io_size(a->io_dtype)) % 16 == 0;
  p.x = a->x; p.w = a->w; p.bias = a->bias; p.xs_in = W > 1 ? a->conv_state_in : nullptr;
  p.du = a->du; p.dx = a->dx; p.dw = a->dw; p.dbias = a->dbias;
  p.dxs_in = W > 1 ? a->dconv_state_in : nullptr;
  p.ws = static_cast<float *>(workspace);
  return cuda_status(msc::launch_conv1d_bwd(p, s), fn);
}

}  // extern "C"
