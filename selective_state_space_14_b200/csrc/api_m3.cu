// api_m3.cu -- extern "C" entry points of the Mamba-3 SISO scan (msc.h).
//
// Argument checks on the host, then the launch on the caller's stream.  Same
// conventions as api.cu: status codes, a thread-local message naming the
// argument, no allocation, no synchronisation.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstddef>
#include <cstdio>

#include "../../include/msc.h"
#include "kernels.h"

static_assert(MSC_M3_CHUNK == MSC_M3_CHUNK_STEPS, "saved-state interval");

namespace msc {
msc_status api_fail(msc_status st, const char *fmt, ...);
msc_status api_ok();
msc_status api_cuda(cudaError_t e, const char *what);
}  // namespace msc

namespace {

using msc::api_cuda;
using msc::api_fail;
using msc::api_ok;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define M3_REQUIRE(fn, name, ptr)                                                        \
  do {                                                                                   \
    if ((ptr) == nullptr) return api_fail(MSC_ERR_INVALID_ARG, "%s: %s is NULL", fn, name); \
    if (!aligned16(ptr))                                                                 \
      return api_fail(MSC_ERR_ALIGNMENT, "%s: %s is not 16-byte aligned", fn, name);     \
  } while (0)

#define M3_OPTIONAL(fn, name, ptr)                                                       \
  do {                                                                                   \
    if ((ptr) != nullptr && !aligned16(ptr))                                             \
      return api_fail(MSC_ERR_ALIGNMENT, "%s: %s is not 16-byte aligned", fn, name);     \
  } while (0)

template <typename Args>
msc_status check_m3(const char *fn, const Args *a, size_t min_size = sizeof(Args)) {
  if (!a) return api_fail(MSC_ERR_INVALID_ARG, "%s: args is NULL", fn);
  if (a->struct_size < min_size)
    return api_fail(MSC_ERR_INVALID_ARG, "%s: struct_size %u is smaller than the struct (%zu)",
                    fn, a->struct_size, min_size);
  if (a->io_dtype != MSC_F32 && a->io_dtype != MSC_BF16 && a->io_dtype != MSC_F16)
    return api_fail(MSC_ERR_INVALID_ARG,
                    "%s: io_dtype %d is not MSC_F32 (0), MSC_BF16 (1) or MSC_F16 (2)",
                    fn, (int)a->io_dtype);
  if (a->batch < 0 || a->seqlen < 0 || a->nheads < 1 || a->ngroups < 1 || a->nangles < 0)
    return api_fail(MSC_ERR_INVALID_ARG,
                    "%s: need batch >= 0, seqlen >= 0, nheads >= 1, ngroups >= 1, nangles >= 0",
                    fn);
  if (a->nheads % a->ngroups != 0)
    return api_fail(MSC_ERR_INVALID_ARG, "%s: ngroups %lld does not divide nheads %lld", fn,
                    (long long)a->ngroups, (long long)a->nheads);
  if (!msc::m3_supported(a->headdim, a->dstate))
    return api_fail(MSC_ERR_UNSUPPORTED,
                    "%s: headdim %lld / dstate %lld not supported (headdim 16, 32 or 64; dstate 16, "
                    "32, 64, 128, 192 or 256)", fn,
                    (long long)a->headdim, (long long)a->dstate);
  if (2 * a->nangles > a->dstate)
    return api_fail(MSC_ERR_INVALID_ARG, "%s: 2 * nangles (%lld) exceeds dstate (%lld)", fn,
                    (long long)(2 * a->nangles), (long long)a->dstate);
  if (a->batch > 65535 || a->nheads > 65535)
    return api_fail(MSC_ERR_UNSUPPORTED, "%s: batch and nheads must be <= 65535", fn);
  return MSC_OK;
}

}  // namespace

extern "C" {

size_t msc_mamba3_siso_saved_states_bytes(int64_t batch, int64_t seqlen, int64_t nheads,
                                          int64_t headdim, int64_t dstate) {
  if (batch <= 0 || seqlen <= 0 || nheads <= 0 || headdim <= 0 || dstate <= 0) return 0;
  const int64_t nc = (seqlen + MSC_M3_CHUNK - 1) / MSC_M3_CHUNK;
  // chunk-start states, then chunk-start cumulative angles
  return sizeof(float) * (size_t)(batch * nheads * nc * (headdim * dstate + dstate / 2));
}

size_t msc_mamba3_siso_scan_fwd_workspace_bytes(int64_t batch, int64_t seqlen, int64_t nheads,
                                                int64_t headdim, int64_t dstate) {
  if (batch <= 0 || seqlen <= 0 || nheads <= 0 || headdim <= 0 || dstate <= msc::kM3Slab) return 0;
  return sizeof(float) * (size_t)(batch * seqlen * nheads * headdim);  // y over the earlier slabs
}

}  // extern "C"

namespace {

// The raw projections' checks for the fused entry points (after the scan
// struct's own checks): bf16 io, d_state 16, 32 or 64 (the tensor-core
// kernels), and the raw rows present wherever there are tokens.
template <typename Scan>
msc_status check_raw(const char *fn, const Scan *a, const msc_m3_raw_args *raw) {
  if (!a) return api_fail(MSC_ERR_INVALID_ARG, "%s: args is NULL", fn);
  if (!raw) return api_fail(MSC_ERR_INVALID_ARG, "%s: raw is NULL", fn);
  if (raw->struct_size < sizeof(msc_m3_raw_args))
    return api_fail(MSC_ERR_INVALID_ARG, "%s: raw struct_size %u is smaller than the struct (%zu)",
                    fn, raw->struct_size, sizeof(msc_m3_raw_args));
  if (a->io_dtype != MSC_BF16)
    return api_fail(MSC_ERR_UNSUPPORTED,
                    "%s: io_dtype %d: the fused path takes bf16 io (use "
                    "msc_mamba3_siso_discretize and the scan)", fn, (int)a->io_dtype);
  // the tensor-core kernels of one 64-state slab
  if (a->dstate != 16 && a->dstate != 32 && a->dstate != 64)
    return api_fail(MSC_ERR_UNSUPPORTED,
                    "%s: dstate %lld: the fused path takes d_state 16, 32 or 64 (use "
                    "msc_mamba3_siso_discretize and the scan)", fn, (long long)a->dstate);
  if (!(raw->A_floor >= 0.f) || !(raw->eps >= 0.f))
    return api_fail(MSC_ERR_INVALID_ARG, "%s: A_floor and eps must be >= 0", fn);
  M3_OPTIONAL(fn, "dt_bias", raw->dt_bias);
  if (a->batch > 0 && a->seqlen > 0) {
    M3_REQUIRE(fn, "dd_dt", raw->dd_dt);
    M3_REQUIRE(fn, "dd_a", raw->dd_a);
    M3_REQUIRE(fn, "trap", raw->trap);
    if (a->nangles > 0) M3_REQUIRE(fn, "angles", raw->angles);
    M3_REQUIRE(fn, "B_raw", raw->B_raw);
    M3_REQUIRE(fn, "C_raw", raw->C_raw);
  }
  return MSC_OK;
}

// BCNorm's rows in the fused entry points' workspace: Bm, Cm bf16 [B, L, G, N]
// each, 256-byte aligned.  BCNorm is per (b, t, g), shared by the group's
// heads, so it runs once per row ahead of the per-head scan kernels.
size_t bcnorm_bytes(int64_t B, int64_t L, int64_t G, int64_t N) {
  return (sizeof(uint16_t) * (size_t)(B * L * G * N) + 255) / 256 * 256;
}

// The BCNorm pass: the discretisation kernel with its B and C outputs alone,
// so the rows are the bits msc_mamba3_siso_discretize writes.
template <typename Scan>
cudaError_t bcnorm_pass(const Scan *a, const msc_m3_raw_args *raw, void *bn, void *cn,
                        cudaStream_t s) {
  msc::M3DiscParams d = {};
  d.io = a->io_dtype;
  d.B = a->batch; d.L = a->seqlen; d.H = a->nheads; d.N = a->dstate; d.G = a->ngroups;
  d.K = a->nangles;
  d.bc_only = true;
  d.A_floor = raw->A_floor; d.eps = raw->eps;
  d.B_raw = raw->B_raw; d.C_raw = raw->C_raw;
  d.Bm = bn; d.Cm = cn;
  return msc::launch_m3_disc_fwd(d, s);
}

// The scan arguments with the derived inputs taken by the raw rows (alpha ..
// theta) and by BCNorm's rows (Bm, Cm), so that the scan's own pointer checks
// test those.
template <typename Scan>
Scan with_raw(const Scan *a, const msc_m3_raw_args *raw, const void *bn, const void *cn) {
  Scan s = *a;
  s.Bm = bn;
  s.Cm = cn;
  s.alpha = raw->dd_dt;
  s.beta = raw->dd_a;
  s.gamma = raw->trap;
  s.theta = raw->angles;
  return s;
}

void set_raw(msc::M3Params &p, const msc_m3_raw_args *raw) {
  p.raw = true;
  p.alpha = p.beta = p.gamma = p.theta = nullptr;
  p.dd_dt = raw->dd_dt;
  p.dd_a = raw->dd_a;
  p.trap = raw->trap;
  p.angles = raw->angles;
  p.dt_bias = raw->dt_bias;
  p.A_floor = raw->A_floor;
  p.eps = raw->eps;
}

// the scan forward; raw non-null: from raw projections (the arguments'
// derived-input pointers already replaced by with_raw)
msc_status m3_fwd_impl(const char *fn, const msc_m3_fwd_args *a, const msc_m3_raw_args *raw,
                       msc_stream_t stream) {
  // callers built before the workspace fields pass a shorter struct: no workspace
  msc_status st = check_m3(fn, a, offsetof(msc_m3_fwd_args, workspace));
  if (st != MSC_OK) return st;
  const bool has_ws_fields = a->struct_size >= sizeof(msc_m3_fwd_args);
  void *const workspace = has_ws_fields ? a->workspace : nullptr;
  const size_t workspace_bytes = has_ws_fields ? a->workspace_bytes : 0;
  if (a->batch == 0) return api_ok();
  M3_OPTIONAL(fn, "D", a->D);
  M3_OPTIONAL(fn, "h0", a->h0);
  M3_OPTIONAL(fn, "final_state", a->final_state);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t B = a->batch, H = a->nheads, P = a->headdim, N = a->dstate;
  if (a->seqlen == 0) {
    if (a->final_state) {
      const size_t bytes = sizeof(float) * (size_t)(B * H * P * N);
      return api_cuda(a->h0 ? cudaMemcpyAsync(a->final_state, a->h0, bytes,
                                              cudaMemcpyDeviceToDevice, s)
                            : cudaMemsetAsync(a->final_state, 0, bytes, s),
                      fn);
    }
    return api_ok();
  }
  M3_REQUIRE(fn, "x", a->x);
  M3_REQUIRE(fn, "Bm", a->Bm);
  M3_REQUIRE(fn, "Cm", a->Cm);
  M3_REQUIRE(fn, "alpha", a->alpha);
  M3_REQUIRE(fn, "beta", a->beta);
  M3_REQUIRE(fn, "gamma", a->gamma);
  if (a->nangles > 0) M3_REQUIRE(fn, "theta", a->theta);
  M3_REQUIRE(fn, "out", a->out);
  M3_OPTIONAL(fn, "z", a->z);
  M3_OPTIONAL(fn, "saved_states", a->saved_states);
  const size_t need = msc_mamba3_siso_scan_fwd_workspace_bytes(B, a->seqlen, H, P, N);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need))
    return api_fail(MSC_ERR_WORKSPACE, "%s: dstate %lld needs a workspace of %zu bytes, %zu given",
                    fn, (long long)N, need, workspace ? workspace_bytes : (size_t)0);
  M3_OPTIONAL(fn, "workspace", workspace);
  msc::M3Params p = {};
  p.io = a->io_dtype;
  p.B = B; p.L = a->seqlen; p.H = H; p.P = P; p.N = N; p.G = a->ngroups; p.K = a->nangles;
  p.x = a->x; p.z = a->z; p.Bm = a->Bm; p.Cm = a->Cm;
  p.alpha = a->alpha; p.beta = a->beta; p.gamma = a->gamma; p.theta = a->theta;
  p.Dp = a->D; p.h0 = a->h0; p.out = a->out; p.final_state = a->final_state;
  p.saved = a->saved_states;
  p.tok_y = need > 0 ? static_cast<float *>(workspace) : nullptr;
  if (raw) set_raw(p, raw);
  return api_cuda(msc::launch_m3_fwd(p, s), fn);
}

}  // namespace

extern "C" {

msc_status msc_mamba3_siso_scan_fwd(const msc_m3_fwd_args *a, msc_stream_t stream) {
  return m3_fwd_impl("msc_mamba3_siso_scan_fwd", a, nullptr, stream);
}

msc_status msc_mamba3_siso_scan_fwd_raw(const msc_m3_fwd_args *a, const msc_m3_raw_args *raw,
                                        msc_stream_t stream) {
  const char *fn = "msc_mamba3_siso_scan_fwd_raw";
  msc_status st = check_m3(fn, a);
  if (st != MSC_OK) return st;
  if ((st = check_raw(fn, a, raw)) != MSC_OK) return st;
  const int64_t B = a->batch, L = a->seqlen, G = a->ngroups, N = a->dstate;
  if (B == 0 || L == 0) return m3_fwd_impl(fn, a, raw, stream);  // no rows to normalise
  const size_t rows = bcnorm_bytes(B, L, G, N);
  if (a->workspace == nullptr || a->workspace_bytes < 2 * rows)
    return api_fail(MSC_ERR_WORKSPACE, "%s: workspace of %zu bytes given, %zu required", fn,
                    a->workspace ? a->workspace_bytes : (size_t)0, 2 * rows);
  M3_REQUIRE(fn, "workspace", a->workspace);
  char *ws = static_cast<char *>(a->workspace);
  msc_m3_fwd_args s = with_raw(a, raw, ws, ws + rows);
  s.workspace = nullptr;  // d_state <= 64: the scan itself needs none
  s.workspace_bytes = 0;
  // the scan's own pointer checks, ahead of the BCNorm launch
  M3_REQUIRE(fn, "x", s.x);
  M3_REQUIRE(fn, "out", s.out);
  M3_OPTIONAL(fn, "z", s.z);
  M3_OPTIONAL(fn, "D", s.D);
  M3_OPTIONAL(fn, "h0", s.h0);
  M3_OPTIONAL(fn, "final_state", s.final_state);
  M3_OPTIONAL(fn, "saved_states", s.saved_states);
  if ((st = api_cuda(bcnorm_pass(a, raw, ws, ws + rows, reinterpret_cast<cudaStream_t>(stream)),
                     fn)) != MSC_OK)
    return st;
  return m3_fwd_impl(fn, &s, raw, stream);
}

size_t msc_mamba3_siso_scan_fwd_raw_workspace_bytes(int64_t batch, int64_t seqlen,
                                                    int64_t nheads, int64_t headdim,
                                                    int64_t dstate, int64_t ngroups,
                                                    int64_t nangles) {
  if (batch <= 0 || seqlen <= 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || ngroups <= 0 ||
      nangles < 0)
    return 0;
  return 2 * bcnorm_bytes(batch, seqlen, ngroups, dstate);
}

size_t msc_mamba3_siso_scan_bwd_workspace_bytes(int64_t batch, int64_t seqlen, int64_t nheads,
                                                int64_t headdim, int64_t dstate,
                                                int64_t ngroups, int64_t nangles) {
  if (batch <= 0 || seqlen <= 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || ngroups <= 0)
    return 0;
  return msc::m3_bwd_workspace_bytes(batch, seqlen, nheads, headdim, dstate, ngroups, nangles);
}

}  // extern "C"

namespace {

// the scan backward (the raw-projection entry point points the derived inputs
// and their gradients into its workspace)
msc_status m3_bwd_impl(const char *fn, const msc_m3_bwd_args *a, void *workspace,
                       size_t workspace_bytes, msc_stream_t stream) {
  msc_status st = check_m3(fn, a);
  if (st != MSC_OK) return st;
  const int64_t B = a->batch, L = a->seqlen, H = a->nheads, P = a->headdim, N = a->dstate;
  const int64_t G = a->ngroups, K = a->nangles;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (B == 0) {
    if (a->dD) return api_cuda(cudaMemsetAsync(a->dD, 0, sizeof(float) * (size_t)H, s), fn);
    return api_ok();
  }
  M3_OPTIONAL(fn, "dD", a->dD);
  M3_OPTIONAL(fn, "dh0", a->dh0);
  if (L == 0) {
    cudaError_t e = cudaSuccess;
    if (a->dD) e = cudaMemsetAsync(a->dD, 0, sizeof(float) * (size_t)H, s);
    if (e == cudaSuccess && a->dh0)
      e = cudaMemsetAsync(a->dh0, 0, sizeof(float) * (size_t)(B * H * P * N), s);
    return api_cuda(e, fn);
  }
  M3_REQUIRE(fn, "x", a->x);
  M3_REQUIRE(fn, "Bm", a->Bm);
  M3_REQUIRE(fn, "Cm", a->Cm);
  M3_REQUIRE(fn, "alpha", a->alpha);
  M3_REQUIRE(fn, "beta", a->beta);
  M3_REQUIRE(fn, "gamma", a->gamma);
  if (K > 0) {
    M3_REQUIRE(fn, "theta", a->theta);
    M3_REQUIRE(fn, "dtheta", a->dtheta);
  }
  M3_REQUIRE(fn, "saved_states", a->saved_states);
  M3_REQUIRE(fn, "dout", a->dout);
  M3_REQUIRE(fn, "dx", a->dx);
  M3_REQUIRE(fn, "dB", a->dB);
  M3_REQUIRE(fn, "dC", a->dC);
  M3_REQUIRE(fn, "dalpha", a->dalpha);
  M3_REQUIRE(fn, "dbeta", a->dbeta);
  M3_REQUIRE(fn, "dgamma", a->dgamma);
  M3_OPTIONAL(fn, "z", a->z);
  M3_OPTIONAL(fn, "dz", a->dz);
  M3_OPTIONAL(fn, "D", a->D);
  M3_OPTIONAL(fn, "h0", a->h0);
  const size_t need = msc::m3_bwd_workspace_bytes(B, L, H, P, N, G, K);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need))
    return api_fail(MSC_ERR_WORKSPACE, "%s: workspace of %zu bytes given, %zu required", fn,
                    workspace ? workspace_bytes : (size_t)0, need);
  if (workspace && !aligned16(workspace))
    return api_fail(MSC_ERR_ALIGNMENT, "%s: workspace is not 16-byte aligned", fn);
  msc::M3Params p = {};
  p.io = a->io_dtype;
  p.B = B; p.L = L; p.H = H; p.P = P; p.N = N; p.G = G; p.K = K;
  p.x = a->x; p.z = a->z; p.Bm = a->Bm; p.Cm = a->Cm;
  p.alpha = a->alpha; p.beta = a->beta; p.gamma = a->gamma; p.theta = a->theta;
  p.Dp = a->D; p.h0 = a->h0; p.saved_in = a->saved_states; p.dout = a->dout;
  p.dx = a->dx; p.dz = a->z ? a->dz : nullptr; p.dB = a->dB; p.dC = a->dC;
  p.dalpha = a->dalpha; p.dbeta = a->dbeta; p.dgamma = a->dgamma; p.dtheta = a->dtheta;
  p.dD = a->dD; p.dh0 = a->dh0; p.ws = workspace; p.ws_bytes = workspace_bytes;
  return api_cuda(msc::launch_m3_bwd(p, s), fn);
}

// the raw-projection backward's workspace: the scan's own, then the scan's
// f32 gradients of the derived inputs: dalpha, dbeta, dgamma [B, L, H],
// dtheta [B, L, H, K], dB, dC [B, L, G, N], then the derived inputs
// themselves (bf16): alpha, beta, gamma [B, L, H], theta [B, L, H, K], Bm,
// Cm [B, L, G, N]
struct RawWs {
  size_t da, db, dg, dth, dB, dC, al, be, ga, th, bn, cn, total;
};
RawWs raw_ws(int64_t B, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G, int64_t K) {
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  RawWs w;
  w.da = up(msc::m3_bwd_workspace_bytes(B, L, H, P, N, G, K));
  const size_t th = up(sizeof(float) * (size_t)(B * L * H));
  w.db = w.da + th;
  w.dg = w.db + th;
  w.dth = w.dg + th;
  w.dB = w.dth + up(sizeof(float) * (size_t)(B * L * H * (K > 0 ? K : 1)));
  w.dC = w.dB + up(sizeof(float) * (size_t)(B * L * G * N));
  // the discretisation's outputs, re-derived from the raw projections (bf16)
  w.al = w.dC + up(sizeof(float) * (size_t)(B * L * G * N));
  const size_t hb = up(sizeof(uint16_t) * (size_t)(B * L * H));
  w.be = w.al + hb;
  w.ga = w.be + hb;
  w.th = w.ga + hb;
  w.bn = w.th + up(sizeof(uint16_t) * (size_t)(B * L * H * (K > 0 ? K : 1)));
  w.cn = w.bn + bcnorm_bytes(B, L, G, N);
  w.total = w.cn + bcnorm_bytes(B, L, G, N);
  return w;
}

}  // namespace

extern "C" {

msc_status msc_mamba3_siso_scan_bwd(const msc_m3_bwd_args *a, void *workspace,
                                    size_t workspace_bytes, msc_stream_t stream) {
  return m3_bwd_impl("msc_mamba3_siso_scan_bwd", a, workspace, workspace_bytes, stream);
}

size_t msc_mamba3_siso_scan_bwd_raw_workspace_bytes(int64_t batch, int64_t seqlen,
                                                    int64_t nheads, int64_t headdim,
                                                    int64_t dstate, int64_t ngroups,
                                                    int64_t nangles) {
  if (batch <= 0 || seqlen <= 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || ngroups <= 0 ||
      nangles < 0)
    return 0;
  return raw_ws(batch, seqlen, nheads, headdim, dstate, ngroups, nangles).total;
}

msc_status msc_mamba3_siso_scan_bwd_raw(const msc_m3_bwd_args *a, const msc_m3_raw_args *raw,
                                        const msc_m3_raw_grads *grads, void *workspace,
                                        size_t workspace_bytes, msc_stream_t stream) {
  const char *fn = "msc_mamba3_siso_scan_bwd_raw";
  msc_status st = check_m3(fn, a);
  if (st != MSC_OK) return st;
  if ((st = check_raw(fn, a, raw)) != MSC_OK) return st;
  if (!grads) return api_fail(MSC_ERR_INVALID_ARG, "%s: grads is NULL", fn);
  if (grads->struct_size < sizeof(msc_m3_raw_grads))
    return api_fail(MSC_ERR_INVALID_ARG,
                    "%s: grads struct_size %u is smaller than the struct (%zu)", fn,
                    grads->struct_size, sizeof(msc_m3_raw_grads));
  M3_OPTIONAL(fn, "ddt_bias", grads->ddt_bias);
  const int64_t B = a->batch, L = a->seqlen, H = a->nheads, P = a->headdim, N = a->dstate;
  const int64_t G = a->ngroups, K = a->nangles;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  msc_m3_bwd_args sa = *a;
  if (B == 0 || L == 0) {  // no tokens: dD, dh0 and the bias gradient are 0
    st = m3_bwd_impl(fn, &sa, workspace, workspace_bytes, stream);
    if (st != MSC_OK || !grads->ddt_bias) return st;
    return api_cuda(cudaMemsetAsync(grads->ddt_bias, 0, sizeof(float) * (size_t)H, s), fn);
  }
  const RawWs w = raw_ws(B, L, H, P, N, G, K);
  if (workspace == nullptr || workspace_bytes < w.total)
    return api_fail(MSC_ERR_WORKSPACE, "%s: workspace of %zu bytes given, %zu required", fn,
                    workspace ? workspace_bytes : (size_t)0, w.total);
  M3_REQUIRE(fn, "workspace", workspace);
  M3_REQUIRE(fn, "ddd_dt", grads->ddd_dt);
  M3_REQUIRE(fn, "ddd_a", grads->ddd_a);
  M3_REQUIRE(fn, "dtrap", grads->dtrap);
  if (K > 0) M3_REQUIRE(fn, "dangles", grads->dangles);
  M3_REQUIRE(fn, "dB_raw", grads->dB_raw);
  M3_REQUIRE(fn, "dC_raw", grads->dC_raw);
  // the scan's own pointer checks, ahead of the first launch
  M3_REQUIRE(fn, "x", a->x);
  M3_REQUIRE(fn, "saved_states", a->saved_states);
  M3_REQUIRE(fn, "dout", a->dout);
  M3_REQUIRE(fn, "dx", a->dx);
  M3_OPTIONAL(fn, "z", a->z);
  M3_OPTIONAL(fn, "dz", a->dz);
  M3_OPTIONAL(fn, "D", a->D);
  M3_OPTIONAL(fn, "h0", a->h0);
  M3_OPTIONAL(fn, "dD", a->dD);
  M3_OPTIONAL(fn, "dh0", a->dh0);
  char *ws = static_cast<char *>(workspace);
  // the discretisation and BCNorm once, into the workspace: the backward's two
  // chunk kernels then read them (deriving the per-head values inside both
  // measured slower than this pass and the reads)
  msc::M3DiscParams f = {};
  f.io = a->io_dtype;
  f.B = B; f.L = L; f.H = H; f.N = N; f.G = G; f.K = K;
  f.A_floor = raw->A_floor; f.eps = raw->eps;
  f.dd_dt = raw->dd_dt; f.dd_a = raw->dd_a; f.trap = raw->trap; f.angles = raw->angles;
  f.dt_bias = raw->dt_bias; f.B_raw = raw->B_raw; f.C_raw = raw->C_raw;
  f.alpha = ws + w.al; f.beta = ws + w.be; f.gamma = ws + w.ga;
  f.theta = K > 0 ? ws + w.th : nullptr;
  f.Bm = ws + w.bn; f.Cm = ws + w.cn;
  if ((st = api_cuda(msc::launch_m3_disc_fwd(f, s), fn)) != MSC_OK) return st;
  sa.alpha = f.alpha; sa.beta = f.beta; sa.gamma = f.gamma; sa.theta = f.theta;
  sa.Bm = f.Bm; sa.Cm = f.Cm;
  sa.dalpha = reinterpret_cast<float *>(ws + w.da);
  sa.dbeta = reinterpret_cast<float *>(ws + w.db);
  sa.dgamma = reinterpret_cast<float *>(ws + w.dg);
  sa.dtheta = reinterpret_cast<float *>(ws + w.dth);
  sa.dB = reinterpret_cast<float *>(ws + w.dB);
  sa.dC = reinterpret_cast<float *>(ws + w.dC);
  st = m3_bwd_impl(fn, &sa, workspace, w.da, stream);
  if (st != MSC_OK) return st;
  // the discretisation's backward on the scan's gradients of its outputs
  msc::M3DiscParams d = {};
  d.io = a->io_dtype;
  d.B = B; d.L = L; d.H = H; d.N = N; d.G = G; d.K = K;
  d.A_floor = raw->A_floor; d.eps = raw->eps;
  d.dd_dt = raw->dd_dt; d.dd_a = raw->dd_a; d.trap = raw->trap; d.angles = raw->angles;
  d.dt_bias = raw->dt_bias; d.B_raw = raw->B_raw; d.C_raw = raw->C_raw;
  d.dalpha = sa.dalpha; d.dbeta = sa.dbeta; d.dgamma = sa.dgamma; d.dtheta = sa.dtheta;
  d.dB = sa.dB; d.dC = sa.dC;
  d.ddd_dt = grads->ddd_dt; d.ddd_a = grads->ddd_a; d.dtrap = grads->dtrap;
  d.dangles = grads->dangles; d.ddt_bias = grads->ddt_bias;
  d.dB_raw = grads->dB_raw; d.dC_raw = grads->dC_raw;
  return api_cuda(msc::launch_m3_disc_bwd(d, s), fn);
}

}  // extern "C"

namespace {
// the decode step; raw non-null: the discretisation and BCNorm fused ahead
msc_status m3_step(const char *fn, const msc_m3_su_args *a, const msc_m3_disc_step_args *raw,
                   msc_stream_t stream) {
  if (!a) return api_fail(MSC_ERR_INVALID_ARG, "%s: args is NULL", fn);
  if (a->struct_size < sizeof(msc_m3_su_args))
    return api_fail(MSC_ERR_INVALID_ARG, "%s: struct_size %u is smaller than the struct (%zu)",
                    fn, a->struct_size, sizeof(msc_m3_su_args));
  if (a->io_dtype != MSC_F32 && a->io_dtype != MSC_BF16 && a->io_dtype != MSC_F16)
    return api_fail(MSC_ERR_INVALID_ARG,
                    "%s: io_dtype %d is not MSC_F32 (0), MSC_BF16 (1) or MSC_F16 (2)",
                    fn, (int)a->io_dtype);
  if (a->batch < 0 || a->nheads < 1 || a->ngroups < 1 || a->nangles < 0)
    return api_fail(MSC_ERR_INVALID_ARG,
                    "%s: need batch >= 0, nheads >= 1, ngroups >= 1, nangles >= 0", fn);
  if (a->nheads % a->ngroups != 0)
    return api_fail(MSC_ERR_INVALID_ARG, "%s: ngroups %lld does not divide nheads %lld", fn,
                    (long long)a->ngroups, (long long)a->nheads);
  if (!msc::m3_supported(a->headdim, a->dstate))
    return api_fail(MSC_ERR_UNSUPPORTED,
                    "%s: headdim %lld / dstate %lld not supported (headdim 16, 32 or 64; dstate 16, "
                    "32, 64, 128, 192 or 256)", fn,
                    (long long)a->headdim, (long long)a->dstate);
  if (2 * a->nangles > a->dstate)
    return api_fail(MSC_ERR_INVALID_ARG, "%s: 2 * nangles (%lld) exceeds dstate (%lld)", fn,
                    (long long)(2 * a->nangles), (long long)a->dstate);
  if (a->batch * a->nheads > ((int64_t)1 << 31))
    return api_fail(MSC_ERR_UNSUPPORTED, "%s: batch * nheads must be <= 2^31", fn);
  if (a->batch == 0) return api_ok();
  M3_REQUIRE(fn, "state", a->state);
  M3_REQUIRE(fn, "x_prev", a->x_prev);
  M3_REQUIRE(fn, "bt_prev", a->bt_prev);
  M3_REQUIRE(fn, "x", a->x);
  M3_REQUIRE(fn, "out", a->out);
  if (a->nangles > 0) M3_REQUIRE(fn, "phi", a->phi);
  if (raw) {
    if (raw->struct_size < sizeof(msc_m3_disc_step_args))
      return api_fail(MSC_ERR_INVALID_ARG, "%s: raw struct_size %u is smaller than the struct "
                      "(%zu)", fn, raw->struct_size, sizeof(msc_m3_disc_step_args));
    if (!(raw->A_floor >= 0.f) || !(raw->eps >= 0.f))
      return api_fail(MSC_ERR_INVALID_ARG, "%s: A_floor and eps must be >= 0", fn);
    M3_REQUIRE(fn, "dd_dt", raw->dd_dt);
    M3_REQUIRE(fn, "dd_a", raw->dd_a);
    M3_REQUIRE(fn, "trap", raw->trap);
    if (a->nangles > 0) M3_REQUIRE(fn, "angles", raw->angles);
    M3_OPTIONAL(fn, "dt_bias", raw->dt_bias);
    M3_REQUIRE(fn, "B_raw", raw->B_raw);
    M3_REQUIRE(fn, "C_raw", raw->C_raw);
  } else {
    M3_REQUIRE(fn, "Bm", a->Bm);
    M3_REQUIRE(fn, "Cm", a->Cm);
    M3_REQUIRE(fn, "alpha", a->alpha);
    M3_REQUIRE(fn, "beta", a->beta);
    M3_REQUIRE(fn, "gamma", a->gamma);
    if (a->nangles > 0) M3_REQUIRE(fn, "theta", a->theta);
  }
  M3_OPTIONAL(fn, "z", a->z);
  M3_OPTIONAL(fn, "D", a->D);
  msc::M3SUParams p = {};
  p.io = a->io_dtype;
  p.B = a->batch; p.H = a->nheads; p.P = a->headdim; p.N = a->dstate; p.G = a->ngroups;
  p.K = a->nangles;
  p.state = a->state; p.x_prev = a->x_prev; p.bt_prev = a->bt_prev; p.phi = a->phi;
  p.x = a->x; p.z = a->z; p.Bm = a->Bm; p.Cm = a->Cm;
  p.alpha = a->alpha; p.beta = a->beta; p.gamma = a->gamma; p.theta = a->theta;
  p.Dp = a->D; p.out = a->out;
  if (raw) {
    p.raw = true;
    p.dd_dt = raw->dd_dt; p.dd_a = raw->dd_a; p.trap = raw->trap; p.angles = raw->angles;
    p.dt_bias = raw->dt_bias; p.B_raw = raw->B_raw; p.C_raw = raw->C_raw;
    p.A_floor = raw->A_floor; p.eps = raw->eps;
  }
  return api_cuda(msc::launch_m3_state_update(p, reinterpret_cast<cudaStream_t>(stream)), fn);
}
}  // namespace

extern "C" {

msc_status msc_mamba3_siso_state_update(const msc_m3_su_args *a, msc_stream_t stream) {
  return m3_step("msc_mamba3_siso_state_update", a, nullptr, stream);
}

msc_status msc_mamba3_siso_disc_state_update(const msc_m3_su_args *step,
                                             const msc_m3_disc_step_args *raw,
                                             msc_stream_t stream) {
  const char *fn = "msc_mamba3_siso_disc_state_update";
  if (!raw) return api_fail(MSC_ERR_INVALID_ARG, "%s: raw is NULL", fn);
  return m3_step(fn, step, raw, stream);
}


}  // extern "C"

namespace {
template <typename Args>
msc_status check_disc(const char *fn, const Args *a) {
  if (!a) return api_fail(MSC_ERR_INVALID_ARG, "%s: args is NULL", fn);
  if (a->struct_size < sizeof(Args))
    return api_fail(MSC_ERR_INVALID_ARG, "%s: struct_size %u is smaller than the struct (%zu)",
                    fn, a->struct_size, sizeof(Args));
  if (a->io_dtype != MSC_F32 && a->io_dtype != MSC_BF16 && a->io_dtype != MSC_F16)
    return api_fail(MSC_ERR_INVALID_ARG,
                    "%s: io_dtype %d is not MSC_F32 (0), MSC_BF16 (1) or MSC_F16 (2)",
                    fn, (int)a->io_dtype);
  if (a->batch < 0 || a->seqlen < 0 || a->nheads < 1 || a->ngroups < 1 || a->dstate < 1 ||
      a->nangles < 0)
    return api_fail(MSC_ERR_INVALID_ARG,
                    "%s: need batch >= 0, seqlen >= 0, nheads >= 1, ngroups >= 1, dstate >= 1, "
                    "nangles >= 0", fn);
  if (2 * a->nangles > a->dstate)
    return api_fail(MSC_ERR_INVALID_ARG, "%s: 2 * nangles (%lld) exceeds dstate (%lld)", fn,
                    (long long)(2 * a->nangles), (long long)a->dstate);
  if (!(a->A_floor >= 0.f) || !(a->eps >= 0.f))
    return api_fail(MSC_ERR_INVALID_ARG, "%s: A_floor and eps must be >= 0", fn);
  // per-warp shared memory holds a token's per-head dt, its angles and (backward)
  // its dtheta rows
  if (a->nheads * (a->nangles + 2) + a->nangles > 6144)
    return api_fail(MSC_ERR_UNSUPPORTED, "%s: nheads * (nangles + 2) + nangles must be <= 6144",
                    fn);
  if (a->batch * a->seqlen == 0) return MSC_OK;
  M3_REQUIRE(fn, "dd_dt", a->dd_dt);
  M3_REQUIRE(fn, "dd_a", a->dd_a);
  M3_REQUIRE(fn, "trap", a->trap);
  if (a->nangles > 0) M3_REQUIRE(fn, "angles", a->angles);
  M3_OPTIONAL(fn, "dt_bias", a->dt_bias);
  M3_REQUIRE(fn, "B_raw", a->B_raw);
  M3_REQUIRE(fn, "C_raw", a->C_raw);
  return MSC_OK;
}

msc::M3DiscParams disc_params(const msc_m3_disc_args *a) {
  msc::M3DiscParams p = {};
  p.io = a->io_dtype;
  p.B = a->batch; p.L = a->seqlen; p.H = a->nheads; p.N = a->dstate; p.G = a->ngroups;
  p.K = a->nangles; p.A_floor = a->A_floor; p.eps = a->eps;
  p.dd_dt = a->dd_dt; p.dd_a = a->dd_a; p.trap = a->trap; p.angles = a->angles;
  p.dt_bias = a->dt_bias; p.B_raw = a->B_raw; p.C_raw = a->C_raw;
  return p;
}
}  // namespace

extern "C" {

msc_status msc_mamba3_siso_discretize(const msc_m3_disc_args *a, msc_stream_t stream) {
  const char *fn = "msc_mamba3_siso_discretize";
  msc_status st = check_disc(fn, a);
  if (st != MSC_OK) return st;
  if (a->batch * a->seqlen == 0) return api_ok();
  M3_REQUIRE(fn, "alpha", a->alpha);
  M3_REQUIRE(fn, "beta", a->beta);
  M3_REQUIRE(fn, "gamma", a->gamma);
  if (a->nangles > 0) M3_REQUIRE(fn, "theta", a->theta);
  M3_REQUIRE(fn, "Bm", a->Bm);
  M3_REQUIRE(fn, "Cm", a->Cm);
  msc::M3DiscParams p = disc_params(a);
  p.alpha = a->alpha; p.beta = a->beta; p.gamma = a->gamma; p.theta = a->theta;
  p.Bm = a->Bm; p.Cm = a->Cm;
  return api_cuda(msc::launch_m3_disc_fwd(p, reinterpret_cast<cudaStream_t>(stream)), fn);
}

msc_status msc_mamba3_siso_discretize_bwd(const msc_m3_disc_bwd_args *a, msc_stream_t stream) {
  const char *fn = "msc_mamba3_siso_discretize_bwd";
  msc_status st = check_disc(fn, a);
  if (st != MSC_OK) return st;
  M3_OPTIONAL(fn, "ddt_bias", a->ddt_bias);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (a->batch * a->seqlen == 0) {  // no tokens: the bias gradient is 0
    return a->ddt_bias ? api_cuda(cudaMemsetAsync(a->ddt_bias, 0, sizeof(float) *
                                                  (size_t)a->nheads, s), fn)
                       : api_ok();
  }
  M3_REQUIRE(fn, "dalpha", a->dalpha);
  M3_REQUIRE(fn, "dbeta", a->dbeta);
  M3_REQUIRE(fn, "dgamma", a->dgamma);
  M3_REQUIRE(fn, "dB", a->dB);
  M3_REQUIRE(fn, "dC", a->dC);
  M3_REQUIRE(fn, "ddd_dt", a->ddd_dt);
  M3_REQUIRE(fn, "ddd_a", a->ddd_a);
  M3_REQUIRE(fn, "dtrap", a->dtrap);
  M3_REQUIRE(fn, "dB_raw", a->dB_raw);
  M3_REQUIRE(fn, "dC_raw", a->dC_raw);
  if (a->nangles > 0) {
    M3_REQUIRE(fn, "dtheta", a->dtheta);
    M3_REQUIRE(fn, "dangles", a->dangles);
  }
  msc_m3_disc_args f = {};
  f.io_dtype = a->io_dtype;
  f.batch = a->batch; f.seqlen = a->seqlen; f.nheads = a->nheads; f.dstate = a->dstate;
  f.ngroups = a->ngroups; f.nangles = a->nangles; f.A_floor = a->A_floor; f.eps = a->eps;
  f.dd_dt = a->dd_dt; f.dd_a = a->dd_a; f.trap = a->trap; f.angles = a->angles;
  f.dt_bias = a->dt_bias; f.B_raw = a->B_raw; f.C_raw = a->C_raw;
  msc::M3DiscParams p = disc_params(&f);
  p.dalpha = a->dalpha; p.dbeta = a->dbeta; p.dgamma = a->dgamma; p.dtheta = a->dtheta;
  p.dB = a->dB; p.dC = a->dC;
  p.ddd_dt = a->ddd_dt; p.ddd_a = a->ddd_a; p.dtrap = a->dtrap; p.dangles = a->dangles;
  p.ddt_bias = a->ddt_bias; p.dB_raw = a->dB_raw; p.dC_raw = a->dC_raw;
  return api_cuda(msc::launch_m3_disc_bwd(p, s), fn);
}

}  // extern "C"
