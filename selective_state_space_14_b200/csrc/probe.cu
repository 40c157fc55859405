// probe.cu -- throughput probes of the two pipes the Mamba-1 scans lean on:
// the SFU's 2^x (ex2.approx.ftz.f32) and the FMA pipe's fused multiply-add
// (scalar fma.rn.f32 and packed fma.rn.f32x2).  They measure the compute
// ceiling that the scan kernels are held against beside the HBM line: every
// state element of every step takes one 2^x (its decay), so the SFU rate sets
// a floor on the scan's time that no memory layout removes.
//
// Each thread runs kChains independent dependency chains for `iters` rounds
// (unrolled by four, so that the loop's own instructions take few issue
// slots), so that the pipe, not the latency of one chain, bounds the rate; the
// results are folded into out[thread] so that no chain is dead code.  The
// chains stay finite: 2^-x maps [0, 1] into [0.5, 1], and x * a + b with
// a = 1 - 2^-10, b = 2^-10 stays in [0, 1].
#include <cuda_runtime.h>

#include "../../include/msc.h"
#include "common.cuh"

namespace msc {
msc_status api_fail(msc_status st, const char *fmt, ...);
msc_status api_ok();
msc_status api_cuda(cudaError_t e, const char *what);
}  // namespace msc

namespace {

constexpr int kChains = 8;
constexpr int kProbeThreads = 256;

__global__ void __launch_bounds__(kProbeThreads) probe_ex2_kernel(float *out, int iters) {
  float x[kChains];
#pragma unroll
  for (int c = 0; c < kChains; ++c) x[c] = 0.125f * (float)c + 1e-3f * (float)(threadIdx.x & 7);
#pragma unroll 4
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int c = 0; c < kChains; ++c) x[c] = msc::ex2(-x[c]);
  }
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < kChains; ++c) s += x[c];
  out[(size_t)blockIdx.x * blockDim.x + threadIdx.x] = s;
}

template <bool kPacked>
__global__ void __launch_bounds__(kProbeThreads) probe_ffma_kernel(float *out, int iters) {
  constexpr float a = 1.f - 1.f / 1024.f, b = 1.f / 1024.f;
  float s = 0.f;
  if constexpr (kPacked) {
    float2 x[kChains];
#pragma unroll
    for (int c = 0; c < kChains; ++c) x[c] = make_float2(0.0625f * (float)c, 0.03125f * (float)c);
#pragma unroll 4
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int c = 0; c < kChains; ++c) x[c] = msc::fma2(x[c], msc::splat2(a), msc::splat2(b));
    }
#pragma unroll
    for (int c = 0; c < kChains; ++c) s += x[c].x + x[c].y;
  } else {
    float x[kChains];
#pragma unroll
    for (int c = 0; c < kChains; ++c) x[c] = 0.0625f * (float)c;
#pragma unroll 4
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int c = 0; c < kChains; ++c) x[c] = fmaf(x[c], a, b);
    }
#pragma unroll
    for (int c = 0; c < kChains; ++c) s += x[c];
  }
  out[(size_t)blockIdx.x * blockDim.x + threadIdx.x] = s;
}

msc_status check_probe(const char *fn, const float *out, int64_t blocks, int64_t iters,
                       int64_t *ops) {
  if (!out) return msc::api_fail(MSC_ERR_INVALID_ARG, "%s: out is NULL", fn);
  if (!ops) return msc::api_fail(MSC_ERR_INVALID_ARG, "%s: ops is NULL", fn);
  if (blocks < 1 || blocks > (1 << 20))
    return msc::api_fail(MSC_ERR_INVALID_ARG, "%s: blocks %lld outside 1..%d", fn,
                         (long long)blocks, 1 << 20);
  if (iters < 1 || iters > (1 << 24))
    return msc::api_fail(MSC_ERR_INVALID_ARG, "%s: iters %lld outside 1..%d", fn,
                         (long long)iters, 1 << 24);
  return MSC_OK;
}

}  // namespace

extern "C" {

int64_t msc_probe_threads_per_block(void) { return kProbeThreads; }

msc_status msc_probe_sfu_ex2(float *out, int64_t blocks, int64_t iters, int64_t *ops,
                             msc_stream_t stream) {
  const char *fn = "msc_probe_sfu_ex2";
  const msc_status st = check_probe(fn, out, blocks, iters, ops);
  if (st != MSC_OK) return st;
  *ops = blocks * kProbeThreads * iters * kChains;
  probe_ex2_kernel<<<(unsigned)blocks, kProbeThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      out, (int)iters);
  return msc::api_cuda(cudaGetLastError(), fn);
}

msc_status msc_probe_ffma(float *out, int64_t blocks, int64_t iters, int32_t packed, int64_t *ops,
                          msc_stream_t stream) {
  const char *fn = "msc_probe_ffma";
  const msc_status st = check_probe(fn, out, blocks, iters, ops);
  if (st != MSC_OK) return st;
  if (packed != 0 && packed != 1)
    return msc::api_fail(MSC_ERR_INVALID_ARG, "%s: packed must be 0 or 1 (got %d)", fn, packed);
  // element FMAs: a packed instruction computes two
  *ops = blocks * kProbeThreads * iters * kChains * (packed ? 2 : 1);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (packed)
    probe_ffma_kernel<true><<<(unsigned)blocks, kProbeThreads, 0, s>>>(out, (int)iters);
  else
    probe_ffma_kernel<false><<<(unsigned)blocks, kProbeThreads, 0, s>>>(out, (int)iters);
  return msc::api_cuda(cudaGetLastError(), fn);
}

}  // extern "C"
