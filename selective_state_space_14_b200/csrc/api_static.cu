// api_static.cu -- msc_selective_scan_bwd_static: the Mamba-1 backward pass
// for callers that cannot allocate device memory.
//
// Some callers are not allowed to call cudaMalloc at the point where they run
// the backward pass: code that executes inside a pre-planned memory budget
// (every byte was reserved up front and nothing may be added later), code
// running under a custom or pooled allocator that must not be bypassed, and
// code paths that may not synchronise the device (cudaMalloc/cudaFree can
// synchronise).  For them this entry point takes its scratch from a fixed
// array in the library's own device memory instead of from the caller.
//
// The array below is part of the library image: every GPU on which the library
// is loaded holds it (MSC_STATIC_SCRATCH_BYTES) until the process exits.
// Host code cannot use the array's name as a device address -- it names a
// host-side shadow -- so the device address is looked up with
// cudaGetSymbolAddress, once per device, with that device current, on the
// first call made on that device.  Make that first call before any stream
// capture.  The address is kept for the life of the process: a
// cudaDeviceReset (or anything else that tears down and rebuilds the device's
// primary context) reloads the module and may move the array, so do not use
// this entry point across such a reset.  All calls share the one array: calls whose executions overlap on
// the GPU (different streams, or different host threads on one stream without
// ordering) race on it and must be serialised by the caller.  The backward
// kernels overwrite every scratch word they later read, so nothing in the
// array needs to start at zero and the previous call's contents are harmless.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/msc.h"
#include "kernels.h"

namespace msc {
msc_status api_fail(msc_status st, const char *fmt, ...);
msc_status m1_bwd_check_sizes(const char *fn, const msc_ss_bwd_args *a);
}  // namespace msc

namespace {

static __device__ __align__(256) unsigned char g_bwd_scratch[MSC_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_lock;
void *g_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" msc_status msc_selective_scan_bwd_static(const msc_ss_bwd_args *args,
                                                    msc_stream_t stream) {
  const char *fn = "msc_selective_scan_bwd_static";
  if (!args) return msc::api_fail(MSC_ERR_INVALID_ARG, "%s: args is NULL", fn);
  if (args->struct_size < sizeof(msc_ss_bwd_args))
    return msc::api_fail(MSC_ERR_INVALID_ARG, "%s: struct_size %u < sizeof(msc_ss_bwd_args) %zu",
                         fn, args->struct_size, sizeof(msc_ss_bwd_args));
  // the backward's own argument checks first: the scratch size is computed
  // from sizes that are known to be valid (ngroups >= 1 and a divisor of dim)
  const msc_status st = msc::m1_bwd_check_sizes(fn, args);
  if (st != MSC_OK) return st;
  const size_t need = msc_selective_scan_bwd_workspace_bytes(
      args->batch, args->dim, args->dstate, args->seqlen, args->ngroups);
  if (need > (size_t)MSC_STATIC_SCRATCH_BYTES)
    return msc::api_fail(MSC_ERR_WORKSPACE,
                         "%s: these sizes need %zu bytes of scratch, more than the %zu bytes of "
                         "the library's static scratch; use msc_selective_scan_bwd with a "
                         "caller-provided workspace",
                         fn, need, (size_t)MSC_STATIC_SCRATCH_BYTES);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return msc::api_fail(MSC_ERR_CUDA, "%s: cudaGetDevice failed: %s", fn, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return msc::api_fail(MSC_ERR_UNSUPPORTED, "%s: device ordinal %d beyond %d", fn, dev,
                         kMaxDevices);
  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> guard(g_lock);
    if (g_scratch_addr[dev] == nullptr) {
      void *ptr = nullptr;
      e = cudaGetSymbolAddress(&ptr, g_bwd_scratch);
      if (e != cudaSuccess || ptr == nullptr)
        return msc::api_fail(MSC_ERR_CUDA, "%s: cudaGetSymbolAddress of the static scratch "
                                           "failed on device %d: %s",
                             fn, dev, cudaGetErrorString(e));
      g_scratch_addr[dev] = ptr;
    }
    scratch = g_scratch_addr[dev];
  }
  return msc_selective_scan_bwd(args, scratch, (size_t)MSC_STATIC_SCRATCH_BYTES, stream);
}
