// api_m3.cu -- extern "C" entry points of the Mamba-3 SISO scan (msc.h).
#include <cuda_runtime.h>

#include <cstdio>

#include "../../include/msc.h"
#include "kernels.h"

namespace {
thread_local char g_m3_err[256];
}

extern "C" {

size_t msc_mamba3_siso_saved_states_bytes(int64_t batch, int64_t seqlen, int64_t nheads,
                                          int64_t headdim, int64_t dstate) {
  if (batch <= 0 || seqlen <= 0 || nheads <= 0 || headdim <= 0 || dstate <= 0) return 0;
  const int64_t nc = (seqlen + MSC_M3_CHUNK - 1) / MSC_M3_CHUNK;
  return sizeof(float) * (size_t)(batch * nheads * nc * headdim * dstate);
}

size_t msc_mamba3_siso_scan_bwd_workspace_bytes(int64_t, int64_t, int64_t, int64_t, int64_t,
                                                int64_t, int64_t) {
  return 0;
}

msc_status msc_mamba3_siso_scan_fwd(const msc_m3_fwd_args *, msc_stream_t) {
  return MSC_ERR_UNSUPPORTED;
}

msc_status msc_mamba3_siso_scan_bwd(const msc_m3_bwd_args *, void *, size_t, msc_stream_t) {
  return MSC_ERR_UNSUPPORTED;
}

}  // extern "C"
