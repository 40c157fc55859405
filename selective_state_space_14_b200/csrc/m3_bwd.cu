// m3_bwd.cu -- Mamba-3 SISO scan, backward (sm_100a).  (in progress)
#include "m3_common.cuh"

namespace msc {

size_t m3_bwd_workspace_bytes(int64_t, int64_t, int64_t, int64_t, int64_t, int64_t, int64_t) {
  return 0;
}

cudaError_t launch_m3_bwd(const M3Params &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace msc
