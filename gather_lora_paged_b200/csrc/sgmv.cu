// sgmv.cu -- SGMV prefill path (placeholder until the tensor-core kernels land).
#include "slora_internal.h"

namespace slora {

size_t sgmv_scratch_bytes(const slora_pool_desc&) { return 0; }

cudaError_t launch_sgmv(const BgmvParams&, int, const int32_t*, const int32_t*, int, int, int,
                        cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace slora
