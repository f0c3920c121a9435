// gemm_sm100.cu -- tensor-core GEMM for the layer's two projections.
// (Not yet enabled: the CUDA-core GEMM in layer.cu serves every shape.)
#include "internal.h"

namespace hstu {

bool gemm_tc_supported(const void *, int64_t, const void *, int64_t, const void *, int64_t,
                       int64_t, int64_t, int64_t) {
  return false;
}

cudaError_t launch_gemm_tc(const void *, int64_t, const void *, int64_t, const float *,
                           const void *, int64_t, void *, int64_t, int64_t, int64_t, int64_t,
                           int, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace hstu
