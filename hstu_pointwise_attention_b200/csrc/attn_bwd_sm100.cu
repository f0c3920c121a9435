// attn_bwd_sm100.cu -- backward HSTU pointwise attention on the tensor cores.
// (Not yet enabled: the CUDA-core backward in attn_simt.cu serves every shape.)
#include "internal.h"

namespace hstu {

bool bwd_tc_supported(const AttnProblem &) { return false; }

cudaError_t launch_bwd_tc(const AttnProblem &, const Scratch &, const void *, void *, void *,
                          void *, float *, float *, const WaitCtl &, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace hstu
