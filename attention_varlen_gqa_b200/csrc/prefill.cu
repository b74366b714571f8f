// prefill.cu -- varlen GQA prefill (placeholder until the tcgen05 kernel lands).
#include "common.cuh"
#include "kernels.h"

namespace attn {
cudaError_t launch_prefill(const PrefillParams &, const CUtensorMap &, const CUtensorMap &,
                           const CUtensorMap &, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace attn
