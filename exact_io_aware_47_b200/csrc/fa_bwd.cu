// Backward pass (placeholder launcher; kernels follow).
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

cudaError_t launch_bwd(int d, bool bf16, const CUtensorMap& tmq, const CUtensorMap& tmk,
                       const CUtensorMap& tmv, const CUtensorMap& tmdo, const BwdParams& p,
                       int num_sms, cudaStream_t stream) {
  return cudaErrorNotSupported;
}

}  // namespace fa
