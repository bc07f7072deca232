// verify_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) tree-verify attention.
#include "kdv_internal.cuh"

namespace kdv {

cudaError_t launch_verify_tc(const VerifyArgs&, const VerifyPlan&, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace kdv
