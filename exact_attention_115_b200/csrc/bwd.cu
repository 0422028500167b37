// Backward kernels (placeholder until the tcgen05 backward lands).
#include "common.cuh"
#include "launch.h"

namespace fa {

cudaError_t launch_bwd(int dtype, int d, bool causal, const BwdLaunch& a) {
  (void)dtype; (void)d; (void)causal; (void)a;
  return cudaErrorNotSupported;
}

FA_ERROR_ACCESSOR(take_error_bwd)

}  // namespace fa
