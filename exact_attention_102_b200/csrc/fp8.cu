// fp8.cu — FP8 prepare + forward (placeholder until the sm_100a kernels land).
#include "prim.cuh"
#include "kernels.h"

namespace fa {
cudaError_t launch_fp8_prepare(const Fp8PrepArgs&, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_fwd_fp8(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                           const Fp8FwdArgs&, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace fa
