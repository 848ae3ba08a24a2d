// attn_bwd_sm100.cu - placeholder until the tcgen05 backward lands.
#include "common.cuh"
#include "sm100_primitives.cuh"

namespace flint {
cudaError_t launch_attn_bwd_sm100_impl(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                       const CUtensorMap&, const Resolved&, const float*,
                                       const float*, const int4*, const int*, int, const int4*,
                                       const int*, int, float*, float*, void*, int*, int,
                                       cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace flint
