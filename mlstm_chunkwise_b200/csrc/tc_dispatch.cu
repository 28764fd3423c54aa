// Support predicates and launchers of the tensor-core kernels.
#include "tc.h"

namespace mlstm {

bool tc_unfused_supported(const Problem&) { return false; }
bool tc_fused_supported(const Problem&) { return false; }

cudaError_t launch_tc_states(const Problem&, const void*, const void*, const float*, const float*,
                             Gates, float*, float*, float*, float*, float*, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_tc_parallel(const Problem&, const void*, const void*, const void*, Gates,
                               const float*, const float*, void*, float*, float*, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_tc_fused(const Problem&, const void*, const void*, const void*, const float*,
                            const float*, Gates, void*, float*, float*, float*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace mlstm
