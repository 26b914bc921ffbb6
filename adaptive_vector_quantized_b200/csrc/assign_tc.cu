// placeholder: tensor-core assignment kernel (added next)
#include "internal.h"
namespace avq {
bool assign_tc_supported(const Shape&, avq_dtype) { return false; }
cudaError_t launch_assign_tc(const Shape&, const void*, const void*, const void*, int32_t*,
                             unsigned int*, cudaStream_t, LaunchLog&) {
  return cudaErrorNotSupported;
}
}  // namespace avq
