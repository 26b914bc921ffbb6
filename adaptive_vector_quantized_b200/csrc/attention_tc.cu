// placeholder: tensor-core attention kernel (added next)
#include "internal.h"
namespace avq {
bool attention_tc_supported(const Shape&, avq_dtype, int, int, int) { return false; }
size_t attention_tc_workspace(const Shape&, int, int, int) { return 0; }
cudaError_t launch_attention_tc(const Shape&, const void*, const void*, const void*, const float*,
                                const int32_t*, int, int, float, int, void*, int32_t*, float*,
                                void*, unsigned int*, cudaStream_t, LaunchLog&) {
  return cudaErrorNotSupported;
}
}  // namespace avq
