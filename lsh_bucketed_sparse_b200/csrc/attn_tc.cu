// Stage 3 on the tensor cores (tcgen05): not built yet in this revision.
#include "internal.h"

namespace lsh {
bool attn_tc_supported(const Problem&) { return false; }
cudaError_t launch_attn_tc(const Problem&, const void*, const void*, const float*,
                           const int32_t*, void*, float*, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace lsh
