// Stage 1 on the tensor cores (tcgen05): not built yet in this revision.
#include "internal.h"

namespace lsh {
bool hash_tc_supported(const Problem&) { return false; }
cudaError_t launch_hash_tc(const Problem&, const void*, const void*, int16_t*, float*,
                           cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace lsh
