// Placeholders for tensor-core kernels not built yet: every problem goes to
// the generic kernels.
#include "tc.h"

namespace gqla {

bool tc_expand_supports(const Problem&) { return false; }
cudaError_t tc_expand(const Problem&, const void*, const void*, const void*, void*, void*, int, int32_t*,
                      cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace gqla
