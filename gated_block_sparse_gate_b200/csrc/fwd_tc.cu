// fwd_tc.cu — tensor-core (tcgen05) gated forward; placeholder until written.
#include "internal.h"

namespace gbs {
bool fwd_tc_supported(const Problem&) { return false; }
cudaError_t launch_fwd_tc(const Problem&, const void*, const void*, const void*, const float*,
                          const Selection&, const int32_t*, int, void*, float*, unsigned int*,
                          cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace gbs
