// persistent.cu -- placeholder until the fused greedy kernel lands.
#include "persistent.h"

namespace domino {

bool use_persistent_greedy(const Shape&) { return false; }

cudaError_t launch_persistent_greedy(const Shape&, const domino_weights_t&, const void*, const void*, const float*,
                                     int32_t*, float*, float*, const Workspace&, int32_t*, uint64_t, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace domino
