// Tensor-core (tcgen05) matching: placeholder until the kernel lands.
#include "common.cuh"
#include "launch.h"

namespace httm {
bool match_tc_supported(const Dims&, bool) { return false; }
cudaError_t launch_match_tc(const Dims&, const BlockDesc*, const int4*, int, const void*, const void*,
                            const Buffers&, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace httm
