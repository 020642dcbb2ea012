// Tensor-core (tcgen05) attention: placeholder until the kernel lands.
#include "common.cuh"
#include "launch.h"

namespace httm {
bool attention_tc_supported(const Dims&, bool) { return false; }
cudaError_t launch_attention_tc(const Dims&, const void*, const void*, const void*, void*, int, const Buffers&,
                                cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace httm
