// Tensor-core (tcgen05) chunked prefill for bf16 inputs, sm_100a.
// Not yet available in this build: every request goes to the CUDA-core kernel.

#include "common.cuh"
#include "launch.h"

namespace gdr {

bool tc_prefill_supported(const PrefillArgs&) { return false; }

size_t tc_prefill_workspace(int, int, int, int, int, bool) { return 0; }

cudaError_t launch_prefill_tc(const PrefillArgs&, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace gdr
