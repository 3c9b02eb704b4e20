// chunk_tc.cu -- tensor-core (tcgen05) chunked forward. Not yet available in
// this build: every problem is routed to the CUDA-core kernel.
#include "common.cuh"
#include "internal.h"

namespace pdn {

int tc_supported(const KParams &) { return 0; }

size_t tc_workspace_bytes(const KParams &) { return 0; }

cudaError_t launch_chunk_tc(const KParams &, void *, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace pdn
