// tcgen05 tensor-core path (bf16).  Not yet enabled: every shape falls back
// to the SIMT kernels.
#include "tc_path.cuh"

namespace monarch {

bool tc_supports(const Problem&) { return false; }

size_t tc_workspace_bytes(const Problem&) { return 0; }

cudaError_t tc_forward(const bf16*, const bf16*, const bf16*, bf16*, const Problem&, char*, int*,
                       cudaStream_t, int*) {
  return cudaErrorNotSupported;
}

}  // namespace monarch
