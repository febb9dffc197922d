// Host-side interface of the tcgen05 tensor-core MonarchAttention path (bf16).
#pragma once

#include <stddef.h>

#include "common.cuh"

namespace monarch {

// True when the tensor-core kernels take this shape.
bool tc_supports(const Problem& pb);

// True when every tensor-core kernel of this shape's forward pass takes q,
// k, v and out in transposed token order (Problem::tr; the later steps of
// some shapes run on SIMT kernels, which do not).
bool tc_takes_transposed(const Problem& pb);

// Workspace bytes the tensor-core path needs for this shape.
size_t tc_workspace_bytes(const Problem& pb);

// Whole forward pass on `stream`.  `ws` is a device buffer of at least
// tc_workspace_bytes(pb); `status` is the device status word that kernels
// with bounded waits set on timeout.  Adds its launch count to *launches.
cudaError_t tc_forward(const bf16* q, const bf16* k, const bf16* v, bf16* out, const Problem& pb,
                       char* ws, int* status, cudaStream_t stream, int* launches);

// Launches one CTA whose bounded wait must expire after limit_ns and set the
// status word (exercises the timeout path without any fault).
cudaError_t tc_selftest_timeout(int* status, unsigned long long limit_ns, cudaStream_t stream);

}  // namespace monarch
