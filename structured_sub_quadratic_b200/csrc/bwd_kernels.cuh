// Host-side interface of the backward-pass kernels (T = 1).
#pragma once

#include <stddef.h>

#include "common.cuh"

namespace monarch {

// fp32 workspace pieces (element counts); layouts in bwd_kernels.cu.
// (qt016, kt16, y16: the bf16 Qt0, Kt and Y of the tensor-core recompute;
// dkt16, dy16: bf16 dKt and dY for the tensor-core R side; counted in floats.)
struct BwdWorkspaceSizes {
  size_t qt0, kt, y, hs, lse, delta, dq1, dkt, dy, dhs, rbuf, dsbuf, dqt0_part, qt016, kt16, y16,
      dkt16, dy16;
};

struct BwdWorkspace {
  float *qt0, *kt, *y, *hs, *lse, *delta, *dq1, *dkt, *dy, *dhs, *rbuf, *dsbuf, *dqt0_part,
      *qt016, *kt16, *y16, *dkt16, *dy16;
};

BwdWorkspaceSizes bwd_workspace_sizes(const Problem& pb);

// Gradients dq, dk, dv of sum(O * dout) for the forward pass with T = 1
// (unpadded), on `stream`; adds its launch count to *launches.  bf16 shapes
// the tensor-core L side takes (bwd_tc.cuh) run it there; `status` is the
// device status word its bounded waits set on timeout.
template <typename TIn>
cudaError_t bwd_forward_t1(const TIn* q, const TIn* k, const TIn* v, const TIn* dout, TIn* dq,
                           TIn* dk, TIn* dv, const Problem& pb, const BwdWorkspace& ws,
                           int* status, cudaStream_t stream, int* launches);

}  // namespace monarch
