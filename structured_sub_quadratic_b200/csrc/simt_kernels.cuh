// Host-side interface of the SIMT (general-shape) MonarchAttention kernels.
#pragma once

#include <algorithm>
#include <stddef.h>

#include "common.cuh"

namespace monarch {

// Element strides of the aggregated-query buffer read by the R-update:
// qt row (g, k, p, q, i) starts at g*g_ + k*k_ + p*p_ + q*q_ + i*i_.
// Step one reads the uniform-L means Qt0[g][p][i] (k and q strides 0).
struct QtStrides {
  long g, k, p, q, i;
};

// Workspace pieces (element counts), see simt_kernels.cu for layouts.  Kt
// and Y hold TW elements (fp32 or bf16), everything else fp32.
struct SimtWorkspaceSizes {
  size_t qt0, qt, kt, y, hs, lse, ybar;
};

struct SimtWorkspace {
  float *qt0, *qt;
  void *kt, *y;
  float *hs, *lse, *ybar;
};

SimtWorkspaceSizes simt_workspace_sizes(const Problem& pb);

// Runs the forward pass on `stream` with TW-typed Kt/Y intermediates; adds
// the number of kernels it launched to *launches.  With final_output false
// it stops after the last R-update (Kt, Y, Hs written), leaving the final
// L-update and output to the caller.
template <typename TIn, typename TW>
cudaError_t simt_forward(const TIn* q, const TIn* k, const TIn* v, TIn* out, const Problem& pb,
                         const SimtWorkspace& ws, cudaStream_t stream, int* launches,
                         bool final_output = true);

// Single steps, for paths that run the other steps elsewhere.
// R-update of one step: qt rows addressed by `st`; writes Kt, Hs (and Y).
template <typename TIn, typename TW>
cudaError_t simt_r_update(const TIn* k, const TIn* v, const float* qt, const QtStrides& st,
                          TW* kt, TW* y, float* hs, const Problem& pb, bool write_y,
                          cudaStream_t stream, int* launches);

// Non-final L-update: row log-sum-exps, then the aggregated queries
// Qt [G][b1 k][c1][c2][b2 i][d] (fp32) of the next step.
template <typename TIn, typename TW>
cudaError_t simt_l_update(const TIn* q, const TW* kt, const float* hs, float* lse, float* qt,
                          const Problem& pb, cudaStream_t stream, int* launches);

}  // namespace monarch
