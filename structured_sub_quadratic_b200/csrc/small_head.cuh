// Whole MonarchAttention forward pass of one small head per CTA (bf16).
#pragma once

#include "common.cuh"

namespace monarch {

// True for the shapes the one-CTA-per-head kernel takes: untiled
// (c1 = c2 = 1), b1, b2 <= 16, b1*b2 <= 216, d = 64, T >= 1.
bool small_head_supports(const Problem& pb);

// The forward pass on `stream` for such a shape; no workspace.  With padding
// (pb.real_lo, pb.real_hi) q, k, v and out hold only the real rows of each
// head (real_hi - real_lo of them), which the kernel reads and writes in place.
cudaError_t small_head_forward(const bf16* q, const bf16* k, const bf16* v, bf16* out,
                               const Problem& pb, cudaStream_t stream, int* launches);

}  // namespace monarch
