// Host-side interface of the CUDA-core kernels for shapes whose groups are
// too small for the tensor-core tiles (bf16 in and out, fp32 arithmetic).
#pragma once

#include "common.cuh"

namespace monarch {

// Step-one aggregation when every row group holds at most 16 rows: one warp
// per (g, p, i).  Unpadded shapes only.
bool small_init_fits(const Problem& pb);
cudaError_t launch_small_init(const bf16* q, bf16* qt0, const Problem& pb, cudaStream_t stream,
                              int* launches);

// R-update when every column group holds at most 8 keys and a chunk at most
// 32 positions: one warp per sub-item (g, p, k, q).  `qt_per_item` selects
// the query rows as in the tensor-core R-update (0: Qt0 [G][c1][b2][d],
// 1: Qt [G][b1][c1][c2][b2][d]); Y is written when `write_y`.  Unpadded
// shapes only.
bool small_r_fits(const Problem& pb);
cudaError_t launch_small_r(const bf16* qt, const bf16* k, const bf16* v, bf16* kt, bf16* y,
                           float* hs, const Problem& pb, bool qt_per_item, bool write_y,
                           cudaStream_t stream, int* launches);

// Final L-update + output when every row has at most 8 keys (b1 c2 <= 8):
// one warp per (g, i, p).  Unpadded shapes only.
bool small_out_fits(const Problem& pb);
cudaError_t launch_small_out(const bf16* q, const bf16* kt, const bf16* y, const float* hs,
                             bf16* out, const Problem& pb, cudaStream_t stream, int* launches);

}  // namespace monarch
