// Host-side interface of the tcgen05 tensor-core MonarchAttention path (bf16).
#pragma once

#include <cuda.h>
#include <stddef.h>

#include "common.cuh"

namespace monarch {

// True when the tensor-core kernels take this shape.
bool tc_supports(const Problem& pb);

// True when the tensor-core kernels of this shape's forward pass take q, k,
// v and out in transposed token order (Problem::tr): every shape they take.
bool tc_takes_transposed(const Problem& pb);

// bf16 TMA tensor map with 128-byte swizzle (dims and box innermost first,
// strides in bytes for dims 1..); encoded maps are cached.  False when the
// driver rejects it.
bool tc_make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                 const cuuint64_t* strides, const cuuint32_t* box);

// 3-D map of q (or of any (G, N, d) bf16 tensor in q's layout) whose box is
// the 128 rows l of one position i, from the coordinates (column, i,
// g b1 + l0) in Monarch order.
bool tc_make_q_slab_map(CUtensorMap* m, const bf16* q, const Problem& pb, int D);

// Step one of the forward pass alone (the step-one aggregation, then the
// R-update): bf16 Qt0 [G][c1][b2][d], Kt and Y [G][b2][c1][b1][c2][d] (Y
// when pb.T == 1), fp32 Hs.  For shapes tc_supports() takes.
cudaError_t tc_step_one(const bf16* q, const bf16* k, const bf16* v, bf16* qt0, bf16* kt, bf16* y,
                        float* hs, const Problem& pb, int* status, cudaStream_t stream,
                        int* launches);

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
