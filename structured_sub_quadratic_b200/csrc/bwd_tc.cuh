// Host-side interface of the tensor-core (tcgen05) L side of the backward
// pass (bf16, T = 1).
#pragma once

#include "common.cuh"

namespace monarch {

// True when the tensor-core L side takes this backward shape: a shape the
// tensor-core forward takes, with d in {64, 128}, rows of at most 128 keys
// (b1 c2 <= 128), row groups of at most 128 rows, Monarch token order and no
// padding.
bool bwd_tc_l_side_supports(const Problem& pb);

// The forward quantities the backward needs, recomputed by the tensor-core
// step one: bf16 Qt0 (qt0_16), Kt and Y (kt16, y16), fp32 Hs, and Qt0 in
// fp32 (qt0) for the SIMT R side, which then recomputes R from the same
// aggregated queries.
cudaError_t bwd_tc_recompute(const bf16* q, const bf16* k, const bf16* v, bf16* qt0_16,
                             bf16* kt16, bf16* y16, float* hs, float* qt0, const Problem& pb,
                             int* status, cudaStream_t stream, int* launches);

// The L side of the backward pass on the tensor cores.  Inputs: q and dO
// (bf16, (G, N, d)), the recomputed bf16 Kt, Y [G][b2][c1][b1][c2][d] and
// fp32 Hs.  Outputs, fp32, in the layouts the R side reads:
//   dq1 [G][N][d]   the L side's part of dq: sc sum_{k,q} dS_L Kt
//   dkt, dy         [G][b2][c1][b1][c2][d]: sc sum_l dS_L q, sum_l L dO
//   dhs             [G][b2][c1][b1][c2]: sum_l dS_L
// with L the final L-update's weights, dS_L = L (dO . Y - delta) and
// delta = dO . O = sum_{k,q} L (dO . Y).  `status` is the device status word
// that the bounded waits set on timeout.  Adds its launches to *launches.
// dkt16 and dy16, when not null, receive bf16 copies of dKt and dY in
// chunk-major order [G][c1][b1 k][c2 q][b2 i][d], the R side's operands.
cudaError_t bwd_tc_l_side(const bf16* q, const bf16* dout, const bf16* kt16, const bf16* y16,
                          const float* hs, float* dq1, float* dkt, float* dy, float* dhs,
                          bf16* dkt16, bf16* dy16, const Problem& pb, int* status,
                          cudaStream_t stream, int* launches);

// True when the tensor-core R side also takes the shape: untiled
// (c1 = c2 = 1) with b2 <= 128 positions.
bool bwd_tc_r_side_supports(const Problem& pb);

// The R side on the tensor cores: from bf16 Qt0 [G][b2][d], k, v and the L
// side's bf16 dKt, dY (chunk-major) and fp32 dHs, writes the partial dQt0
// [G][b2 i][b1 k][d] (fp32) and the final dk, dv (bf16, (G, N, d)).
cudaError_t bwd_tc_r_side(const bf16* qt0_16, const bf16* k, const bf16* v, const bf16* dkt16,
                          const bf16* dy16, const float* dhs, float* dqt0_part, bf16* dk,
                          bf16* dv, const Problem& pb, int* status, cudaStream_t stream,
                          int* launches);

}  // namespace monarch
