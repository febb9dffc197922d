// Host-side pieces shared by the C-ABI entry points (monarch_api.cu and
// noalloc.cu): argument validation, the choice of kernels for a bf16 shape,
// and the per-device status word.
#pragma once

#include "common.cuh"

namespace monarch {

// MONARCH_OK or the status the header documents for these sizes
// (INVALID_ARG for counts out of range or a size overflow, UNSUPPORTED for
// d outside [1, 256]).  Checks d before any size arithmetic.
int validate_args(int B, int H, int b1, int b2, int d, int T, int c1, int c2);

Problem make_problem(int B, int H, int b1, int b2, int d, int T, int c1, int c2);

// Which kernels run a bf16 forward pass of this shape: the one-CTA-per-head
// kernel (small untiled heads, T >= 2; no workspace), the tcgen05 path
// (workspace of tc_workspace_bytes), or the SIMT kernels (every other shape).
enum class Bf16Kernels { kSmallHead, kTensorCore, kSimt };
Bf16Kernels choose_bf16_kernels(const Problem& pb);

// Device address of the status word of device `dev` (which must be
// current): a static device variable that kernels with bounded waits set on
// a timeout.  Nothing is allocated for it.  Returns a MONARCH_* status.
int device_status_word(int dev, int** out);

}  // namespace monarch
